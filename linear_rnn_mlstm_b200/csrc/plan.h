// Launch plan of the chunkwise forward and the workspace layout it implies.
//
// The forward follows the chunkwise-parallel form of the mLSTM recurrence: a
// head's sequence is cut into chunks of L tokens; inside a chunk the outputs
// are a masked, gate-decayed quadratic form (like attention), and across
// chunks a d x d state is carried.  To run long sequences on all SMs, each
// head's chunks are grouped into P segments that run concurrently:
//   phase 0 (gates)    per-chunk prefix sums of log f and maxima of log i - b;
//   phase 1 (summary)  per segment g < P-1, the segment's own contribution to
//                      the state at its end, with its own stabiliser;
//   phase 3 (outputs)  per (segment, value-row tile): fold the summaries of
//                      segments 0..g-1 into the incoming state, then walk the
//                      segment's chunks, writing h and, for the last segment,
//                      the final state.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace xlstm {

struct FwdPlan {
    int B, NH, S, DH, L;      // L = chunk
    int BH;
    int nchunks;              // ceil(S / L)
    int P;                    // segments per head
    int cps;                  // chunks per segment
    int path;                 // 1 = SIMT, 2 = tensor core
    int rows;                 // value rows per output CTA
    int ntiles;               // ceil(DH / rows)
    int Spad;                 // S rounded up to 64 tokens (row stride of off_upad)
    // workspace layout, in floats from the workspace base
    size_t off_bcum;          // [BH, S]        chunk-local inclusive cumsum of log f
    size_t off_pmax;          // [BH, S]        chunk-local inclusive prefix max of log i - b
    // the same per-token gate values with rows padded to Spad (256-byte aligned
    // 64-token tiles, fetched by bulk copies):
    size_t off_upad;          // [BH, Spad]     log i - b
    size_t off_bpad;          // [BH, Spad]     b
    size_t off_xpad;          // [BH, Spad]     chunk-local prefix max of log i - b
    size_t off_cstat;         // [BH, nchunks, 2]  (chunk total of log f, chunk max of log i - b)
    size_t off_sstat;         // [BH, P, 2]     (segment total of log f, segment stabiliser)
    size_t off_summ;          // [BH, P-1, DH*DH + DH]  segment summaries (C part then n part)
    // DH 512 on the tensor path (key columns split over two CTAs):
    size_t off_part;          // [2, BH, S, DH]  each key half's numerator
    size_t off_dpart;         // [2, BH, S]      each key half's denominator
    size_t off_tok;           // [BH, S, 2]      row factor and floor per token
    size_t total_floats;
    size_t bytes() const { return total_floats * sizeof(float); }
};

// Fills `p`; returns false if the configuration cannot be planned.
bool make_fwd_plan(int B, int NH, int S, int DH, int L, int path, int forced_segments,
                   int num_sms, FwdPlan *p);
// Recomputes the workspace offsets of `p` from its sizes and P (make_fwd_plan
// calls it; a caller that changes P afterwards calls it again).
void layout_fwd_workspace(FwdPlan *p);

}  // namespace xlstm
