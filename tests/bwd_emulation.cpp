// Host emulation of the mLSTM backward kernels (test infrastructure).
//
// Runs the kernels' own per-thread bodies (linear_rnn_mlstm_b200/csrc/bwd_body.cuh)
// on the CPU, one "thread" after another in launch order, on fp32 inputs read
// from a file, and writes the gradients to another file.  Every buffer is its
// own exact-size heap allocation, so a build with AddressSanitizer reports any
// access outside the buffers the kernels are given.
//
// usage: bwd_emulation IN OUT
//   IN : int32 B, NH, S, DH, L, fgate_exp, has_dC, has_dn; then float32
//        q, k, v [BH*S*DH], itilde, ftilde [BH*S], otilde, dh [BH*S*DH],
//        dC [BH*DH*DH] (if has_dC), dn [BH*DH] (if has_dn)
//   OUT: float32 dq, dk, dv [BH*S*DH], ditilde, dftilde [BH*S], dotilde [BH*S*DH]
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "bwd_body.cuh"

using xlstm::bwd::BwdPtrs;

static std::vector<float> read_floats(FILE *f, size_t n) {
    std::vector<float> v(n);
    if (n && fread(v.data(), sizeof(float), n, f) != n) {
        fprintf(stderr, "short read\n");
        exit(2);
    }
    return v;
}

int main(int argc, char **argv) {
    if (argc != 3) return 2;
    FILE *in = fopen(argv[1], "rb");
    if (!in) return 2;
    int hdr[8];
    if (fread(hdr, sizeof(int), 8, in) != 8) return 2;
    const int B = hdr[0], NH = hdr[1], S = hdr[2], DH = hdr[3], L = hdr[4];
    const int BH = B * NH, NC = (S + L - 1) / L;
    const size_t nx = (size_t)BH * S * DH, ng = (size_t)BH * S, DD = (size_t)DH * DH;
    std::vector<float> q = read_floats(in, nx), k = read_floats(in, nx), v = read_floats(in, nx);
    std::vector<float> ip = read_floats(in, ng), fp = read_floats(in, ng);
    std::vector<float> op = read_floats(in, nx), dh = read_floats(in, nx);
    std::vector<float> dC, dn;
    if (hdr[6]) dC = read_floats(in, (size_t)BH * DD);
    if (hdr[7]) dn = read_floats(in, (size_t)BH * DH);
    fclose(in);

    std::vector<float> dq(nx), dk(nx), dv(nx), di(ng), df(ng), dO(nx);
    std::vector<float> logf(ng), b(ng), mt(ng), den(ng), nq(ng), A(ng), dF(ng), dnq(ng);
    std::vector<float> mprev((size_t)BH * NC), mend((size_t)BH * NC), Bsum((size_t)BH * NC);
    std::vector<float> Cst((size_t)BH * (NC + 1) * DD), nst((size_t)BH * (NC + 1) * DH);
    std::vector<float> num(nx), dnum(nx);
    std::vector<float> dCb((size_t)BH * NC * DD), dnb((size_t)BH * NC * DH);

    BwdPtrs p;
    p.q = q.data(); p.k = k.data(); p.v = v.data();
    p.ip = ip.data(); p.fp = fp.data(); p.op = op.data(); p.dh = dh.data();
    p.dC = hdr[6] ? dC.data() : nullptr;
    p.dn = hdr[7] ? dn.data() : nullptr;
    p.dq = dq.data(); p.dk = dk.data(); p.dv = dv.data();
    p.di = di.data(); p.df = df.data(); p.dO = dO.data();
    p.logf = logf.data(); p.b = b.data(); p.mt = mt.data(); p.den = den.data();
    p.nq = nq.data(); p.A = A.data(); p.dF = dF.data(); p.dnq = dnq.data();
    p.mprev = mprev.data(); p.mend = mend.data(); p.Bsum = Bsum.data();
    p.Cst = Cst.data(); p.nst = nst.data(); p.num = num.data(); p.dnum = dnum.data();
    p.dCb = dCb.data(); p.dnb = dnb.data();
    p.BH = BH; p.S = S; p.DH = DH; p.L = L; p.NC = NC; p.fgate_exp = hdr[5];
    p.dnhl = nullptr; p.dki = nullptr; p.dvi = nullptr; p.tc = 0;

    if (S > 0) {
        for (int h = 0; h < BH; ++h) xlstm::bwd::gates_head(p, h);
        for (int h = 0; h < BH; ++h)
            for (int r = 0; r <= DH; ++r) xlstm::bwd::states_row<float>(p, h, r);
        for (int h = 0; h < BH; ++h)
            for (int t = 0; t < S; ++t) xlstm::bwd::token_fwd<float>(p, h, t);
        for (int h = 0; h < BH; ++h)
            for (int r = 0; r <= DH; ++r) xlstm::bwd::reverse_row<float>(p, h, r);
        for (int h = 0; h < BH; ++h)
            for (int t = 0; t < S; ++t) xlstm::bwd::token_grad<float>(p, h, t);
        for (int h = 0; h < BH; ++h) xlstm::bwd::forget_head(p, h);
    }

    FILE *out = fopen(argv[2], "wb");
    if (!out) return 2;
    for (const std::vector<float> *a : {&dq, &dk, &dv, &di, &df, &dO})
        if (!a->empty()) fwrite(a->data(), sizeof(float), a->size(), out);
    fclose(out);
    return 0;
}
