// Host emulation of the sLSTM forward kernel (test infrastructure).
//
// Runs the kernel's own per-unit code (linear_rnn_mlstm_b200/csrc/slstm_body.cuh)
// on the CPU: for each head, every unit's step t runs one after another, then
// the "barrier", exactly the order of dependencies the kernel's one barrier
// per step enforces.  Every buffer is its own exact-size allocation, so a build
// with AddressSanitizer reports any access outside them.
//
// usage: slstm_emulation IN OUT
//   IN : int32 B, NH, S, DH, fgate_exp, has_state; float32 zx, ix, fx, ox
//        [BH*S*DH], R [NH*4*DH*DH], then c0, n0, m0, h0 [BH*DH] if has_state
//   OUT: float32 h [BH*S*DH], c, n, m, h_last [BH*DH]
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "slstm_body.cuh"

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
    int hdr[6];
    if (fread(hdr, sizeof(int), 6, in) != 6) return 2;
    const int B = hdr[0], NH = hdr[1], S = hdr[2], DH = hdr[3];
    const int BH = B * NH;
    const size_t nx = (size_t)BH * S * DH, ns = (size_t)BH * DH;
    std::vector<float> zx = read_floats(in, nx), ix = read_floats(in, nx),
                       fx = read_floats(in, nx), ox = read_floats(in, nx);
    std::vector<float> R = read_floats(in, (size_t)NH * 4 * DH * DH);
    std::vector<float> c0, n0, m0, h0;
    if (hdr[5]) {
        c0 = read_floats(in, ns); n0 = read_floats(in, ns);
        m0 = read_floats(in, ns); h0 = read_floats(in, ns);
    }
    fclose(in);
    std::vector<float> h(nx), c_out(ns), n_out(ns), m_out(ns), h_out(ns);
    xlstm::slstm::SlstmPtrs p;
    p.zx = zx.data(); p.ix = ix.data(); p.fx = fx.data(); p.ox = ox.data(); p.R = R.data();
    p.h = h.data();
    p.c0 = hdr[5] ? c0.data() : nullptr; p.n0 = hdr[5] ? n0.data() : nullptr;
    p.m0 = hdr[5] ? m0.data() : nullptr; p.h0 = hdr[5] ? h0.data() : nullptr;
    p.c_out = c_out.data(); p.n_out = n_out.data(); p.m_out = m_out.data(); p.h_out = h_out.data();
    p.BH = BH; p.NH = NH; p.S = S; p.DH = DH; p.fgate_exp = hdr[4];
    for (int bh = 0; bh < BH; ++bh) {
        std::vector<float> hbuf0(DH), hbuf1(DH);        // the two shared arrays
        std::vector<float> c(DH), n(DH), m(DH);
        float *bufs[2] = {hbuf0.data(), hbuf1.data()};
        for (int j = 0; j < DH; ++j) xlstm::slstm::unit_init(p, bh, j, c[j], n[j], m[j], bufs[0]);
        for (int t = 0; t < S; ++t)
            for (int j = 0; j < DH; ++j)
                xlstm::slstm::unit_step(p, bh, j, t, bufs[t & 1], bufs[(t + 1) & 1], c[j], n[j], m[j]);
        for (int j = 0; j < DH; ++j) xlstm::slstm::unit_final(p, bh, j, c[j], n[j], m[j], bufs[S & 1]);
    }
    FILE *out = fopen(argv[2], "wb");
    if (!out) return 2;
    for (const std::vector<float> *a : {&h, &c_out, &n_out, &m_out, &h_out})
        if (!a->empty()) fwrite(a->data(), sizeof(float), a->size(), out);
    fclose(out);
    return 0;
}
