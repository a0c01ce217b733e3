// Test-only shim: exposes the fused engine's host-side tile schedule (csrc/schedule.cu,
// compiled here as plain C++) to the CPU tests through a C function.
#include <string.h>

#include <vector>

#include "fused.cuh"

extern "C" int kda_test_schedule(int B, int H, int nh, int dk, int dv, int r, int num_ctas, size_t cap,
                                 uint8_t *mat, uint8_t *flags, uint16_t *rb, uint16_t *kb, uint32_t *seg,
                                 uint32_t *seg0, uint16_t *nseg, uint32_t *off, uint32_t *rbinfo, size_t rbcap,
                                 size_t *ntiles, size_t *nseg_total)
{
    std::vector<kda::TileEntry> t;
    std::vector<uint32_t> o, info;
    size_t ns = 0;
    kda::fused_build_schedule(kda::Dims{B, H, nh, dk, dv, r}, num_ctas, &t, &o, &ns, &info);
    *ntiles = t.size();
    *nseg_total = ns;
    if (t.size() > cap || info.size() > rbcap) return 1;
    for (size_t i = 0; i < t.size(); ++i) {
        mat[i] = t[i].mat;
        flags[i] = t[i].flags;
        rb[i] = t[i].rb;
        kb[i] = t[i].kb;
        seg[i] = t[i].seg;
        seg0[i] = t[i].seg0;
        nseg[i] = t[i].nseg;
    }
    memcpy(off, o.data(), o.size() * 4);
    memcpy(rbinfo, info.data(), info.size() * 4);
    return 0;
}
