// Test-only shim: exposes the fused engine's host-side tile schedule (csrc/schedule.cu) and
// status-word decoding (csrc/status.cu), compiled here as plain C++, to the CPU tests through
// C functions.
#include <string.h>

#include <stdio.h>

#include <string>
#include <vector>

#include "fused.cuh"
#include "status.h"

extern "C" int kda_test_schedule(int BP, int H, int nh, int dk, int dv, int r, int num_ctas, size_t cap,
                                 uint8_t *mat, uint8_t *flags, uint16_t *rb, uint16_t *kb, uint32_t *seg,
                                 uint32_t *seg0, uint16_t *nseg, uint32_t *off, uint32_t *rbinfo, size_t rbcap,
                                 size_t *ntiles, size_t *nseg_total)
{
    std::vector<kda::TileEntry> t;
    std::vector<uint32_t> o, info;
    size_t ns = 0;
    const kda::Dims d{BP, H, nh, dk, dv, r};
    kda::fused_build_schedule(d, num_ctas, kda::fused_sched_geo(d, BP), &t, &o, &ns, &info);
    *ntiles = t.size();
    *nseg_total = ns;
    if (t.size() > cap || info.size() > rbcap) return 1;
    for (size_t i = 0; i < t.size(); ++i) {
        mat[i] = t[i].mat;
        flags[i] = t[i].flags;
        rb[i] = t[i].rg;
        kb[i] = t[i].kb;
        seg[i] = t[i].seg;
        seg0[i] = t[i].seg0;
        nseg[i] = t[i].nseg;
    }
    memcpy(off, o.data(), o.size() * 4);
    memcpy(rbinfo, info.data(), info.size() * 4);
    return 0;
}

// Schedule shape for padded batch BP: rows per q/k/v tile, rows per W_o tile, run length.
extern "C" void kda_test_sched_geo(int BP, int H, int nh, int dk, int dv, int r, int *nx, int *no, int *run)
{
    const kda::SchedGeo g = kda::fused_sched_geo(kda::Dims{BP, H, nh, dk, dv, r}, BP);
    *nx = g.nx;
    *no = g.no;
    *run = g.run;
}

// Decodes three status words in place; returns the status, *fatal and the message.
extern "C" int kda_test_take_status(int *words, int *fatal, char *msg, size_t cap)
{
    bool f = *fatal != 0;
    std::string m;
    const int st = kda::take_status(words, &f, &m);
    *fatal = f ? 1 : 0;
    snprintf(msg, cap, "%s", m.c_str());
    return st;
}
