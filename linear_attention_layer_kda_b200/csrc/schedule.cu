// schedule.cu -- host-only: the fused engine's tile schedule (which CTA streams which weight
// tiles, in which order, and where each run's partial sum goes).  Kept apart from the kernel
// so that its invariants can be checked on a machine without a GPU.
#include <stdlib.h>

#include <algorithm>
#include <vector>

#include "fused.cuh"

namespace kda {

// Row groups of N = 256 weight rows while the epilogue's running sums allow it (fewer for
// 32 and 64 sequences).  Runs: short ones spread each row group over more SMs, so its last
// partial sum lands sooner, but every run writes a partial sum (BP x N fp32) and adds one to
// the consumers' reads.  Measured at hidden 4096 (32 heads of 128 x 128): 2 tiles for 8
// sequences (31.9 us against 32.5 us with 4), 4 for 16 (41.6 us against 48.7 us with 8); 8 for
// 32 sequences lies between.  At 64 sequences and hidden 6144 (48 K blocks): two runs of 24
// (209 us) against 32 + 16 (233 us), 12 (220 us), 8 (235 us) or 48 (247 us).
SchedGeo fused_sched_geo(const Dims &dmax, int BP)
{
    const ActGeo g = act_geo(BP);
    const int nkb = std::max(1, dmax.H / 128);
    // longest run per padded batch (measured), then the K blocks of a row group cut into the
    // fewest runs of equal length that respect it (48 blocks at 64 rows: 2 x 24, not 32 + 16)
    const int longest = BP <= 8 ? 2 : (BP <= 16 ? 4 : (BP <= 32 ? 8 : BP / 2));
    const int nrun = (nkb + longest - 1) / longest;
    return SchedGeo{g.nx, g.no, (nkb + nrun - 1) / nrun};
}

// Tile order and segments.
//
// A tile is `rows` weight rows (a row group) x one 128-wide K block.  The q, k and v row
// groups are listed in the order of the first head they hold (q, k, v of the same heads side
// by side), each with all its K blocks; then the W_o tiles, in chunks of `run` consecutive K
// blocks (o blocks, i.e. heads): chunk 0 for every output row group, then chunk 1, ...
//
// The list is dealt out in waves: wave w gives CTA c the `run` tiles at list positions
// (w * P + c) * run ..., so all SMs stream the earliest heads' weights first and those heads'
// q/k/v are final long before the stream ends; the state units of early heads, and the W_o
// tiles that read their o blocks, then overlap the rest of the stream.  The tiles left over
// after the last full wave are split into P contiguous pieces of equal size (+-1), so every
// CTA streams the same number of tiles to within one.
//
// A segment is a CTA's run of consecutive tiles of one row group; its partial sum goes to its
// own slot.  Slots are numbered row group by row group, so the slots of a row group are
// adjacent (rbinfo: first slot, count).
void fused_build_schedule(const Dims &d, int P, const SchedGeo &g, std::vector<TileEntry> *tiles,
                          std::vector<uint32_t> *off, size_t *nseg_total, std::vector<uint32_t> *rbinfo)
{
    const int nKBx = d.H / 128, nKBo = d.Dv() / 128;
    const int nRGq = (d.Dk() + g.nx - 1) / g.nx, nRGv = (d.Dv() + g.nx - 1) / g.nx, nRGo = (d.H + g.no - 1) / g.no;
    int run = std::max(1, g.run);
    if (const char *e = getenv("KDA_RUN")) run = std::max(1, atoi(e));
    struct T { uint8_t mat; uint16_t rg, kb; };
    std::vector<T> list;
    list.reserve((size_t)(2 * nRGq + nRGv) * nKBx + (size_t)nRGo * nKBo);
    // q/k/v row groups by first head, then matrix
    struct G { int head, mat, rg; };
    std::vector<G> groups;
    for (int rg = 0; rg < nRGq; ++rg) {
        groups.push_back(G{rg * g.nx / d.dk, 0, rg});
        groups.push_back(G{rg * g.nx / d.dk, 1, rg});
    }
    for (int rg = 0; rg < nRGv; ++rg) groups.push_back(G{rg * g.nx / d.dv, 2, rg});
    std::stable_sort(groups.begin(), groups.end(),
                     [](const G &a, const G &b) { return a.head != b.head ? a.head < b.head : a.mat < b.mat; });
    for (const G &x : groups)
        for (int kb = 0; kb < nKBx; ++kb) list.push_back(T{(uint8_t)x.mat, (uint16_t)x.rg, (uint16_t)kb});
    for (int k0 = 0; k0 < nKBo; k0 += run)
        for (int rg = 0; rg < nRGo; ++rg)
            for (int kb = k0; kb < std::min(nKBo, k0 + run); ++kb) list.push_back(T{3, (uint16_t)rg, (uint16_t)kb});

    std::vector<std::vector<T>> per_cta(P);
    const size_t n = list.size();
    size_t pos = 0;
    while (n - pos >= (size_t)P * run) {  // full waves
        for (int c = 0; c < P; ++c)
            for (int i = 0; i < run; ++i) per_cta[c].push_back(list[pos++]);
    }
    {  // the rest, in P contiguous pieces of equal size (+-1)
        const size_t rest = n - pos, base = rest / P, extra = rest % P;
        for (int c = 0; c < P; ++c) {
            const size_t len = base + ((size_t)c < extra ? 1 : 0);
            for (size_t i = 0; i < len; ++i) per_cta[c].push_back(list[pos++]);
        }
    }

    // row-group keys: q 0.., k nRGq.., v 2 nRGq.., o 2 nRGq + nRGv..
    auto key = [&](const T &t) {
        return t.mat == 3 ? 2 * nRGq + nRGv + t.rg : (t.mat == 2 ? 2 * nRGq + t.rg : t.mat * nRGq + t.rg);
    };
    const int nkeys = 2 * nRGq + nRGv + nRGo;
    std::vector<uint32_t> nseg(nkeys, 0), seg0(nkeys, 0);
    for (int c = 0; c < P; ++c) {
        const auto &L = per_cta[c];
        for (size_t i = 0; i < L.size(); ++i)
            if (i == 0 || key(L[i]) != key(L[i - 1])) nseg[key(L[i])]++;
    }
    size_t total = 0;
    for (int k = 0; k < nkeys; ++k) {
        seg0[k] = (uint32_t)total;
        total += nseg[k];
    }
    std::vector<uint32_t> next(seg0);
    tiles->clear();
    off->assign(P + 1, 0);
    for (int c = 0; c < P; ++c) {
        (*off)[c] = (uint32_t)tiles->size();
        const auto &L = per_cta[c];
        uint32_t cur = 0;
        for (size_t i = 0; i < L.size(); ++i) {
            const int k = key(L[i]);
            TileEntry e{};
            e.mat = L[i].mat;
            e.rg = L[i].rg;
            e.kb = L[i].kb;
            const bool start = i == 0 || key(L[i - 1]) != k;
            const bool end = i + 1 == L.size() || key(L[i + 1]) != k;
            if (start) cur = next[k]++;
            e.flags = (start ? kSegStart : 0) | (end ? kSegEnd : 0);
            e.nseg = (uint16_t)nseg[k];
            e.seg = cur;
            e.seg0 = seg0[k];
            tiles->push_back(e);
        }
    }
    (*off)[P] = (uint32_t)tiles->size();
    *nseg_total = total;
    if (rbinfo) {
        rbinfo->resize(2 * (size_t)nkeys);
        for (int k = 0; k < nkeys; ++k) {
            (*rbinfo)[2 * k] = seg0[k];
            (*rbinfo)[2 * k + 1] = nseg[k];
        }
    }
}

}  // namespace kda
