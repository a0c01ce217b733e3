// schedule.cu -- host-only: the fused engine's tile schedule (which CTA streams which weight
// tiles, in which order, and where each run's partial sum goes).  Kept apart from the kernel
// so that its invariants can be checked on a machine without a GPU.
#include <stdlib.h>

#include <algorithm>
#include <vector>

#include "fused.cuh"

namespace kda {
namespace {

constexpr int kHeadsPerGroup = 8;
// Head groups of q/k/v tiles between a group's q/k/v tiles and its W_o tiles (-1: all W_o
// tiles after all q/k/v tiles).  Measured at batch 8: interleaving (1, 2, 3) stalls the MMA on
// o blocks whose state units are still running, so the default keeps W_o last.
constexpr int kWoLag = -1;

}  // namespace

// Tile order and segments.  Heads are taken in groups of eight; group g contributes the
// q, k and v row blocks of its heads (all K blocks), split into contiguous equal runs over
// the CTAs; then the W_o tiles whose K blocks belong to group g, split the same way.  A
// segment is a CTA's run inside one row block; its partial-sum slot is numbered row block
// by row block so the segments of a row block are adjacent.
void fused_build_schedule(const Dims &d, int P, std::vector<TileEntry> *tiles, std::vector<uint32_t> *off,
                          size_t *nseg_total, std::vector<uint32_t> *rbinfo)
{
    const int nKBx = d.H / 128, nKBo = d.Dv() / 128, nRBq = d.Dk() / 128, nRBv = d.Dv() / 128, nRBo = d.H / 128;
    const int hpu = std::max(128 / d.dk, 128 / d.dv);
    int heads_per_group = kHeadsPerGroup, wo_lag = kWoLag;
    if (const char *e = getenv("KDA_HEADS_PER_GROUP")) heads_per_group = std::max(1, atoi(e));
    if (const char *e = getenv("KDA_WO_LAG")) wo_lag = atoi(e);
    const int hpg = std::max(hpu, heads_per_group / hpu * hpu);
    const int G = (d.nh + hpg - 1) / hpg;
    struct T { uint8_t mat; uint16_t rb, kb; };
    std::vector<std::vector<T>> per_cta(P);
    // Contiguous runs in CTA order; the n % P longer runs go to the CTAs with the fewest
    // tiles so far, so that the totals over all groups differ by at most one tile.
    auto split = [&](const std::vector<T> &list) {
        const size_t n = list.size(), base = n / P, extra = n % P;
        std::vector<int> order(P);
        for (int c = 0; c < P; ++c) order[c] = c;
        std::stable_sort(order.begin(), order.end(),
                         [&](int a, int b) { return per_cta[a].size() < per_cta[b].size(); });
        std::vector<size_t> len(P, base);
        for (size_t j = 0; j < extra; ++j) len[order[j]]++;
        size_t pos = 0;
        for (int c = 0; c < P; ++c)
            for (size_t i = 0; i < len[c]; ++i) per_cta[c].push_back(list[pos++]);
    };
    auto qkv_group = [&](int g) {
        const int h0 = g * hpg, h1 = std::min(d.nh, h0 + hpg);
        std::vector<T> list;
        for (int m = 0; m < 3; ++m) {
            const int hd = m == 2 ? d.dv : d.dk;
            for (int rb = h0 * hd / 128; rb < h1 * hd / 128; ++rb)
                for (int kb = 0; kb < nKBx; ++kb) list.push_back(T{(uint8_t)m, (uint16_t)rb, (uint16_t)kb});
        }
        split(list);
    };
    auto wo_group = [&](int g) {
        const int h0 = g * hpg, h1 = std::min(d.nh, h0 + hpg);
        std::vector<T> list;
        for (int rb = 0; rb < nRBo; ++rb)
            for (int kb = h0 * d.dv / 128; kb < h1 * d.dv / 128; ++kb) list.push_back(T{3, (uint16_t)rb, (uint16_t)kb});
        split(list);
    };
    // The W_o tiles of group g follow the q/k/v tiles of group g + lag, so the state units of
    // group g run while the weight stream carries later groups' q/k/v.
    const int lag = wo_lag < 0 ? G : wo_lag;
    for (int g = 0; g < G; ++g) {
        qkv_group(g);
        if (g - lag >= 0) wo_group(g - lag);
    }
    for (int g = std::max(0, G - lag); g < G; ++g) wo_group(g);
    // row-block keys: q 0.., k nRBq.., v 2nRBq.., o 2nRBq+nRBv..
    auto key = [&](const T &t) {
        return t.mat == 3 ? 2 * nRBq + nRBv + t.rb : (t.mat == 2 ? 2 * nRBq + t.rb : t.mat * nRBq + t.rb);
    };
    const int nkeys = 2 * nRBq + nRBv + nRBo;
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
            e.rb = L[i].rb;
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
    (void)nKBo;
}

}  // namespace kda
