// fused.cuh -- interface of the FUSED engine (one persistent kernel per decode step).
#pragma once

#include <cuda.h>

#include <vector>

#include "common.cuh"

namespace kda {

// One 128 x 128 FP8 weight tile of the projection stream (16 bytes, read by every role).
struct TileEntry {
    uint8_t mat;    // 0 W_q, 1 W_k, 2 W_v, 3 W_o
    uint8_t flags;  // kSegStart | kSegEnd
    uint16_t rb;    // row block (128 output rows) within the matrix
    uint16_t kb;    // K block (128 input columns)
    uint16_t nseg;  // segments (partial sums) of this row block per step
    uint32_t seg;   // partial-sum slot of this tile's segment
    uint32_t seg0;  // first partial-sum slot of this row block
};
constexpr uint8_t kSegStart = 1, kSegEnd = 2;
constexpr int kTraceSlots = 192;  // timeline stamps per CTA in builds with KDA_TRACE (32 events + 5 x 32 tiles)

struct FusedState {
    // device areas inside the handle's scratch
    void *base = nullptr;
    size_t bytes = 0;
    uint8_t *xq = nullptr;      // x planes  [2 * BP + scale rows][H]: E4M3 codes, then fp32 block scales
    uint8_t *oq = nullptr;      // o planes  [4 * BP + scale rows][Dv]
    float *part = nullptr;      // partial sums [nseg_total][BPmax][128]
    uint32_t *ctr = nullptr;    // flags and counters
    size_t ctr_bytes = 0;
    TileEntry *tiles = nullptr;  // per-CTA tile lists, concatenated
    uint32_t *cta_off = nullptr; // [num_ctas + 1]
    uint32_t *rbinfo = nullptr;  // per row block: first partial slot, segments
    uint64_t *trace = nullptr;   // [num_ctas][kTraceSlots] (KDA_TRACE builds only)
    // host side
    int num_ctas = 0;
    int bp_max = 0;
    size_t ntiles = 0, nseg_total = 0;
    int max_tiles_per_cta = 0;
    std::vector<TileEntry> h_tiles;
    std::vector<uint32_t> h_off;
    std::vector<uint32_t> h_rbinfo;
    uint32_t epoch = 0;  // steps issued since the last reset
    uint32_t cum_b = 0;  // sum of batch sizes of those steps
    bool needs_reset = false;
    bool uploaded = false;
    uint64_t timeout_ns = 2000000000ull;
    int debug_skip_gate_release = 0;
    int stages_override = 0;  // KDA_STAGES: cap on ring stages (tuning)
    // tensor-map cache for the weights (keyed by the four FP8 pointers)
    const void *map_keys[4][4] = {};
    CUtensorMap wmaps[4][4];
    int map_next = 0;
    // counter offsets
    int off_oready = 0, off_rb = 0;
};

bool fused_supports(const Dims &d, int num_sms);
size_t fused_scratch_bytes(const Dims &dmax, int num_sms);
void fused_bind_scratch(const Dims &dmax, int num_sms, void *base, size_t bytes, FusedState *fs);
cudaError_t fused_init(const Dims &dmax, FusedState *fs);
void fused_destroy(FusedState *fs);
int fused_launches();
cudaError_t fused_step(const Dims &d, const kda_weights &w, const void *x, float *state, void *out, int out_dtype,
                       FusedState &fs, const Scratch &s, int *status, cudaStream_t stream);

// Schedule of the projection stream (host only; exposed for self-checks).
void fused_build_schedule(const Dims &d, int num_ctas, std::vector<TileEntry> *tiles, std::vector<uint32_t> *off,
                          size_t *nseg_total, std::vector<uint32_t> *rbinfo);

}  // namespace kda
