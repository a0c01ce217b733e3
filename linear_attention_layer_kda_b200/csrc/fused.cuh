// fused.cuh -- interface of the FUSED engine (one persistent kernel per decode step).
#pragma once

#include <cuda.h>

#include <vector>

#include "common.cuh"

namespace kda {

// One weight tile of the projection stream: `rows` weight rows (a row group) x one 128-wide
// K block (16 bytes, read by every role).
struct TileEntry {
    uint8_t mat;    // 0 W_q, 1 W_k, 2 W_v, 3 W_o
    uint8_t flags;  // kSegStart | kSegEnd
    uint16_t rg;    // row group within the matrix
    uint16_t kb;    // K block (128 input columns)
    uint16_t nseg;  // segments (partial sums) of this row group per step
    uint32_t seg;   // partial-sum slot of this tile's segment
    uint32_t seg0;  // first partial-sum slot of this row group
};
constexpr uint8_t kSegStart = 1, kSegEnd = 2;
constexpr int kTraceSlots = 192;  // timeline stamps per CTA in builds with KDA_TRACE (32 events + 5 x 32 tiles)

// Shape of the schedule: weight rows per q/k/v tile and per W_o tile, tiles per run.
struct SchedGeo {
    int nx, no, run;
};

// Padded batch and the activation-tile geometry that follows from it (host and device).
//
// Activations enter the tensor cores as the M-side operand: FP8 "planes" whose rows are
// (plane, sequence) pairs.  Rows come in groups of 16 -- two planes of eight sequences -- and
// group slot v sits at row rowbase(v), lanes 0-15 or 16-31 of TMEM lane quarter v % 4, so
// that the 16x256b TMEM loads of one warp quarter hand each thread both planes of one
// sequence.  With fewer than four groups the groups are repeated in the empty quarters
// (slot v holds group v % groups) and the four epilogue warps split the columns instead.
struct ActGeo {
    int BP;           // padded batch: 8, 16, 32 or 64
    int gx, go;       // row groups of the x planes (2 planes) and of the o planes (4 planes)
    int sr;           // scale rows: ceil(BP / 32), 32 fp32 scales per 128-byte row
    int rsx, rso;     // first scale row of an x tile and of an o tile
    int mhx, mho;     // M halves (128 rows each) of an x and an o tile
    int nx, no;       // weight rows per q/k/v tile and per W_o tile (the MMA's N)
};
__host__ __device__ constexpr int act_rowbase(int v) { return 128 * (v / 8) + 32 * (v % 4) + 16 * ((v % 8) / 4); }
__host__ __device__ constexpr int act_slots(int groups) { return groups < 4 ? 4 : groups; }
// Scale rows sit in the unused half of quarter 0 while at most four slots exist, else after
// the last M half.
__host__ __device__ constexpr int act_scale_row(int groups) { return groups <= 4 ? 16 : 128 * ((groups + 7) / 8); }
// Rows an activation tile occupies (planes, replicas and scale rows).
__host__ __device__ constexpr int act_rows(int groups, int sr)
{
    return groups <= 4 ? act_rowbase(act_slots(groups) - 1) + 16 : act_scale_row(groups) + sr;
}
__host__ __device__ constexpr int act_n_for(int groups)
{
    // at most 64 running sums per epilogue thread: (groups per warp) x N / 4 <= 64
    return 256 / ((groups + 3) / 4);
}
__host__ __device__ constexpr ActGeo act_geo(int BP)
{
    return ActGeo{BP,
                  BP / 8,
                  BP / 4,
                  (BP + 31) / 32,
                  act_scale_row(BP / 8),
                  act_scale_row(BP / 4),
                  (BP / 8 + 7) / 8,
                  (BP / 4 + 7) / 8,
                  act_n_for(BP / 8),
                  act_n_for(BP / 4)};
}

struct FusedState {
    // device areas inside the handle's scratch
    void *base = nullptr;
    size_t bytes = 0;
    uint8_t *xq = nullptr;       // x planes  [act_rows(gx) rows][H]: E4M3 codes and fp32 block scales
    uint8_t *oq = nullptr;       // o planes  [act_rows(go) rows][Dv]
    float *part = nullptr;       // partial sums [nseg_total][2][BPmax][256]
    float *gbuf = nullptr;       // gates of every single-token state unit [units][260]
    uint32_t *ctr = nullptr;     // flags and counters
    size_t ctr_bytes = 0;
    // one schedule per padded-batch class (BP 8, 16, 32, 64 up to the handle's largest)
    TileEntry *tiles[4] = {};     // per-CTA tile lists, concatenated
    uint32_t *cta_off[4] = {};    // [num_ctas + 1]
    uint32_t *rbinfo[4] = {};     // per row group: first partial slot, segments
    uint64_t *trace = nullptr;   // [num_ctas][kTraceSlots] (KDA_TRACE builds only)
    // host side
    int num_ctas = 0;
    int bp_max = 0;
    int nclass = 0;                 // schedules built: classes 0 .. nclass-1
    size_t nseg_total = 0;          // partial-sum slots of the largest schedule
    int max_tiles_per_cta[4] = {};
    std::vector<TileEntry> h_tiles[4];
    std::vector<uint32_t> h_off[4];
    std::vector<uint32_t> h_rbinfo[4];
    int last_class = -1;            // class of the previous step (counters are per class)
    uint32_t epoch = 0;  // steps issued since the last reset
    uint32_t cum_b = 0;  // sum of rows (sequences x tokens) of those steps
    uint32_t cum_s = 0;  // sum of sequences of those steps
    bool needs_reset = false;
    bool uploaded = false;
    uint64_t timeout_ns = 2000000000ull;
    int debug_skip_gate_release = 0;
    int stages_override = 0;  // KDA_STAGES: ring stages (tuning)
    int early_tiles = 0;      // KDA_EARLY_TILES: weight copies issued before x is split (tuning)
    bool overlap = true;      // launch with programmatic stream serialization (kda_decode_set_launch_overlap)
    int device = -1;
    // tensor-map cache for the weights (keyed by the four FP8 pointers)
    const void *map_keys[4][4] = {};
    int map_box[4][4] = {};  // box rows each map was encoded with
    CUtensorMap wmaps[4][4];
    int map_next = 0;
    // tensor maps of the activation planes (fixed per handle and padded batch)
    CUtensorMap amaps[4][5];
    bool amap_ok[4] = {};
    // counter offsets
    int off_oready = 0, off_rb = 0;
    // tensor parallelism by heads: exchange regions of the group's ranks (slots, then flags)
    int tp_world = 0, tp_rank = 0, tp_bmax = 0;
    bool tp_ready = false;          // every rank's region is mapped
    uint32_t tp_epoch = 0;          // fused steps run in the group (never reset)
    void *tp_region[8] = {};        // [rank]: slots [2][world][bmax][H] fp32, flags [2][world][H/32]
    size_t tp_slot_bytes = 0;
};

bool fused_supports(const Dims &d, int num_sms);
size_t fused_scratch_bytes(const Dims &dmax, int num_sms);
void fused_bind_scratch(const Dims &dmax, int num_sms, void *base, size_t bytes, FusedState *fs);
cudaError_t fused_init(const Dims &dmax, FusedState *fs);
void fused_destroy(FusedState *fs);
int fused_launches();
int fused_max_tokens();
// d.B rows = sequences x tokens (row b * tokens + t); tokens <= fused_max_tokens().
cudaError_t fused_step(const Dims &d, int tokens, const kda_weights &w, const void *x, float *state, void *out,
                       int out_dtype, FusedState &fs, const Scratch &s, int *status, cudaStream_t stream);

// Schedule shape of a step whose padded batch is BP (host only).
SchedGeo fused_sched_geo(const Dims &dmax, int BP);

// Schedule of the projection stream (host only; exposed for self-checks).
void fused_build_schedule(const Dims &d, int num_ctas, const SchedGeo &g, std::vector<TileEntry> *tiles,
                          std::vector<uint32_t> *off, size_t *nseg_total, std::vector<uint32_t> *rbinfo);

}  // namespace kda
