// fused.cu -- the FUSED engine: the whole decode step as one persistent kernel on sm_100a.
//
// Design (the TrnRT story's megakernel rules restated for B200: the working set stays on
// chip and only x, the state, the streamed weights and out cross HBM; the weight stream is
// split over every SM; Kiln's "one scale per kernel tile" for the FP8 weights):
//
//  * One CTA per SM, 16 warps, cooperative launch (all CTAs co-resident).
//  * Projection pipeline (warps 0-7).  Every projection is a stream of weight tiles of N
//    rows (256 while the batch allows) x one 128-wide K block; each 128 x 128 sub-block has
//    one fp32 scale.  Warp 0 lane 0 loads the weight tiles with TMA into a shared-memory
//    ring, each followed by the activation tile of its K block (x planes, or o planes once
//    the state units have released them).  Warp 2 lane 0 issues tcgen05.mma kind::f8f6f4 with the
//    ACTIVATIONS as the M = 128 operand and the WEIGHTS as the N operand (K = 128 in four
//    K = 32 steps) into one of two TMEM accumulators, and commits once per tile: a
//    tcgen05.mma costs about the same whatever its N, so 256 weight rows per instruction and
//    one commit per 32 KB keep the tensor pipe ahead of HBM.  Warps 4-7 (one per TMEM lane
//    quarter) read the accumulator with 16x256b loads, which hand each thread both planes of
//    one sequence, apply weight scale x activation scale per 128 x 128 block and keep
//    running sums in registers; a CTA's run of tiles in one row group ends in a partial sum.
//    Warp 3 lane 0 publishes it with a release increment of the row group's counter, so the
//    fence that the release implies never holds up the epilogue; consumers add a row group's
//    partials in slot order (deterministic).
//  * Activations enter the tensor cores as FP8 "planes": a K-block of 128 values v with a
//    power-of-two scale s is split v/s = p0 + p1 (+ p2 + p3) with every p an E4M3 value
//    (each plane is the round-to-nearest residual of the previous ones).  Two planes hold
//    a bf16 x exactly (up to the E4M3 subnormal floor, 2^-10 of the scale), four hold the
//    fp32 readout o to about 2^-16 of its block maximum.  Products of E4M3 values are
//    exact and accumulate in fp32, so no weight is ever dequantised in registers.
//  * Vector warps (8-15): split x into planes (a share per CTA), compute the beta and
//    alpha-down gate rows (bf16, CUDA cores), then run (sequence, o K-block) state units,
//    assigned statically in head order: load the unit's fp32 state, wait until its heads'
//    q/k/v are final, apply the gated delta rule in registers, split o into planes and
//    release the K-block to the output projection, write the state back in place; the next
//    unit's gates are computed while the current one waits.  Last, they add the W_o
//    partials of their output rows into out.
//  * Order: the weight tiles are dealt to the SMs in waves, earliest heads first (see
//    schedule.cu), so early heads' state units and W_o tiles overlap the rest of the
//    stream.  Few stages are kept in flight per SM: HBM is saturated with less, and every
//    extra byte queued in the memory system delays the flags and partial sums the step's
//    dependency chain runs on.  For the same reason the weight stream holds after its first
//    tiles until x is split (bounded).
//  * Every wait is bounded (global timer); on expiry the kernel records
//    KDA_ERR_DEVICE_TIMEOUT, raises an abort flag every CTA polls, waits for its own
//    copies and MMAs in flight, frees TMEM and returns.
#include <math.h>
#include <stdlib.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

#include "fused.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int kThreads = 512;
// Register shares per warpgroup (the block launches with 128 per thread): the single-lane
// roles of warps 0-3 need few, the epilogue keeps 128, the state units get the rest.
// 128 * (48 + 128 + 168 + 168) = 65536 = 512 * 128.
constexpr int kRegsControl = 48, kRegsVector = 168;
static_assert(kRegsControl + 128 + 2 * kRegsVector <= 4 * 128, "register shares exceed the launch budget");
constexpr int kMaxBP = 64;
constexpr int kMaxStages = 8;    // ring stages (weight tile + activation tile)
constexpr int kMaxAcc = 4;       // TMEM accumulator buffers
constexpr int kEpiWarps = 4;     // warps 4-7, one per TMEM lane quarter
constexpr int kMaxTilesPerCta = 512;
constexpr int kTmemCols = 512;
constexpr int kMaxStagesDefault = 3;  // stages in flight unless KDA_STAGES says otherwise
constexpr int kEarlyTilesDefault = 1;  // weight copies issued before x is known final (KDA_EARLY_TILES)
constexpr uint64_t kEarlyHoldNs = 6000;  // longest hold of the rest of the stream
constexpr int kSegBars = 32;          // segment hand-off barriers (epilogue -> publisher), reused mod 32

// Optional timeline (compile with -DKDA_TRACE): per CTA, kTraceSlots global-timer stamps.
#ifdef KDA_TRACE
#define KDA_TR(P, slot)                                                                       \
    do {                                                                                      \
        if ((P).trace) (P).trace[(size_t)blockIdx.x * kTraceSlots + (slot)] = globaltimer_ns(); \
    } while (0)
#else
#define KDA_TR(P, slot) \
    do {                \
    } while (0)
#endif
enum TraceSlot {
    TR_START = 0, TR_XREADY, TR_FIRST_MMA, TR_QKV_DONE, TR_EPI_DONE, TR_XQ_DONE, TR_GATES_DONE,
    TR_UNIT0 = 7,  /* units 0, 1: claimed, (unused), done */
    TR_GRID_WAIT = 13, /* the preceding grid has completed (griddepcontrol.wait returned) */
    TR_UNIT_HAND = 15, /* units 0, 1: o handed off */
    TR_PUB0 = 25, /* publisher: release of segment k issued and done, k < 7 */
    TR_O_WAIT0 = 19, TR_O_READY0, TR_O_READY_LAST, TR_END, TR_LAST_REDUCE_START, TR_LAST_REDUCE_END,
    TR_TILE_TMA = 32, TR_TILE_MMA = 64, TR_TILE_EPI = 96, TR_USUB = 128, /* 16 stamps per state unit, units < 2 */
    TR_TILE_ACT = 160 /* per tile i < 32 */
};

// counters (uint32, monotonic across steps; targets are multiples of the step count)
//   C_XQ          x K-blocks split into planes (B per K block per step)
//   C_GATE        gate rows finished
//   (words 2 and 3 are unused)
//   C_ABORT       set by any wait that gives up
//   off_oready+kb state units done for o K-block kb (B per step)
//   off_rb+key    segments published for row group key (q, k, v, o row groups)
constexpr int C_XQ = 0, C_GATE = 1, C_ABORT = 4, C_FIXED = 16;
// Gate buffer: per state unit, alpha of its rows at [0, 256) and beta of its heads at kGateBeta.
constexpr int kGateBeta = 256, kGateStride = 260;

// Status words in mapped host memory: [0] status, [1] wait site, [2] set when a drain of
// copies in flight gave up (the handle can no longer be trusted).
constexpr int ST_CODE = 0, ST_WHERE = 1, ST_DRAIN = 2;

constexpr int kOHand = 8;  // o-block hand-off barriers (state unit -> o publisher), reused mod 8

constexpr int kMaxT = 8;  // tokens per sequence in one multi-token step
constexpr int kMaxTp = 8;  // ranks of a tensor-parallel group

// NT: tokens per unit (1, or kMaxT in the multi-token kernels).
template <int NT>
struct __align__(16) VecSmemT {
    static constexpr int NA = NT < 2 ? 2 : NT;  // gate slots (one token: the current and the next unit)
    uint64_t ohand[kOHand];        // unit k's o planes are stored (arrival of vector warp 0)
    int opub;                      // units whose o block the o publisher has released
    int pad_[3];
    float q[NT][256], k[NT][256];  // per token and head of the unit: q, k^ (heads_per_unit * dk)
    float a[NA][256];              // alpha per gate slot
    float v[NT][128];              // per token and virtual column of the unit
    float u[128], o[128];
    float red_w[8][128], red_p[8][128];  // adjacent: also the t rows of token_gates
    float beta[NA][2], kq[NT][2], inv[NT][2];
    int unit, ok, fail;
};

struct FusedParams {
    CUtensorMap tm_w[4];  // W_q, W_k, W_v (box nx rows), W_o (box no rows): uint8 [rows, K], 128B swizzle
    CUtensorMap tm_xq;    // x planes + scale rows (one box)
    CUtensorMap tm_xrep;  // one 16-row group of x planes, copied into the empty quarters
    CUtensorMap tm_oq;    // o planes (+ scale rows when they fit in one 256-row box)
    CUtensorMap tm_osc;   // o scale rows alone, used when the o tile is taller than 256 rows
    CUtensorMap tm_orep;  // one 16-row group of o planes, copied into the empty quarters
    const float *wscale[4];
    const uint16_t *x, *wa_down, *wa_up, *wb;
    float *state;
    void *out;
    uint8_t *xq, *oq;  // x and o planes + scale rows
    float *part;
    float *gbuf;  // single-token gates of every state unit [units][kGateStride]
    float *q, *k, *v, *bpre, *t;
    uint32_t *ctr;
    uint64_t *trace;  // null unless built with KDA_TRACE
    const TileEntry *tiles;
    const uint32_t *cta_off;
    int *status;
    const uint2 *rbinfo;  // per row-group key: (first partial slot, segments)
    int B, H, nh, dk, dv, r;  // B: rows (sequences x tokens)
    int T, Bs;                // tokens per sequence, sequences (B = Bs * T; row b * T + t)
    int nKBx, nKBo, nRGq, nRGv, nRGo;
    int off_oready, off_rb;
    uint32_t epoch, t_xq, t_gate, t_o;
    uint64_t timeout_ns;
    int out_bf16, stages, a_bytes, w_bytes, nacc, cols, skip_gate_release, early_tiles;
    // tensor parallelism by heads (tp_world > 0): this rank's partial out goes to every rank's
    // exchange slots [parity][src][tp_bmax][H] fp32 and their flags [parity][src][H / 32]
    int tp_world, tp_rank, tp_bmax;
    uint32_t tp_epoch;
    float *tp_slots[kMaxTp];
    uint32_t *tp_flags[kMaxTp];
};

// Floats per partial-sum slot: [pair][BP][N <= 256]; pair 1 only for the o planes 2 and 3.
template <int BP>
__host__ __device__ constexpr size_t slot_floats() { return (size_t)2 * BP * 256; }

struct Ctl {
    const FusedParams &P;
    volatile int *sh_abort;
};

// Abort check on the shared-memory flag; the global flag (set by another CTA) is read at
// most every 20 us per waiting thread, via poll_abort.
__device__ __forceinline__ bool should_stop(const Ctl &c) { return *c.sh_abort != 0; }

__device__ __forceinline__ bool poll_abort(const Ctl &c, uint64_t now, uint64_t &next)
{
    if (*c.sh_abort) return true;
    if (now < next) return false;
    next = now + 20000;
    if (*(volatile uint32_t *)(c.P.ctr + C_ABORT) != 0u) {
        *c.sh_abort = 1;
        return true;
    }
    return false;
}

__device__ void raise_abort(const Ctl &c, int where)
{
    *c.sh_abort = 1;
    atomicExch(c.P.ctr + C_ABORT, 1u);
    volatile int *st = c.P.status;  // mapped host memory: plain stores, no atomics
    st[ST_WHERE] = where;           // the site first, so a host that sees the code sees its site
    __threadfence_system();
    st[ST_CODE] = KDA_ERR_DEVICE_TIMEOUT;
    __threadfence_system();
}

__device__ bool wait_bar(uint64_t *b, uint32_t parity, const Ctl &c, int where)
{
    if (mbar_try_wait(b, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    uint64_t next = t0 + 20000;
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(b, parity)) return true;
        if ((it & 15u) == 0u) {
            const uint64_t now = globaltimer_ns();
            if (poll_abort(c, now, next)) return false;
            if (now - t0 > c.P.timeout_ns) {
                raise_abort(c, where);
                return false;
            }
        }
    }
}

// Bounded wait for the phase a barrier is known to reach (exit path only).  If it gives up,
// copies or MMAs of this CTA may still be in flight: record that the handle is unusable.
__device__ void drain_bar(const FusedParams &P, uint64_t *b, uint32_t parity)
{
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(b, parity)) {
        if (globaltimer_ns() - t0 > P.timeout_ns) {
            volatile int *st = P.status;
            st[ST_DRAIN] = 1;
            __threadfence_system();
            return;
        }
    }
}

__device__ bool wait_count(const uint32_t *p, uint32_t target, const Ctl &c, int where)
{
    if ((int32_t)(ld_acquire(p) - target) >= 0) return true;
    const uint64_t t0 = globaltimer_ns();
    uint64_t next = t0 + 20000;
    for (;;) {
        __nanosleep(32);
        if ((int32_t)(ld_acquire(p) - target) >= 0) return true;
        const uint64_t now = globaltimer_ns();
        if (poll_abort(c, now, next)) return false;
        if (now - t0 > c.P.timeout_ns) {
            raise_abort(c, where);
            return false;
        }
    }
}

// Bounded wait until a flag that another GPU writes equals `want` (system-scope acquire).
__device__ bool wait_flag_sys(const uint32_t *p, uint32_t want, const Ctl &c, int where)
{
    auto ld = [](const uint32_t *q) {
        uint32_t v;
        asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(q) : "memory");
        return v;
    };
    if (ld(p) == want) return true;
    const uint64_t t0 = globaltimer_ns();
    uint64_t next = t0 + 20000;
    for (;;) {
        __nanosleep(64);
        if (ld(p) == want) return true;
        const uint64_t now = globaltimer_ns();
        if (poll_abort(c, now, next)) return false;
        if (now - t0 > c.P.timeout_ns) {
            raise_abort(c, where);
            return false;
        }
    }
}

__device__ __forceinline__ void st_release_sys(uint32_t *p, uint32_t v)
{
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ int rg_key(const FusedParams &P, int mat, int rg)
{
    return mat < 2 ? mat * P.nRGq + rg : (mat == 2 ? 2 * P.nRGq + rg : 2 * P.nRGq + P.nRGv + rg);
}

// Two sums over the segments of a row group, element `off` of each slot, in slot order, with
// all loads of 8 slots per item issued together; items with has[j] false are skipped.
template <int BP>
__device__ __forceinline__ void sum_segs2(const FusedParams &P, const int (&key)[2], const int (&off)[2],
                                          const bool (&has)[2], float (&out)[2])
{
    constexpr size_t SLOT = slot_floats<BP>();
    uint2 info[2];
    const float *base[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        info[j] = has[j] ? __ldg(P.rbinfo + key[j]) : make_uint2(0u, 0u);
        base[j] = P.part + (size_t)info[j].x * SLOT + off[j];
        out[j] = 0.f;
    }
    const uint32_t nmax = info[0].y > info[1].y ? info[0].y : info[1].y;
    for (uint32_t g0 = 0; g0 < nmax; g0 += 8) {
        float v[2][8];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int g = 0; g < 8; ++g) v[j][g] = g0 + g < info[j].y ? __ldcg(base[j] + (size_t)(g0 + g) * SLOT) : 0.f;
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int g = 0; g < 8; ++g) out[j] += v[j][g];
    }
}

__device__ __forceinline__ bool wait_rb(const FusedParams &P, int key, const Ctl &c, int where)
{
    const uint32_t nseg = __ldg(P.rbinfo + key).y;
    return wait_count(P.ctr + P.off_rb + key, nseg * P.epoch, c, where);
}

// ---------------------------------------------------------------- activation planes

// Smallest power of two s with amax / s <= 448 (s = 1 for amax == 0), from the exponent
// bits of amax / 448: that exponent, or the next one when amax / 448 is not itself a power of
// two.  Below the normal range the scale stays at 2^-126.
__device__ __forceinline__ float pow2_scale(float amax)
{
    if (!(amax > 0.f)) return 1.f;
    const uint32_t y = __float_as_uint(amax * (1.f / 448.f));
    uint32_t e = y >> 23;
    if (e == 0u) return __uint_as_float(1u << 23);
    if (y & 0x7FFFFFu) ++e;
    return __uint_as_float(e << 23);
}

// 1 / s for a power of two s in [2^-126, 2^126] (exact).
__device__ __forceinline__ float pow2_inv(float s) { return __uint_as_float((254u - (__float_as_uint(s) >> 23)) << 23); }

// 1 / (1 + e^z) (the hardware exponential and reciprocal: a few ulp; 0 once e^z overflows).
__device__ __forceinline__ float inv_one_plus_exp(float z) { return __fdividef(1.f, 1.f + __expf(z)); }

// Row of plane p of sequence b in an x tile (2 planes; group b / 8) and in an o tile (4
// planes; group 2 (b / 8) + p / 2).
__device__ __forceinline__ int x_row(int p, int b) { return act_rowbase(b / 8) + 8 * p + (b % 8); }
__device__ __forceinline__ int o_row(int p, int b) { return act_rowbase(2 * (b / 8) + p / 2) + 8 * (p % 2) + (b % 8); }

// Rows of the first TMA box of an activation tile with `groups` groups: its groups and
// scale rows, at most 256 rows (the scale rows past 256 come in a second box).
__host__ __device__ constexpr int act_main_rows(int groups, int sr)
{
    return groups <= 4 ? (act_rowbase(groups - 1) + 16 > 16 + sr ? act_rowbase(groups - 1) + 16 : 16 + sr)
                       : (act_rows(groups, sr) > 256 ? 256 : act_rows(groups, sr));
}

// Byte offset of (row r, byte c) in a 128-byte-swizzled tile: 16-byte chunk c / 16 of row r
// sits at chunk (c / 16) ^ (r % 8).
__device__ __forceinline__ int swz(int r, int c) { return r * 128 + ((((c >> 4) ^ (r & 7))) << 4) + (c & 15); }

// Splits four values (already divided by their scale) into NP E4M3 planes, 4 codes per word.
template <int NP>
__device__ __forceinline__ void split_planes(float v0, float v1, float v2, float v3, uint32_t (&w)[NP])
{
    float r[4] = {v0, v1, v2, v3};
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(r[0], r[1]), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(r[2], r[3]), __NV_SATFINITE, __NV_E4M3);
        w[p] = (uint32_t)lo | ((uint32_t)hi << 16);
        const float2 flo = e4m3x2_to_float2(lo), fhi = e4m3x2_to_float2(hi);
        r[0] -= flo.x;
        r[1] -= flo.y;
        r[2] -= fhi.x;
        r[3] -= fhi.y;
    }
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float4 ld_stream_f4(const float *p)
{
    float4 v;
    asm volatile("ld.global.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ void st_stream_f4(float *p, float4 v)
{
    asm volatile("st.global.cs.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

// This CTA's 1/gridDim share of [p, p + bytes) -> L2 (bulk prefetch, 16-byte granules).
__device__ __forceinline__ void prefetch_l2_slice(const void *p, size_t bytes)
{
    const size_t gran = (bytes / 16 + gridDim.x - 1) / gridDim.x * 16;
    const size_t lo = (size_t)blockIdx.x * gran;
    if (lo >= bytes) return;
    const size_t n = (bytes - lo < gran ? bytes - lo : gran) & ~(size_t)15;
    if (n) bulk_prefetch_l2(static_cast<const char *>(p) + lo, (uint32_t)n);
}

// ---------------------------------------------------------------- vector warps

template <int BP>
__device__ void quantize_x(const FusedParams &P, int gw, int ngw, int lane)
{
    constexpr ActGeo G = act_geo(BP);
    const int items = P.B * P.nKBx;
#pragma unroll 1
    for (int it = gw; it < items; it += ngw) {
        const int b = it / P.nKBx, kb = it % P.nKBx;
        const uint2 raw = *reinterpret_cast<const uint2 *>(P.x + (size_t)b * P.H + kb * 128 + lane * 4);
        const float v0 = bf16_bits_to_float(raw.x & 0xFFFFu), v1 = bf16_bits_to_float(raw.x >> 16);
        const float v2 = bf16_bits_to_float(raw.y & 0xFFFFu), v3 = bf16_bits_to_float(raw.y >> 16);
        const float amax = warp_max(fmaxf(fmaxf(fabsf(v0), fabsf(v1)), fmaxf(fabsf(v2), fabsf(v3))));
        const float s = pow2_scale(amax), inv = pow2_inv(s);  // exact: s is a power of two
        uint32_t w[2];
        split_planes<2>(v0 * inv, v1 * inv, v2 * inv, v3 * inv, w);
#pragma unroll
        for (int p = 0; p < 2; ++p)
            *reinterpret_cast<uint32_t *>(P.xq + (size_t)x_row(p, b) * P.H + kb * 128 + lane * 4) = w[p];
        if (lane == 0)
            *reinterpret_cast<float *>(P.xq + (size_t)(G.rsx + b / 32) * P.H + kb * 128 + (b % 32) * 4) = s;
        fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) red_release_add(P.ctr + C_XQ, 1u);
    }
}

// Gate rows (W_b and W_a_down, bf16): one row per CTA at a time, its K range split over the
// eight vector warps, partial sums added in warp order through shared memory.
template <int BP, class VS>
__device__ void gate_rows(const FusedParams &P, VS *vs, int vt)
{
    const int vw = vt >> 5, lane = vt & 31;
    const int rows = P.nh + P.r;
    const int kchunk = P.H / 8;  // multiple of 16
#pragma unroll 1
    for (int it = blockIdx.x; it < rows; it += gridDim.x) {
        const uint16_t *wrow = it < P.nh ? P.wb + (size_t)it * P.H : P.wa_down + (size_t)(it - P.nh) * P.H;
        float acc[BP];
#pragma unroll
        for (int b = 0; b < BP; ++b) acc[b] = 0.f;
#pragma unroll 1
        for (int k0 = vw * kchunk + lane * 8; k0 < (vw + 1) * kchunk; k0 += 256) {
            const uint4 wr = ld_stream_v4(wrow + k0);
            const uint32_t wv[4] = {wr.x, wr.y, wr.z, wr.w};
            float wf[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                wf[2 * j] = bf16_bits_to_float(wv[j] & 0xFFFFu);
                wf[2 * j + 1] = bf16_bits_to_float(wv[j] >> 16);
            }
#pragma unroll
            for (int b0 = 0; b0 < BP; b0 += 8) {  // eight independent x loads in flight
                uint4 xr[8];
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    xr[j] = b0 + j < P.B ? __ldg(reinterpret_cast<const uint4 *>(P.x + (size_t)(b0 + j) * P.H + k0))
                                         : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t xv[4] = {xr[j].x, xr[j].y, xr[j].z, xr[j].w};
                    float a = acc[b0 + j];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        a = fmaf(wf[2 * e], bf16_bits_to_float(xv[e] & 0xFFFFu), a);
                        a = fmaf(wf[2 * e + 1], bf16_bits_to_float(xv[e] >> 16), a);
                    }
                    acc[b0 + j] = a;
                }
            }
        }
#pragma unroll
        for (int b = 0; b < BP; ++b) {
            const float v = warp_sum(acc[b]);
            if (lane == 0) vs->red_w[vw][b] = v;
        }
        named_bar(2, 256);
        if (vt < P.B) {
            float sum = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) sum += vs->red_w[j][vt];
            if (it < P.nh) P.bpre[(size_t)vt * P.nh + it] = sum;
            else P.t[(size_t)vt * P.r + (it - P.nh)] = sum;
        }
        named_bar(2, 256);
        if (vt == 0 && !P.skip_gate_release) red_release_add(P.ctr + C_GATE, 1u);
    }
}

// Gates of two units (u1 < 0: none) into their rows of the gate buffer (alpha of the unit's
// rows at [0, hpu * dk), beta of its heads at kGateBeta), by all 256 vector threads with every
// load issued in one batch: t of the two sequences into shared memory, beta, and one W_a_up row
// per thread and unit.  t and W_b x must be final.
template <int DK, int DV, class VS>
__device__ void pair_gates(const FusedParams &P, VS *vs, int u0, int u1, int vt)
{
    constexpr int hpu = 128 / DV, rows = hpu * DK;
    const int r4 = P.r / 4;
    const int us[2] = {u0, u1};
    float *ts = &vs->red_w[0][0];  // [2][r] (r <= 256)
    if (vt < 2 * r4) {
        const int j = vt / r4, c4 = vt % r4;
        if (us[j] >= 0)
            *reinterpret_cast<float4 *>(ts + j * P.r + 4 * c4) =
                __ldcg(reinterpret_cast<const float4 *>(P.t + (size_t)(us[j] % P.Bs) * P.r) + c4);
    } else if (vt >= 128 && vt < 128 + 2 * hpu) {
        const int j = (vt - 128) / hpu, hh = (vt - 128) % hpu;
        if (us[j] >= 0) {
            const int b = us[j] % P.Bs, h = (us[j] / P.Bs) * hpu + hh;
            P.gbuf[(size_t)us[j] * kGateStride + kGateBeta + hh] = inv_one_plus_exp(-__ldcg(P.bpre + (size_t)b * P.nh + h));
        }
    }
    for (int idx0 = 0; idx0 < 2 * rows; idx0 += 256) {
        const int idx = idx0 + vt, j = idx / rows, i = idx % rows;
        const bool has = idx < 2 * rows && us[j < 2 ? j : 0] >= 0;
        const uint16_t *wr = P.wa_up + ((size_t)((has ? us[j] : 0) / P.Bs) * hpu * DK + i) * P.r;
        float z = 0.f;
        for (int j0 = 0; j0 < P.r; j0 += 64) {
            uint4 w4[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                w4[q] = has && j0 + q * 8 < P.r ? __ldg(reinterpret_cast<const uint4 *>(wr + j0 + q * 8))
                                                : make_uint4(0, 0, 0, 0);
            if (j0 == 0) named_bar(2, 256);  // t is in shared memory
            if (has) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    if (j0 + q * 8 >= P.r) break;
                    const uint32_t wv[4] = {w4[q].x, w4[q].y, w4[q].z, w4[q].w};
                    const float *tv = ts + j * P.r + j0 + q * 8;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        z = fmaf(bf16_bits_to_float(wv[e] & 0xFFFFu), tv[2 * e], z);
                        z = fmaf(bf16_bits_to_float(wv[e] >> 16), tv[2 * e + 1], z);
                    }
                }
            }
        }
        if (has) P.gbuf[(size_t)us[j] * kGateStride + i] = inv_one_plus_exp(z);
    }
    named_bar(2, 256);
}

// Gates of every token of a multi-token unit (sequence bs, o K-block kb): alpha into a[t],
// beta into beta[t].  Each thread loads one W_a_up row once and dots it with the T rows of t
// (staged in shared memory).  t and W_b x must be final.
template <int DK, int DV, class VS>
__device__ void token_gates(const FusedParams &P, VS *vs, int bs, int kb, int vt)
{
    constexpr int hpu = 128 / DV, rows = hpu * DK;
    const int T = P.T, h0 = kb * hpu, r4 = P.r / 4;
    float *ts = &vs->red_w[0][0];  // [T][r], T * r <= 2048 (red_w and red_p)
    for (int idx = vt; idx < T * r4; idx += 256) {
        const int t = idx / r4, c4 = idx % r4;
        *reinterpret_cast<float4 *>(ts + t * P.r + 4 * c4) =
            __ldcg(reinterpret_cast<const float4 *>(P.t + (size_t)(bs * T + t) * P.r) + c4);
    }
    for (int idx = vt; idx < T * hpu; idx += 256) {
        const int t = idx / hpu, hh = idx % hpu;
        vs->beta[t][hh] = inv_one_plus_exp(-__ldcg(P.bpre + (size_t)(bs * T + t) * P.nh + h0 + hh));
    }
    for (int i0 = 0; i0 < rows; i0 += 256) {
        const int i = i0 + vt;
        const bool has = i < rows;
        const uint16_t *wr = P.wa_up + ((size_t)h0 * DK + (has ? i : 0)) * P.r;
        float z[kMaxT];
#pragma unroll
        for (int t = 0; t < kMaxT; ++t) z[t] = 0.f;
        for (int j0 = 0; j0 < P.r; j0 += 64) {
            uint4 w4[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                w4[q] = has && j0 + q * 8 < P.r ? __ldg(reinterpret_cast<const uint4 *>(wr + j0 + q * 8))
                                                : make_uint4(0, 0, 0, 0);
            if (i0 == 0 && j0 == 0) named_bar(2, 256);  // the t rows are in shared memory
            if (!has) continue;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (j0 + q * 8 >= P.r) break;
                const uint32_t wv[4] = {w4[q].x, w4[q].y, w4[q].z, w4[q].w};
                float wf[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    wf[2 * e] = bf16_bits_to_float(wv[e] & 0xFFFFu);
                    wf[2 * e + 1] = bf16_bits_to_float(wv[e] >> 16);
                }
#pragma unroll
                for (int t = 0; t < kMaxT; ++t) {
                    if (t >= T) break;
                    const float *tv = ts + t * P.r + j0 + q * 8;
#pragma unroll
                    for (int e = 0; e < 8; ++e) z[t] = fmaf(wf[e], tv[e], z[t]);
                }
            }
        }
        if (has)
#pragma unroll
            for (int t = 0; t < kMaxT; ++t)
                if (t < T) vs->a[t][i] = inv_one_plus_exp(z[t]);
    }
    named_bar(2, 256);
}

// One state unit: sequence bs, o K-block kb (heads kb*128/dv ..), all dk rows, and its T
// tokens applied in order (rows bs*T + t) with the state held in registers.  With one token
// the first unit computes the gates of all of this CTA's units into the gate buffer (once
// every CTA's gate rows are final) and each unit copies its own into slot nu & 1 while it
// waits for its q/k/v; with several tokens every token's gates are computed here.
template <int BP, int DK, int DV, bool MT, class VS>
__device__ bool state_unit(const FusedParams &P, VS *vs, const Ctl &c, int u, int vt, int nu)
{
    constexpr ActGeo G = act_geo(BP);
    const int T = MT ? P.T : 1, bs = u % P.Bs, kb = u / P.Bs, slot = nu & 1;
    constexpr int RPW = DK / 8;  // rows per warp
    const int vw = vt >> 5, lane = vt & 31;
    constexpr int dv = DV, hpu = 128 / DV;
    const int h0 = kb * hpu;
    const int vc = lane * 4, hh = vc / dv, cc = vc % dv, h = h0 + hh;
    const int Dk = P.nh * DK, Dv = P.nh * dv;
    float *S = P.state + (((size_t)bs * P.nh + h) * DK) * dv + cc;

    float4 s[RPW];
    if (!MT) {
#pragma unroll
        for (int r = 0; r < RPW; ++r) s[r] = ld_stream_f4(S + (size_t)(vw * RPW + r) * dv);
    }

    if (vt == 0) vs->fail = 0;
    named_bar(2, 256);
    if (vt == 0 && nu < 2) KDA_TR(P, TR_USUB + 16 * nu);
    if (nu == 0) {
        // first unit, its state loads in flight: every CTA's gate rows (t and W_b x) final,
        // then this unit's and the next unit's gates (with several tokens: per unit, below)
        if (vt == 0 && !wait_count(P.ctr + C_GATE, P.t_gate, c, 10)) vs->fail = 1;
        named_bar(2, 256);
        if (vs->fail) return false;
        if (!MT)
            for (int u2 = u; u2 < P.Bs * P.nKBo; u2 += 2 * (int)gridDim.x)
                pair_gates<DK, DV>(P, vs, u2, u2 + (int)gridDim.x < P.Bs * P.nKBo ? u2 + (int)gridDim.x : -1, vt);
    }
    float ga = 0.f, gb = 0.f;  // this unit's gates (written by this CTA, read through L2)
    if (!MT) {
        if (vt < hpu * DK) ga = __ldcg(P.gbuf + (size_t)u * kGateStride + vt);
        if (vt < hpu) gb = __ldcg(P.gbuf + (size_t)u * kGateStride + kGateBeta + vt);
    }
    // then the heads' q, k, v: wait for every segment of their row groups (one thread per
    // counter, so the round trips overlap), add the partials
    {
        const int glo = h0 * DK / G.nx, nq = ((h0 + hpu) * DK - 1) / G.nx - glo + 1;
        const int vlo = kb * 128 / G.nx, nv = (kb * 128 + 127) / G.nx - vlo + 1;
        if (vt < 2 * nq + nv) {
            const int key = vt < nq ? glo + vt
                                    : (vt < 2 * nq ? P.nRGq + glo + (vt - nq) : 2 * P.nRGq + vlo + (vt - 2 * nq));
            if (!wait_rb(P, key, c, 11)) vs->fail = 1;
        }
    }
    named_bar(2, 256);
    if (vt == 0 && nu < 2) KDA_TR(P, TR_USUB + 16 * nu + 1);
    if (vs->fail) return false;
    if (!MT) {  // read after the items' barrier below
        if (vt < hpu * DK) vs->a[slot][vt] = ga;
        if (vt < hpu) vs->beta[slot][vt] = gb;
    }
    if (MT) {
        token_gates<DK, DV>(P, vs, bs, kb, vt);
#pragma unroll
        for (int r = 0; r < RPW; ++r) s[r] = ld_stream_f4(S + (size_t)(vw * RPW + r) * dv);
    }
    constexpr int nqk = hpu * DK, per = 2 * nqk + 128;
    {
        // items (token t, i): q and k rows of the unit's heads, then its 128 v columns; a
        // thread's items are loaded together (one memory round trip), then summed in slot order
        const int nitems = T * per;
        for (int it0 = 0; it0 < nitems; it0 += 512) {
            int key[2], off[2];
            bool has[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int it = it0 + vt + 256 * j, t = it / per, i = it % per, row = bs * T + t;
                has[j] = it < nitems;
                if (i < 2 * nqk) {
                    const int qrow = h0 * DK + i % nqk;
                    key[j] = (i / nqk) * P.nRGq + qrow / G.nx;
                    off[j] = row * G.nx + qrow % G.nx;
                } else {
                    const int col = kb * 128 + (i - 2 * nqk);
                    key[j] = 2 * P.nRGq + col / G.nx;
                    off[j] = row * G.nx + col % G.nx;
                }
            }
            float val[2];
            sum_segs2<BP>(P, key, off, has, val);
            if (vt == 0 && nu < 2 && it0 == 0) KDA_TR(P, TR_USUB + 16 * nu + 2);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int it = it0 + vt + 256 * j, t = it / per, i = it % per, row = bs * T + t;
                if (!has[j]) continue;
                if (i < 2 * nqk) {
                    const int ii = i % nqk, isk = i / nqk, qrow = h0 * DK + ii;
                    (isk ? vs->k[t] : vs->q[t])[ii] = val[j];
                    (isk ? P.k : P.q)[(size_t)row * Dk + qrow] = val[j];  // kept for kda_decode_debug_copy
                } else {
                    const int ii = i - 2 * nqk;
                    vs->v[t][ii] = val[j];
                    P.v[(size_t)row * Dv + (size_t)kb * 128 + ii] = val[j];
                }
            }
        }
    }
    named_bar(2, 256);
    if (vt == 0 && nu < 2) KDA_TR(P, TR_USUB + 16 * nu + 3);
    // ||k|| and k.q per token and head (one warp per pair)
    for (int pr = vw; pr < T * hpu; pr += 8) {
        const int t = pr / hpu, hd = pr % hpu;
        float ss = 0.f, kq = 0.f;
        for (int i = lane; i < DK; i += 32) {
            const float kv = vs->k[t][hd * DK + i];
            ss = fmaf(kv, kv, ss);
            kq = fmaf(kv, vs->q[t][hd * DK + i], kq);
        }
        ss = warp_sum(ss);
        kq = warp_sum(kq);
        if (lane == 0) {
            const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
            vs->inv[t][hd] = inv;
            vs->kq[t][hd] = kq * inv;
        }
    }
    named_bar(2, 256);
    for (int i = vt; i < T * nqk; i += 256) vs->k[i / nqk][i % nqk] *= vs->inv[i / nqk][(i % nqk) / DK];
    named_bar(2, 256);
    if (vt == 0 && nu < 2) KDA_TR(P, TR_USUB + 16 * nu + 4);
    for (int t = 0; t < T; ++t) {
        const float *al = vs->a[MT ? t : slot];
        const float *kt = vs->k[t], *qt = vs->q[t];
        // S~ = diag(alpha) S; partial w = S~^T k^, p = S~^T q over this warp's rows
        float4 pw = make_float4(0.f, 0.f, 0.f, 0.f), pp = pw;
        const int i0 = hh * DK + vw * RPW;  // this warp's rows, four at a time (16-byte loads)
#pragma unroll
        for (int r4 = 0; r4 < RPW; r4 += 4) {
            const float4 a4 = *reinterpret_cast<const float4 *>(al + i0 + r4);
            const float4 k4 = *reinterpret_cast<const float4 *>(kt + i0 + r4);
            const float4 q4 = *reinterpret_cast<const float4 *>(qt + i0 + r4);
            const float av[4] = {a4.x, a4.y, a4.z, a4.w}, kv[4] = {k4.x, k4.y, k4.z, k4.w};
            const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float4 &sr = s[r4 + j];
                const float a = av[j], kk = kv[j], qq = qv[j];
                sr.x *= a; sr.y *= a; sr.z *= a; sr.w *= a;
                pw.x = fmaf(kk, sr.x, pw.x); pw.y = fmaf(kk, sr.y, pw.y);
                pw.z = fmaf(kk, sr.z, pw.z); pw.w = fmaf(kk, sr.w, pw.w);
                pp.x = fmaf(qq, sr.x, pp.x); pp.y = fmaf(qq, sr.y, pp.y);
                pp.z = fmaf(qq, sr.z, pp.z); pp.w = fmaf(qq, sr.w, pp.w);
            }
        }
        *reinterpret_cast<float4 *>(&vs->red_w[vw][vc]) = pw;
        *reinterpret_cast<float4 *>(&vs->red_p[vw][vc]) = pp;
        named_bar(2, 256);
        if (vt == 0 && nu < 2 && t == 0) KDA_TR(P, TR_USUB + 16 * nu + 9);
        if (vt < 128) {
            float w = 0.f, p = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                w += vs->red_w[j][vt];
                p += vs->red_p[j][vt];
            }
            const int hx = vt / dv;
            const float uu = vs->beta[MT ? t : slot][hx] * (vs->v[t][vt] - w);
            vs->u[vt] = uu;
            vs->o[vt] = fmaf(uu, vs->kq[t][hx], p);
        }
        named_bar(2, 256);
        if (vt == 0 && nu < 2 && t == 0) KDA_TR(P, TR_USUB + 16 * nu + 5);
        // o of row bs*T + t -> four E4M3 planes with one power-of-two scale for the K-block
        if (vw == 0) {
            const int row = bs * T + t;
            const float4 o4 = *reinterpret_cast<const float4 *>(&vs->o[vc]);
            const float amax = warp_max(fmaxf(fmaxf(fabsf(o4.x), fabsf(o4.y)), fmaxf(fabsf(o4.z), fabsf(o4.w))));
            const float sc = pow2_scale(amax), inv = pow2_inv(sc);
            uint32_t wq[4];
            split_planes<4>(o4.x * inv, o4.y * inv, o4.z * inv, o4.w * inv, wq);
#pragma unroll
            for (int p = 0; p < 4; ++p)
                *reinterpret_cast<uint32_t *>(P.oq + (size_t)o_row(p, row) * Dv + (size_t)kb * 128 + vc) = wq[p];
            if (lane == 0)
                *reinterpret_cast<float *>(P.oq + (size_t)(G.rso + row / 32) * Dv + (size_t)kb * 128 + (row % 32) * 4) = sc;
            if (lane == 0 && nu < 2 && t == 0) KDA_TR(P, TR_USUB + 16 * nu + 6);
        }
        // S' = S~ + k^ u^T (kept in registers for the next token)
        const float4 u4 = *reinterpret_cast<const float4 *>(&vs->u[vc]);
#pragma unroll
        for (int r4 = 0; r4 < RPW; r4 += 4) {
            const float4 k4 = *reinterpret_cast<const float4 *>(kt + i0 + r4);
            const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float4 &sr = s[r4 + j];
                sr.x = fmaf(kv[j], u4.x, sr.x); sr.y = fmaf(kv[j], u4.y, sr.y);
                sr.z = fmaf(kv[j], u4.z, sr.z); sr.w = fmaf(kv[j], u4.w, sr.w);
            }
        }
        if (t + 1 < T) named_bar(2, 256);  // u, o and the reductions are reused by the next token
    }
    if (vw == 0) {
        fence_proxy_async_global();  // every token's planes, read by other SMs' TMA copies
        __syncwarp();
        if (lane == 0) {
            // hand the release of the o block (every token's planes) to the o publisher (its
            // fence then never holds up the unit); at most kOHand units may wait for it
            const uint64_t t0 = globaltimer_ns();
            while (nu - *(volatile int *)&vs->opub >= kOHand && globaltimer_ns() - t0 < P.timeout_ns) __nanosleep(64);
            mbar_arrive(&vs->ohand[nu % kOHand]);
            if (nu < 2) KDA_TR(P, TR_UNIT_HAND + nu);
        }
    }
    // the updated state, written back in place (after the hand-off: nothing reads it this step)
#pragma unroll
    for (int r = 0; r < RPW; ++r) st_stream_f4(S + (size_t)(vw * RPW + r) * dv, s[r]);
    named_bar(2, 256);
    if (vt == 0 && nu < 2) KDA_TR(P, TR_USUB + 16 * nu + 7);
    return true;
}

// Warp 1, lane 0: releases the o blocks of this CTA's state units, in unit order, once vector
// warp 0 has stored their planes.
template <class VS>
__device__ void o_publisher(const FusedParams &P, VS *vs, const Ctl &c)
{
    const int units = P.Bs * P.nKBo;
    for (int k = 0, u = blockIdx.x; u < units; ++k, u += gridDim.x) {
        if (!wait_bar(&vs->ohand[k % kOHand], (uint32_t)(k / kOHand) & 1u, c, 14)) return;
        if (!*c.sh_abort) red_release_add(P.ctr + P.off_oready + u / P.Bs, 1u);
        *(volatile int *)&vs->opub = k + 1;
    }
}

// State of unit u (sequence u % B, the heads of o K-block u / B) -> L2, in 32 KB bulk prefetches.
__device__ void prefetch_unit_state(const FusedParams &P, int u)
{
    const int b = u % P.Bs, kb = u / P.Bs, hpu = 128 / P.dv;
    const size_t bytes = (size_t)hpu * P.dk * P.dv * 4;
    const char *p = reinterpret_cast<const char *>(P.state + (((size_t)b * P.nh + (size_t)kb * hpu) * P.dk) * P.dv);
    const uint64_t pol = policy_evict_last();
    for (size_t o = 0; o < bytes; o += 32768)
        bulk_prefetch_l2_hint(p + o, (uint32_t)(bytes - o < 32768 ? bytes - o : 32768), pol);
}

template <int BP, int DK, int DV, bool MT, class VS>
__device__ void vector_role(const FusedParams &P, VS *vs, const Ctl &c)
{
    constexpr ActGeo G = act_geo(BP);
    const int vt = threadIdx.x - 256, vw = vt >> 5, lane = vt & 31;
    quantize_x<BP>(P, blockIdx.x * 8 + vw, gridDim.x * 8, lane);
    if (vt == 0) KDA_TR(P, TR_XQ_DONE);
    if (vt == 0 && (int)blockIdx.x < P.Bs * P.nKBo) prefetch_unit_state(P, blockIdx.x);
    gate_rows<BP>(P, vs, vt);
    if (vt == 0) KDA_TR(P, TR_GATES_DONE);
    // State units (sequence u % B, o K-block u / B) in head order, CTA c taking c, c + grid,
    // ...: the same units every step, so the next unit's gates are computed while the
    // current one waits for its q/k/v.
    const int units = P.Bs * P.nKBo;
    for (int nu = 0, u = blockIdx.x; u < units; ++nu, u += gridDim.x) {
        if (vt == 0) vs->unit = should_stop(c) ? 1 : 0;
        named_bar(2, 256);
        if (vs->unit) return;
        if (vt == 0 && nu < 2) KDA_TR(P, TR_UNIT0 + 3 * nu);
        const int next = u + (int)gridDim.x < units ? u + (int)gridDim.x : -1;
        if (vt == 0 && next >= 0) prefetch_unit_state(P, next);  // its state streams in meanwhile
        if (!state_unit<BP, DK, DV, MT>(P, vs, c, u, vt, nu)) return;
        if (vt == 0 && nu < 2) KDA_TR(P, TR_UNIT0 + 3 * nu + 2);
    }
    // out = sum of the W_o partials (both plane pairs): items of 32 output rows.  With tensor
    // parallelism the sum is this rank's partial out: it is pushed to every rank's exchange
    // slot (peer stores over NVLink), the item's flag is raised in every rank, and each rank
    // then adds the ranks' partials in rank order (the same bits everywhere).
    const int nitems = P.H / 32, par = (int)(P.tp_epoch & 1u);
    const size_t slot_sz = (size_t)P.tp_world * P.tp_bmax * P.H;
    for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
        const int grow0 = item * 32, rg = grow0 / G.no, key = 2 * P.nRGq + P.nRGv + rg;
        if (vt == 0 && item == (int)blockIdx.x) KDA_TR(P, TR_LAST_REDUCE_START);
        if (vt == 0) vs->ok = wait_rb(P, key, c, 12);
        named_bar(2, 256);
        if (!vs->ok) return;
        if (vt == 0 && item == (int)blockIdx.x) KDA_TR(P, TR_O_WAIT0);
        const int grow = grow0 + lane, n = grow % G.no;
        for (int b = vw; b < P.B; b += 8) {
            const int kk[2] = {key, key}, off[2] = {b * G.no + n, (BP + b) * G.no + n};
            const bool has[2] = {true, true};
            float val[2];
            sum_segs2<BP>(P, kk, off, has, val);
            const float v = val[0] + val[1];
            if (P.tp_world > 0) {
                const size_t o = par * slot_sz + ((size_t)P.tp_rank * P.tp_bmax + b) * P.H + grow;
                for (int r = 0; r < P.tp_world; ++r) P.tp_slots[r][o] = v;
            } else if (P.out_bf16) {
                static_cast<__nv_bfloat16 *>(P.out)[(size_t)b * P.H + grow] = __float2bfloat16_rn(v);
            } else {
                static_cast<float *>(P.out)[(size_t)b * P.H + grow] = v;
            }
        }
        if (P.tp_world > 0) __threadfence_system();  // the pushed rows before the flags
        named_bar(2, 256);
        if (P.tp_world > 0 && vt < P.tp_world)
            st_release_sys(P.tp_flags[vt] + ((size_t)par * P.tp_world + P.tp_rank) * nitems + item, P.tp_epoch);
        if (vt == 0 && item == (int)blockIdx.x) KDA_TR(P, TR_LAST_REDUCE_END);
    }
    if (P.tp_world == 0) return;
    const float *mine = P.tp_slots[P.tp_rank] + par * slot_sz;
    const uint32_t *flags = P.tp_flags[P.tp_rank] + (size_t)par * P.tp_world * nitems;
    for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
        if (vt == 0) vs->fail = 0;
        named_bar(2, 256);
        if (vt < P.tp_world && !wait_flag_sys(flags + (size_t)vt * nitems + item, P.tp_epoch, c, 15)) vs->fail = 1;
        named_bar(2, 256);
        if (vs->fail) return;
        const int grow = item * 32 + lane;
        for (int b = vw; b < P.B; b += 8) {
            float v = 0.f;
            for (int r = 0; r < P.tp_world; ++r) v += __ldcv(mine + ((size_t)r * P.tp_bmax + b) * P.H + grow);
            if (P.out_bf16) static_cast<__nv_bfloat16 *>(P.out)[(size_t)b * P.H + grow] = __float2bfloat16_rn(v);
            else static_cast<float *>(P.out)[(size_t)b * P.H + grow] = v;
        }
    }
}

// ---------------------------------------------------------------- projection pipeline

// Shared-memory ring.  Stage s: an activation region (1024-aligned), then a weight region.
// The MMA reads 128 activation rows from a region's start; rows past the ones loaded are junk
// (the stage's weights), which only fill accumulator lanes nobody reads.
struct Ring {
    uint8_t *a0;
    int S, a_bytes, w_bytes, nacc, cols;
    uint64_t *full, *mmad, *empty, *accempty, *segdone;
    __device__ uint8_t *a(int s) const { return a0 + (size_t)s * (a_bytes + w_bytes); }
    __device__ uint8_t *w(int s) const { return a0 + (size_t)s * (a_bytes + w_bytes) + a_bytes; }
};

// fp32 scale of sequence b in an activation tile whose scale rows start at row R.
__device__ __forceinline__ float staged_scale(const uint8_t *a, int R, int b)
{
    return *reinterpret_cast<const float *>(a + swz(R + b / 32, (b % 32) * 4));
}

// One activation tile into stage s: the first box (groups and scale rows, up to 256 rows),
// the scale rows past 256, and a 16-row copy of group v % groups into each empty slot v.
template <int GR, int SR>
__device__ __forceinline__ uint32_t act_copy(uint8_t *dst, const CUtensorMap *main, const CUtensorMap *sc,
                                             const CUtensorMap *rep, int kb, uint64_t *bar, uint64_t pol)
{
    constexpr int RO = act_rows(GR, SR), RMAIN = act_main_rows(GR, SR), RSC = RO > 256 ? RO - 256 : 0;
    constexpr int NREP = act_slots(GR) - GR;
    const uint32_t bytes = (uint32_t)(RMAIN + RSC + 16 * NREP) * 128u;
    mbar_expect_tx(bar, bytes);
    tma_load_2d(dst, main, kb * 128, 0, bar, pol);
    if (RSC > 0) tma_load_2d(dst + 256 * 128, sc, kb * 128, 256, bar, pol);
#pragma unroll
    for (int v = GR; v < GR + NREP; ++v)
        tma_load_2d(dst + act_rowbase(v) * 128, rep, kb * 128, act_rowbase(v % GR), bar, pol);
    return bytes;
}

// Warp 0, lane 0.  Weight copies run up to S tiles ahead; the activation copy of tile i is
// issued right after its weight copy once its input is final (x split into planes, or an
// o K-block whose state units are done).  An activation that is not ready yet is deferred
// and polled only when no weight copy can be issued, so weights keep streaming.
template <int BP>
__device__ __forceinline__ void weight_copy(const FusedParams &P, const Ring &R, const TileEntry &e, int i, uint64_t pol)
{
    constexpr ActGeo G = act_geo(BP);
    const int N = e.mat < 3 ? G.nx : G.no;
    if (i < 32) KDA_TR(P, TR_TILE_TMA + i);
    mbar_expect_tx(&R.full[i % R.S], N * 128);
    tma_load_2d(R.w(i % R.S), &P.tm_w[e.mat], e.kb * 128, e.rg * N, &R.full[i % R.S], pol);
}

// The weight copies of the first stages (all free at launch); returns how many were issued.
template <int BP>
__device__ int preissue_weights(const FusedParams &P, const Ring &R, const TileEntry *my, int n)
{
    const uint64_t pol_w = policy_evict_first();
    const int k = n < R.S ? n : R.S;
    for (int i = 0; i < k; ++i) weight_copy<BP>(P, R, my[i], i, pol_w);
    return k;
}

template <int BP>
__device__ void producer(const FusedParams &P, const Ring &R, const TileEntry *my, int n, const Ctl &c, int pre)
{
    constexpr ActGeo G = act_geo(BP);
    const uint64_t pol_w = policy_evict_first(), pol_a = policy_evict_last();
    int nw = pre, na = 0;  // weight copies issued, activation copies issued (na <= nw)
    bool x_ok = false;
    uint32_t o_ok[16] = {};  // bit kb: o K-block kb known final (kb < 512)
    uint64_t t_stall = 0, t_poll = 0, t_abort = globaltimer_ns() + 20000;
    auto known_ready = [&](const TileEntry &e) {
        return e.mat < 3 ? x_ok : ((o_ok[e.kb >> 5] >> (e.kb & 31)) & 1u) != 0u;
    };
    auto poll_ready = [&](const TileEntry &e) {
        if (e.mat < 3) {
            if ((int32_t)(ld_acquire(P.ctr + C_XQ) - P.t_xq) < 0) return false;
            x_ok = true;
            KDA_TR(P, TR_XREADY);
        } else {
            if ((int32_t)(ld_acquire(P.ctr + P.off_oready + e.kb) - P.t_o) < 0) return false;
            o_ok[e.kb >> 5] |= 1u << (e.kb & 31);
            KDA_TR(P, TR_O_READY_LAST);
        }
        fence_proxy_async_global();  // planes written by other SMs, read by the async proxy
        return true;
    };
    // Hold the weight stream back after the first early_tiles copies until x is split into
    // planes (or kEarlyHoldNs passed): the x loads of the splitting CTAs then do not queue
    // behind a full ring of weight copies from every SM, and the MMA starts sooner.
    const uint64_t hold_until = globaltimer_ns() + kEarlyHoldNs;
    while (na < n) {
        bool progress = false;
        if (!x_ok && nw >= P.early_tiles && nw < n && my[nw].mat < 3 && globaltimer_ns() < hold_until) {
            if (!poll_ready(my[nw])) {
                __nanosleep(128);
                continue;
            }
        }
        while (na < nw && known_ready(my[na])) {
            const TileEntry e = my[na];
            uint64_t *bar = &R.full[na % R.S];
            uint8_t *dst = R.a(na % R.S);
            if (na < 32) KDA_TR(P, TR_TILE_ACT + na);
            if (e.mat < 3) act_copy<G.gx, G.sr>(dst, &P.tm_xq, &P.tm_xq, &P.tm_xrep, e.kb, bar, pol_a);
            else act_copy<G.go, G.sr>(dst, &P.tm_oq, &P.tm_osc, &P.tm_orep, e.kb, bar, pol_a);
            ++na;
            progress = true;
        }
        if (nw < n && nw - na < R.S && mbar_test_wait(&R.empty[nw % R.S], ((uint32_t)(nw / R.S) & 1u) ^ 1u)) {
            weight_copy<BP>(P, R, my[nw], nw, pol_w);
            ++nw;
            t_stall = 0;
            continue;
        }
        const uint64_t now = globaltimer_ns();
        if (na < nw && now >= t_poll) {  // a poll is a global round trip: at most one per 0.2 us
            if (poll_ready(my[na])) progress = true;
            else t_poll = globaltimer_ns() + 200;
        }
        if (progress) {
            t_stall = 0;
            continue;
        }
        // nothing could be issued: give up after the timeout
        if (poll_abort(c, now, t_abort)) break;
        if (t_stall == 0) t_stall = now;
        else if (now - t_stall > P.timeout_ns) {
            raise_abort(c, 1);
            break;
        }
    }
    // Every issued copy must land before the CTA may exit.  Stages whose activation copy was
    // never issued get the missing arrival, so their phase completes when the weight lands.
    for (int i = na; i < nw; ++i) mbar_arrive(&R.full[i % R.S]);
    for (int i = nw > R.S ? nw - R.S : 0; i < nw; ++i) drain_bar(P, &R.full[i % R.S], (uint32_t)(i / R.S) & 1u);
}

template <int BP>
__device__ void mma_issuer(const FusedParams &P, const Ring &R, const TileEntry *my, int n, uint32_t tmem,
                           const Ctl &c)
{
    constexpr ActGeo G = act_geo(BP);
    int issued = 0;
    for (int i = 0; i < n; ++i) {
        const TileEntry e = my[i];
        const int s = i % R.S, buf = i % R.nacc;
        if (!wait_bar(&R.full[s], (uint32_t)(i / R.S) & 1u, c, 5)) break;
        if (i >= R.nacc && !wait_bar(&R.accempty[buf], ((uint32_t)(i / R.nacc) & 1u) ^ 1u, c, 7)) break;
        tc_fence_after();
        const bool isx = e.mat < 3;
        const int N = isx ? G.nx : G.no, MH = isx ? G.mhx : G.mho;
        const uint32_t idesc = idesc_e4m3_f32(128, (uint32_t)N);
        const uint32_t aa = smem_u32(R.a(s)), wa = smem_u32(R.w(s));
        const uint32_t d = tmem + (uint32_t)(buf * R.cols);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            for (int h = 0; h < MH; ++h)
                mma_f8f6f4(d + (uint32_t)(h * N), sdesc_k128_sw128(aa + h * 16384 + ks * 32),
                           sdesc_k128_sw128(wa + ks * 32), idesc, ks > 0 ? 1u : 0u);
        mma_commit(&R.mmad[s]);
        if (issued == 0) KDA_TR(P, TR_FIRST_MMA);
        if (i < 32) KDA_TR(P, TR_TILE_MMA + i);
        ++issued;
    }
    if (issued > 0) {  // the last MMAs must finish before TMEM is freed
        const int i = issued - 1;
        drain_bar(P, &R.mmad[i % R.S], (uint32_t)(i / R.S) & 1u);
    }
}

// 16x256b TMEM load, 8 repetitions: for repetition r, registers 4r, 4r+1 hold lane
// (base + t/4) and 4r+2, 4r+3 lane (base + 8 + t/4), columns 8r + 2 (t % 4) + {0, 1}.
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// Slots of warp quarter q: v = q, q + 4, ...  Slot v holds row group g = v % GR (x: sequences
// 8g..8g+7, planes 0-1; o: sequences 8(g/2).., planes 2(g%2), 2(g%2)+1).  With fewer than
// four groups, the copies of a group split its N columns: slot v takes part v / GR.
template <int GR, int N>
struct EpiGeo {
    static constexpr int SL = GR < 4 ? 4 : GR;       // slots
    static constexpr int CS = GR < 4 ? 4 / GR : 1;   // column parts per group
    static constexpr int NW = N / CS;                // columns per slot
    static constexpr int GPW = SL / 4;               // slots per warp
    static constexpr int KPS = NW / 4;               // running sums per slot and thread
    static_assert(GPW * KPS <= 64, "running sums exceed the register budget");
    static_assert(NW % 64 == 0, "a slot's columns come in 64-column loads");
};

// The activation scales thread t of warp quarter q needs from a stage (one per slot): read
// before the stage is handed back, so that its refill does not wait for the TMEM reads.
template <int GR, int N, bool O>
__device__ __forceinline__ void epi_scales(int q, int t, const uint8_t *as, int RS, float (&sa)[4])
{
    using E = EpiGeo<GR, N>;
#pragma unroll
    for (int gi = 0; gi < E::GPW; ++gi) {
        const int v = q + 4 * gi, g = v % GR;
        const int b = (O ? 8 * (g / 2) : 8 * g) + (t >> 2);
        sa[gi] = v < E::SL ? staged_scale(as, RS, b) : 0.f;
    }
}

// One tile into the running sums of warp quarter q.  Thread t owns sequence (first of the
// group) + t/4 and KPS columns; both of its planes arrive in the same load and are added
// before the scale.
template <int GR, int N, bool O>
__device__ __forceinline__ void epi_accumulate(uint32_t tq, int q, int t, const float (&sa)[4], float fw0, float fw1,
                                               float (&acc)[64])
{
    using E = EpiGeo<GR, N>;
#pragma unroll
    for (int gi = 0; gi < E::GPW; ++gi) {
        const int v = q + 4 * gi, part = v / GR;
        if (v < E::SL) {
            const int h = v / 8;
            const uint32_t lofs = (uint32_t)(16 * ((v % 8) / 4));
            const float f0 = fw0 * sa[gi], f1 = fw1 * sa[gi];
            const int col0 = GR < 4 ? part * E::NW : 0;
#pragma unroll
            for (int c8 = 0; c8 < E::NW / 64; ++c8) {
                uint32_t r[32];
                tmem_ld_16x256b_x8(tq + (lofs << 16) + (uint32_t)(h * N + col0 + c8 * 64), r);
                tmem_wait_ld();
#pragma unroll
                for (int rep = 0; rep < 8; ++rep) {
                    const float f = (col0 + c8 * 64 + rep * 8 < 128) ? f0 : f1;
                    const int k = gi * E::KPS + (c8 * 8 + rep) * 2;
                    acc[k] = fmaf(f, __uint_as_float(r[4 * rep]) + __uint_as_float(r[4 * rep + 2]), acc[k]);
                    acc[k + 1] = fmaf(f, __uint_as_float(r[4 * rep + 1]) + __uint_as_float(r[4 * rep + 3]), acc[k + 1]);
                }
            }
        }
    }
}

// The running sums of warp quarter q -> partial-sum slot [pair][BP][N].
template <int BP, int GR, int N, bool O>
__device__ __forceinline__ void epi_publish(float *slot, int q, int t, int B, const float (&acc)[64])
{
    using E = EpiGeo<GR, N>;
#pragma unroll
    for (int gi = 0; gi < E::GPW; ++gi) {
        const int v = q + 4 * gi, g = v % GR, part = v / GR;
        if (v < E::SL) {
            const int b = (O ? 8 * (g / 2) : 8 * g) + (t >> 2), pair = O ? (g & 1) : 0;
            const int col0 = GR < 4 ? part * E::NW : 0;
            if (b < B) {
                float *dst = slot + ((size_t)pair * BP + b) * N + col0 + 2 * (t & 3);
#pragma unroll
                for (int cc = 0; cc < E::NW / 8; ++cc) {
                    const int k = gi * E::KPS + 2 * cc;
                    __stcg(reinterpret_cast<float2 *>(dst + 8 * cc), make_float2(acc[k], acc[k + 1]));
                }
            }
        }
    }
}

// Lane 0 waits, the warp shares the result (a warp-uniform decision).
__device__ __forceinline__ bool warp_wait_bar(uint64_t *b, uint32_t parity, const Ctl &c, int where)
{
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = wait_bar(b, parity, c, where) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Warps 4-7: per tile, read the fp32 accumulator from TMEM, scale it and add it to the
// running segment sums in registers; at a segment end store the partials and hand the
// segment to the publisher.  Nothing here waits on global memory, so the MMA (up to nacc
// buffers ahead) never idles behind a publication.  After an abort the loop keeps running
// with the work skipped, so that the publisher still sees every hand-off.
template <int BP>
__device__ void epilogue_role(const FusedParams &P, const Ring &R, const TileEntry *my, int n, uint32_t tmem,
                              const Ctl &c)
{
    constexpr ActGeo G = act_geo(BP);
    const int q = ((int)threadIdx.x >> 5) & 3;  // TMEM lane quarter of this warp
    const int t = threadIdx.x & 31;
    const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
    bool dead = false;
    int nseg = 0;
    float acc[64];
#pragma unroll
    for (int k = 0; k < 64; ++k) acc[k] = 0.f;
    auto wscales = [&](const TileEntry &e, float &w0, float &w1) {
        const int N = e.mat < 3 ? G.nx : G.no;
        const int rows = e.mat < 2 ? P.nh * P.dk : (e.mat == 2 ? P.nh * P.dv : P.H);
        const int nkb = e.mat < 3 ? P.nKBx : P.nKBo, rb0 = e.rg * N / 128;
        w0 = __ldg(P.wscale[e.mat] + (size_t)rb0 * nkb + e.kb);
        w1 = (N == 256 && (rb0 + 1) * 128 < rows) ? __ldg(P.wscale[e.mat] + (size_t)(rb0 + 1) * nkb + e.kb) : 0.f;
    };
    float w0n = 0.f, w1n = 0.f;
    if (n > 0) wscales(my[0], w0n, w1n);
    for (int i = 0; i < n; ++i) {
        const TileEntry e = my[i];
        const int s = i % R.S, buf = i % R.nacc;
        const float w0 = w0n, w1 = w1n;
        if (i + 1 < n) wscales(my[i + 1], w0n, w1n);  // one tile ahead
        if (e.flags & kSegStart) {
#pragma unroll
            for (int k = 0; k < 64; ++k) acc[k] = 0.f;
        }
        if (threadIdx.x == 128 && e.mat == 3 && (i == 0 || my[i - 1].mat != 3)) KDA_TR(P, TR_QKV_DONE);
        if (!dead && !warp_wait_bar(&R.mmad[s], (uint32_t)(i / R.S) & 1u, c, 8)) dead = true;
        if (!dead) {
            tc_fence_after();
            float sa[4];
            if (e.mat < 3) epi_scales<G.gx, G.nx, false>(q, t, R.a(s), G.rsx, sa);
            else epi_scales<G.go, G.no, true>(q, t, R.a(s), G.rso, sa);
            __syncwarp();
            if (t == 0) mbar_arrive(&R.empty[s]);  // the MMA is done and the stage's scales are read
            const uint32_t tb = tq + (uint32_t)(buf * R.cols);
            if (e.mat < 3) epi_accumulate<G.gx, G.nx, false>(tb, q, t, sa, w0, w1, acc);
            else epi_accumulate<G.go, G.no, true>(tb, q, t, sa, w0, w1, acc);
            tc_fence_before();
            __syncwarp();
            if (t == 0) mbar_arrive(&R.accempty[buf]);  // the accumulator is read
            if (threadIdx.x == 128 && i < 32) KDA_TR(P, TR_TILE_EPI + i);
        }
        if (!(e.flags & kSegEnd)) continue;
        if (!dead) {
            float *slot = P.part + (size_t)e.seg * slot_floats<BP>();
            if (e.mat < 3) epi_publish<BP, G.gx, G.nx, false>(slot, q, t, P.B, acc);
            else epi_publish<BP, G.go, G.no, true>(slot, q, t, P.B, acc);
        }
        __syncwarp();  // the warp's partial stores come before lane 0's arrival
        if (t == 0) mbar_arrive(&R.segdone[nseg % kSegBars]);
        ++nseg;
    }
}

// Warp 3, lane 0: in tile order, each segment's partials are released to the consumers once
// the four epilogue warps have stored them (the release fence runs here, off the epilogue).
__device__ void publisher(const FusedParams &P, const Ring &R, const TileEntry *my, int n, const Ctl &c)
{
    int k = 0;
    for (int i = 0; i < n; ++i) {
        const TileEntry e = my[i];
        if (!(e.flags & kSegEnd)) continue;
        const bool ok = wait_bar(&R.segdone[k % kSegBars], (uint32_t)(k / kSegBars) & 1u, c, 9);
        ++k;
        if (!ok) break;
        if (!*c.sh_abort) red_release_add(P.ctr + P.off_rb + rg_key(P, e.mat, e.rg), 1u);
        if (k - 1 < 7) KDA_TR(P, TR_PUB0 + k - 1);
    }
}

// MT: several tokens per sequence (multi-token steps; a separate instantiation keeps the
// single-token state unit's registers to itself)
template <int BP, int DK, int DV, bool MT>
__global__ void __launch_bounds__(kThreads, 1) k_fused(const __grid_constant__ FusedParams P)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Ring R;
    R.S = P.stages;
    R.a_bytes = P.a_bytes;
    R.w_bytes = P.w_bytes;
    R.nacc = P.nacc;
    R.cols = P.cols;
    R.a0 = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)P.stages * (P.a_bytes + P.w_bytes));
    R.full = bars;
    R.mmad = bars + kMaxStages;
    R.empty = bars + 2 * kMaxStages;
    R.accempty = bars + 3 * kMaxStages;
    R.segdone = bars + 3 * kMaxStages + kMaxAcc;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3 * kMaxStages + kMaxAcc + kSegBars);
    volatile int *sh_abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    using VS = VecSmemT<MT ? kMaxT : 1>;
    VS *vs = reinterpret_cast<VS *>(bars + 3 * kMaxStages + kMaxAcc + kSegBars + 2);
    TileEntry *stiles = reinterpret_cast<TileEntry *>(reinterpret_cast<uint8_t *>(vs) + sizeof(VS));

    // this CTA's tile list -> shared memory (read by every role, once per tile)
    const uint32_t t_begin = P.cta_off[blockIdx.x];
    const int n = (int)(P.cta_off[blockIdx.x + 1] - t_begin);
    for (int i = threadIdx.x; i < n; i += kThreads) stiles[i] = P.tiles[t_begin + i];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < P.stages; ++s) {
            mbar_init(&R.full[s], 2);           // weight copy + activation copy
            mbar_init(&R.mmad[s], 1);           // the tile's MMA commit
            mbar_init(&R.empty[s], kEpiWarps);  // the epilogue warps are done with the stage
        }
        for (int b = 0; b < P.nacc; ++b) mbar_init(&R.accempty[b], kEpiWarps);
        for (int b = 0; b < kSegBars; ++b) mbar_init(&R.segdone[b], kEpiWarps);
        for (int b = 0; b < kOHand; ++b) mbar_init(&vs->ohand[b], 1);
        vs->opub = 0;
        *sh_abort = 0;
        mbar_fence_init();
    }
    if (warp == 3 && lane == 0) {
        // small weights every CTA reads soon: pull them into L2 before the weight stream queues up
        prefetch_l2_slice(P.wb, (size_t)P.nh * P.H * 2);
        prefetch_l2_slice(P.wa_down, (size_t)P.r * P.H * 2);
        prefetch_l2_slice(P.wa_up, (size_t)P.nh * P.dk * P.r * 2);
    }
    if (warp == 0 && lane == 0) {
        for (int m = 0; m < 4; ++m) prefetch_tmap(&P.tm_w[m]);
        prefetch_tmap(&P.tm_xq);
        prefetch_tmap(&P.tm_xrep);
        prefetch_tmap(&P.tm_oq);
        prefetch_tmap(&P.tm_orep);
        if (act_rows(act_geo(BP).go, act_geo(BP).sr) > 256) prefetch_tmap(&P.tm_osc);
    }
    if (warp == 2) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0) KDA_TR(P, TR_START);
    const uint32_t tmem = *tmem_slot;
    const Ctl c{P, sh_abort};
    const TileEntry *my = stiles;

    // Launched with programmatic stream serialization, the next step's grid may start on the
    // SMs this grid frees.  Before waiting for this grid to finish, it only reads inputs no
    // kernel writes -- the weights (the first stages of the stream) and its tile lists;
    // x, the state and every scratch buffer are touched after the wait.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    int pre = 0;
    if (warp == 0 && lane == 0) pre = preissue_weights<BP>(P, R, my, n);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0) KDA_TR(P, TR_GRID_WAIT);
    if (warp == 3 && lane == 0) prefetch_l2_slice(P.x, (size_t)P.B * P.H * 2);

    if (warp < 4) {  // single-lane roles: few registers
        regs_dec<kRegsControl>();
        if (warp == 0) {
            if (lane == 0) producer<BP>(P, R, my, n, c, pre);
        } else if (warp == 1) {
            if (lane == 0) o_publisher(P, vs, c);
        } else if (warp == 2) {
            if (lane == 0) mma_issuer<BP>(P, R, my, n, tmem, c);
        } else {
            if (lane == 0) publisher(P, R, my, n, c);
        }
        __syncwarp();
    } else if (warp < 4 + kEpiWarps) {
        epilogue_role<BP>(P, R, my, n, tmem, c);
        if (threadIdx.x == 128) KDA_TR(P, TR_EPI_DONE);
    } else {  // state units: the registers the others gave up
        regs_inc<kRegsVector>();
        vector_role<BP, DK, DV, MT>(P, vs, c);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (threadIdx.x == 0) KDA_TR(P, TR_END);
}

// ---------------------------------------------------------------- host side

typedef CUresult (*PFN_encodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                    const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

PFN_encodeTiled get_encode()
{
    static PFN_encodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_encodeTiled>(p);
        else
            (void)cudaGetLastError();
    });
    return fn;
}

// uint8 matrix [rows, cols] (row-major), box [box_rows, 128 bytes], 128-byte swizzle.  Rows
// of a box past the matrix read as zero.
bool encode_u8_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    PFN_encodeTiled enc = get_encode();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {128, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int bp_for(int B)
{
    int bp = 8;
    while (bp < B) bp *= 2;
    return bp;
}
int class_of(int BP) { return BP <= 8 ? 0 : BP <= 16 ? 1 : BP <= 32 ? 2 : 3; }

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// shared-memory regions of one ring stage: activation tile, weight tile
size_t a_bytes_for(int BP)
{
    const ActGeo g = act_geo(BP);
    return align_up((size_t)std::max(act_rows(g.gx, g.sr), act_rows(g.go, g.sr)) * 128, 1024);
}
size_t w_bytes_for(int BP)
{
    const ActGeo g = act_geo(BP);
    return (size_t)std::max(g.nx, g.no) * 128;
}
size_t stage_bytes_for(int BP) { return a_bytes_for(BP) + w_bytes_for(BP); }
int tmem_cols_for(int BP)
{
    const ActGeo g = act_geo(BP);
    return std::max(g.mhx * g.nx, g.mho * g.no);
}

int row_group_keys(const Dims &d, const SchedGeo &g)
{
    return 2 * ((d.Dk() + g.nx - 1) / g.nx) + (d.Dv() + g.nx - 1) / g.nx + (d.H + g.no - 1) / g.no;
}

size_t ctr_words(const Dims &d, int max_keys) { return C_FIXED + (size_t)d.Dv() / 128 + max_keys + 16; }

template <int BP, int DK, int DV, bool MT>
void *kernel_ptr() { return reinterpret_cast<void *>(&k_fused<BP, DK, DV, MT>); }

template <bool MT>
void *pick_kernel_t(int BP, int DK, int DV)
{
    switch (BP * 1000000 + DK * 1000 + DV) {
    case 8064064: return kernel_ptr<8, 64, 64, MT>();
    case 8064128: return kernel_ptr<8, 64, 128, MT>();
    case 8128064: return kernel_ptr<8, 128, 64, MT>();
    case 8128128: return kernel_ptr<8, 128, 128, MT>();
    case 16064064: return kernel_ptr<16, 64, 64, MT>();
    case 16064128: return kernel_ptr<16, 64, 128, MT>();
    case 16128064: return kernel_ptr<16, 128, 64, MT>();
    case 16128128: return kernel_ptr<16, 128, 128, MT>();
    case 32064064: return kernel_ptr<32, 64, 64, MT>();
    case 32064128: return kernel_ptr<32, 64, 128, MT>();
    case 32128064: return kernel_ptr<32, 128, 64, MT>();
    case 32128128: return kernel_ptr<32, 128, 128, MT>();
    case 64064064: return kernel_ptr<64, 64, 64, MT>();
    case 64064128: return kernel_ptr<64, 64, 128, MT>();
    case 64128064: return kernel_ptr<64, 128, 64, MT>();
    case 64128128: return kernel_ptr<64, 128, 128, MT>();
    default: return nullptr;
    }
}
void *pick_kernel(int BP, int DK, int DV, bool multi)
{
    return multi ? pick_kernel_t<true>(BP, DK, DV) : pick_kernel_t<false>(BP, DK, DV);
}

// Shared memory past the ring: barriers, the vector warps' area, the tile list (+ the 1 KB
// alignment slack of the dynamic allocation).
size_t fixed_smem_bytes(int max_tiles, bool multi)
{
    return 1024 /*alignment slack*/ + (3 * kMaxStages + kMaxAcc + kSegBars + 2) * 8 +
           (multi ? sizeof(VecSmemT<kMaxT>) : sizeof(VecSmemT<1>)) + (size_t)max_tiles * sizeof(TileEntry);
}

constexpr size_t kSmemBudget = 227 * 1024;

// Schedules of every padded-batch class up to bpm; false if one does not fit the kernel.
struct ClassPlan {
    std::vector<TileEntry> tiles;
    std::vector<uint32_t> off, rbinfo;
    size_t nseg = 0;
    int max_tiles = 0, keys = 0;
};
bool plan_classes(const Dims &dmax, int num_ctas, int bpm, std::vector<ClassPlan> *plans)
{
    plans->clear();
    for (int BP = 8; BP <= bpm; BP *= 2) {
        ClassPlan cp;
        const SchedGeo g = fused_sched_geo(dmax, BP);
        fused_build_schedule(dmax, num_ctas, g, &cp.tiles, &cp.off, &cp.nseg, &cp.rbinfo);
        for (int c = 0; c < num_ctas; ++c) cp.max_tiles = std::max(cp.max_tiles, (int)(cp.off[c + 1] - cp.off[c]));
        if (cp.max_tiles > kMaxTilesPerCta) return false;
        if (fixed_smem_bytes(cp.max_tiles, true) + 2 * stage_bytes_for(BP) > kSmemBudget) return false;
        cp.keys = row_group_keys(dmax, g);
        plans->push_back(std::move(cp));
    }
    return true;
}

}  // namespace

bool fused_supports(const Dims &d, int num_sms)
{
    if (num_sms < 1 || d.B < 1 || d.B > kMaxBP) return false;
    if (d.H % 128 || d.Dk() % 128 || d.Dv() % 128) return false;
    if ((d.dk != 64 && d.dk != 128) || (d.dv != 64 && d.dv != 128)) return false;
    if (d.r < 16 || d.r > 256 || d.r % 16) return false;
    if (d.nh > 65535 || d.H / 128 > 65535) return false;
    return true;
}

static int num_ctas_for(int num_sms) { return num_sms; }

size_t fused_scratch_bytes(const Dims &dmax, int num_sms)
{
    if (!fused_supports(Dims{std::min(dmax.B, kMaxBP), dmax.H, dmax.nh, dmax.dk, dmax.dv, dmax.r}, num_sms)) return 0;
    const int bpm = bp_for(std::min(dmax.B, kMaxBP));
    std::vector<ClassPlan> plans;
    if (!plan_classes(dmax, num_ctas_for(num_sms), bpm, &plans)) return 0;  // too many tiles: simple engine
    const ActGeo g = act_geo(bpm);
    size_t part = 0, sched = 0;
    int keys = 0;
    for (size_t ci = 0; ci < plans.size(); ++ci) {
        const int BP = 8 << ci;
        part = std::max(part, plans[ci].nseg * (size_t)2 * BP * 256 * 4);
        sched += align_up(plans[ci].tiles.size() * sizeof(TileEntry), 256) + align_up(plans[ci].off.size() * 4, 256) +
                 align_up(plans[ci].rbinfo.size() * 4, 256);
        keys = std::max(keys, plans[ci].keys);
    }
    size_t n = 0;
    n += align_up((size_t)act_rows(g.gx, g.sr) * dmax.H, 1024);     // x planes + scale rows
    n += align_up((size_t)act_rows(g.go, g.sr) * dmax.Dv(), 1024);  // o planes + scale rows
    n += align_up((size_t)std::min(dmax.B, kMaxBP) * (dmax.Dv() / 128) * kGateStride * 4, 256);  // gate buffer
    n += align_up(part, 256);                                // partial sums
    n += align_up(ctr_words(dmax, keys) * 4, 256);           // counters
    n += sched;                                              // tile lists, offsets, row-group info
    return n + 1024;
}

void fused_bind_scratch(const Dims &dmax, int num_sms, void *base, size_t bytes, FusedState *fs)
{
    fs->base = base;
    fs->bytes = bytes;
    if (!bytes) return;
    const int bpm = bp_for(std::min(dmax.B, kMaxBP));
    fs->bp_max = bpm;
    fs->num_ctas = num_ctas_for(num_sms);
    std::vector<ClassPlan> plans;
    plan_classes(dmax, fs->num_ctas, bpm, &plans);
    fs->nclass = (int)plans.size();
    const ActGeo g = act_geo(bpm);
    size_t part = 0;
    int keys = 0;
    for (int ci = 0; ci < fs->nclass; ++ci) {
        const int BP = 8 << ci;
        part = std::max(part, plans[ci].nseg * (size_t)2 * BP * 256 * 4);
        keys = std::max(keys, plans[ci].keys);
        fs->max_tiles_per_cta[ci] = plans[ci].max_tiles;
        fs->nseg_total = std::max(fs->nseg_total, plans[ci].nseg);
        fs->h_tiles[ci] = std::move(plans[ci].tiles);
        fs->h_off[ci] = std::move(plans[ci].off);
        fs->h_rbinfo[ci] = std::move(plans[ci].rbinfo);
    }
    char *p = reinterpret_cast<char *>(align_up(reinterpret_cast<uintptr_t>(base), 1024));
    auto take = [&](size_t n, size_t a) { char *r = p; p += align_up(n, a); return r; };
    fs->xq = (uint8_t *)take((size_t)act_rows(g.gx, g.sr) * dmax.H, 1024);
    fs->oq = (uint8_t *)take((size_t)act_rows(g.go, g.sr) * dmax.Dv(), 1024);
    fs->gbuf = (float *)take((size_t)std::min(dmax.B, kMaxBP) * (dmax.Dv() / 128) * kGateStride * 4, 256);
    fs->part = (float *)take(part, 256);
    fs->ctr_bytes = ctr_words(dmax, keys) * 4;
    fs->ctr = (uint32_t *)take(fs->ctr_bytes, 256);
    for (int ci = 0; ci < fs->nclass; ++ci) {
        fs->tiles[ci] = (TileEntry *)take(fs->h_tiles[ci].size() * sizeof(TileEntry), 256);
        fs->cta_off[ci] = (uint32_t *)take(fs->h_off[ci].size() * 4, 256);
        fs->rbinfo[ci] = (uint32_t *)take(fs->h_rbinfo[ci].size() * 4, 256);
    }
    fs->off_oready = C_FIXED;
    fs->off_rb = fs->off_oready + dmax.Dv() / 128;
}

cudaError_t fused_init(const Dims &, FusedState *fs)
{
    if (!fs->bytes) return cudaSuccess;
    if (const char *e = getenv("KDA_WAIT_LIMIT_MS")) {
        const double ms = atof(e);
        if (ms > 0) fs->timeout_ns = (uint64_t)(ms * 1e6);
    }
    if (const char *e = getenv("KDA_DEBUG_SKIP_GATE_RELEASE")) fs->debug_skip_gate_release = atoi(e) != 0;
    if (const char *e = getenv("KDA_STAGES")) fs->stages_override = atoi(e);
    fs->early_tiles = kEarlyTilesDefault;
    if (const char *e = getenv("KDA_EARLY_TILES")) fs->early_tiles = std::max(0, atoi(e));
    cudaError_t err = cudaGetDevice(&fs->device);
    for (int ci = 0; ci < fs->nclass && err == cudaSuccess; ++ci) {
        err = cudaMemcpy(fs->tiles[ci], fs->h_tiles[ci].data(), fs->h_tiles[ci].size() * sizeof(TileEntry),
                         cudaMemcpyHostToDevice);
        if (err == cudaSuccess)
            err = cudaMemcpy(fs->cta_off[ci], fs->h_off[ci].data(), fs->h_off[ci].size() * 4, cudaMemcpyHostToDevice);
        if (err == cudaSuccess)
            err = cudaMemcpy(fs->rbinfo[ci], fs->h_rbinfo[ci].data(), fs->h_rbinfo[ci].size() * 4,
                             cudaMemcpyHostToDevice);
    }
#ifdef KDA_TRACE
    if (err == cudaSuccess) err = cudaMalloc(&fs->trace, (size_t)fs->num_ctas * kTraceSlots * 8);
    if (err == cudaSuccess) err = cudaMemset(fs->trace, 0, (size_t)fs->num_ctas * kTraceSlots * 8);
#endif
    fs->uploaded = err == cudaSuccess;
    return err;
}

void fused_destroy(FusedState *fs)
{
    if (fs->trace) cudaFree(fs->trace);
    fs->trace = nullptr;
}

int fused_launches() { return 1; }

int fused_max_tokens() { return kMaxT; }

cudaError_t fused_step(const Dims &d, int tokens, const kda_weights &w, const void *x, float *state, void *out,
                       int out_dtype, FusedState &fs, const Scratch &s, int *status, cudaStream_t stream)
{
    if (!fs.uploaded) return cudaErrorNotReady;
    if (tokens < 1 || tokens > kMaxT || d.B % tokens) return cudaErrorNotSupported;
    const int BP = bp_for(d.B), cls = class_of(BP);
    const bool multi = tokens > 1;
    void *kern = pick_kernel(BP, d.dk, d.dv, multi);
    if (!kern || cls >= fs.nclass) return cudaErrorNotSupported;
    const ActGeo g = act_geo(BP);
    const SchedGeo sg = fused_sched_geo(d, BP);
    if (fs.last_class >= 0 && fs.last_class != cls) fs.needs_reset = true;  // row-group counters differ per class
    if (fs.needs_reset) {
        cudaError_t e = cudaMemsetAsync(fs.ctr, 0, fs.ctr_bytes, stream);
        if (e != cudaSuccess) return e;
        fs.epoch = 0;
        fs.cum_b = 0;
        fs.cum_s = 0;
        fs.needs_reset = false;
    }
    static thread_local FusedParams P;
    memset(&P, 0, sizeof P);
    // weight maps (cached by pointer and tile rows)
    const void *keys[4] = {w.wq, w.wk, w.wv, w.wo};
    const int box[4] = {g.nx, g.nx, g.nx, g.no};
    int slot = -1;
    for (int i = 0; i < 4 && slot < 0; ++i) {
        bool hit = true;
        for (int m = 0; m < 4; ++m) hit = hit && fs.map_keys[i][m] == keys[m] && fs.map_box[i][m] == box[m];
        if (hit) slot = i;
    }
    if (slot < 0) {
        slot = fs.map_next;
        fs.map_next = (fs.map_next + 1) & 3;
        const uint64_t rows[4] = {(uint64_t)d.Dk(), (uint64_t)d.Dk(), (uint64_t)d.Dv(), (uint64_t)d.H};
        const uint64_t cols[4] = {(uint64_t)d.H, (uint64_t)d.H, (uint64_t)d.H, (uint64_t)d.Dv()};
        for (int m = 0; m < 4; ++m) {
            fs.map_keys[slot][m] = nullptr;
            if (!encode_u8_map(&fs.wmaps[slot][m], keys[m], rows[m], cols[m], (uint32_t)box[m]))
                return cudaErrorInvalidValue;
        }
        for (int m = 0; m < 4; ++m) {
            fs.map_keys[slot][m] = keys[m];
            fs.map_box[slot][m] = box[m];
        }
    }
    for (int m = 0; m < 4; ++m) P.tm_w[m] = fs.wmaps[slot][m];
    // activation-plane maps (fixed per handle and class): x tile and one x group; o tile, its
    // scale rows past 256 and one o group
    if (!fs.amap_ok[cls]) {
        const ActGeo gm = act_geo(fs.bp_max);  // buffer rows are sized for the largest class
        const int xrows = act_rows(gm.gx, gm.sr), orows = act_rows(gm.go, gm.sr), ro = act_rows(g.go, g.sr);
        if (!encode_u8_map(&fs.amaps[cls][0], fs.xq, xrows, d.H, act_main_rows(g.gx, g.sr)) ||
            !encode_u8_map(&fs.amaps[cls][1], fs.xq, xrows, d.H, 16) ||
            !encode_u8_map(&fs.amaps[cls][2], fs.oq, orows, d.Dv(), act_main_rows(g.go, g.sr)) ||
            !encode_u8_map(&fs.amaps[cls][3], fs.oq, orows, d.Dv(), ro > 256 ? ro - 256 : 16) ||
            !encode_u8_map(&fs.amaps[cls][4], fs.oq, orows, d.Dv(), 16))
            return cudaErrorInvalidValue;
        fs.amap_ok[cls] = true;
    }
    P.tm_xq = fs.amaps[cls][0];
    P.tm_xrep = fs.amaps[cls][1];
    P.tm_oq = fs.amaps[cls][2];
    P.tm_osc = fs.amaps[cls][3];
    P.tm_orep = fs.amaps[cls][4];
    P.wscale[0] = w.sq;
    P.wscale[1] = w.sk;
    P.wscale[2] = w.sv;
    P.wscale[3] = w.so;
    P.x = static_cast<const uint16_t *>(x);
    P.wa_down = w.wa_down;
    P.wa_up = w.wa_up;
    P.wb = w.wb;
    P.state = state;
    P.out = out;
    P.xq = fs.xq;
    P.oq = fs.oq;
    P.part = fs.part;
    P.gbuf = fs.gbuf;
    P.q = s.q;
    P.k = s.k;
    P.v = s.v;
    P.bpre = s.bpre;
    P.t = s.t;
    P.ctr = fs.ctr;
    P.trace = fs.trace;
    P.tiles = fs.tiles[cls];
    P.cta_off = fs.cta_off[cls];
    P.status = status;
    P.B = d.B;
    P.T = tokens;
    P.Bs = d.B / tokens;
    P.H = d.H;
    P.nh = d.nh;
    P.dk = d.dk;
    P.dv = d.dv;
    P.r = d.r;
    P.nKBx = d.H / 128;
    P.nKBo = d.Dv() / 128;
    P.nRGq = (d.Dk() + sg.nx - 1) / sg.nx;
    P.nRGv = (d.Dv() + sg.nx - 1) / sg.nx;
    P.nRGo = (d.H + sg.no - 1) / sg.no;
    P.off_oready = fs.off_oready;
    P.off_rb = fs.off_rb;
    P.rbinfo = reinterpret_cast<const uint2 *>(fs.rbinfo[cls]);
    const uint32_t epoch = fs.epoch + 1;
    P.epoch = epoch;
    P.t_xq = (fs.cum_b + (uint32_t)d.B) * (uint32_t)P.nKBx;
    P.early_tiles = fs.early_tiles;
    P.t_gate = epoch * (uint32_t)(d.nh + d.r);
    P.t_o = fs.cum_s + (uint32_t)P.Bs;
    P.timeout_ns = fs.timeout_ns;
    P.out_bf16 = out_dtype == KDA_OUT_BF16;
    P.skip_gate_release = fs.debug_skip_gate_release;
    if (fs.tp_world > 0) {
        if (!fs.tp_ready) return cudaErrorNotReady;
        P.tp_world = fs.tp_world;
        P.tp_rank = fs.tp_rank;
        P.tp_bmax = fs.tp_bmax;
        P.tp_epoch = fs.tp_epoch + 1;
        for (int r = 0; r < fs.tp_world; ++r) {
            P.tp_slots[r] = static_cast<float *>(fs.tp_region[r]);
            P.tp_flags[r] = reinterpret_cast<uint32_t *>(static_cast<char *>(fs.tp_region[r]) + fs.tp_slot_bytes);
        }
    }
    P.a_bytes = (int)a_bytes_for(BP);
    P.w_bytes = (int)w_bytes_for(BP);
    P.cols = tmem_cols_for(BP);
    P.nacc = std::min(kMaxAcc, kTmemCols / P.cols);
    const size_t sbytes = stage_bytes_for(BP);
    const size_t fixed = fixed_smem_bytes(fs.max_tiles_per_cta[cls], multi);
    if (fixed + 2 * sbytes > kSmemBudget) return cudaErrorNotSupported;
    int stages = (int)std::min<size_t>(kMaxStagesDefault, (kSmemBudget - fixed) / sbytes);
    if (fs.stages_override > 0)
        stages = (int)std::min<size_t>({(size_t)kMaxStages, (kSmemBudget - fixed) / sbytes,
                                        (size_t)std::max(2, fs.stages_override)});
    P.stages = stages;
    const size_t smem = (size_t)stages * sbytes + fixed;

    // the dynamic shared-memory limit is a per-device attribute of the kernel
    static std::mutex mu;
    static std::map<std::pair<int, void *>, size_t> configured;
    {
        std::lock_guard<std::mutex> lk(mu);
        const auto key = std::make_pair(fs.device, kern);
        auto it = configured.find(key);
        if (it == configured.end() || it->second < smem) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            configured[key] = smem;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(fs.num_ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    // Every CTA must be resident at once (they wait on one another, with bounded waits): one
    // CTA per SM and a grid of one CTA per SM.  A cooperative launch makes the runtime check
    // that; with launch overlap the grid instead starts on the SMs the previous step frees.
    cudaLaunchAttribute attr[1];
    if (fs.overlap) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
    } else {
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void *args[1] = {&P};
    cudaError_t e = cudaLaunchKernelExC(&cfg, kern, args);
    if (e != cudaSuccess) return e;
    fs.last_class = cls;
    if (fs.tp_world > 0) fs.tp_epoch += 1;
    fs.epoch = epoch;
    fs.cum_b += (uint32_t)d.B;
    fs.cum_s += (uint32_t)P.Bs;
    return cudaSuccess;
}

}  // namespace kda
