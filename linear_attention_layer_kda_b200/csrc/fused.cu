// fused.cu -- the FUSED engine: the whole decode step as one persistent kernel on sm_100a.
//
// Design (the TrnRT story's megakernel rules restated for B200: the working set stays on
// chip and only x, the state, the streamed weights and out cross HBM; the weight stream is
// split over every SM; Kiln's "one scale per kernel tile" for the FP8 weights):
//
//  * One CTA per SM, 16 warps, cooperative launch (all CTAs co-resident).
//  * Projection pipeline (warps 0-7).  Every projection is a stream of 128 x 128 FP8 E4M3
//    weight tiles (one fp32 block scale each).  Warp 0 lane 0 loads tiles with TMA into an
//    S-stage shared-memory ring, each followed by the matching activation slice; warp 2 lane
//    0 issues tcgen05.mma kind::f8f6f4 (M=128 weight rows, N = planes x padded batch, K=128
//    in four K=32 steps) into one of eight TMEM accumulators; warps 4-7 read TMEM, apply
//    weight scale x activation scale to the 128-wide K-block partial and accumulate in
//    registers.  A CTA's run of tiles in one row block ends in a partial sum, published with
//    a release increment of the row block's counter; the consumers (state units for q, k, v;
//    the output reduction for W_o) add a row block's partials in slot order (deterministic).
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
//  * Order: the q/k/v tiles of head group 0, 1, ..., then the W_o tiles of head group
//    0, 1, ...  The weight stream holds after its first tiles until x is split (bounded),
//    so the x loads are not queued behind every SM's ring fill.
//  * Every wait is bounded (global timer); on expiry the kernel records
//    KDA_ERR_DEVICE_TIMEOUT, raises an abort flag every CTA polls, waits for its own
//    copies and MMAs in flight, frees TMEM and returns.
#include <math.h>
#include <stdlib.h>

#include <algorithm>
#include <map>
#include <mutex>

#include "fused.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int kThreads = 512;
constexpr int kMaxBP = 64;
constexpr int kTileBytes = 128 * 128;
constexpr int kMaxStages = 12;   // ring stages (weight tile + activation planes)
constexpr int kMaxAcc = 8;       // TMEM accumulator buffers
constexpr int kMaxTilesPerCta = 512;
constexpr int kTmemCols = 512;
constexpr int kEarlyTiles = 2;                 // weight copies issued before x is known final
constexpr uint64_t kEarlyHoldNs = 6000;        // longest hold of the rest of the stream

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
    TR_UNIT0 = 7,  /* 3 stamps per unit: claimed, inputs ready, done; 4 units */
    TR_O_WAIT0 = 19, TR_O_READY0, TR_O_READY_LAST, TR_END, TR_LAST_REDUCE_START, TR_LAST_REDUCE_END,
    TR_TILE_TMA = 32, TR_TILE_MMA = 64, TR_TILE_EPI = 96, TR_TILE_TMA_RET = 128, TR_TILE_ACT = 160 /* per tile i < 32 */
};

// counters (uint32, monotonic across steps; targets are multiples of the step count)
//   C_XQ          x K-blocks split into planes (B per K block per step)
//   C_GATE        gate rows finished
//   (words 2 and 3 are unused)
//   C_ABORT       set by any wait that gives up
//   off_oready+kb state units done for o K-block kb (B per step)
//   off_rb+key    segments published for row block key (q, k, v, o row blocks)
constexpr int C_XQ = 0, C_GATE = 1, C_ABORT = 4, C_FIXED = 16;

struct __align__(16) VecSmem {
    float q[256], k[256];          // per head of the unit: q, k^  (heads_per_unit * dk)
    float a[2][256];               // alpha of the current and the next unit (by unit parity)
    float v[128], u[128], o[128];  // per virtual column of the unit
    float red_w[8][128], red_p[8][128];
    float beta[2][2], kq[2], inv[2];  // beta: [unit parity][head of the unit]
    int unit, ok, fail;
};

struct FusedParams {
    CUtensorMap tm_w[4];  // W_q, W_k, W_v, W_o: uint8 [rows, K], box 128 x 128, 128B swizzle
    CUtensorMap tm_xq;    // x planes: [2*BP, H], box [2*BP, 128]
    CUtensorMap tm_oq;    // o planes (+ scale rows when they fit in one 256-row box)
    CUtensorMap tm_osc;   // o scale rows alone, used when 4*BP + scale rows > 256
    const float *wscale[4];
    const uint16_t *x, *wa_down, *wa_up, *wb;
    float *state;
    void *out;
    uint8_t *xq, *oq;  // planes + scale rows
    float *part;
    float *q, *k, *v, *bpre, *t;
    uint32_t *ctr;
    uint64_t *trace;  // null unless built with KDA_TRACE
    const TileEntry *tiles;
    const uint32_t *cta_off;
    int *status;
    const uint2 *rbinfo;  // per row-block key: (first partial slot, segments)
    int B, H, nh, dk, dv, r;
    int nKBx, nKBo, nRBq, nRBv, nRBo;
    int off_oready, off_rb;
    uint32_t epoch, t_xq, t_gate, t_o;
    uint64_t timeout_ns;
    int out_bf16, stages, stage_bytes, nacc, skip_gate_release;
};

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
    st[0] = KDA_ERR_DEVICE_TIMEOUT;
    st[1] = where;
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

// Bounded wait for the phase a barrier is known to reach (used on the exit path only).
__device__ void drain_bar(uint64_t *b, uint32_t parity, uint64_t limit_ns)
{
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(b, parity))
        if (globaltimer_ns() - t0 > limit_ns) return;
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

__device__ __forceinline__ int rb_key(const FusedParams &P, int mat, int rb)
{
    return mat < 2 ? mat * P.nRBq + rb : (mat == 2 ? 2 * P.nRBq + rb : 2 * P.nRBq + P.nRBv + rb);
}

// Sum of the published partials of row `r` (0..127), sequence b, of row block `key`, in slot order.
template <int BP>
__device__ __forceinline__ float sum_partials(const FusedParams &P, int key, int b, int r)
{
    const uint2 info = __ldg(P.rbinfo + key);
    const float *base = P.part + ((size_t)info.x * BP + b) * 128 + r;
    float s = 0.f;
    for (uint32_t g0 = 0; g0 < info.y; g0 += 8) {
        float v[8];
#pragma unroll
        for (int g = 0; g < 8; ++g) v[g] = g0 + g < info.y ? __ldcg(base + (size_t)(g0 + g) * BP * 128) : 0.f;
#pragma unroll
        for (int g = 0; g < 8; ++g) s += v[g];
    }
    return s;
}

// Two sums of the kind above with all their loads issued together (8 slots per item at a
// time); items with has[j] false are skipped.  Same slot order, so the same bits.
template <int BP>
__device__ __forceinline__ void sum_partials2(const FusedParams &P, const int (&key)[2], const int (&r)[2],
                                              const bool (&has)[2], int b, float (&out)[2])
{
    uint2 info[2];
    const float *base[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        info[j] = has[j] ? __ldg(P.rbinfo + key[j]) : make_uint2(0u, 0u);
        base[j] = P.part + ((size_t)info[j].x * BP + b) * 128 + r[j];
        out[j] = 0.f;
    }
    const uint32_t nmax = info[0].y > info[1].y ? info[0].y : info[1].y;
    for (uint32_t g0 = 0; g0 < nmax; g0 += 8) {
        float v[2][8];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int g = 0; g < 8; ++g)
                v[j][g] = g0 + g < info[j].y ? __ldcg(base[j] + (size_t)(g0 + g) * BP * 128) : 0.f;
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

// Smallest power of two s with amax / s <= 448 (s = 1 for amax == 0).
__device__ __forceinline__ float pow2_scale(float amax)
{
    if (!(amax > 0.f)) return 1.f;
    int e;
    const float m = frexpf(amax * (1.f / 448.f), &e);
    return ldexpf(1.f, m == 0.5f ? e - 1 : e);
}

// Plane buffers hold, per K block (128 bytes of every row), NP planes of BP rows and then
// the BP fp32 scales of the block in ceil(BP/32) extra rows ("scale rows"), so one TMA
// copy brings a tile's activation planes and their scales.
__host__ __device__ constexpr int scale_rows(int BP) { return (BP + 31) / 32; }
__device__ __forceinline__ float *scale_slot(uint8_t *rowbase0, size_t pitch, int NP, int BP, int b)
{
    return reinterpret_cast<float *>(rowbase0 + (size_t)(NP * BP + b / 32) * pitch + (b % 32) * 4);
}

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
    const int items = P.B * P.nKBx;
    for (int it = gw; it < items; it += ngw) {
        const int b = it / P.nKBx, kb = it % P.nKBx;
        const uint2 raw = *reinterpret_cast<const uint2 *>(P.x + (size_t)b * P.H + kb * 128 + lane * 4);
        const float v0 = bf16_bits_to_float(raw.x & 0xFFFFu), v1 = bf16_bits_to_float(raw.x >> 16);
        const float v2 = bf16_bits_to_float(raw.y & 0xFFFFu), v3 = bf16_bits_to_float(raw.y >> 16);
        const float amax = warp_max(fmaxf(fmaxf(fabsf(v0), fabsf(v1)), fmaxf(fabsf(v2), fabsf(v3))));
        const float s = pow2_scale(amax), inv = 1.f / s;  // exact: s is a power of two
        uint32_t w[2];
        split_planes<2>(v0 * inv, v1 * inv, v2 * inv, v3 * inv, w);
#pragma unroll
        for (int p = 0; p < 2; ++p)
            *reinterpret_cast<uint32_t *>(P.xq + (size_t)(p * BP + b) * P.H + kb * 128 + lane * 4) = w[p];
        if (lane == 0) *scale_slot(P.xq + kb * 128, P.H, 2, BP, b) = s;
        fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) red_release_add(P.ctr + C_XQ, 1u);
    }
}

// Gate rows (W_b and W_a_down, bf16): one row per CTA at a time, its K range split over the
// eight vector warps, partial sums added in warp order through shared memory.
template <int BP>
__device__ void gate_rows(const FusedParams &P, VecSmem *vs, int vt)
{
    const int vw = vt >> 5, lane = vt & 31;
    const int rows = P.nh + P.r;
    const int kchunk = P.H / 8;  // multiple of 16
    for (int it = blockIdx.x; it < rows; it += gridDim.x) {
        const uint16_t *wrow = it < P.nh ? P.wb + (size_t)it * P.H : P.wa_down + (size_t)(it - P.nh) * P.H;
        float acc[BP];
#pragma unroll
        for (int b = 0; b < BP; ++b) acc[b] = 0.f;
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

// Gates of state unit u (sequence u % B, o K-block u / B) into slot `slot`: beta of its
// heads and alpha = exp(-softplus(z)) = 1 / (1 + e^z), z = W_a_up[row] . t, of its rows,
// computed by vector threads [t0, t0 + nt).  t and W_b x must be final (C_GATE acquired).
template <int DK>
__device__ void unit_gates(const FusedParams &P, VecSmem *vs, int u, int slot, int vt, int t0, int nt)
{
    const int b = u % P.B, kb = u / P.B, hpu = 128 / P.dv, h0 = kb * hpu;
    const int me = vt - t0;
    if (me < 0 || me >= nt) return;
    if (me < hpu) vs->beta[slot][me] = 1.f / (1.f + expf(-__ldcg(P.bpre + (size_t)b * P.nh + h0 + me)));
    const float *t = P.t + (size_t)b * P.r;
    for (int i = me; i < hpu * DK; i += nt) {
        const uint16_t *wr = P.wa_up + ((size_t)h0 * DK + i) * P.r;
        float z = 0.f;
        for (int j0 = 0; j0 < P.r; j0 += 32) {
            uint4 w4[4];
            float4 t4[8];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                w4[q] = j0 + q * 8 < P.r ? __ldg(reinterpret_cast<const uint4 *>(wr + j0 + q * 8)) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                t4[q] = j0 + q * 4 < P.r ? __ldcg(reinterpret_cast<const float4 *>(t + j0 + q * 4)) : make_float4(0, 0, 0, 0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t wv[4] = {w4[q].x, w4[q].y, w4[q].z, w4[q].w};
                const float tv[8] = {t4[2 * q].x, t4[2 * q].y, t4[2 * q].z, t4[2 * q].w,
                                     t4[2 * q + 1].x, t4[2 * q + 1].y, t4[2 * q + 1].z, t4[2 * q + 1].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    z = fmaf(bf16_bits_to_float(wv[e] & 0xFFFFu), tv[2 * e], z);
                    z = fmaf(bf16_bits_to_float(wv[e] >> 16), tv[2 * e + 1], z);
                }
            }
        }
        vs->a[slot][i] = 1.f / (1.f + expf(z));
    }
}

// One state unit: sequence b, o K-block kb (heads kb*128/dv ..), all dk rows.  Its gates are
// in slot nu & 1; while warp 0 waits for the unit's q/k/v, warps 1-7 compute the gates of
// this CTA's next unit (next_u >= 0) into the other slot.
template <int BP, int DK>
__device__ bool state_unit(const FusedParams &P, VecSmem *vs, const Ctl &c, int u, int next_u, int vt, int nu)
{
    const int b = u % P.B, kb = u / P.B, slot = nu & 1;
    constexpr int RPW = DK / 8;  // rows per warp
    const int vw = vt >> 5, lane = vt & 31;
    const int dv = P.dv, hpu = 128 / dv, h0 = kb * hpu;
    const int vc = lane * 4, hh = vc / dv, cc = vc % dv, h = h0 + hh;
    const int Dk = P.nh * DK, Dv = P.nh * dv;
    float *S = P.state + (((size_t)b * P.nh + h) * DK) * dv + cc;

    float4 s[RPW];
#pragma unroll
    for (int r = 0; r < RPW; ++r) s[r] = ld_stream_f4(S + (size_t)(vw * RPW + r) * dv);

    if (vt == 0) vs->fail = 0;
    named_bar(2, 256);
    // then the heads' q, k, v: wait for every segment of their row blocks (one thread per
    // counter, so the round trips overlap), add the partials
    {
        const int rlo = h0 * DK / 128, nq = ((h0 + hpu) * DK - 1) / 128 - rlo + 1;
        if (vt < 2 * nq + 1) {
            const int key = vt < nq ? rlo + vt : (vt < 2 * nq ? P.nRBq + rlo + (vt - nq) : 2 * P.nRBq + kb);
            if (!wait_rb(P, key, c, 11)) vs->fail = 1;
        }
        if (next_u >= 0) unit_gates<DK>(P, vs, next_u, slot ^ 1, vt, 32, 224);
    }
    named_bar(2, 256);
    if (vt == 0 && nu < 4) KDA_TR(P, TR_UNIT0 + 3 * nu + 1);
    if (vs->fail) return false;
    {
        // items: q and k rows of the unit's heads, then its 128 v columns; a thread's items
        // are loaded together (one memory round trip), then summed in slot order
        const int nqk = hpu * DK, nitems = 2 * nqk + 128;
        for (int it0 = 0; it0 < nitems; it0 += 512) {  // 384 items (dk = 128) or 640 (dk = 128, dv = 64)
            int key[2], r[2];
            bool has[2];
    #pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int it = it0 + vt + 256 * j;
                has[j] = it < nitems;
                if (it < 2 * nqk) {
                    const int row = h0 * DK + it % nqk;
                    key[j] = (it / nqk) * P.nRBq + row / 128;
                    r[j] = row % 128;
                } else {
                    key[j] = 2 * P.nRBq + kb;
                    r[j] = it - 2 * nqk;
                }
            }
            float val[2];
            sum_partials2<BP>(P, key, r, has, b, val);
    #pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int it = it0 + vt + 256 * j;
                if (!has[j]) continue;
                if (it < 2 * nqk) {
                    const int i = it % nqk, isk = it / nqk, row = h0 * DK + i;
                    (isk ? vs->k : vs->q)[i] = val[j];
                    (isk ? P.k : P.q)[(size_t)b * Dk + row] = val[j];  // kept for kda_decode_debug_copy
                } else {
                    const int i = it - 2 * nqk;
                    vs->v[i] = val[j];
                    P.v[(size_t)b * Dv + (size_t)kb * 128 + i] = val[j];
                }
            }
        }
    }
    named_bar(2, 256);
    // ||k|| and k.q per head (one warp per head)
    if (vw < hpu) {
        float ss = 0.f, kq = 0.f;
        for (int i = lane; i < DK; i += 32) {
            const float kv = vs->k[vw * DK + i];
            ss = fmaf(kv, kv, ss);
            kq = fmaf(kv, vs->q[vw * DK + i], kq);
        }
        ss = warp_sum(ss);
        kq = warp_sum(kq);
        if (lane == 0) {
            const float inv = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
            vs->inv[vw] = inv;
            vs->kq[vw] = kq * inv;
        }
    }
    named_bar(2, 256);
    for (int i = vt; i < hpu * DK; i += 256) vs->k[i] *= vs->inv[i / DK];
    named_bar(2, 256);

    // S~ = diag(alpha) S; partial w = S~^T k^, p = S~^T q over this warp's rows
    float4 pw = make_float4(0.f, 0.f, 0.f, 0.f), pp = pw;
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        const int i = hh * DK + vw * RPW + r;
        const float a = vs->a[slot][i], kk = vs->k[i], qq = vs->q[i];
        s[r].x *= a; s[r].y *= a; s[r].z *= a; s[r].w *= a;
        pw.x = fmaf(kk, s[r].x, pw.x); pw.y = fmaf(kk, s[r].y, pw.y);
        pw.z = fmaf(kk, s[r].z, pw.z); pw.w = fmaf(kk, s[r].w, pw.w);
        pp.x = fmaf(qq, s[r].x, pp.x); pp.y = fmaf(qq, s[r].y, pp.y);
        pp.z = fmaf(qq, s[r].z, pp.z); pp.w = fmaf(qq, s[r].w, pp.w);
    }
    *reinterpret_cast<float4 *>(&vs->red_w[vw][vc]) = pw;
    *reinterpret_cast<float4 *>(&vs->red_p[vw][vc]) = pp;
    named_bar(2, 256);
    if (vt < 128) {
        float w = 0.f, p = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            w += vs->red_w[j][vt];
            p += vs->red_p[j][vt];
        }
        const int hx = vt / dv;
        const float uu = vs->beta[slot][hx] * (vs->v[vt] - w);
        vs->u[vt] = uu;
        vs->o[vt] = fmaf(uu, vs->kq[hx], p);
    }
    named_bar(2, 256);
    // o -> four E4M3 planes with one power-of-two scale for the K-block; release it
    if (vw == 0) {
        const float4 o4 = *reinterpret_cast<const float4 *>(&vs->o[vc]);
        const float amax = warp_max(fmaxf(fmaxf(fabsf(o4.x), fabsf(o4.y)), fmaxf(fabsf(o4.z), fabsf(o4.w))));
        const float sc = pow2_scale(amax), inv = 1.f / sc;
        uint32_t wq[4];
        split_planes<4>(o4.x * inv, o4.y * inv, o4.z * inv, o4.w * inv, wq);
#pragma unroll
        for (int p = 0; p < 4; ++p)
            *reinterpret_cast<uint32_t *>(P.oq + (size_t)(p * BP + b) * Dv + (size_t)kb * 128 + vc) = wq[p];
        if (lane == 0) *scale_slot(P.oq + (size_t)kb * 128, Dv, 4, BP, b) = sc;
        fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) red_release_add(P.ctr + P.off_oready + kb, 1u);
    }
    // S' = S~ + k^ u^T, written back in place (after the release: nothing reads it this step)
    const float4 u4 = *reinterpret_cast<const float4 *>(&vs->u[vc]);
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        const float kk = vs->k[hh * DK + vw * RPW + r];
        float4 o;
        o.x = fmaf(kk, u4.x, s[r].x); o.y = fmaf(kk, u4.y, s[r].y);
        o.z = fmaf(kk, u4.z, s[r].z); o.w = fmaf(kk, u4.w, s[r].w);
        st_stream_f4(S + (size_t)(vw * RPW + r) * dv, o);
    }
    named_bar(2, 256);
    return true;
}

template <int BP, int DK>
__device__ void vector_role(const FusedParams &P, VecSmem *vs, const Ctl &c)
{
    const int vt = threadIdx.x - 256, vw = vt >> 5, lane = vt & 31;
    const int gw = blockIdx.x * 8 + vw, ngw = gridDim.x * 8;
    quantize_x<BP>(P, gw, ngw, lane);
    if (vt == 0) KDA_TR(P, TR_XQ_DONE);
    gate_rows<BP>(P, vs, vt);
    if (vt == 0) KDA_TR(P, TR_GATES_DONE);
    if (vt == 0) {
        // warm L2 with this CTA's share of the recurrent state: units read it from L2 later
        const size_t sbytes = (size_t)P.B * P.nh * P.dk * P.dv * 4;
        const size_t gran = (sbytes / 16 + gridDim.x - 1) / gridDim.x * 16;
        const size_t lo = (size_t)blockIdx.x * gran;
        if (lo < sbytes) {
            const size_t nb = (sbytes - lo < gran ? sbytes - lo : gran) & ~(size_t)15;
            const uint64_t pol = policy_evict_last();
            for (size_t o = 0; o < nb; o += 32768)
                bulk_prefetch_l2_hint(reinterpret_cast<const char *>(P.state) + lo + o,
                                      (uint32_t)(nb - o < 32768 ? nb - o : 32768), pol);
        }
    }
    // State units (sequence u % B, o K-block u / B) in head order, CTA c taking c, c + grid,
    // ...: the same units every step, so the next unit's gates are computed while the
    // current one waits for its q/k/v.
    const int units = P.B * P.nKBo;
    if ((int)blockIdx.x < units) {
        if (vt == 0) vs->ok = wait_count(P.ctr + C_GATE, P.t_gate, c, 10);  // t and W_b x final
        named_bar(2, 256);
        if (!vs->ok) return;
        unit_gates<DK>(P, vs, blockIdx.x, 0, vt, 0, 256);
        named_bar(2, 256);
    }
    for (int nu = 0, u = blockIdx.x; u < units; ++nu, u += gridDim.x) {
        if (vt == 0) vs->unit = should_stop(c) ? 1 : 0;
        named_bar(2, 256);
        if (vs->unit) return;
        if (vt == 0 && nu < 4) KDA_TR(P, TR_UNIT0 + 3 * nu);
        const int next = u + (int)gridDim.x < units ? u + (int)gridDim.x : -1;
        if (!state_unit<BP, DK>(P, vs, c, u, next, vt, nu)) return;
        if (vt == 0 && nu < 4) KDA_TR(P, TR_UNIT0 + 3 * nu + 2);
    }
    // out = sum of the W_o partials: items of (row block, 32-row quarter)
    for (int item = blockIdx.x; item < 4 * P.nRBo; item += gridDim.x) {
        const int rb = item >> 2, key = 2 * P.nRBq + P.nRBv + rb;
        if (vt == 0) vs->ok = wait_rb(P, key, c, 12);
        named_bar(2, 256);
        if (!vs->ok) return;
        const int r = (item & 3) * 32 + lane, grow = rb * 128 + r;
        for (int b = vw; b < P.B; b += 8) {
            const float v = sum_partials<BP>(P, key, b, r);
            if (P.out_bf16) static_cast<__nv_bfloat16 *>(P.out)[(size_t)b * P.H + grow] = __float2bfloat16_rn(v);
            else static_cast<float *>(P.out)[(size_t)b * P.H + grow] = v;
        }
        named_bar(2, 256);
    }
}

// ---------------------------------------------------------------- projection pipeline

// Shared-memory ring.  Stage s holds the weight tile (16 KB), the activation planes of the
// same tile (up to 4 planes x BP rows x 128 bytes) and their BP scales; one producer issues
// both copies back to back, so they sit next to each other in the TMA queue.
struct Ring {
    uint8_t *base;
    int S, sbytes, NACC;
    uint64_t *full, *empty, *accfull, *accempty;
    __device__ uint8_t *w(int s) const { return base + (size_t)s * sbytes; }
    __device__ uint8_t *a(int s) const { return base + (size_t)s * sbytes + kTileBytes; }
    // scale of sequence b in the staged activation tile: row NP*BP + b/32 of a 128B-swizzled
    // tile, 16-byte chunk ((b%32)/4) XOR (row % 8)
    __device__ float scale(int s, int NP, int BP, int b) const
    {
        const int row = NP * BP + b / 32, chunk = ((b % 32) >> 2) ^ (row & 7);
        return *reinterpret_cast<const float *>(a(s) + row * 128 + chunk * 16 + (b & 3) * 4);
    }
};

// Warp 0, lane 0.  Weight copies run up to S tiles ahead; the activation copy of tile i is
// issued right after its weight copy once its input is final (x split into planes, or an
// o K-block whose state units are done).  An activation that is not ready yet is deferred
// and polled only when no weight copy can be issued, so weights keep streaming.
template <int BP>
__device__ void producer(const FusedParams &P, const Ring &R, const TileEntry *my, int n, const Ctl &c)
{
    const uint64_t pol_w = policy_evict_first(), pol_a = policy_evict_last();
    int nw = 0, na = 0;  // weight copies issued, activation copies issued (na <= nw)
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
    // Hold the weight stream back after the first kEarlyTiles copies until x is split into
    // planes (or kEarlyHoldNs passed): the x loads of the splitting CTAs then do not queue
    // behind a full ring of weight copies from every SM, and the MMA starts sooner.
    const uint64_t hold_until = globaltimer_ns() + kEarlyHoldNs;
    while (na < n) {
        bool progress = false;
        if (!x_ok && nw >= kEarlyTiles && nw < n && my[nw].mat < 3 && globaltimer_ns() < hold_until) {
            if (!poll_ready(my[nw])) {
                __nanosleep(128);
                continue;
            }
        }
        while (na < nw && known_ready(my[na])) {
            const TileEntry e = my[na];
            const int s = na % R.S;
            const int np = e.mat < 3 ? 2 : 4;
            if (na < 32) KDA_TR(P, TR_TILE_ACT + na);
            mbar_expect_tx(&R.full[s], (np * BP + scale_rows(BP)) * 128);
            tma_load_2d(R.a(s), e.mat < 3 ? &P.tm_xq : &P.tm_oq, e.kb * 128, 0, &R.full[s], pol_a);
            if (e.mat == 3 && 4 * BP + scale_rows(BP) > 256)
                tma_load_2d(R.a(s) + 4 * BP * 128, &P.tm_osc, e.kb * 128, 4 * BP, &R.full[s], pol_a);
            ++na;
            progress = true;
        }
        if (nw < n && nw - na < R.S && mbar_test_wait(&R.empty[nw % R.S], ((uint32_t)(nw / R.S) & 1u) ^ 1u)) {
            const TileEntry e = my[nw];
            if (nw < 32) KDA_TR(P, TR_TILE_TMA + nw);
            mbar_expect_tx(&R.full[nw % R.S], kTileBytes);
            tma_load_2d(R.w(nw % R.S), &P.tm_w[e.mat], e.kb * 128, e.rb * 128, &R.full[nw % R.S], pol_w);
            if (nw < 32) KDA_TR(P, TR_TILE_TMA_RET + nw);
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
    for (int i = nw > R.S ? nw - R.S : 0; i < nw; ++i)
        drain_bar(&R.full[i % R.S], (uint32_t)(i / R.S) & 1u, P.timeout_ns);
}

template <int BP>
__device__ void mma_issuer(const FusedParams &P, const Ring &R, const TileEntry *my, int n, uint32_t tmem,
                           const Ctl &c)
{
    int issued = 0;
    for (int i = 0; i < n; ++i) {
        const TileEntry e = my[i];
        const int s = i % R.S, buf = i % R.NACC;
        const uint32_t ph = (uint32_t)(i / R.S) & 1u, bph = (uint32_t)(i / R.NACC) & 1u;
        if (!wait_bar(&R.full[s], ph, c, 5)) break;
        if (!wait_bar(&R.accempty[buf], bph ^ 1u, c, 7)) break;
        tc_fence_after();
        const uint32_t idesc = e.mat < 3 ? idesc_e4m3_f32(128, 2 * BP) : idesc_e4m3_f32(128, 4 * BP);
        const uint32_t aa = smem_u32(R.w(s)), ba = smem_u32(R.a(s));
        const uint32_t d = tmem + (uint32_t)(buf * 4 * BP);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_f8f6f4(d, sdesc_k128_sw128(aa + ks * 32), sdesc_k128_sw128(ba + ks * 32), idesc, ks > 0 ? 1u : 0u);
        mma_commit(&R.empty[s]);
        mma_commit(&R.accfull[buf]);
        if (issued == 0) KDA_TR(P, TR_FIRST_MMA);
        if (i < 32) KDA_TR(P, TR_TILE_MMA + i);
        ++issued;
    }
    if (issued > 0) {  // the last MMAs must finish before TMEM is freed
        const int i = issued - 1;
        drain_bar(&R.accfull[i % R.NACC], (uint32_t)(i / R.NACC) & 1u, P.timeout_ns);
    }
}

template <int NPL, int BP>
__device__ __forceinline__ void accumulate_tile(uint32_t taddr, const Ring &R, int s, float ws, float (&acc)[BP])
{
    constexpr int N = NPL * BP;
    constexpr bool kCache = BP <= 32;  // keep the BP combined scales in registers
    float as[kCache ? BP : 1];
    if (kCache) {
#pragma unroll
        for (int b = 0; b < (kCache ? BP : 1); ++b) as[b] = ws * R.scale(s, NPL, BP, b);
    }
#pragma unroll
    for (int c0 = 0; c0 < N; c0 += 16) {
        float v[16];
        tmem_ld16(taddr + (uint32_t)c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int b = (c0 + j) % BP;
            const float f = kCache ? as[kCache ? b : 0] : ws * R.scale(s, NPL, BP, b);
            acc[b] = fmaf(f, v[j], acc[b]);
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
// running segment sum in registers; at a segment end publish the partial and release it.
// Nothing here waits on global memory, so the MMA (up to NACC buffers ahead) never idles
// behind a publication.  After an abort the loop keeps running with the work skipped, so
// that all 128 threads pass the same named barriers.
template <int BP>
__device__ void epilogue_role(const FusedParams &P, const Ring &R, const TileEntry *my, int n, uint32_t tmem,
                              const Ctl &c)
{
    const int et = threadIdx.x - 128;  // 0..127
    const int quarter = (threadIdx.x >> 5) & 3;
    const int lane = threadIdx.x & 31;
    const int row = quarter * 32 + lane;  // TMEM lane = weight row within the tile
    const uint32_t taddr_base = tmem + ((uint32_t)(quarter * 32) << 16);
    bool dead = false;
    float acc[BP];
#pragma unroll
    for (int b = 0; b < BP; ++b) acc[b] = 0.f;
    auto wscale_of = [&](const TileEntry &t) {
        return __ldg(P.wscale[t.mat] + (size_t)t.rb * (t.mat < 3 ? P.nKBx : P.nKBo) + t.kb);
    };
    float ws_next = n > 0 ? wscale_of(my[0]) : 0.f;
    for (int i = 0; i < n; ++i) {
        const TileEntry e = my[i];
        const int s = i % R.S, buf = i % R.NACC;
        const uint32_t bph = (uint32_t)(i / R.NACC) & 1u;
        const float ws = ws_next;
        if (i + 1 < n) ws_next = wscale_of(my[i + 1]);  // one tile ahead
        if (e.flags & kSegStart) {
#pragma unroll
            for (int b = 0; b < BP; ++b) acc[b] = 0.f;
        }
        if (et == 0 && e.mat == 3 && (i == 0 || my[i - 1].mat != 3)) KDA_TR(P, TR_QKV_DONE);
        if (!dead && !warp_wait_bar(&R.accfull[buf], bph, c, 8)) dead = true;
        if (!dead) {
            tc_fence_after();
            const uint32_t taddr = taddr_base + (uint32_t)(buf * 4 * BP);
            if (e.mat < 3) accumulate_tile<2, BP>(taddr, R, s, ws, acc);
            else accumulate_tile<4, BP>(taddr, R, s, ws, acc);
            mbar_arrive(&R.empty[s]);  // the stage's scales are read
            tc_fence_before();
            mbar_arrive(&R.accempty[buf]);
            if (et == 0 && i < 32) KDA_TR(P, TR_TILE_EPI + i);
        }
        if (!(e.flags & kSegEnd)) continue;
        if (!dead) {
            float *part = P.part + (size_t)e.seg * BP * 128;
#pragma unroll
            for (int b = 0; b < BP; ++b)
                if (b < P.B) part[b * 128 + row] = acc[b];
        }
        named_bar(1, 128);  // all 128 partial rows are stored before the release
        if (et == 0 && !dead && !*c.sh_abort) red_release_add(P.ctr + P.off_rb + rb_key(P, e.mat, e.rb), 1u);
    }
}

template <int BP, int DK>
__global__ void __launch_bounds__(kThreads, 1) k_fused(const __grid_constant__ FusedParams P)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Ring R;
    R.S = P.stages;
    R.sbytes = P.stage_bytes;
    R.NACC = P.nacc;
    R.base = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)P.stages * P.stage_bytes);
    R.full = bars;
    R.empty = bars + kMaxStages;
    R.accfull = bars + 2 * kMaxStages;
    R.accempty = bars + 2 * kMaxStages + kMaxAcc;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * kMaxStages + 2 * kMaxAcc);
    volatile int *sh_abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    VecSmem *vs = reinterpret_cast<VecSmem *>(bars + 2 * kMaxStages + 2 * kMaxAcc + 2);
    TileEntry *stiles = reinterpret_cast<TileEntry *>(reinterpret_cast<uint8_t *>(vs) + sizeof(VecSmem));

    // this CTA's tile list -> shared memory (read by every role, once per tile)
    const uint32_t t_begin = P.cta_off[blockIdx.x];
    const int n = (int)(P.cta_off[blockIdx.x + 1] - t_begin);
    for (int i = threadIdx.x; i < n; i += kThreads) stiles[i] = P.tiles[t_begin + i];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < P.stages; ++s) {
            mbar_init(&R.full[s], 2);          // weight copy + activation copy
            mbar_init(&R.empty[s], 1 + 128);   // MMA commit + the epilogue's 128 threads
        }
        for (int b = 0; b < P.nacc; ++b) {
            mbar_init(&R.accfull[b], 1);
            mbar_init(&R.accempty[b], 128);
        }
        *sh_abort = 0;
        mbar_fence_init();
    }
    if (warp == 3 && lane == 0) {
        // small inputs every CTA reads soon: pull them into L2 before the weight stream queues up
        prefetch_l2_slice(P.x, (size_t)P.B * P.H * 2);
        prefetch_l2_slice(P.wb, (size_t)P.nh * P.H * 2);
        prefetch_l2_slice(P.wa_down, (size_t)P.r * P.H * 2);
        prefetch_l2_slice(P.wa_up, (size_t)P.nh * P.dk * P.r * 2);
    }
    if (warp == 0 && lane == 0) {
        for (int m = 0; m < 4; ++m) prefetch_tmap(&P.tm_w[m]);
        prefetch_tmap(&P.tm_xq);
        prefetch_tmap(&P.tm_oq);
        if (4 * BP + scale_rows(BP) > 256) prefetch_tmap(&P.tm_osc);
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

    if (warp == 0) {
        if (lane == 0) producer<BP>(P, R, my, n, c);
    } else if (warp == 2) {
        if (lane == 0) mma_issuer<BP>(P, R, my, n, tmem, c);
    } else if (warp >= 4 && warp < 8) {
        epilogue_role<BP>(P, R, my, n, tmem, c);
        if (threadIdx.x == 128) KDA_TR(P, TR_EPI_DONE);
    } else if (warp >= 8) {
        vector_role<BP, DK>(P, vs, c);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        __syncwarp();
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

// uint8 matrix [rows, cols] (row-major), box [box_rows, 128 bytes], 128-byte swizzle.
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

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ring stage: weight tile, then up to four activation planes of BP rows and the scale rows
size_t stage_bytes_for(int BP) { return align_up((size_t)kTileBytes + (4 * BP + scale_rows(BP)) * 128, 1024); }

size_t ctr_words(const Dims &d)
{
    return C_FIXED + (size_t)d.Dv() / 128 + 2 * (d.Dk() / 128) + d.Dv() / 128 + d.H / 128 + 16;
}

template <int BP, int DK>
void *kernel_ptr() { return reinterpret_cast<void *>(&k_fused<BP, DK>); }

void *pick_kernel(int BP, int DK)
{
    switch (BP * 1000 + DK) {
    case 8064: return kernel_ptr<8, 64>();
    case 8128: return kernel_ptr<8, 128>();
    case 16064: return kernel_ptr<16, 64>();
    case 16128: return kernel_ptr<16, 128>();
    case 32064: return kernel_ptr<32, 64>();
    case 32128: return kernel_ptr<32, 128>();
    case 64064: return kernel_ptr<64, 64>();
    case 64128: return kernel_ptr<64, 128>();
    default: return nullptr;
    }
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
    std::vector<TileEntry> t;
    std::vector<uint32_t> o;
    size_t nseg = 0;
    fused_build_schedule(dmax, num_ctas_for(num_sms), &t, &o, &nseg, nullptr);
    for (size_t c = 0; c + 1 < o.size(); ++c)
        if (o[c + 1] - o[c] > (uint32_t)kMaxTilesPerCta) return 0;  // too many tiles per CTA: simple engine
    size_t n = 0;
    n += align_up((size_t)(2 * bpm + scale_rows(bpm)) * dmax.H, 1024);    // x planes + scale rows
    n += align_up((size_t)(4 * bpm + scale_rows(bpm)) * dmax.Dv(), 1024);  // o planes + scale rows
    n += align_up(nseg * bpm * 128 * 4, 256);                             // partial sums
    n += align_up(ctr_words(dmax) * 4, 256);                              // counters
    n += align_up(t.size() * sizeof(TileEntry), 256);                     // tile lists
    n += align_up(o.size() * 4, 256);
    n += align_up((size_t)2 * (2 * (dmax.Dk() / 128) + 2 * (dmax.Dv() / 128) + dmax.H / 128) * 4, 256);  // rbinfo
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
    fused_build_schedule(dmax, fs->num_ctas, &fs->h_tiles, &fs->h_off, &fs->nseg_total, &fs->h_rbinfo);
    fs->ntiles = fs->h_tiles.size();
    fs->max_tiles_per_cta = 0;
    for (int c = 0; c < fs->num_ctas; ++c)
        fs->max_tiles_per_cta = std::max(fs->max_tiles_per_cta, (int)(fs->h_off[c + 1] - fs->h_off[c]));
    char *p = reinterpret_cast<char *>(align_up(reinterpret_cast<uintptr_t>(base), 1024));
    auto take = [&](size_t n, size_t a) { char *r = p; p += align_up(n, a); return r; };
    fs->xq = (uint8_t *)take((size_t)(2 * bpm + scale_rows(bpm)) * dmax.H, 1024);
    fs->oq = (uint8_t *)take((size_t)(4 * bpm + scale_rows(bpm)) * dmax.Dv(), 1024);
    fs->part = (float *)take(fs->nseg_total * bpm * 128 * 4, 256);
    fs->ctr_bytes = ctr_words(dmax) * 4;
    fs->ctr = (uint32_t *)take(fs->ctr_bytes, 256);
    fs->tiles = (TileEntry *)take(fs->h_tiles.size() * sizeof(TileEntry), 256);
    fs->cta_off = (uint32_t *)take(fs->h_off.size() * 4, 256);
    fs->rbinfo = (uint32_t *)take(fs->h_rbinfo.size() * 4, 256);
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
    cudaError_t err = cudaMemcpy(fs->tiles, fs->h_tiles.data(), fs->h_tiles.size() * sizeof(TileEntry),
                                 cudaMemcpyHostToDevice);
    if (err == cudaSuccess)
        err = cudaMemcpy(fs->cta_off, fs->h_off.data(), fs->h_off.size() * 4, cudaMemcpyHostToDevice);
    if (err == cudaSuccess)
        err = cudaMemcpy(fs->rbinfo, fs->h_rbinfo.data(), fs->h_rbinfo.size() * 4, cudaMemcpyHostToDevice);
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

cudaError_t fused_step(const Dims &d, const kda_weights &w, const void *x, float *state, void *out, int out_dtype,
                       FusedState &fs, const Scratch &s, int *status, cudaStream_t stream)
{
    if (!fs.uploaded) return cudaErrorNotReady;
    const int BP = bp_for(d.B);
    void *kern = pick_kernel(BP, d.dk);
    if (!kern || BP > fs.bp_max) return cudaErrorNotSupported;
    if (fs.needs_reset) {
        cudaError_t e = cudaMemsetAsync(fs.ctr, 0, fs.ctr_bytes, stream);
        if (e != cudaSuccess) return e;
        fs.epoch = 0;
        fs.cum_b = 0;
        fs.needs_reset = false;
    }
    static thread_local FusedParams P;
    memset(&P, 0, sizeof P);
    // weight maps (cached by pointer)
    const void *keys[4] = {w.wq, w.wk, w.wv, w.wo};
    int slot = -1;
    for (int i = 0; i < 4 && slot < 0; ++i)
        if (fs.map_keys[i][0] == keys[0] && fs.map_keys[i][1] == keys[1] && fs.map_keys[i][2] == keys[2] &&
            fs.map_keys[i][3] == keys[3])
            slot = i;
    if (slot < 0) {
        slot = fs.map_next;
        fs.map_next = (fs.map_next + 1) & 3;
        const uint64_t rows[4] = {(uint64_t)d.Dk(), (uint64_t)d.Dk(), (uint64_t)d.Dv(), (uint64_t)d.H};
        const uint64_t cols[4] = {(uint64_t)d.H, (uint64_t)d.H, (uint64_t)d.H, (uint64_t)d.Dv()};
        for (int m = 0; m < 4; ++m) {
            fs.map_keys[slot][m] = nullptr;
            if (!encode_u8_map(&fs.wmaps[slot][m], keys[m], rows[m], cols[m], 128)) return cudaErrorInvalidValue;
        }
        for (int m = 0; m < 4; ++m) fs.map_keys[slot][m] = keys[m];
    }
    for (int m = 0; m < 4; ++m) P.tm_w[m] = fs.wmaps[slot][m];
    const int sr = scale_rows(BP);
    if (!encode_u8_map(&P.tm_xq, fs.xq, 2 * BP + sr, d.H, 2 * BP + sr)) return cudaErrorInvalidValue;
    if (4 * BP + sr <= 256) {
        if (!encode_u8_map(&P.tm_oq, fs.oq, 4 * BP + sr, d.Dv(), 4 * BP + sr)) return cudaErrorInvalidValue;
    } else {
        if (!encode_u8_map(&P.tm_oq, fs.oq, 4 * BP + sr, d.Dv(), 4 * BP)) return cudaErrorInvalidValue;
        if (!encode_u8_map(&P.tm_osc, fs.oq, 4 * BP + sr, d.Dv(), sr)) return cudaErrorInvalidValue;
    }
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
    P.q = s.q;
    P.k = s.k;
    P.v = s.v;
    P.bpre = s.bpre;
    P.t = s.t;
    P.ctr = fs.ctr;
    P.trace = fs.trace;
    P.tiles = fs.tiles;
    P.cta_off = fs.cta_off;
    P.status = status;
    P.B = d.B;
    P.H = d.H;
    P.nh = d.nh;
    P.dk = d.dk;
    P.dv = d.dv;
    P.r = d.r;
    P.nKBx = d.H / 128;
    P.nKBo = d.Dv() / 128;
    P.nRBq = d.Dk() / 128;
    P.nRBv = d.Dv() / 128;
    P.off_oready = fs.off_oready;
    P.off_rb = fs.off_rb;
    P.rbinfo = reinterpret_cast<const uint2 *>(fs.rbinfo);
    P.nRBo = d.H / 128;
    const uint32_t epoch = fs.epoch + 1;
    P.epoch = epoch;
    P.t_xq = (fs.cum_b + (uint32_t)d.B) * (uint32_t)P.nKBx;
    P.t_gate = epoch * (uint32_t)(d.nh + d.r);
    P.t_o = fs.cum_b + (uint32_t)d.B;
    P.timeout_ns = fs.timeout_ns;
    P.out_bf16 = out_dtype == KDA_OUT_BF16;
    P.skip_gate_release = fs.debug_skip_gate_release;
    const size_t sbytes = stage_bytes_for(BP);
    P.nacc = std::min(kMaxAcc, kTmemCols / (4 * BP));
    const size_t fixed = 1024 /*alignment slack*/ + (2 * kMaxStages + 2 * kMaxAcc + 2) * 8 + sizeof(VecSmem) +
                         (size_t)fs.max_tiles_per_cta * sizeof(TileEntry);
    const size_t budget = 227 * 1024;
    if (fixed + 2 * sbytes > budget) return cudaErrorNotSupported;
    int stages = (int)std::min<size_t>(kMaxStages, (budget - fixed) / sbytes);
    if (fs.stages_override > 0) stages = std::min(stages, std::max(2, fs.stages_override));
    P.stages = stages;
    P.stage_bytes = (int)sbytes;
    const size_t smem = (size_t)stages * sbytes + fixed;

    static std::mutex mu;
    static std::map<void *, size_t> configured;
    {
        std::lock_guard<std::mutex> lk(mu);
        auto it = configured.find(kern);
        if (it == configured.end() || it->second < smem) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            configured[kern] = smem;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(fs.num_ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void *args[1] = {&P};
    cudaError_t e = cudaLaunchKernelExC(&cfg, kern, args);
    if (e != cudaSuccess) return e;
    fs.epoch = epoch;
    fs.cum_b += (uint32_t)d.B;
    return cudaSuccess;
}

}  // namespace kda
