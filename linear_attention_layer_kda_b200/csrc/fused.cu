// fused.cu -- the FUSED engine: the whole decode step as one persistent kernel on sm_100a.
//
// Design (the TrnRT story's megakernel rules restated for B200: the working set stays on
// chip and only x, the state, the streamed weights and out cross HBM; the weight stream is
// split over every SM; Kiln's "one scale per kernel tile" for the FP8 weights):
//
//  * One CTA per SM, 16 warps, cooperative launch (all CTAs co-resident).
//  * Projection pipeline (warps 0-7).  Every projection is a stream of 128 x 128 FP8 E4M3
//    weight tiles (one fp32 block scale each).  Warp 0 loads tiles with TMA into an
//    S-stage shared-memory ring; warp 1 loads the matching activation slice; warp 2 issues
//    tcgen05.mma kind::f8f6f4 (M=128 weight rows, N = planes x padded batch, K=128 in four
//    K=32 steps) into a double-buffered TMEM accumulator; warps 4-7 read TMEM, apply
//    weight scale x activation scale to the 128-wide K-block partial and accumulate in
//    registers.  A CTA's run of tiles in one row block ends in a partial sum; the last of
//    the row block's contributors adds the partials in a fixed order (deterministic).
//  * Activations enter the tensor cores as FP8 "planes": a K-block of 128 values v with a
//    power-of-two scale s is split v/s = p0 + p1 (+ p2 + p3) with every p an E4M3 value
//    (each plane is the round-to-nearest residual of the previous ones).  Two planes hold
//    a bf16 x exactly (up to the E4M3 subnormal floor, 2^-10 of the scale), four hold the
//    fp32 readout o to about 2^-16 of its block maximum.  Products of E4M3 values are
//    exact and accumulate in fp32, so no weight is ever dequantised in registers.
//  * Vector warps (8-15): split x into planes, compute the beta and alpha-down gate rows
//    (bf16, CUDA cores), then claim (sequence, o K-block) state units in head order: load
//    the unit's fp32 state, wait until its heads' q/k/v are final, apply the gated delta
//    rule in registers, write the state back in place, split o into planes and release
//    the K-block to the output projection.
//  * Order: the q/k/v tiles of head group 0, 1, ..., then the W_o tiles of head group
//    0, 1, ...  Heads become final group by group, so state traffic and the output
//    projection overlap the weight stream instead of following it.
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
constexpr int kHeadsPerGroup = 8;
constexpr int kMaxStages = 8;
constexpr int kTmemCols = 512;

// counters
constexpr int C_XQ = 0, C_GATE = 1, C_CLAIM0 = 2, C_ABORT = 4, C_FIXED = 16;

struct VecSmem {
    float q[256], k[256], a[256];  // per head of the unit: q, k^, alpha  (heads_per_unit * dk)
    float v[128], u[128], o[128];  // per virtual column of the unit
    float t[256];                  // W_a_down x of the unit's sequence
    float red_w[8][128], red_p[8][128];
    float beta[2], kq[2], inv[2];
    int unit, ok;
};

struct FusedParams {
    CUtensorMap tm_w[4];  // W_q, W_k, W_v, W_o: uint8 [rows, K], box 128 x 128, 128B swizzle
    CUtensorMap tm_xq;    // x planes: [2*BP, H], box [2*BP, 128]
    CUtensorMap tm_oq;    // o planes: [4*BP, Dv], box [4*BP, 128]
    const float *wscale[4];
    const uint16_t *x, *wa_down, *wa_up, *wb;
    float *state;
    void *out;
    uint8_t *xq, *oq;
    float *xscale, *oscale, *part;
    float *q, *k, *v, *bpre, *t;
    uint32_t *ctr;
    const TileEntry *tiles;
    const uint32_t *cta_off;
    int *status;
    int B, H, nh, dk, dv, r;
    int nKBx, nKBo, nRBq, nRBv;
    int off_head, off_oready, off_rb, off_out;
    uint32_t epoch, t_xq, t_gate, t_head, t_o;
    uint64_t timeout_ns;
    int out_bf16, stages, stage_bytes, skip_gate_release;
};

struct Ctl {
    const FusedParams &P;
    volatile int *sh_abort;
};

__device__ __forceinline__ bool should_stop(const Ctl &c)
{
    if (*c.sh_abort) return true;
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
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(b, parity)) return true;
        if ((it & 15u) == 0u) {
            if (should_stop(c)) return false;
            if (globaltimer_ns() - t0 > c.P.timeout_ns) {
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
    for (uint32_t it = 1;; ++it) {
        __nanosleep(64);
        if ((int32_t)(ld_acquire(p) - target) >= 0) return true;
        if ((it & 15u) == 0u) {
            if (should_stop(c)) return false;
            if (globaltimer_ns() - t0 > c.P.timeout_ns) {
                raise_abort(c, where);
                return false;
            }
        }
    }
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
        if (lane == 0) P.xscale[kb * BP + b] = s;
        __threadfence();
        fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) red_release_add(P.ctr + C_XQ, 1u);
    }
}

template <int BP>
__device__ void gate_rows(const FusedParams &P, int gw, int ngw, int lane)
{
    const int rows = P.nh + P.r;
    for (int it = gw; it < rows; it += ngw) {
        const uint16_t *wrow = it < P.nh ? P.wb + (size_t)it * P.H : P.wa_down + (size_t)(it - P.nh) * P.H;
        float acc[BP];
#pragma unroll
        for (int b = 0; b < BP; ++b) acc[b] = 0.f;
        for (int k0 = lane * 8; k0 < P.H; k0 += 256) {
            const uint4 wr = ld_stream_v4(wrow + k0);
            const uint32_t wv[4] = {wr.x, wr.y, wr.z, wr.w};
            float wf[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                wf[2 * j] = bf16_bits_to_float(wv[j] & 0xFFFFu);
                wf[2 * j + 1] = bf16_bits_to_float(wv[j] >> 16);
            }
#pragma unroll
            for (int b = 0; b < BP; ++b) {
                if (b < P.B) {
                    const uint4 xr = __ldg(reinterpret_cast<const uint4 *>(P.x + (size_t)b * P.H + k0));
                    const uint32_t xv[4] = {xr.x, xr.y, xr.z, xr.w};
                    float a = acc[b];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        a = fmaf(wf[2 * j], bf16_bits_to_float(xv[j] & 0xFFFFu), a);
                        a = fmaf(wf[2 * j + 1], bf16_bits_to_float(xv[j] >> 16), a);
                    }
                    acc[b] = a;
                }
            }
        }
#pragma unroll
        for (int b = 0; b < BP; ++b) {
            const float v = warp_sum(acc[b]);
            if (lane == 0 && b < P.B) {
                if (it < P.nh) P.bpre[(size_t)b * P.nh + it] = v;
                else P.t[(size_t)b * P.r + (it - P.nh)] = v;
            }
        }
        __threadfence();
        __syncwarp();
        if (lane == 0 && !P.skip_gate_release) red_release_add(P.ctr + C_GATE, 1u);
    }
}

// One state unit: sequence b, o K-block kb (heads kb*128/dv ..), all dk rows.
template <int BP, int DK>
__device__ bool state_unit(const FusedParams &P, VecSmem *vs, const Ctl &c, int b, int kb, int vt)
{
    constexpr int RPW = DK / 8;  // rows per warp
    const int vw = vt >> 5, lane = vt & 31;
    const int dv = P.dv, hpu = 128 / dv, h0 = kb * hpu;
    const int vc = lane * 4, hh = vc / dv, cc = vc % dv, h = h0 + hh;
    const int Dk = P.nh * DK, Dv = P.nh * dv;
    float *S = P.state + (((size_t)b * P.nh + h) * DK) * dv + cc;

    float4 s[RPW];
#pragma unroll
    for (int r = 0; r < RPW; ++r) s[r] = ld_stream_f4(S + (size_t)(vw * RPW + r) * dv);

    if (vt == 0) {
        bool ok = wait_count(P.ctr + C_GATE, P.t_gate, c, 10);
        for (int j = 0; ok && j < hpu; ++j) ok = wait_count(P.ctr + P.off_head + h0 + j, P.t_head, c, 11);
        vs->ok = ok;
    }
    named_bar(2, 256);
    if (!vs->ok) return false;

    for (int i = vt; i < hpu * DK; i += 256) {
        const size_t row = (size_t)h0 * DK + i;
        vs->q[i] = __ldcg(P.q + (size_t)b * Dk + row);
        vs->k[i] = __ldcg(P.k + (size_t)b * Dk + row);
    }
    for (int i = vt; i < 128; i += 256) vs->v[i] = __ldcg(P.v + (size_t)b * Dv + (size_t)kb * 128 + i);
    for (int j = vt; j < P.r; j += 256) vs->t[j] = __ldcg(P.t + (size_t)b * P.r + j);
    if (vt < hpu) vs->beta[vt] = 1.f / (1.f + expf(-__ldcg(P.bpre + (size_t)b * P.nh + h0 + vt)));
    named_bar(2, 256);

    // alpha = exp(-softplus(z)) = 1 / (1 + e^z),  z = W_a_up[row] . t
    for (int i = vt; i < hpu * DK; i += 256) {
        const uint16_t *wr = P.wa_up + ((size_t)h0 * DK + i) * P.r;
        float z = 0.f;
        for (int j = 0; j < P.r; j += 8) {
            const uint4 w8 = __ldg(reinterpret_cast<const uint4 *>(wr + j));
            const uint32_t wv[4] = {w8.x, w8.y, w8.z, w8.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                z = fmaf(bf16_bits_to_float(wv[e] & 0xFFFFu), vs->t[j + 2 * e], z);
                z = fmaf(bf16_bits_to_float(wv[e] >> 16), vs->t[j + 2 * e + 1], z);
            }
        }
        vs->a[i] = 1.f / (1.f + expf(z));
    }
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
        const float a = vs->a[i], kk = vs->k[i], qq = vs->q[i];
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
        const float u = vs->beta[hx] * (vs->v[vt] - w);
        vs->u[vt] = u;
        vs->o[vt] = fmaf(u, vs->kq[hx], p);
    }
    named_bar(2, 256);
    // S' = S~ + k^ u^T, written back in place
    const float4 u4 = *reinterpret_cast<const float4 *>(&vs->u[vc]);
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        const float kk = vs->k[hh * DK + vw * RPW + r];
        float4 o;
        o.x = fmaf(kk, u4.x, s[r].x); o.y = fmaf(kk, u4.y, s[r].y);
        o.z = fmaf(kk, u4.z, s[r].z); o.w = fmaf(kk, u4.w, s[r].w);
        st_stream_f4(S + (size_t)(vw * RPW + r) * dv, o);
    }
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
        if (lane == 0) P.oscale[kb * BP + b] = sc;
        __threadfence();
        fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) red_release_add(P.ctr + P.off_oready + kb, 1u);
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
    gate_rows<BP>(P, gw, ngw, lane);
    const int units = P.B * P.nKBo;
    uint32_t *claim = P.ctr + C_CLAIM0 + (P.epoch & 1u);
    for (;;) {
        if (vt == 0) vs->unit = should_stop(c) ? units : (int)atomicAdd(claim, 1u);
        named_bar(2, 256);
        const int u = vs->unit;
        named_bar(2, 256);
        if (u >= units) break;
        if (!state_unit<BP, DK>(P, vs, c, u % P.B, u / P.B, vt)) break;
    }
}

// ---------------------------------------------------------------- projection pipeline

struct Ring {
    uint8_t *base;
    int stages, stage_bytes;
    uint64_t *wfull, *afull, *wempty, *aempty, *accfull, *accempty;
    __device__ uint8_t *w(int s) const { return base + (size_t)s * stage_bytes; }
    __device__ uint8_t *a(int s) const { return base + (size_t)s * stage_bytes + kTileBytes; }
    __device__ float *as(int s, int BP) const
    {
        return reinterpret_cast<float *>(base + (size_t)s * stage_bytes + kTileBytes + 4 * BP * 128);
    }
};

template <int BP>
__device__ void weight_producer(const FusedParams &P, const Ring &R, const TileEntry *my, int n, const Ctl &c)
{
    const uint64_t pol = policy_evict_first();
    int issued = 0;
    for (int i = 0; i < n; ++i) {
        const TileEntry e = my[i];
        const int s = i % R.stages;
        const uint32_t ph = (uint32_t)(i / R.stages) & 1u;
        if (!wait_bar(&R.wempty[s], ph ^ 1u, c, 1)) break;
        mbar_expect_tx(&R.wfull[s], kTileBytes);
        tma_load_2d(R.w(s), &P.tm_w[e.mat], e.kb * 128, e.rb * 128, &R.wfull[s], pol);
        ++issued;
    }
    // every issued copy must land before the CTA may exit
    for (int i = issued > R.stages ? issued - R.stages : 0; i < issued; ++i)
        drain_bar(&R.wfull[i % R.stages], (uint32_t)(i / R.stages) & 1u, P.timeout_ns);
}

template <int BP>
__device__ void act_producer(const FusedParams &P, const Ring &R, const TileEntry *my, int n, const Ctl &c)
{
    const uint64_t pol = policy_evict_last();
    bool x_ready = false;
    int issued = 0;
    for (int i = 0; i < n; ++i) {
        const TileEntry e = my[i];
        const int s = i % R.stages;
        const uint32_t ph = (uint32_t)(i / R.stages) & 1u;
        if (!wait_bar(&R.aempty[s], ph ^ 1u, c, 2)) break;
        if (e.mat < 3) {
            if (!x_ready) {
                if (!wait_count(P.ctr + C_XQ, P.t_xq, c, 3)) break;
                fence_proxy_async_global();
                x_ready = true;
            }
            mbar_expect_tx(&R.afull[s], 2 * BP * 128 + BP * 4);
            tma_load_2d(R.a(s), &P.tm_xq, e.kb * 128, 0, &R.afull[s], pol);
            bulk_load(R.as(s, BP), P.xscale + (size_t)e.kb * BP, BP * 4, &R.afull[s]);
        } else {
            if (!wait_count(P.ctr + P.off_oready + e.kb, P.t_o, c, 4)) break;
            fence_proxy_async_global();
            mbar_expect_tx(&R.afull[s], 4 * BP * 128 + BP * 4);
            tma_load_2d(R.a(s), &P.tm_oq, e.kb * 128, 0, &R.afull[s], pol);
            bulk_load(R.as(s, BP), P.oscale + (size_t)e.kb * BP, BP * 4, &R.afull[s]);
        }
        ++issued;
    }
    for (int i = issued > R.stages ? issued - R.stages : 0; i < issued; ++i)
        drain_bar(&R.afull[i % R.stages], (uint32_t)(i / R.stages) & 1u, P.timeout_ns);
}

template <int BP>
__device__ void mma_issuer(const FusedParams &P, const Ring &R, const TileEntry *my, int n, uint32_t tmem,
                           const Ctl &c)
{
    int issued = 0;
    for (int i = 0; i < n; ++i) {
        const TileEntry e = my[i];
        const int s = i % R.stages, buf = i & 1;
        const uint32_t ph = (uint32_t)(i / R.stages) & 1u, bph = (uint32_t)(i >> 1) & 1u;
        if (!wait_bar(&R.wfull[s], ph, c, 5)) break;
        if (!wait_bar(&R.afull[s], ph, c, 6)) break;
        if (!wait_bar(&R.accempty[buf], bph ^ 1u, c, 7)) break;
        tc_fence_after();
        const uint32_t idesc = e.mat < 3 ? idesc_e4m3_f32(128, 2 * BP) : idesc_e4m3_f32(128, 4 * BP);
        const uint32_t aa = smem_u32(R.w(s)), ba = smem_u32(R.a(s));
        const uint32_t d = tmem + (uint32_t)buf * 256u;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_f8f6f4(d, sdesc_k128_sw128(aa + ks * 32), sdesc_k128_sw128(ba + ks * 32), idesc, ks > 0 ? 1u : 0u);
        mma_commit(&R.wempty[s]);
        mma_commit(&R.aempty[s]);
        mma_commit(&R.accfull[buf]);
        ++issued;
    }
    if (issued > 0) {  // the last MMAs must finish before TMEM is freed
        const int i = issued - 1;
        drain_bar(&R.accfull[i & 1], (uint32_t)(i >> 1) & 1u, P.timeout_ns);
    }
}

template <int NPL, int BP>
__device__ __forceinline__ void accumulate_tile(uint32_t taddr, const float *as, float ws, float (&acc)[BP])
{
    constexpr int N = NPL * BP;
#pragma unroll
    for (int c0 = 0; c0 < N; c0 += 16) {
        float v[16];
        tmem_ld16(taddr + (uint32_t)c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int b = (c0 + j) % BP;
            acc[b] = fmaf(ws * as[b], v[j], acc[b]);
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

// Warps 4-7.  After an abort the loop keeps running with the work skipped, so that all
// 128 threads pass the same named barriers.
template <int BP>
__device__ void epilogue_role(const FusedParams &P, const Ring &R, const TileEntry *my, int n, uint32_t tmem,
                              volatile int *sh_last, const Ctl &c)
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
    for (int i = 0; i < n; ++i) {
        const TileEntry e = my[i];
        const int s = i % R.stages, buf = i & 1;
        const uint32_t bph = (uint32_t)(i >> 1) & 1u;
        const int nkb = e.mat < 3 ? P.nKBx : P.nKBo;
        const float ws = __ldg(P.wscale[e.mat] + (size_t)e.rb * nkb + e.kb);
        if (e.flags & kSegStart) {
#pragma unroll
            for (int b = 0; b < BP; ++b) acc[b] = 0.f;
        }
        if (!dead && !warp_wait_bar(&R.accfull[buf], bph, c, 8)) dead = true;
        if (!dead) {
            tc_fence_after();
            const float *as = R.as(s, BP);
            const uint32_t taddr = taddr_base + (uint32_t)buf * 256u;
            if (e.mat < 3) accumulate_tile<2, BP>(taddr, as, ws, acc);
            else accumulate_tile<4, BP>(taddr, as, ws, acc);
            mbar_arrive(&R.aempty[s]);
            tc_fence_before();
            mbar_arrive(&R.accempty[buf]);
        }
        if (!(e.flags & kSegEnd)) continue;

        // segment done: publish the partial; the last contributor of the row block sums them
        if (!dead) {
            float *part = P.part + (size_t)e.seg * BP * 128;
#pragma unroll
            for (int b = 0; b < BP; ++b)
                if (b < P.B) part[b * 128 + row] = acc[b];
        }
        __threadfence();
        named_bar(1, 128);
        if (et == 0) {
            int last = 0;
            if (!dead && !should_stop(c)) {
                uint32_t *cnt = e.mat < 3 ? P.ctr + P.off_rb + (e.mat < 2 ? e.mat * P.nRBq : 2 * P.nRBq) + e.rb
                                          : P.ctr + P.off_out + e.rb;
                const uint32_t old = atom_acq_rel_add(cnt, 1u);
                last = (old + 1u == (uint32_t)e.nseg * P.epoch) ? 1 : 0;
            }
            *sh_last = last;
        }
        named_bar(1, 128);
        const bool last = *sh_last != 0;
        named_bar(1, 128);
        if (last) {
            __threadfence();
            const int grow = e.rb * 128 + row;
            for (int b = 0; b < P.B; ++b) {
                float sum = 0.f;
                for (int g = 0; g < e.nseg; ++g)
                    sum += __ldcg(P.part + ((size_t)(e.seg0 + g) * BP + b) * 128 + row);
                if (e.mat == 3) {
                    if (P.out_bf16) static_cast<__nv_bfloat16 *>(P.out)[(size_t)b * P.H + grow] = __float2bfloat16_rn(sum);
                    else static_cast<float *>(P.out)[(size_t)b * P.H + grow] = sum;
                } else if (e.mat == 2) {
                    P.v[(size_t)b * P.nh * P.dv + grow] = sum;
                } else {
                    (e.mat == 0 ? P.q : P.k)[(size_t)b * P.nh * P.dk + grow] = sum;
                }
            }
            if (e.mat < 3) {
                __threadfence();
                named_bar(1, 128);
                if (et == 0) {
                    const int hd = e.mat == 2 ? P.dv : P.dk;
                    for (int h = e.rb * 128 / hd; h < (e.rb + 1) * 128 / hd; ++h) red_release_add(P.ctr + P.off_head + h, 1u);
                }
            }
        }
    }
}

template <int BP, int DK>
__global__ void __launch_bounds__(kThreads, 1) k_fused(const __grid_constant__ FusedParams P)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Ring R;
    R.base = smem;
    R.stages = P.stages;
    R.stage_bytes = P.stage_bytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)P.stages * P.stage_bytes);
    R.wfull = bars;
    R.afull = bars + kMaxStages;
    R.wempty = bars + 2 * kMaxStages;
    R.aempty = bars + 3 * kMaxStages;
    R.accfull = bars + 4 * kMaxStages;
    R.accempty = bars + 4 * kMaxStages + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4 * kMaxStages + 4);
    volatile int *sh_abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *sh_last = reinterpret_cast<volatile int *>(tmem_slot + 2);
    VecSmem *vs = reinterpret_cast<VecSmem *>(bars + 4 * kMaxStages + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < P.stages; ++s) {
            mbar_init(&R.wfull[s], 1);
            mbar_init(&R.afull[s], 1);
            mbar_init(&R.wempty[s], 1);
            mbar_init(&R.aempty[s], 1 + 128);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&R.accfull[b], 1);
            mbar_init(&R.accempty[b], 128);
        }
        *sh_abort = 0;
        *sh_last = 0;
        mbar_fence_init();
        if (blockIdx.x == 0) P.ctr[C_CLAIM0 + ((P.epoch + 1u) & 1u)] = 0u;  // next step's unit counter
    }
    if (warp == 0 && lane == 0) {
        for (int m = 0; m < 4; ++m) prefetch_tmap(&P.tm_w[m]);
        prefetch_tmap(&P.tm_xq);
        prefetch_tmap(&P.tm_oq);
    }
    if (warp == 2) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Ctl c{P, sh_abort};
    const TileEntry *my = P.tiles + P.cta_off[blockIdx.x];
    const int n = (int)(P.cta_off[blockIdx.x + 1] - P.cta_off[blockIdx.x]);

    if (warp == 0) {
        if (lane == 0) weight_producer<BP>(P, R, my, n, c);
    } else if (warp == 1) {
        if (lane == 0) act_producer<BP>(P, R, my, n, c);
    } else if (warp == 2) {
        if (lane == 0) mma_issuer<BP>(P, R, my, n, tmem, c);
    } else if (warp >= 4 && warp < 8) {
        epilogue_role<BP>(P, R, my, n, tmem, sh_last, c);
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

size_t stage_bytes_for(int BP) { return align_up((size_t)kTileBytes + 4 * BP * 128 + 256, 1024); }

size_t ctr_words(const Dims &d)
{
    return C_FIXED + (size_t)d.nh + d.Dv() / 128 + 2 * (d.Dk() / 128) + d.Dv() / 128 + d.H / 128 + 16;
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

// Tile order and segments.  Heads are taken in groups of eight; group g contributes the
// q, k and v row blocks of its heads (all K blocks), split into contiguous equal runs over
// the CTAs; then the W_o tiles whose K blocks belong to group g, split the same way.  A
// segment is a CTA's run inside one row block; its partial-sum slot is numbered row block
// by row block so the segments of a row block are adjacent.
void fused_build_schedule(const Dims &d, int P, std::vector<TileEntry> *tiles, std::vector<uint32_t> *off,
                          size_t *nseg_total)
{
    const int nKBx = d.H / 128, nKBo = d.Dv() / 128, nRBq = d.Dk() / 128, nRBv = d.Dv() / 128, nRBo = d.H / 128;
    const int hpu = std::max(128 / d.dk, 128 / d.dv);
    const int hpg = std::max(hpu, kHeadsPerGroup / hpu * hpu);
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
    for (int g = 0; g < G; ++g) {
        const int h0 = g * hpg, h1 = std::min(d.nh, h0 + hpg);
        std::vector<T> list;
        for (int m = 0; m < 3; ++m) {
            const int hd = m == 2 ? d.dv : d.dk;
            for (int rb = h0 * hd / 128; rb < h1 * hd / 128; ++rb)
                for (int kb = 0; kb < nKBx; ++kb) list.push_back(T{(uint8_t)m, (uint16_t)rb, (uint16_t)kb});
        }
        split(list);
    }
    for (int g = 0; g < G; ++g) {
        const int h0 = g * hpg, h1 = std::min(d.nh, h0 + hpg);
        std::vector<T> list;
        for (int rb = 0; rb < nRBo; ++rb)
            for (int kb = h0 * d.dv / 128; kb < h1 * d.dv / 128; ++kb) list.push_back(T{3, (uint16_t)rb, (uint16_t)kb});
        split(list);
    }
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
    (void)nRBo;
    (void)nKBo;
}

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
    fused_build_schedule(dmax, num_ctas_for(num_sms), &t, &o, &nseg);
    size_t n = 0;
    n += align_up((size_t)2 * bpm * dmax.H, 1024);                       // x planes
    n += align_up((size_t)(dmax.H / 128) * bpm * 4, 256);                // x scales
    n += align_up((size_t)4 * bpm * dmax.Dv(), 1024);                     // o planes
    n += align_up((size_t)(dmax.Dv() / 128) * bpm * 4, 256);             // o scales
    n += align_up(nseg * bpm * 128 * 4, 256);                             // partial sums
    n += align_up(ctr_words(dmax) * 4, 256);                              // counters
    n += align_up(t.size() * sizeof(TileEntry), 256);                     // tile lists
    n += align_up(o.size() * 4, 256);
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
    fused_build_schedule(dmax, fs->num_ctas, &fs->h_tiles, &fs->h_off, &fs->nseg_total);
    fs->ntiles = fs->h_tiles.size();
    char *p = reinterpret_cast<char *>(align_up(reinterpret_cast<uintptr_t>(base), 1024));
    auto take = [&](size_t n, size_t a) { char *r = p; p += align_up(n, a); return r; };
    fs->xq = (uint8_t *)take((size_t)2 * bpm * dmax.H, 1024);
    fs->xscale = (float *)take((size_t)(dmax.H / 128) * bpm * 4, 256);
    fs->oq = (uint8_t *)take((size_t)4 * bpm * dmax.Dv(), 1024);
    fs->oscale = (float *)take((size_t)(dmax.Dv() / 128) * bpm * 4, 256);
    fs->part = (float *)take(fs->nseg_total * bpm * 128 * 4, 256);
    fs->ctr_bytes = ctr_words(dmax) * 4;
    fs->ctr = (uint32_t *)take(fs->ctr_bytes, 256);
    fs->tiles = (TileEntry *)take(fs->h_tiles.size() * sizeof(TileEntry), 256);
    fs->cta_off = (uint32_t *)take(fs->h_off.size() * 4, 256);
    fs->off_head = C_FIXED;
    fs->off_oready = fs->off_head + dmax.nh;
    fs->off_rb = fs->off_oready + dmax.Dv() / 128;
    fs->off_out = fs->off_rb + 2 * (dmax.Dk() / 128) + dmax.Dv() / 128;
}

cudaError_t fused_init(const Dims &, FusedState *fs)
{
    if (!fs->bytes) return cudaSuccess;
    if (const char *e = getenv("KDA_WAIT_LIMIT_MS")) {
        const double ms = atof(e);
        if (ms > 0) fs->timeout_ns = (uint64_t)(ms * 1e6);
    }
    if (const char *e = getenv("KDA_DEBUG_SKIP_GATE_RELEASE")) fs->debug_skip_gate_release = atoi(e) != 0;
    cudaError_t err = cudaMemcpy(fs->tiles, fs->h_tiles.data(), fs->h_tiles.size() * sizeof(TileEntry),
                                 cudaMemcpyHostToDevice);
    if (err == cudaSuccess)
        err = cudaMemcpy(fs->cta_off, fs->h_off.data(), fs->h_off.size() * 4, cudaMemcpyHostToDevice);
    fs->uploaded = err == cudaSuccess;
    return err;
}

void fused_destroy(FusedState *) {}

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
    if (!encode_u8_map(&P.tm_xq, fs.xq, 2 * BP, d.H, 2 * BP)) return cudaErrorInvalidValue;
    if (!encode_u8_map(&P.tm_oq, fs.oq, 4 * BP, d.Dv(), 4 * BP)) return cudaErrorInvalidValue;
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
    P.xscale = fs.xscale;
    P.oscale = fs.oscale;
    P.part = fs.part;
    P.q = s.q;
    P.k = s.k;
    P.v = s.v;
    P.bpre = s.bpre;
    P.t = s.t;
    P.ctr = fs.ctr;
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
    P.off_head = fs.off_head;
    P.off_oready = fs.off_oready;
    P.off_rb = fs.off_rb;
    P.off_out = fs.off_out;
    const uint32_t epoch = fs.epoch + 1;
    P.epoch = epoch;
    P.t_xq = (fs.cum_b + (uint32_t)d.B) * (uint32_t)P.nKBx;
    P.t_gate = epoch * (uint32_t)(d.nh + d.r);
    P.t_head = epoch * 3u;
    P.t_o = fs.cum_b + (uint32_t)d.B;
    P.timeout_ns = fs.timeout_ns;
    P.out_bf16 = out_dtype == KDA_OUT_BF16;
    P.skip_gate_release = fs.debug_skip_gate_release;
    const size_t sb = stage_bytes_for(BP);
    const size_t fixed = 1024 /*align slack*/ + (4 * kMaxStages + 8) * 8 + sizeof(VecSmem) + 64;
    const size_t budget = 227 * 1024;
    int stages = (int)std::min<size_t>(kMaxStages, (budget - fixed) / sb);
    if (stages < 2) return cudaErrorNotSupported;
    P.stages = stages;
    P.stage_bytes = (int)sb;
    const size_t smem = (size_t)stages * sb + fixed;

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
