// chunk.cu -- the chunked (parallel-in-time) form of the gated delta rule, for prefill.
//
// One CTA per (head, sequence) carries the head's state S (dk x dv, fp32) in shared memory
// through the sequence's tokens, C at a time.  Inside a chunk that starts from S0, with
// gamma(t, i) = prod_{i < j <= t} alpha_j the decay from token i to token t (a diagonal over
// key channels) and g_t = gamma(t, start), unrolling the recurrence over the chunk gives
//
//   u_t = beta_t (v_t - S0^T (g_t k^_t) - sum_{i < t} u_i k^_i^T gamma(t, i) k^_t)
//   o_t = S0^T (g_t q_t) + sum_{i <= t} u_i k^_i^T gamma(t, i) q_t
//   S'  = g_C S0 + sum_i (gamma(C, i) k^_i) u_i^T
//
// so the C values u_t solve one unit lower-triangular system (I + A) U = diag(beta)(V - G K S0)
// with A[t, i] = beta_t k^_i^T gamma(t, i) k^_t, and the readouts and the state are dense
// products.  The decays are taken in log space, L_t = sum_{j <= t} log alpha_j from the chunk
// start, and every factor used is exp of a difference that is <= 0 (no overflow, whatever the
// decay); log alpha = -softplus(z) is clamped at -30, below which a channel's memory is gone to
// fp32 precision anyway.  Everything is fp32 on CUDA cores: the chunk products are fp32
// products, which the tensor cores would only reach through several TF32 passes.
//
// Phases per chunk (256 threads):
//   A  load k, q, log alpha, v, beta of the chunk's tokens; normalise k; prefix-sum log alpha
//   B  A[t, i] and Q[t, i] = k^_i^T gamma(t, i) q_t for i <= t (a warp per pair, lanes over
//      channels); then, in place, k^ -> g k^, q -> g q and log alpha -> gamma(C, t) k^_t
//   C  rhs U = beta (V - (G K^) S0) and P = (G Q) S0 (4 x 4 register tiles per thread)
//   D  forward substitution of (I + A) U = rhs, a thread per value column
//   E  o_t = P_t + sum_{i <= t} Q[t, i] u_i (stored), S = g_C S + W^T U (in place)
#include <math.h>

#include "common.cuh"

namespace kda {
namespace {

constexpr int kChunkThreads = 256;
constexpr float kLogAlphaFloor = -30.f;

// Shared-memory layout of one CTA (floats): S [DK][DV], then per chunk KH, QS, LG [C][DK],
// U [C][DV], AKK, AKQ [C][C], beta [C], gC [DK].
template <int DK, int DV, int C>
struct ChunkSmem {
    static constexpr int S = 0;
    static constexpr int KH = S + DK * DV;
    static constexpr int QS = KH + C * DK;
    static constexpr int LG = QS + C * DK;
    static constexpr int U = LG + C * DK;
    static constexpr int AKK = U + C * DV;
    static constexpr int AKQ = AKK + C * C;
    static constexpr int BETA = AKQ + C * C;
    static constexpr int GC = BETA + C;
    static constexpr int TOTAL = GC + DK;
    static constexpr size_t bytes = (size_t)TOTAL * 4;
};

__device__ __forceinline__ float log_alpha(float z)
{
    // log alpha = -softplus(z) = -(max(z, 0) + log1p(e^-|z|))
    const float lz = -(fmaxf(z, 0.f) + log1pf(expf(-fabsf(z))));
    return fmaxf(lz, kLogAlphaFloor);
}

// Phase A: the chunk's tokens [c0, c0 + n) of sequence b, head h; tokens past n are padding
// (k = q = v = 0, beta = 0, alpha = 1), which changes neither the outputs nor the state.
template <int DK, int DV, int C>
__device__ void chunk_load(float *sm, const float *q, const float *k, const float *v, const float *bpre,
                           const float *z, int nh, size_t row0, int n, int h)
{
    using L = ChunkSmem<DK, DV, C>;
    float *KH = sm + L::KH, *QS = sm + L::QS, *LG = sm + L::LG, *U = sm + L::U, *BT = sm + L::BETA;
    const int tid = threadIdx.x;
    for (int e = tid; e < C * (DK / 4); e += kChunkThreads) {
        const int t = e / (DK / 4), c4 = e % (DK / 4);
        float4 kk = make_float4(0.f, 0.f, 0.f, 0.f), qq = kk, lg = kk;
        if (t < n) {
            const size_t off = (row0 + t) * (size_t)nh * DK + (size_t)h * DK + 4 * c4;
            kk = __ldg(reinterpret_cast<const float4 *>(k + off));
            qq = __ldg(reinterpret_cast<const float4 *>(q + off));
            const float4 zz = __ldg(reinterpret_cast<const float4 *>(z + off));
            lg = make_float4(log_alpha(zz.x), log_alpha(zz.y), log_alpha(zz.z), log_alpha(zz.w));
        }
        *reinterpret_cast<float4 *>(KH + t * DK + 4 * c4) = kk;
        *reinterpret_cast<float4 *>(QS + t * DK + 4 * c4) = qq;
        *reinterpret_cast<float4 *>(LG + t * DK + 4 * c4) = lg;
    }
    for (int e = tid; e < C * (DV / 4); e += kChunkThreads) {
        const int t = e / (DV / 4), c4 = e % (DV / 4);
        float4 vv = make_float4(0.f, 0.f, 0.f, 0.f);
        if (t < n)
            vv = __ldg(reinterpret_cast<const float4 *>(v + (row0 + t) * (size_t)nh * DV + (size_t)h * DV + 4 * c4));
        *reinterpret_cast<float4 *>(U + t * DV + 4 * c4) = vv;
    }
    for (int t = tid; t < C; t += kChunkThreads)
        BT[t] = t < n ? 1.f / (1.f + expf(-__ldg(bpre + (row0 + t) * (size_t)nh + h))) : 0.f;
    __syncthreads();
    // k -> k^ (a warp per token; a zero key stays zero)
    const int warp = tid >> 5, lane = tid & 31;
    for (int t = warp; t < C; t += kChunkThreads / 32) {
        float ss = 0.f;
        for (int d = lane; d < DK; d += 32) ss = fmaf(KH[t * DK + d], KH[t * DK + d], ss);
        ss = warp_sum(ss);
        const float inv = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
        for (int d = lane; d < DK; d += 32) KH[t * DK + d] *= inv;
    }
    // log alpha -> prefix sums from the chunk start (a thread per channel)
    for (int d = tid; d < DK; d += kChunkThreads) {
        float acc = 0.f;
        for (int t = 0; t < C; ++t) {
            acc += LG[t * DK + d];
            LG[t * DK + d] = acc;
        }
    }
    __syncthreads();
}

// Phase B: A[t, i] = beta_t k^_i^T gamma(t, i) k^_t for i < t, Q[t, i] = k^_i^T gamma(t, i) q_t
// for i <= t (a warp per pair, lanes over key channels); then, in place, k^_t -> g_t k^_t,
// q_t -> g_t q_t, L_t -> gamma(C, t) k^_t (the weights of the chunk's state update), and
// gC = g of the chunk's last token.
template <int DK, int DV, int C>
__device__ void chunk_pairs(float *sm)
{
    using L = ChunkSmem<DK, DV, C>;
    float *KH = sm + L::KH, *QS = sm + L::QS, *LG = sm + L::LG, *AKK = sm + L::AKK, *AKQ = sm + L::AKQ;
    const float *BT = sm + L::BETA;
    float *GC = sm + L::GC;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int NP = C * (C + 1) / 2;
    for (int p = warp; p < NP; p += kChunkThreads / 32) {
        // pair p -> (t, i), i <= t, enumerated row by row
        int t = (int)((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
        while ((t + 1) * (t + 2) / 2 <= p) ++t;
        while (t * (t + 1) / 2 > p) --t;
        const int i = p - t * (t + 1) / 2;
        float kk = 0.f, kq = 0.f;
#pragma unroll
        for (int d0 = 0; d0 < DK; d0 += 32) {
            const int d = d0 + lane;
            const float e = expf(LG[t * DK + d] - LG[i * DK + d]);  // gamma(t, i) <= 1
            const float ki = KH[i * DK + d] * e;
            kk = fmaf(ki, KH[t * DK + d], kk);
            kq = fmaf(ki, QS[t * DK + d], kq);
        }
        kk = warp_sum(kk);
        kq = warp_sum(kq);
        if (lane == 0) {
            AKK[t * C + i] = i < t ? BT[t] * kk : 0.f;
            AKQ[t * C + i] = kq;
        }
    }
    for (int d = tid; d < DK; d += kChunkThreads) GC[d] = LG[(C - 1) * DK + d];  // L of the last token
    __syncthreads();
    for (int e = tid; e < C * DK; e += kChunkThreads) {
        const int d = e % DK;
        const float kh = KH[e], qs = QS[e], l = LG[e];
        const float g = expf(l);
        KH[e] = kh * g;
        QS[e] = qs * g;
        LG[e] = kh * expf(GC[d] - l);  // gamma(C, t) <= 1
    }
    __syncthreads();
    for (int d = tid; d < DK; d += kChunkThreads) GC[d] = expf(GC[d]);
}

// Register tiles of the [C x DV] products: a thread owns R token rows x 4 value columns.
template <int DV, int C>
struct Tile {
    static constexpr int JB = DV / 4;                // column blocks
    static constexpr int TB = kChunkThreads / JB;    // row blocks
    static constexpr int R = C / TB;                 // rows per thread
    static_assert(R >= 1 && C % TB == 0, "chunk too small for the tiling");
};

__device__ __forceinline__ void fma4(float4 &a, float s, const float4 &b)
{
    a.x = fmaf(s, b.x, a.x);
    a.y = fmaf(s, b.y, a.y);
    a.z = fmaf(s, b.z, a.z);
    a.w = fmaf(s, b.w, a.w);
}

template <int DK, int DV, int C>
__global__ void __launch_bounds__(kChunkThreads, 1)
    k_chunk(const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v,
            const float *__restrict__ bpre, const float *__restrict__ z, float *__restrict__ state,
            float *__restrict__ o, int nh, int T)
{
    extern __shared__ __align__(16) float sm[];
    using L = ChunkSmem<DK, DV, C>;
    using TL = Tile<DV, C>;
    float *S = sm + L::S, *KH = sm + L::KH, *QS = sm + L::QS, *LG = sm + L::LG, *U = sm + L::U;
    const float *AKK = sm + L::AKK, *AKQ = sm + L::AKQ, *BT = sm + L::BETA, *GC = sm + L::GC;
    const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    float *Sg = state + ((size_t)b * nh + h) * DK * DV;
    for (int e = tid; e < DK * DV / 4; e += kChunkThreads)
        reinterpret_cast<float4 *>(S)[e] = reinterpret_cast<const float4 *>(Sg)[e];
    const int j0 = 4 * (tid % TL::JB), t0 = (tid / TL::JB) * TL::R;
    for (int c0 = 0; c0 < T; c0 += C) {
        const int n = T - c0 < C ? T - c0 : C;
        const size_t row0 = (size_t)b * T + c0;
        __syncthreads();  // the previous chunk is done with every buffer
        chunk_load<DK, DV, C>(sm, q, k, v, bpre, z, nh, row0, n, h);
        chunk_pairs<DK, DV, C>(sm);
        // C: rhs = beta (V - (G K^) S0), P = (G Q) S0
        float4 acc[TL::R], pq[TL::R];
#pragma unroll
        for (int r = 0; r < TL::R; ++r) acc[r] = pq[r] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int d = 0; d < DK; ++d) {
            const float4 s4 = *reinterpret_cast<const float4 *>(S + d * DV + j0);
#pragma unroll
            for (int r = 0; r < TL::R; ++r) {
                fma4(acc[r], KH[(t0 + r) * DK + d], s4);
                fma4(pq[r], QS[(t0 + r) * DK + d], s4);
            }
        }
#pragma unroll
        for (int r = 0; r < TL::R; ++r) {
            float4 *u = reinterpret_cast<float4 *>(U + (t0 + r) * DV + j0);
            const float be = BT[t0 + r];
            float4 x = *u;
            x.x = be * (x.x - acc[r].x);
            x.y = be * (x.y - acc[r].y);
            x.z = be * (x.z - acc[r].z);
            x.w = be * (x.w - acc[r].w);
            *u = x;
        }
        __syncthreads();
        // D: (I + A) U = rhs, A strictly lower triangular: forward substitution per column
        for (int j = tid; j < DV; j += kChunkThreads) {
            for (int t = 1; t < C; ++t) {
                float x = U[t * DV + j];
                for (int i = 0; i < t; ++i) x = fmaf(-AKK[t * C + i], U[i * DV + j], x);
                U[t * DV + j] = x;
            }
        }
        __syncthreads();
        // E: o_t = P_t + sum_{i <= t} Q[t, i] u_i
#pragma unroll
        for (int r = 0; r < TL::R; ++r) acc[r] = pq[r];
        for (int i = 0; i < t0 + TL::R; ++i) {
            const float4 u4 = *reinterpret_cast<const float4 *>(U + i * DV + j0);
#pragma unroll
            for (int r = 0; r < TL::R; ++r)
                if (i <= t0 + r) fma4(acc[r], AKQ[(t0 + r) * C + i], u4);
        }
#pragma unroll
        for (int r = 0; r < TL::R; ++r)
            if (t0 + r < n)
                *reinterpret_cast<float4 *>(o + (row0 + t0 + r) * (size_t)nh * DV + (size_t)h * DV + j0) = acc[r];
        // S = g_C S + W^T U, W = gamma(C, t) k^_t (in LG): a thread owns RD key rows x 4 columns
        constexpr int RD = DK / TL::TB;
        const int d0 = (tid / TL::JB) * RD;
        float4 sa[RD];
#pragma unroll
        for (int r = 0; r < RD; ++r) sa[r] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int t = 0; t < C; ++t) {
            const float4 u4 = *reinterpret_cast<const float4 *>(U + t * DV + j0);
#pragma unroll
            for (int r = 0; r < RD; ++r) fma4(sa[r], LG[t * DK + d0 + r], u4);
        }
#pragma unroll
        for (int r = 0; r < RD; ++r) {
            float4 *sp = reinterpret_cast<float4 *>(S + (d0 + r) * DV + j0);
            const float g = GC[d0 + r];
            float4 x = *sp;
            x.x = fmaf(g, x.x, sa[r].x);
            x.y = fmaf(g, x.y, sa[r].y);
            x.z = fmaf(g, x.z, sa[r].z);
            x.w = fmaf(g, x.w, sa[r].w);
            *sp = x;
        }
    }
    __syncthreads();
    for (int e = tid; e < DK * DV / 4; e += kChunkThreads)
        reinterpret_cast<float4 *>(Sg)[e] = reinterpret_cast<const float4 *>(S)[e];
}

template <int DK, int DV, int C>
cudaError_t launch_chunk(const Dims &d, int nseq, int T, const Scratch &s, float *state, cudaStream_t st)
{
    const size_t smem = ChunkSmem<DK, DV, C>::bytes;
    static bool configured = false;  // the attribute only grows; setting it again is harmless
    if (!configured) {
        const cudaError_t e = cudaFuncSetAttribute(k_chunk<DK, DV, C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)smem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    k_chunk<DK, DV, C><<<dim3(d.nh, nseq), kChunkThreads, smem, st>>>(s.q, s.k, s.v, s.bpre, s.z, state, s.o, d.nh,
                                                                      T);
    return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_chunk_c(const Dims &d, int nseq, int T, int chunk, const Scratch &s, float *state,
                           cudaStream_t st)
{
    switch (chunk) {
    case 16: return launch_chunk<DK, DV, 16>(d, nseq, T, s, state, st);
    case 32: return launch_chunk<DK, DV, 32>(d, nseq, T, s, state, st);
    case 64: return launch_chunk<DK, DV, 64>(d, nseq, T, s, state, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool chunk_supported(int dk, int dv, int chunk)
{
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return false;
    if (chunk != 16 && chunk != 32 && chunk != 64) return false;
    if (chunk < kChunkThreads / (dv / 4)) return false;  // at least one row per thread of the tiling
    return chunk_smem_bytes(dk, dv, chunk) <= 227 * 1024;
}

size_t chunk_smem_bytes(int dk, int dv, int C)
{
    return (size_t)(dk * dv + 3 * C * dk + C * dv + 2 * C * C + C + dk) * 4;
}

cudaError_t chunk_state(const Dims &d, int nseq, int T, int chunk, const Scratch &s, float *state, cudaStream_t st)
{
    if (!chunk_supported(d.dk, d.dv, chunk)) return cudaErrorInvalidValue;
    if (d.dk == 128 && d.dv == 128) return launch_chunk_c<128, 128>(d, nseq, T, chunk, s, state, st);
    if (d.dk == 64 && d.dv == 64) return launch_chunk_c<64, 64>(d, nseq, T, chunk, s, state, st);
    if (d.dk == 128 && d.dv == 64) return launch_chunk_c<128, 64>(d, nseq, T, chunk, s, state, st);
    return launch_chunk_c<64, 128>(d, nseq, T, chunk, s, state, st);
}

}  // namespace kda
