// chunk.cu -- the chunked (parallel-in-time) form of the gated delta rule, for prefill.
//
// The state S (dk x dv, fp32) of a head is carried through the sequence's tokens C at a time.
// Inside a chunk that starts from S0, with gamma(t, i) = prod_{i < j <= t} alpha_j the decay
// from token i to token t (a diagonal over key channels) and g_t = gamma(t, start), unrolling
// the recurrence over the chunk gives
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
// Everything that involves only keys, queries and gates -- the normalised keys, the decays,
// A, Q[t, i] = k^_i^T gamma(t, i) q_t and the inverse of I + A -- is independent from chunk to
// chunk, so a first kernel prepares it for every chunk at once (one CTA per sequence, head and
// chunk) into a chunk record.  Only the parts that touch the state are sequential; and the
// value columns are independent of one another (every quantity that involves v, u, o or S is
// linear in them, column by column), so the second kernel runs one CTA per sequence, head and
// slice of DVS value columns, walking the chunks in order with the next record in flight:
//
//   prepare  (a) load k, q, log alpha, beta of the chunk's tokens; normalise k; prefix-sum
//                log alpha;  (b) A[t, i] and Q[t, i] for i <= t (a warp per pair, lanes over
//                channels), then k^ -> g k^, q -> g q, log alpha -> gamma(C, t) k^_t;
//            (c) X = (I + A)^-1 by forward substitution (a thread per column), TB = X diag(beta)
//   scan     R = V - (G K^) S0, P = (G Q) S0;  U = TB R;  o = P + Q U;  S = g_C S + W^T U
#include <math.h>

#include <atomic>

#include "common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int kChunkThreads = 256;
constexpr float kLogAlphaFloor = -30.f;

// Chunk record (floats), one per (sequence, head, chunk): KH = g k^, QS = g q, LG = gamma(C, t)
// k^_t [C][DK]; TB = (I + A)^-1 diag(beta), AKQ = Q (zero above the diagonal) [C][C]; GC = g_C
// [DK].  16-byte multiple, so records are bulk-copy aligned back to back.
template <int DK, int C>
struct ChunkRec {
    static constexpr int KH = 0;
    static constexpr int QS = KH + C * DK;
    static constexpr int LG = QS + C * DK;
    static constexpr int TB = LG + C * DK;
    static constexpr int AKQ = TB + C * C;
    static constexpr int GC = AKQ + C * C;
    static constexpr int TOTAL = GC + DK;
    static_assert(TOTAL % 4 == 0, "records must stay 16-byte aligned");
};

// Preparation kernel shared memory: a record, then AKK [C][C] and beta [C].
template <int DK, int C>
struct PrepSmem {
    using R = ChunkRec<DK, C>;
    static constexpr int AKK = R::TOTAL;
    static constexpr int BETA = AKK + C * C;
    static constexpr int TOTAL = BETA + C;
    static constexpr size_t bytes = (size_t)TOTAL * 4;
};

__device__ __forceinline__ float log_alpha(float z)
{
    // log alpha = -softplus(z) = -(max(z, 0) + log1p(e^-|z|))
    const float lz = -(fmaxf(z, 0.f) + log1pf(expf(-fabsf(z))));
    return fmaxf(lz, kLogAlphaFloor);
}

// (a): the chunk's tokens [c0, c0 + n) of sequence b, head h; tokens past n are padding
// (k = q = 0, beta = 0, alpha = 1), which changes neither the outputs nor the state.
template <int DK, int C>
__device__ void prep_load(float *sm, const float *q, const float *k, const float *bpre, const float *z, int nh,
                          size_t row0, int n, int h)
{
    using L = PrepSmem<DK, C>;
    using R = ChunkRec<DK, C>;
    float *KH = sm + R::KH, *QS = sm + R::QS, *LG = sm + R::LG, *BT = sm + L::BETA;
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

// (b): A[t, i] = beta_t k^_i^T gamma(t, i) k^_t for i < t and Q[t, i] = k^_i^T gamma(t, i) q_t
// for i <= t, zero elsewhere (a warp per pair, lanes over key channels); then, in place,
// k^_t -> g_t k^_t, q_t -> g_t q_t, L_t -> gamma(C, t) k^_t (the weights of the chunk's state
// update), and GC = g of the chunk's last token.
template <int DK, int C>
__device__ void prep_pairs(float *sm)
{
    using L = PrepSmem<DK, C>;
    using R = ChunkRec<DK, C>;
    float *KH = sm + R::KH, *QS = sm + R::QS, *LG = sm + R::LG, *AKK = sm + L::AKK, *AKQ = sm + R::AKQ;
    const float *BT = sm + L::BETA;
    float *GC = sm + R::GC;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int e = tid; e < C * C; e += kChunkThreads) AKK[e] = AKQ[e] = 0.f;
    __syncthreads();
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
            if (i < t) AKK[t * C + i] = BT[t] * kk;
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

// One chunk of one head of one sequence -> its record (grid: chunks x heads x sequences).
template <int DK, int C>
__global__ void __launch_bounds__(kChunkThreads)
    k_chunk_prep(const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ bpre,
                 const float *__restrict__ z, float *__restrict__ rec, int nh, int T)
{
    extern __shared__ __align__(128) float sm[];
    using L = PrepSmem<DK, C>;
    using R = ChunkRec<DK, C>;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const int c0 = c * C, n = T - c0 < C ? T - c0 : C;
    prep_load<DK, C>(sm, q, k, bpre, z, nh, (size_t)b * T + c0, n, h);
    prep_pairs<DK, C>(sm);
    // (c): X = (I + A)^-1, A strictly lower triangular: column j by forward substitution,
    // X[t][j] = -sum_{j <= i < t} A[t][i] X[i][j]; then TB = X diag(beta)
    float *X = sm + R::TB;
    const float *AKK = sm + L::AKK, *BT = sm + L::BETA;
    for (int j = tid; j < C; j += kChunkThreads) {
        for (int t = 0; t <= j; ++t) X[t * C + j] = t == j ? 1.f : 0.f;
        for (int t = j + 1; t < C; ++t) {
            float x = 0.f;
            for (int i = j; i < t; ++i) x = fmaf(-AKK[t * C + i], X[i * C + j], x);
            X[t * C + j] = x;
        }
    }
    __syncthreads();
    for (int e = tid; e < C * C; e += kChunkThreads) X[e] *= BT[e % C];
    __syncthreads();
    const int nchunks = gridDim.x;
    float4 *dst = reinterpret_cast<float4 *>(rec + (((size_t)b * nh + h) * nchunks + c) * R::TOTAL);
    for (int e = tid; e < R::TOTAL / 4; e += kChunkThreads) dst[e] = reinterpret_cast<const float4 *>(sm)[e];
}

// The scan's shared memory (floats): S [DK][DV], NBUF record buffers, the chunk's R / U
// [C][DV], then the mbarriers.
template <int DK, int DV, int C, int NBUF>
struct ScanSmem {
    using R = ChunkRec<DK, C>;
    static constexpr int REC = (DK * DV + 31) / 32 * 32;  // S at offset 0
    static constexpr int RSTRIDE = (R::TOTAL + 31) / 32 * 32;
    static constexpr int UB = REC + NBUF * RSTRIDE;
    static constexpr int BARS = UB + C * DV;
    static constexpr size_t bytes = (size_t)BARS * 4 + 2 * 8;
};

// Thread 0 waits (bounded) for the record copy completing phase `parity` of `bar`; false
// after the limit, with the wait site in the status words.
__device__ bool wait_record(uint64_t *bar, uint32_t parity, int *status, uint64_t timeout_ns)
{
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > timeout_ns) {
            if (status) {
                volatile int *st = status;
                st[1] = 30;  // the site first, so a host that sees the code sees its site
                __threadfence_system();
                st[0] = KDA_ERR_DEVICE_TIMEOUT;
                __threadfence_system();
            }
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ void fma4(float4 &a, float s, const float4 &b)
{
    a.x = fmaf(s, b.x, a.x);
    a.y = fmaf(s, b.y, a.y);
    a.z = fmaf(s, b.z, a.z);
    a.w = fmaf(s, b.w, a.w);
}

// The sequential part for one slice of DV value columns of one head of one sequence (grid:
// heads x sequences x slices).  Thread (t0, j0) owns token row t0 of the chunk and value
// columns j0 .. j0 + 3 of R, U and o, and key rows d0 .. d0 + RD - 1 of those columns of S.
// With two record buffers the next chunk's record is copied in while this one is used.
template <int DK, int DV, int C, int NBUF>
__global__ void __launch_bounds__(kChunkThreads, 1)
    k_chunk_scan(const float *__restrict__ rec, const float *__restrict__ v, float *__restrict__ state,
                 float *__restrict__ o, int nh, int dv_all, int T, int nchunks, int *status, uint64_t timeout_ns)
{
    extern __shared__ __align__(128) float sm[];
    using R = ChunkRec<DK, C>;
    using L = ScanSmem<DK, DV, C, NBUF>;
    constexpr int JB = DV / 4, TB = kChunkThreads / JB, RD = DK / TB;
    static_assert(TB == C, "one token row per thread");
    float *S = sm, *UB = sm + L::UB;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BARS);
    __shared__ int stop;
    const int h = blockIdx.x, b = blockIdx.y, col0 = blockIdx.z * DV, tid = threadIdx.x;
    const int j0 = 4 * (tid % JB), t0 = tid / JB, d0 = t0 * RD;
    float *Sg = state + ((size_t)b * nh + h) * DK * dv_all + col0;  // row d of the slice at Sg + d * dv_all
    const float *recs = rec + ((size_t)b * nh + h) * nchunks * R::TOTAL;
    constexpr uint32_t rec_bytes = (uint32_t)R::TOTAL * 4;
    int issued = 0;  // record copies issued (thread 0)
    if (tid == 0) {
        for (int i = 0; i < NBUF; ++i) mbar_init(&bars[i], 1);
        mbar_fence_init();
        stop = 0;
        mbar_expect_tx(&bars[0], rec_bytes);
        bulk_load(sm + L::REC, recs, rec_bytes, &bars[0]);
        issued = 1;
    }
    for (int e = tid; e < DK * DV / 4; e += kChunkThreads) {
        const int d = e / (DV / 4), c4 = e % (DV / 4);
        reinterpret_cast<float4 *>(S)[e] = *reinterpret_cast<const float4 *>(Sg + (size_t)d * dv_all + 4 * c4);
    }
    for (int c = 0; c < nchunks; ++c) {
        const int buf = c % NBUF;
        const float *RC = sm + L::REC + buf * L::RSTRIDE;
        const float *KH = RC + R::KH, *QS = RC + R::QS, *LG = RC + R::LG, *TBm = RC + R::TB, *AKQ = RC + R::AKQ,
                    *GC = RC + R::GC;
        if (tid == 0) {
            // the buffer of the copy issued here was last read before the barrier that ended the
            // previous chunk
            const int cn = NBUF == 1 ? c : c + 1;
            if (cn >= issued && cn < nchunks) {
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_expect_tx(&bars[cn % NBUF], rec_bytes);
                bulk_load(sm + L::REC + (cn % NBUF) * L::RSTRIDE, recs + (size_t)cn * R::TOTAL, rec_bytes,
                          &bars[cn % NBUF]);
                issued = cn + 1;
            }
            if (!wait_record(&bars[buf], (uint32_t)(c / NBUF) & 1u, status, timeout_ns)) stop = 1;
        }
        const int n = T - c * C < C ? T - c * C : C;
        const size_t row = (size_t)b * T + (size_t)c * C + t0;
        float4 vv = make_float4(0.f, 0.f, 0.f, 0.f);
        if (t0 < n) vv = __ldg(reinterpret_cast<const float4 *>(v + row * nh * dv_all + (size_t)h * dv_all + col0 + j0));
        __syncthreads();
        if (stop) break;
        while (!mbar_try_wait(&bars[buf], (uint32_t)(c / NBUF) & 1u)) {
        }  // complete (thread 0 saw it): every thread's own wait ends at once
        // R = V - (G K^) S0 and P = (G Q) S0 for row t0
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f), pq = acc;
#pragma unroll 8
        for (int d = 0; d < DK; ++d) {
            const float4 s4 = *reinterpret_cast<const float4 *>(S + d * DV + j0);
            fma4(acc, KH[t0 * DK + d], s4);
            fma4(pq, QS[t0 * DK + d], s4);
        }
        *reinterpret_cast<float4 *>(UB + t0 * DV + j0) =
            make_float4(vv.x - acc.x, vv.y - acc.y, vv.z - acc.z, vv.w - acc.w);
        __syncthreads();
        // U = TB R (TB = (I + A)^-1 diag(beta), lower triangular)
        float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i = 0; i <= t0; ++i) fma4(u, TBm[t0 * C + i], *reinterpret_cast<const float4 *>(UB + i * DV + j0));
        __syncthreads();
        *reinterpret_cast<float4 *>(UB + t0 * DV + j0) = u;
        __syncthreads();
        // o = P + Q U (Q lower triangular with its diagonal)
        for (int i = 0; i <= t0; ++i) fma4(pq, AKQ[t0 * C + i], *reinterpret_cast<const float4 *>(UB + i * DV + j0));
        if (t0 < n) *reinterpret_cast<float4 *>(o + row * nh * dv_all + (size_t)h * dv_all + col0 + j0) = pq;
        // S = g_C S + W^T U, W = gamma(C, t) k^_t (in LG): key rows d0 .. d0 + RD - 1
        float4 sa[RD];
#pragma unroll
        for (int r = 0; r < RD; ++r) sa[r] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int t = 0; t < C; ++t) {
            const float4 u4 = *reinterpret_cast<const float4 *>(UB + t * DV + j0);
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
        __syncthreads();  // the chunk is done with S, U and its record buffer
    }
    if (stop) {
        // a copy may still be in flight: it must land before the CTA exits
        if (tid == 0)
            for (int i = issued - NBUF > 0 ? issued - NBUF : 0; i < issued; ++i)
                (void)wait_record(&bars[i % NBUF], (uint32_t)(i / NBUF) & 1u, nullptr, timeout_ns);
        __syncthreads();
        return;
    }
    for (int e = tid; e < DK * DV / 4; e += kChunkThreads) {
        const int d = e / (DV / 4), c4 = e % (DV / 4);
        *reinterpret_cast<float4 *>(Sg + (size_t)d * dv_all + 4 * c4) = reinterpret_cast<const float4 *>(S)[e];
    }
}

// Slice width: the narrowest that gives every thread of the [C x DVS] tiling one token row
// (DVS / 4 column blocks x C rows = 256 threads), so that a head spreads over the most SMs.
template <int DV, int C>
constexpr int slice_width()
{
    return (kChunkThreads * 4 / C) > DV ? DV : kChunkThreads * 4 / C;
}

template <int DK, int DV, int C>
constexpr int scan_buffers()
{
    return ScanSmem<DK, slice_width<DV, C>(), C, 2>::bytes <= 227 * 1024 ? 2 : 1;
}

template <int DK, int DV, int C>
cudaError_t launch_chunk(const Dims &d, int nseq, int T, const Scratch &s, float *state, void *ws, int *status,
                         uint64_t timeout_ns, cudaStream_t st)
{
    constexpr int DVS = slice_width<DV, C>(), NB = scan_buffers<DK, DV, C>();
    static_assert(DV % DVS == 0 && kChunkThreads / (DVS / 4) == C, "slices must tile the value columns");
    const size_t prep_smem = PrepSmem<DK, C>::bytes, scan_smem = ScanSmem<DK, DVS, C, NB>::bytes;
    // the shared-memory limit is a per-device attribute of each kernel (setting it twice is harmless)
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev < 64 ? 1ull << dev : 0ull;
    if (!bit || !(configured.load() & bit)) {
        e = cudaFuncSetAttribute(k_chunk_prep<DK, C>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep_smem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_chunk_scan<DK, DVS, C, NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)scan_smem);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit);
    }
    const int nchunks = (T + C - 1) / C;
    float *rec = static_cast<float *>(ws);
    k_chunk_prep<DK, C><<<dim3(nchunks, d.nh, nseq), kChunkThreads, prep_smem, st>>>(s.q, s.k, s.bpre, s.z, rec,
                                                                                    d.nh, T);
    k_chunk_scan<DK, DVS, C, NB><<<dim3(d.nh, nseq, DV / DVS), kChunkThreads, scan_smem, st>>>(
        rec, s.v, state, s.o, d.nh, DV, T, nchunks, status, timeout_ns);
    return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_chunk_c(const Dims &d, int nseq, int T, int chunk, const Scratch &s, float *state, void *ws,
                           int *status, uint64_t timeout_ns, cudaStream_t st)
{
    switch (chunk) {
    case 16: return launch_chunk<DK, DV, 16>(d, nseq, T, s, state, ws, status, timeout_ns, st);
    case 32: return launch_chunk<DK, DV, 32>(d, nseq, T, s, state, ws, status, timeout_ns, st);
    case 64: return launch_chunk<DK, DV, 64>(d, nseq, T, s, state, ws, status, timeout_ns, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool chunk_supported(int dk, int dv, int chunk)
{
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return false;
    return chunk == 16 || chunk == 32 || chunk == 64;
}

size_t chunk_ws_bytes(int dk, int nh, int nseq, int T, int chunk)
{
    const size_t rec = (size_t)(3 * chunk * dk + 2 * chunk * chunk + dk) * 4;
    return (size_t)nseq * nh * ((T + chunk - 1) / chunk) * rec;
}

cudaError_t chunk_state(const Dims &d, int nseq, int T, int chunk, const Scratch &s, float *state, void *ws,
                        int *status, uint64_t timeout_ns, cudaStream_t st)
{
    if (!chunk_supported(d.dk, d.dv, chunk)) return cudaErrorInvalidValue;
    if (d.dk == 128 && d.dv == 128) return launch_chunk_c<128, 128>(d, nseq, T, chunk, s, state, ws, status, timeout_ns, st);
    if (d.dk == 64 && d.dv == 64) return launch_chunk_c<64, 64>(d, nseq, T, chunk, s, state, ws, status, timeout_ns, st);
    if (d.dk == 128 && d.dv == 64) return launch_chunk_c<128, 64>(d, nseq, T, chunk, s, state, ws, status, timeout_ns, st);
    return launch_chunk_c<64, 128>(d, nseq, T, chunk, s, state, ws, status, timeout_ns, st);
}

}  // namespace kda
