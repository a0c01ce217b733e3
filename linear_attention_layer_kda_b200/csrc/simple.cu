// simple.cu -- the SIMPLE engine: five plain CUDA-core kernels per decode step.
//
// It is the correctness baseline of the library and the engine for shapes the
// fused kernel does not cover.  Every stage writes fp32 activations to the
// handle's scratch, so each stage can be checked on its own:
//   1. q, k, v   = FP8 block-scaled projections of x           (k_proj_fp8, one launch, 3 matrices)
//   2. W_b x, W_a_down x                                          (k_gemv_bf16, one launch, 2 matrices)
//   3. z = W_a_up t                                               (k_gemv_bf16)
//   4. gates, k normalisation, delta-rule update in place, o     (k_state)
//   5. out = W_o o                                                (k_proj_fp8)
// Projections follow the Kiln post's FP8 format ("How was Kiln measured":
// 128 x 128 block scales) with the scale applied once per 16-code chunk, which
// never straddles a block.  The state update is the rank-1 form of the gated
// delta rule: S~ = diag(alpha) S, w = S~^T k^, u = beta (v - w),
// S' = S~ + k^ u^T, o = S~^T q + u (k^ . q).
#include "common.cuh"

namespace kda {
namespace {

constexpr int kRowsPerBlock = 8;  // one warp per output row
constexpr int kBatchChunk = 8;    // batch rows per block (gridDim.y covers the rest)

template <typename T>
struct In16;  // 16 consecutive inputs -> floats

template <>
struct In16<float> {
    static __device__ __forceinline__ void load(const float *p, float f[16])
    {
        const float4 *q = reinterpret_cast<const float4 *>(p);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float4 a = __ldg(q + i);
            f[4 * i] = a.x; f[4 * i + 1] = a.y; f[4 * i + 2] = a.z; f[4 * i + 3] = a.w;
        }
    }
};

template <>
struct In16<uint16_t> {  // bf16 bits
    static __device__ __forceinline__ void load(const uint16_t *p, float f[16])
    {
        const uint4 *q = reinterpret_cast<const uint4 *>(p);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            uint4 a = __ldg(q + i);
            uint32_t r[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                f[8 * i + 2 * j] = bf16_bits_to_float(r[j] & 0xFFFFu);
                f[8 * i + 2 * j + 1] = bf16_bits_to_float(r[j] >> 16);
            }
        }
    }
};

__device__ __forceinline__ void store_out(float *p, float v) { *p = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

struct ProjJob {
    const uint8_t *W;  // [N, K] E4M3
    const float *S;    // [N/128, K/128]
    float *y;          // [B, N] (row stride ldy)
};

// y[b, n] = sum_k decode(W[n, k]) * S[n/128][k/128] * x[b, k]; blockIdx.z picks the job.
template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kRowsPerBlock * 32)
    k_proj_fp8(ProjJob j0, ProjJob j1, ProjJob j2, int N, int K, const TIn *__restrict__ xin, int batch,
               TOut *__restrict__ yout)
{
    const ProjJob jb = blockIdx.z == 0 ? j0 : (blockIdx.z == 1 ? j1 : j2);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = blockIdx.x * kRowsPerBlock + warp;
    const int b0 = blockIdx.y * kBatchChunk;
    if (n >= N) return;
    const int nb = min(kBatchChunk, batch - b0);
    float acc[kBatchChunk];
#pragma unroll
    for (int b = 0; b < kBatchChunk; ++b) acc[b] = 0.f;
    const uint8_t *wrow = jb.W + (size_t)n * K;
    const float *srow = jb.S + (size_t)(n / kBlk) * (K / kBlk);
    for (int k0 = lane * 16; k0 < K; k0 += 32 * 16) {
        const uint4 wv = ld_stream_v4(wrow + k0);
        const float s = __ldg(srow + k0 / kBlk);
        float wf[16];
        const uint32_t r[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 lo = e4m3x2_to_float2(r[i] & 0xFFFFu), hi = e4m3x2_to_float2(r[i] >> 16);
            wf[4 * i] = lo.x; wf[4 * i + 1] = lo.y; wf[4 * i + 2] = hi.x; wf[4 * i + 3] = hi.y;
        }
#pragma unroll
        for (int b = 0; b < kBatchChunk; ++b) {
            if (b < nb) {
                float xs[16];
                In16<TIn>::load(xin + (size_t)(b0 + b) * K + k0, xs);
                float p = 0.f;
#pragma unroll
                for (int e = 0; e < 16; ++e) p = fmaf(wf[e], xs[e], p);
                acc[b] = fmaf(s, p, acc[b]);
            }
        }
    }
#pragma unroll
    for (int b = 0; b < kBatchChunk; ++b) {
        const float v = warp_sum(acc[b]);
        if (lane == 0 && b < nb) {
            if (yout) store_out(yout + (size_t)(b0 + b) * N + n, v);
            else jb.y[(size_t)(b0 + b) * N + n] = v;
        }
    }
}

struct GemvJob {
    const uint16_t *W;  // bf16 [N, K]
    float *y;           // [B, N]
    int N;
};

// y[b, n] = sum_k W[n, k] x[b, k] with bf16 W; blockIdx.z picks the job.
template <typename TIn>
__global__ void __launch_bounds__(kRowsPerBlock * 32)
    k_gemv_bf16(GemvJob j0, GemvJob j1, int K, const TIn *__restrict__ xin, int batch)
{
    const GemvJob jb = blockIdx.z == 0 ? j0 : j1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = blockIdx.x * kRowsPerBlock + warp;
    const int b0 = blockIdx.y * kBatchChunk;
    if (n >= jb.N) return;
    const int nb = min(kBatchChunk, batch - b0);
    float acc[kBatchChunk];
#pragma unroll
    for (int b = 0; b < kBatchChunk; ++b) acc[b] = 0.f;
    const uint16_t *wrow = jb.W + (size_t)n * K;
    for (int k0 = lane * 16; k0 < K; k0 += 32 * 16) {
        float wf[16];
        In16<uint16_t>::load(wrow + k0, wf);
#pragma unroll
        for (int b = 0; b < kBatchChunk; ++b) {
            if (b < nb) {
                float xs[16];
                In16<TIn>::load(xin + (size_t)(b0 + b) * K + k0, xs);
                float p = 0.f;
#pragma unroll
                for (int e = 0; e < 16; ++e) p = fmaf(wf[e], xs[e], p);
                acc[b] += p;
            }
        }
    }
#pragma unroll
    for (int b = 0; b < kBatchChunk; ++b) {
        const float v = warp_sum(acc[b]);
        if (lane == 0 && b < nb) jb.y[(size_t)(b0 + b) * jb.N + n] = v;
    }
}

// One block per (head, sequence); thread j owns value column j of S_h (dk x dv, row-major).
template <int DK, int DV>
__global__ void __launch_bounds__(DV)
    k_state(const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v,
            const float *__restrict__ bpre, const float *__restrict__ z, float *__restrict__ state,
            float *__restrict__ o, int nh)
{
    __shared__ float s_q[DK], s_k[DK], s_a[DK];
    const int h = blockIdx.x, b = blockIdx.y, j = threadIdx.x;
    const size_t hk = (size_t)b * nh * DK + (size_t)h * DK;
    for (int i = j; i < DK; i += DV) {
        s_q[i] = q[hk + i];
        s_k[i] = k[hk + i];
        s_a[i] = 1.f / (1.f + expf(z[hk + i]));  // exp(-softplus(z)) = sigmoid(-z)
    }
    __syncthreads();
    float ss = 0.f;
    for (int i = 0; i < DK; ++i) ss = fmaf(s_k[i], s_k[i], ss);
    const float inv = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
    __syncthreads();
    for (int i = j; i < DK; i += DV) s_k[i] *= inv;
    __syncthreads();
    const float beta = 1.f / (1.f + expf(-bpre[(size_t)b * nh + h]));
    float *S = state + ((size_t)b * nh + h) * DK * DV;
    float w = 0.f, p = 0.f, kq = 0.f;
#pragma unroll 8
    for (int i = 0; i < DK; ++i) {
        const float st = s_a[i] * S[(size_t)i * DV + j];
        w = fmaf(s_k[i], st, w);
        p = fmaf(s_q[i], st, p);
        kq = fmaf(s_k[i], s_q[i], kq);
    }
    const float u = beta * (v[(size_t)b * nh * DV + (size_t)h * DV + j] - w);
#pragma unroll 8
    for (int i = 0; i < DK; ++i) {
        float *e = S + (size_t)i * DV + j;
        *e = fmaf(s_k[i], u, s_a[i] * *e);
    }
    o[(size_t)b * nh * DV + (size_t)h * DV + j] = fmaf(u, kq, p);
}

// Several consecutive tokens of one sequence: one block per (head, sequence) runs the
// single-token update above once per token, in token order, on the same state column.
// Row b*T + t of the activations is token t of sequence b; o row b*T + t is the readout
// after token t.  Thread j only ever touches column j of S, so the in-place updates of
// consecutive tokens need no synchronisation beyond the shared vectors' reloads.
template <int DK, int DV>
__global__ void __launch_bounds__(DV)
    k_state_tokens(const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v,
                   const float *__restrict__ bpre, const float *__restrict__ z, float *__restrict__ state,
                   float *__restrict__ o, int nh, int T)
{
    __shared__ float s_q[DK], s_k[DK], s_a[DK];
    const int h = blockIdx.x, b = blockIdx.y, j = threadIdx.x;
    float *S = state + ((size_t)b * nh + h) * DK * DV;
    for (int t = 0; t < T; ++t) {
        const size_t row = (size_t)b * T + t;
        const size_t hk = row * nh * DK + (size_t)h * DK;
        __syncthreads();  // the previous token's readers of s_q, s_k, s_a are done
        for (int i = j; i < DK; i += DV) {
            s_q[i] = q[hk + i];
            s_k[i] = k[hk + i];
            s_a[i] = 1.f / (1.f + expf(z[hk + i]));  // exp(-softplus(z)) = sigmoid(-z)
        }
        __syncthreads();
        float ss = 0.f;
        for (int i = 0; i < DK; ++i) ss = fmaf(s_k[i], s_k[i], ss);
        const float inv = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
        __syncthreads();
        for (int i = j; i < DK; i += DV) s_k[i] *= inv;
        __syncthreads();
        const float beta = 1.f / (1.f + expf(-bpre[row * nh + h]));
        float w = 0.f, p = 0.f, kq = 0.f;
#pragma unroll 8
        for (int i = 0; i < DK; ++i) {
            const float st = s_a[i] * S[(size_t)i * DV + j];
            w = fmaf(s_k[i], st, w);
            p = fmaf(s_q[i], st, p);
            kq = fmaf(s_k[i], s_q[i], kq);
        }
        const float u = beta * (v[row * nh * DV + (size_t)h * DV + j] - w);
#pragma unroll 8
        for (int i = 0; i < DK; ++i) {
            float *e = S + (size_t)i * DV + j;
            *e = fmaf(s_k[i], u, s_a[i] * *e);
        }
        o[row * nh * DV + (size_t)h * DV + j] = fmaf(u, kq, p);
    }
}

template <int DK, int DV>
void launch_state(const Dims &d, const Scratch &s, float *state, cudaStream_t st)
{
    k_state<DK, DV><<<dim3(d.nh, d.B), DV, 0, st>>>(s.q, s.k, s.v, s.bpre, s.z, state, s.o, d.nh);
}

template <int DK, int DV>
void launch_state_tokens(const Dims &d, int nseq, int T, const Scratch &s, float *state, cudaStream_t st)
{
    k_state_tokens<DK, DV><<<dim3(d.nh, nseq), DV, 0, st>>>(s.q, s.k, s.v, s.bpre, s.z, state, s.o, d.nh, T);
}

}  // namespace

// Stages 1-3 for d.B activation rows: q, k, v, W_b x, t = W_a_down x and z = W_a_up t.
cudaError_t simple_projections(const Dims &d, const kda_weights &w, const void *x, const Scratch &s, cudaStream_t st)
{
    const int H = d.H, Dk = d.Dk(), Dv = d.Dv();
    const int by = (d.B + kBatchChunk - 1) / kBatchChunk;
    const uint16_t *xb = static_cast<const uint16_t *>(x);
    // 1. q, k, v
    {
        ProjJob jq{w.wq, w.sq, s.q}, jk{w.wk, w.sk, s.k}, jv{w.wv, w.sv, s.v};
        if (Dk == Dv) {
            k_proj_fp8<uint16_t, float><<<dim3((Dk + 7) / 8, by, 3), 256, 0, st>>>(jq, jk, jv, Dk, H, xb, d.B,
                                                                                  (float *)nullptr);
        } else {
            k_proj_fp8<uint16_t, float><<<dim3((Dk + 7) / 8, by, 2), 256, 0, st>>>(jq, jk, jk, Dk, H, xb, d.B,
                                                                                  (float *)nullptr);
            k_proj_fp8<uint16_t, float><<<dim3((Dv + 7) / 8, by, 1), 256, 0, st>>>(jv, jv, jv, Dv, H, xb, d.B,
                                                                                  (float *)nullptr);
        }
    }
    // 2. beta pre-activation and t = W_a_down x
    {
        GemvJob jb{w.wb, s.bpre, d.nh}, jt{w.wa_down, s.t, d.r};
        const int n = d.nh > d.r ? d.nh : d.r;
        k_gemv_bf16<uint16_t><<<dim3((n + 7) / 8, by, 2), 256, 0, st>>>(jb, jt, H, xb, d.B);
    }
    // 3. z = W_a_up t
    {
        GemvJob jz{w.wa_up, s.z, Dk};
        k_gemv_bf16<float><<<dim3((Dk + 7) / 8, by, 1), 256, 0, st>>>(jz, jz, d.r, s.t, d.B);
    }
    return cudaGetLastError();
}

// Stage 5 for d.B rows: out = W_o o.
cudaError_t simple_out_projection(const Dims &d, const kda_weights &w, const float *o, void *out, int out_dtype,
                                  cudaStream_t st)
{
    const int H = d.H, Dv = d.Dv();
    const int by = (d.B + kBatchChunk - 1) / kBatchChunk;
    ProjJob jo{w.wo, w.so, nullptr};
    if (out_dtype == KDA_OUT_BF16)
        k_proj_fp8<float, __nv_bfloat16><<<dim3((H + 7) / 8, by, 1), 256, 0, st>>>(
            jo, jo, jo, H, Dv, o, d.B, static_cast<__nv_bfloat16 *>(out));
    else
        k_proj_fp8<float, float><<<dim3((H + 7) / 8, by, 1), 256, 0, st>>>(jo, jo, jo, H, Dv, o, d.B,
                                                                          static_cast<float *>(out));
    return cudaGetLastError();
}

namespace {

// The five stages for d.B activation rows; the state stage covers nseq sequences of T
// tokens each (d.B = nseq * T; T == 1 is the single-token step).
cudaError_t simple_run(const Dims &d, int nseq, int T, const kda_weights &w, const void *x, float *state,
                       void *out, int out_dtype, const Scratch &s, cudaStream_t st)
{
    cudaError_t e = simple_projections(d, w, x, s, st);
    if (e != cudaSuccess) return e;
    // 4. state update and readout
    if (T == 1) {
        if (d.dk == 128 && d.dv == 128) launch_state<128, 128>(d, s, state, st);
        else if (d.dk == 64 && d.dv == 64) launch_state<64, 64>(d, s, state, st);
        else if (d.dk == 128 && d.dv == 64) launch_state<128, 64>(d, s, state, st);
        else launch_state<64, 128>(d, s, state, st);
    } else {
        if (d.dk == 128 && d.dv == 128) launch_state_tokens<128, 128>(d, nseq, T, s, state, st);
        else if (d.dk == 64 && d.dv == 64) launch_state_tokens<64, 64>(d, nseq, T, s, state, st);
        else if (d.dk == 128 && d.dv == 64) launch_state_tokens<128, 64>(d, nseq, T, s, state, st);
        else launch_state_tokens<64, 128>(d, nseq, T, s, state, st);
    }
    // 5. out = W_o o
    return simple_out_projection(d, w, s.o, out, out_dtype, st);
}

}  // namespace

int simple_launches() { return 5; }

cudaError_t simple_step(const Dims &d, const kda_weights &w, const void *x, float *state, void *out,
                        int out_dtype, const Scratch &s, cudaStream_t st)
{
    return simple_run(d, d.B, 1, w, x, state, out, out_dtype, s, st);
}

cudaError_t simple_step_tokens(const Dims &d, int tokens, const kda_weights &w, const void *x, float *state,
                               void *out, int out_dtype, const Scratch &s, cudaStream_t st)
{
    Dims rows = d;
    rows.B = d.B * tokens;
    return simple_run(rows, d.B, tokens, w, x, state, out, out_dtype, s, st);
}

}  // namespace kda
