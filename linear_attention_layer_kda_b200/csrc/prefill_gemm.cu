// prefill_gemm.cu -- the projections of a prefill (many rows per weight read) as tensor-core
// GEMMs through cuBLASLt, in bf16 with fp32 accumulation.
//
// The projections are plain dense contractions once the operands are in one format: x is
// bf16 already; an FP8 weight with its 128 x 128 block scale, w = code * scale, is split into
// two bf16 numbers hi = bf16(w), lo = bf16(w - hi) whose sum carries w to about 2^-17 of its
// size, and an fp32 activation (o, t) is split the same way.  Each projection is then a sum
// of bf16 GEMMs (x W_hi + x W_lo; o_hi W_hi + o_hi W_lo + o_lo W_hi, the lo x lo term being
// below 2^-17 of the rest), accumulated in fp32 by the library's beta = 1 epilogue.  The
// splits are rebuilt from the caller's weights on every call (no cache that could go stale
// when the weights change in place).
#include <cublasLt.h>

#include <map>
#include <tuple>

#include "common.cuh"
#include "prefill_gemm.cuh"

namespace kda {
namespace {

__device__ __forceinline__ uint16_t bf16_rn_bits(float v)
{
    const __nv_bfloat16 b = __float2bfloat16_rn(v);
    return *reinterpret_cast<const uint16_t *>(&b);
}

// FP8 E4M3 weight [rows, cols] with fp32 block scales [rows / 128][cols / 128] -> hi, lo bf16.
__global__ void k_split_weight(const uint8_t *__restrict__ w, const float *__restrict__ sc, int rows, int cols,
                               uint16_t *__restrict__ hi, uint16_t *__restrict__ lo)
{
    const size_t n4 = (size_t)rows * cols / 4, nkb = (size_t)cols / 128;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
        const size_t e = 4 * i, r = e / cols, c = e % cols;
        const float s = __ldg(sc + (r / 128) * nkb + c / 128);
        const uint32_t codes = __ldg(reinterpret_cast<const uint32_t *>(w) + i);
        const float2 a = e4m3x2_to_float2(codes & 0xFFFFu), b = e4m3x2_to_float2(codes >> 16);
        const float v[4] = {a.x * s, a.y * s, b.x * s, b.y * s};
        uint16_t h[4], l[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            h[j] = bf16_rn_bits(v[j]);
            l[j] = bf16_rn_bits(v[j] - __uint_as_float((uint32_t)h[j] << 16));
        }
        reinterpret_cast<uint2 *>(hi)[i] = make_uint2(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16));
        reinterpret_cast<uint2 *>(lo)[i] = make_uint2(l[0] | ((uint32_t)l[1] << 16), l[2] | ((uint32_t)l[3] << 16));
    }
}

// fp32 [n] (n a multiple of 4) -> hi, lo bf16.
__global__ void k_split_f32(const float *__restrict__ x, size_t n, uint16_t *__restrict__ hi, uint16_t *__restrict__ lo)
{
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n / 4; i += (size_t)gridDim.x * blockDim.x) {
        const float4 v4 = __ldg(reinterpret_cast<const float4 *>(x) + i);
        const float v[4] = {v4.x, v4.y, v4.z, v4.w};
        uint16_t h[4], l[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            h[j] = bf16_rn_bits(v[j]);
            l[j] = bf16_rn_bits(v[j] - __uint_as_float((uint32_t)h[j] << 16));
        }
        reinterpret_cast<uint2 *>(hi)[i] = make_uint2(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16));
        reinterpret_cast<uint2 *>(lo)[i] = make_uint2(l[0] | ((uint32_t)l[1] << 16), l[2] | ((uint32_t)l[3] << 16));
    }
}

__global__ void k_f32_to_bf16(const float *__restrict__ x, size_t n, __nv_bfloat16 *__restrict__ y)
{
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        y[i] = __float2bfloat16_rn(x[i]);
}

int grid_for(size_t n) { return (int)(n < (size_t)148 * 64 ? (n + 255) / 256 : 148 * 16); }

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

cudaError_t lt_error(cublasStatus_t st) { return st == CUBLAS_STATUS_SUCCESS ? cudaSuccess : cudaErrorUnknown; }

}  // namespace

struct LtGemm {
    cublasLtHandle_t lt = nullptr;
    void *ws = nullptr;
    size_t ws_bytes = 0;
    std::map<std::tuple<int, int, int, int>, cublasLtMatmulAlgo_t> algos;  // (M, N, K, C type)
};

cudaError_t lt_create(LtGemm **out)
{
    *out = nullptr;
    LtGemm *g = new LtGemm;
    if (cublasLtCreate(&g->lt) != CUBLAS_STATUS_SUCCESS) {
        delete g;
        return cudaErrorUnknown;
    }
    g->ws_bytes = (size_t)32 << 20;
    if (cudaMalloc(&g->ws, g->ws_bytes) != cudaSuccess) {
        (void)cudaGetLastError();
        cublasLtDestroy(g->lt);
        delete g;
        return cudaErrorMemoryAllocation;
    }
    *out = g;
    return cudaSuccess;
}

void lt_destroy(LtGemm *g)
{
    if (!g) return;
    if (g->ws && cudaFree(g->ws) != cudaSuccess) (void)cudaGetLastError();
    if (g->lt) cublasLtDestroy(g->lt);
    delete g;
}

// C[M, N] (row-major, fp32) = beta C + A[M, K] B[N, K]^T (row-major bf16 operands).  In the
// library's column-major terms C^T [N x M] = B [N x K] A^T [K x M]: B is stored as a
// [K x N] column-major matrix and taken transposed, A as a [K x M] one taken as it is.
cudaError_t lt_gemm(LtGemm *g, const uint16_t *A, const uint16_t *B, float *C, int M, int N, int K, float beta,
                    cudaStream_t st)
{
    cublasLtMatmulDesc_t op = nullptr;
    cublasLtMatrixLayout_t lb = nullptr, la = nullptr, lc = nullptr;
    cublasStatus_t s = cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F);
    const cublasOperation_t tb = CUBLAS_OP_T, ta = CUBLAS_OP_N;
    if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &tb, sizeof tb);
    if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &ta, sizeof ta);
    if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatrixLayoutCreate(&lb, CUDA_R_16BF, K, N, K);  // B^T stored [K x N]
    if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatrixLayoutCreate(&la, CUDA_R_16BF, K, M, K);  // A^T stored [K x M]
    if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatrixLayoutCreate(&lc, CUDA_R_32F, N, M, N);   // C^T [N x M]
    cublasLtMatmulAlgo_t algo;
    bool have = false;
    if (s == CUBLAS_STATUS_SUCCESS) {
        const auto key = std::make_tuple(M, N, K, 0);
        auto it = g->algos.find(key);
        if (it != g->algos.end()) {
            algo = it->second;
            have = true;
        } else {
            cublasLtMatmulPreference_t pref = nullptr;
            s = cublasLtMatmulPreferenceCreate(&pref);
            if (s == CUBLAS_STATUS_SUCCESS)
                s = cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &g->ws_bytes,
                                                         sizeof g->ws_bytes);
            cublasLtMatmulHeuristicResult_t res = {};
            int nres = 0;
            if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatmulAlgoGetHeuristic(g->lt, op, lb, la, lc, lc, pref, 1, &res, &nres);
            if (pref) cublasLtMatmulPreferenceDestroy(pref);
            if (s == CUBLAS_STATUS_SUCCESS && nres > 0) {
                algo = res.algo;
                have = true;
                g->algos[key] = algo;
            } else if (s == CUBLAS_STATUS_SUCCESS) {
                s = CUBLAS_STATUS_NOT_SUPPORTED;
            }
        }
    }
    const float alpha = 1.f;
    if (s == CUBLAS_STATUS_SUCCESS && have)
        s = cublasLtMatmul(g->lt, op, &alpha, B, lb, A, la, &beta, C, lc, C, lc, &algo, g->ws, g->ws_bytes, st);
    if (lc) cublasLtMatrixLayoutDestroy(lc);
    if (la) cublasLtMatrixLayoutDestroy(la);
    if (lb) cublasLtMatrixLayoutDestroy(lb);
    if (op) cublasLtMatmulDescDestroy(op);
    return lt_error(s);
}

namespace {

// The workspace of one prefill: bf16 hi/lo splits of the four FP8 weights and of the fp32
// activations o and t, then (bf16 out only) the fp32 sum of the output projection.
struct GemmWs {
    uint16_t *qh, *ql, *kh, *kl, *vh, *vl, *wh, *wl, *oh, *ol, *th, *tl;
    float *acc;
    size_t bytes;
};

GemmWs gemm_ws(const Dims &d, void *base)
{
    const size_t H = d.H, Dk = d.Dk(), Dv = d.Dv(), M = d.B, r = d.r;
    const size_t n[12] = {Dk * H, Dk * H, Dk * H, Dk * H, Dv * H, Dv * H, H * Dv, H * Dv, M * Dv, M * Dv, M * r, M * r};
    GemmWs g;
    uint16_t **dst[12] = {&g.qh, &g.ql, &g.kh, &g.kl, &g.vh, &g.vl, &g.wh, &g.wl, &g.oh, &g.ol, &g.th, &g.tl};
    char *p = static_cast<char *>(base);
    size_t off = 0;
    for (int i = 0; i < 12; ++i) {
        *dst[i] = reinterpret_cast<uint16_t *>(p + off);
        off += align_up(n[i] * 2, 256);
    }
    g.acc = reinterpret_cast<float *>(p + off);
    off += align_up(M * H * 4, 256);
    g.bytes = off;
    return g;
}

}  // namespace

size_t prefill_gemm_ws_bytes(const Dims &d) { return gemm_ws(d, nullptr).bytes; }

cudaError_t prefill_projections(LtGemm *g, const Dims &d, const kda_weights &w, const void *x, const Scratch &s,
                                void *ws, cudaStream_t st)
{
    const int H = d.H, Dk = d.Dk(), Dv = d.Dv(), M = d.B, r = d.r;
    const GemmWs b = gemm_ws(d, ws);
    const uint16_t *xb = static_cast<const uint16_t *>(x);
    k_split_weight<<<grid_for((size_t)Dk * H / 4), 256, 0, st>>>(w.wq, w.sq, Dk, H, b.qh, b.ql);
    k_split_weight<<<grid_for((size_t)Dk * H / 4), 256, 0, st>>>(w.wk, w.sk, Dk, H, b.kh, b.kl);
    k_split_weight<<<grid_for((size_t)Dv * H / 4), 256, 0, st>>>(w.wv, w.sv, Dv, H, b.vh, b.vl);
    cudaError_t e = cudaGetLastError();
    const struct {
        const uint16_t *hi, *lo;
        float *out;
        int n;
    } jobs[3] = {{b.qh, b.ql, s.q, Dk}, {b.kh, b.kl, s.k, Dk}, {b.vh, b.vl, s.v, Dv}};
    for (const auto &j : jobs) {
        if (e == cudaSuccess) e = lt_gemm(g, xb, j.hi, j.out, M, j.n, H, 0.f, st);
        if (e == cudaSuccess) e = lt_gemm(g, xb, j.lo, j.out, M, j.n, H, 1.f, st);
    }
    // beta pre-activation and t: bf16 weights and x, exact operands
    if (e == cudaSuccess) e = lt_gemm(g, xb, w.wb, s.bpre, M, d.nh, H, 0.f, st);
    if (e == cudaSuccess) e = lt_gemm(g, xb, w.wa_down, s.t, M, r, H, 0.f, st);
    // z = W_a_up t, t split into hi + lo
    if (e == cudaSuccess) {
        k_split_f32<<<grid_for((size_t)M * r / 4), 256, 0, st>>>(s.t, (size_t)M * r, b.th, b.tl);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = lt_gemm(g, b.th, w.wa_up, s.z, M, Dk, r, 0.f, st);
    if (e == cudaSuccess) e = lt_gemm(g, b.tl, w.wa_up, s.z, M, Dk, r, 1.f, st);
    return e;
}

cudaError_t prefill_out_projection(LtGemm *g, const Dims &d, const kda_weights &w, const float *o, void *out,
                                   int out_dtype, void *ws, cudaStream_t st)
{
    const int H = d.H, Dv = d.Dv(), M = d.B;
    const GemmWs b = gemm_ws(d, ws);
    float *acc = out_dtype == KDA_OUT_BF16 ? b.acc : static_cast<float *>(out);
    k_split_weight<<<grid_for((size_t)H * Dv / 4), 256, 0, st>>>(w.wo, w.so, H, Dv, b.wh, b.wl);
    k_split_f32<<<grid_for((size_t)M * Dv / 4), 256, 0, st>>>(o, (size_t)M * Dv, b.oh, b.ol);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = lt_gemm(g, b.oh, b.wh, acc, M, H, Dv, 0.f, st);
    if (e == cudaSuccess) e = lt_gemm(g, b.oh, b.wl, acc, M, H, Dv, 1.f, st);
    if (e == cudaSuccess) e = lt_gemm(g, b.ol, b.wh, acc, M, H, Dv, 1.f, st);
    if (e == cudaSuccess && out_dtype == KDA_OUT_BF16) {
        k_f32_to_bf16<<<grid_for((size_t)M * H), 256, 0, st>>>(acc, (size_t)M * H, static_cast<__nv_bfloat16 *>(out));
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace kda
