// common.cuh -- internal definitions shared by the CUDA sources of the library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include <string>

#include "kda_decode.h"

namespace kda {

constexpr int kBlk = 128;  // FP8 scale block edge (128 x 128)

// Device scratch of one handle.  Every activation between stages is fp32.
struct Scratch {
    float *q = nullptr;     // [B, nh*dk]
    float *k = nullptr;     // [B, nh*dk]  (unnormalised)
    float *v = nullptr;     // [B, nh*dv]
    float *bpre = nullptr;  // [B, nh]     W_b x
    float *t = nullptr;     // [B, r]      W_a_down x
    float *z = nullptr;     // [B, nh*dk]  W_a_up t
    float *o = nullptr;     // [B, nh*dv]  readout
};

struct Dims {
    int B, H, nh, dk, dv, r;
    int Dk() const { return nh * dk; }
    int Dv() const { return nh * dv; }
};

// Launch the simple engine (five kernels) on `stream`.  Returns cudaSuccess or the launch error.
cudaError_t simple_step(const Dims &d, const kda_weights &w, const void *x, float *state, void *out,
                        int out_dtype, const Scratch &s, cudaStream_t stream);
int simple_launches();
// `tokens` consecutive tokens of each of d.B sequences (x, out: [d.B * tokens, H], row
// b*tokens + t); the state advances token by token.
cudaError_t simple_step_tokens(const Dims &d, int tokens, const kda_weights &w, const void *x, float *state,
                               void *out, int out_dtype, const Scratch &s, cudaStream_t stream);

// Stages of the simple engine, for d.B activation rows (used by the chunked prefill):
// q, k, v, W_b x, t and z into s; and out = W_o o.
cudaError_t simple_projections(const Dims &d, const kda_weights &w, const void *x, const Scratch &s, cudaStream_t st);
cudaError_t simple_out_projection(const Dims &d, const kda_weights &w, const float *o, void *out, int out_dtype,
                                  cudaStream_t st);

// Chunked form of the recurrence for nseq sequences of T tokens (activations of row b*T + t in
// s, as the projections leave them): o of every token into s.o, the state advanced by T
// tokens.  chunk: tokens per chunk (chunk_supported says which); ws: chunk_ws_bytes of device
// workspace (the per-chunk records); a wait that exceeds timeout_ns is recorded in status.
bool chunk_supported(int dk, int dv, int chunk);
size_t chunk_ws_bytes(int dk, int nh, int nseq, int T, int chunk);
cudaError_t chunk_state(const Dims &d, int nseq, int T, int chunk, const Scratch &s, float *state, void *ws,
                        int *status, uint64_t timeout_ns, cudaStream_t st);

// ---------------------------------------------------------------- device helpers
#ifdef __CUDACC__

__device__ __forceinline__ uint4 ld_stream_v4(const void *p)
{
    // weights are read once per step: no L1 allocation
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// 2 E4M3 codes (low byte = first element) -> 2 floats, via the hardware
// e4m3x2 -> f16x2 conversion (exact: every E4M3 value is an fp16 value).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t two_codes)
{
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two_codes & 0xFFFFu), __NV_E4M3);
    return __half22float2(*reinterpret_cast<__half2 *>(&h));
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

#endif

}  // namespace kda
