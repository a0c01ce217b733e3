// prefill_gemm.cuh -- the prefill's projections as bf16 tensor-core GEMMs (cuBLASLt).
#pragma once

#include "common.cuh"

namespace kda {

struct LtGemm;
cudaError_t lt_create(LtGemm **g);
void lt_destroy(LtGemm *g);

// Device bytes of the workspace the two calls below use for d.B rows.
size_t prefill_gemm_ws_bytes(const Dims &d);

// q, k, v, W_b x, t = W_a_down x and z = W_a_up t of d.B rows of x into s (fp32).
cudaError_t prefill_projections(LtGemm *g, const Dims &d, const kda_weights &w, const void *x, const Scratch &s,
                                void *ws, cudaStream_t st);
// out = W_o o for d.B rows (fp32 or bf16 out).
cudaError_t prefill_out_projection(LtGemm *g, const Dims &d, const kda_weights &w, const float *o, void *out,
                                   int out_dtype, void *ws, cudaStream_t st);

}  // namespace kda
