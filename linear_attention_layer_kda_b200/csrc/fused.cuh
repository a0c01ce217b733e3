// fused.cuh -- interface of the FUSED engine (one persistent kernel per decode step).
#pragma once

#include "common.cuh"

namespace kda {

struct FusedState {
    void *base = nullptr;  // inside the handle's scratch
    size_t bytes = 0;
};

bool fused_supports(const Dims &d, int num_sms);
size_t fused_scratch_bytes(const Dims &dmax);
void fused_bind_scratch(const Dims &dmax, void *base, size_t bytes, FusedState *fs);
cudaError_t fused_init(const Dims &dmax, FusedState *fs);
void fused_destroy(FusedState *fs);
int fused_launches();
cudaError_t fused_step(const Dims &d, const kda_weights &w, const void *x, float *state, void *out, int out_dtype,
                       FusedState &fs, int *status, int num_sms, cudaStream_t stream);

}  // namespace kda
