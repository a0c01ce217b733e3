// fused.cu -- the FUSED engine (not yet enabled: fused_supports() is false).
#include "fused.cuh"

namespace kda {

bool fused_supports(const Dims &, int) { return false; }
size_t fused_scratch_bytes(const Dims &) { return 0; }
void fused_bind_scratch(const Dims &, void *base, size_t bytes, FusedState *fs)
{
    fs->base = base;
    fs->bytes = bytes;
}
cudaError_t fused_init(const Dims &, FusedState *) { return cudaSuccess; }
void fused_destroy(FusedState *) {}
int fused_launches() { return 1; }
cudaError_t fused_step(const Dims &, const kda_weights &, const void *, float *, void *, int, FusedState &, int *, int,
                       cudaStream_t)
{
    return cudaErrorNotSupported;
}

}  // namespace kda
