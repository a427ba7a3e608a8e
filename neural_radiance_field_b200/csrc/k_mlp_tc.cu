// bf16 tensor-core (tcgen05/TMEM) evaluation of the NeRF scene MLP.
#include "nerf_ctx.h"

namespace nerfb {

cudaError_t tc_alloc(nerf_ctx* ctx) { ctx->tc_enabled = false; return cudaSuccess; }
void tc_free(nerf_ctx* ctx) { (void)ctx; }
cudaError_t tc_pack(nerf_ctx*, const void*, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t tc_run(nerf_ctx*, const float*, const float*, int64_t, const SampleSpec&, float*,
                   cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace nerfb
