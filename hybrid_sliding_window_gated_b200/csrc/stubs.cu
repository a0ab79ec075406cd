// stubs.cu -- placeholders for entry points whose kernels are not built yet.
#include "swa_internal.h"

namespace swa {
int swa_bwd_impl(const swa_params_t*, const swa_bf16_t*, const swa_bf16_t*, const swa_bf16_t*,
                 const swa_bf16_t*, const float*, const float*, const float*, const swa_bf16_t*,
                 swa_bf16_t*, swa_bf16_t*, swa_bf16_t*, swa_bf16_t*, float*, float*, void*, size_t,
                 cudaStream_t) {
  return SWA_ERR_UNSUPPORTED;
}
size_t swa_bwd_workspace_bytes(const swa_params_t*) { return 0; }
}  // namespace swa
