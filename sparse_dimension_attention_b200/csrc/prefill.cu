// Chunked causal prefill (tcgen05 path) -- entry point placeholder until the
// tensor-core kernel lands; reports AQUA_ERR_UNSUPPORTED without launching.
#include "aqua_internal.cuh"

namespace aqua {

size_t prefill_workspace_bytes(const aqua_cache* /*c*/, int /*Hq*/, int /*L*/) { return 256; }

int launch_prefill(const aqua_cache*, const void*, int, int, const float*, int, int, float, void*, int, int32_t*,
                   void*, cudaStream_t) {
  return set_error(AQUA_ERR_UNSUPPORTED, "aqua_prefill_attn: not built yet");
}

}  // namespace aqua
