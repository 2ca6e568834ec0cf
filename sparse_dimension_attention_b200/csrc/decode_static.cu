// aqua_decode_attn_static: the decode step without a caller-provided workspace.
//
// Some callers cannot hand the library a scratch buffer: their device memory
// is owned by another allocator (a framework's pool or a fixed memory budget
// they may not bypass with cudaMalloc), or their calling convention has no
// place for an extra buffer.  This entry point runs the same kernels as
// aqua_decode_attn, with the scratch placed in a fixed-size array that is part
// of the library's own device image.
//
// Properties:
//   * The array holds kStaticScratchBytes (8 MiB).  Every GPU that loads the
//     library keeps this array for as long as the library stays loaded.
//   * The first call on a device looks up the array's device address for that
//     device (cudaGetSymbolAddress, with that device current); make that first
//     call before any stream capture.
//   * All calls share the array and it keeps the previous call's contents.  The
//     kernels re-initialise the state they rely on (the per-unit merge tickets)
//     at the start of every call, so nothing has to be cleared by the caller.
//     Calls that overlap on the GPU (for example on two streams) race on the
//     array and must be ordered by the caller.
//   * A shape whose scratch would exceed the array is rejected with
//     AQUA_ERR_WORKSPACE before anything is launched.  No device memory is
//     allocated or freed.
#include <cmath>
#include <mutex>

#include "aqua_internal.cuh"

namespace aqua {

namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_static_scratch on the current device (looked up once per device).
int static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(AQUA_ERR_CUDA, "aqua_decode_attn_static: cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return set_error(AQUA_ERR_UNSUPPORTED, "aqua_decode_attn_static: device %d", dev);
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_static_scratch);
    if (e != cudaSuccess || ptr == nullptr)
      return set_error(AQUA_ERR_CUDA, "aqua_decode_attn_static: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return AQUA_OK;
}

}  // namespace
}  // namespace aqua

extern "C" int aqua_decode_attn_static(aqua_cache* cache, const void* q, const void* k_new, const void* v_new,
                                       const float* P, int Hq, int k, float scale, void* out, int out_dtype,
                                       int32_t* sel_out, float* qproj_out, float* scores_out, float* lse_out,
                                       aqua_stream_t stream) {
  using aqua::set_error;
  aqua::clear_error();
  // Every argument check of aqua_decode_attn, in the same order and with the
  // same status codes; then the scratch this shape needs against the array.
  aqua::DecodeArgs a;
  a.q = q; a.k_new = k_new; a.v_new = v_new; a.P = P; a.Hq = Hq; a.k = k; a.scale = scale;
  a.out = out; a.out_dtype = out_dtype; a.sel_out = sel_out; a.qproj_out = qproj_out;
  a.scores_out = scores_out; a.lse_out = lse_out; a.appended = k_new != nullptr;
  int rc = aqua::check_decode_args(cache, a, "aqua_decode_attn_static");
  if (rc != AQUA_OK) return rc;
  const size_t need = aqua::decode_workspace_bytes(cache->B * cache->Hkv, Hq / cache->Hkv, cache->dv_store > 0);
  if (need > aqua::kStaticScratchBytes)
    return set_error(AQUA_ERR_WORKSPACE,
                     "aqua_decode_attn_static: this shape needs %zu bytes of scratch; the built-in array holds %zu "
                     "(use aqua_decode_attn with a workspace)",
                     need, aqua::kStaticScratchBytes);
  rc = aqua::static_scratch(&a.ws);
  if (rc != AQUA_OK) return rc;
  if (!(a.scale > 0.f)) a.scale = 1.0f / std::sqrt((float)cache->d);
  rc = aqua::launch_decode(cache, a, aqua::kPhaseSelect | aqua::kPhaseAttend, reinterpret_cast<cudaStream_t>(stream));
  if (rc == AQUA_OK && k_new != nullptr) cache->max_len += 1;
  return rc;
}
