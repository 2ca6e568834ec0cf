// extern "C" entry points: argument checks on the host (nothing is launched on
// a failed check), workspace sizing, and dispatch to the kernel launchers.
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>

#include <cudaTypedefs.h>
#include <atomic>
#include <map>
#include <mutex>
#include <utility>

#include "aqua_internal.cuh"

namespace aqua {

static thread_local char g_err[512] = "";

int set_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

void clear_error() { g_err[0] = '\0'; }

int check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(AQUA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return AQUA_OK;
}

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static std::atomic<int> cache[64];
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

int set_smem_limit(const void* kernel, int bytes, const char* name) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(AQUA_ERR_CUDA, "%s: cudaGetDevice: %s", name, cudaGetErrorString(e));
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> limit_set;   // (kernel, device) -> bytes
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(kernel, dev);
  const auto it = limit_set.find(key);
  if (it != limit_set.end() && it->second >= bytes) return AQUA_OK;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess)
    return set_error(AQUA_ERR_CUDA, "cudaFuncSetAttribute(%s, %d bytes): %s", name, bytes, cudaGetErrorString(e));
  limit_set[key] = bytes;
  return AQUA_OK;
}

namespace {
// cuTensorMapEncodeTiled from the driver, resolved once through the runtime
PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return encode;
}

int encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                     const cuuint64_t* strides_bytes, const cuuint32_t* box, bool swizzle128) {
  const PFN_cuTensorMapEncodeTiled_v12000 encode = tmap_encoder();
  if (encode == nullptr) return set_error(AQUA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims,
                            strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(AQUA_ERR_CUDA, "cuTensorMapEncodeTiled (rank %d) failed (%d)", rank, (int)r);
  return AQUA_OK;
}
}  // namespace

int encode_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                        uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows, bool swizzle128) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  return encode_tmap_bf16(map, base, 2, dims, strides, box, swizzle128);
}

int encode_tmap_bf16_3d(CUtensorMap* map, const void* base, const uint64_t dims[3], const uint64_t strides_bytes[2],
                        const uint32_t box[3], bool swizzle128) {
  const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  const cuuint64_t st[2] = {strides_bytes[0], strides_bytes[1]};
  const cuuint32_t bx[3] = {box[0], box[1], box[2]};
  return encode_tmap_bf16(map, base, 3, d, st, bx, swizzle128);
}

// launchers (defined next to their kernels)
int launch_project_keys(aqua_cache* c, const void* k_new, const void* v_new, const float* P, int L,
                        cudaStream_t st);
size_t prefill_workspace_bytes(const aqua_cache* c, int Hq, int L);
int launch_prefill(const aqua_cache* c, const void* q, int pos0, int L, const float* P, int Hq, int k,
                   float scale, void* out, int out_dtype, int32_t* sel_out, float* qproj_out, void* ws,
                   cudaStream_t st);
int launch_h2o_update(aqua_cache* c, const float* scores, const float* lse, int Hq, int budget, int recent,
                      int32_t* evicted_out, cudaStream_t st);
size_t calibrate_workspace_bytes(int n, int d);
int launch_calibrate(const float* X, int n, float* P_out, float* sigma_out, void* ws, cudaStream_t st);

}  // namespace aqua

using aqua::set_error;

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int validate_cache(const aqua_cache* c) {
  if (c == nullptr) return set_error(AQUA_ERR_ARG, "cache descriptor is NULL");
  if (c->k_proj == nullptr || c->v == nullptr || c->len == nullptr || c->ctrl == nullptr)
    return set_error(AQUA_ERR_ARG, "cache: k_proj, v, len and ctrl must be non-NULL");
  if (c->d != aqua::kHeadDim) return set_error(AQUA_ERR_UNSUPPORTED, "cache: head dim %d (only 128)", c->d);
  if (c->d_store < 1 || c->d_store > c->d)
    return set_error(AQUA_ERR_ARG, "cache: d_store %d outside [1, d]", c->d_store);
  if (c->B < 1 || c->Hkv < 1) return set_error(AQUA_ERR_ARG, "cache: B=%d Hkv=%d", c->B, c->Hkv);
  if (c->Tcap < 16 || c->Tcap % 16 != 0)
    return set_error(AQUA_ERR_ARG, "cache: Tcap %d must be a positive multiple of 16", c->Tcap);
  if (c->dtype != AQUA_F32 && c->dtype != AQUA_BF16)
    return set_error(AQUA_ERR_UNSUPPORTED, "cache: dtype %d", c->dtype);
  if (c->max_len < 0 || c->max_len > c->Tcap)
    return set_error(AQUA_ERR_ARG, "cache: max_len %d outside [0, Tcap=%d]", c->max_len, c->Tcap);
  if (!aligned(c->k_proj, 16) || !aligned(c->v, 16))
    return set_error(AQUA_ERR_ARG, "cache: k_proj and v must be 16-byte aligned");
  if (c->pos != nullptr && (c->score == nullptr || c->n_abs == nullptr))
    return set_error(AQUA_ERR_ARG, "cache: pos requires score and n_abs");
  if ((long long)c->B * c->Hkv > (1LL << 24))
    return set_error(AQUA_ERR_UNSUPPORTED, "cache: B*Hkv too large");
  if (c->dv_store < 0 || c->dv_store > c->d || c->dv_store % 16 != 0)
    return set_error(AQUA_ERR_ARG, "cache: dv_store %d must be 0 or a multiple of 16 up to d", c->dv_store);
  return AQUA_OK;
}

int check_out_dtype(int out_dtype) {
  if (out_dtype != AQUA_F32 && out_dtype != AQUA_BF16)
    return set_error(AQUA_ERR_UNSUPPORTED, "out_dtype %d", out_dtype);
  return AQUA_OK;
}

// Head grouping shared by every decode entry point.
int check_heads(const aqua_cache* c, int Hq, const char* who) {
  if (Hq < 1 || Hq % c->Hkv != 0)
    return set_error(AQUA_ERR_ARG, "%s: Hq=%d not a multiple of Hkv=%d", who, Hq, c->Hkv);
  const int G = Hq / c->Hkv;
  if (G != 1 && G != 2 && G != 4) return set_error(AQUA_ERR_UNSUPPORTED, "%s: Hq/Hkv=%d not in {1,2,4}", who, G);
  return AQUA_OK;
}

// Arguments of the selection phase (query projection, top-k, optional append).
int check_select_args(const aqua_cache* c, const aqua::DecodeArgs& a, const char* who) {
  if (a.q == nullptr || a.P == nullptr) return set_error(AQUA_ERR_ARG, "%s: NULL q or P", who);
  if (a.k < 1 || a.k > c->d_store)
    return set_error(AQUA_ERR_ARG, "%s: k=%d outside [1, d_store=%d]", who, a.k, c->d_store);
  if (!aligned(a.q, 16) || !aligned(a.P, 16)) return set_error(AQUA_ERR_ARG, "%s: q, P must be 16-byte aligned", who);
  if ((a.k_new == nullptr) != (a.v_new == nullptr))
    return set_error(AQUA_ERR_ARG, "%s: k_new and v_new must both be given or both be NULL", who);
  if (a.k_new != nullptr) {
    if ((long long)c->max_len + 1 > c->Tcap)
      return set_error(AQUA_ERR_ARG, "%s: appending to a full cache (max_len %d, Tcap %d)", who, c->max_len, c->Tcap);
    if (!aligned(a.k_new, 16) || !aligned(a.v_new, 16))
      return set_error(AQUA_ERR_ARG, "%s: k_new, v_new must be 16-byte aligned", who);
  }
  return AQUA_OK;
}

// Arguments of the attention phase (output, optional scores and lse).
int check_attend_args(const aqua::DecodeArgs& a, const char* who) {
  int rc = check_out_dtype(a.out_dtype);
  if (rc != AQUA_OK) return rc;
  if (a.out == nullptr) return set_error(AQUA_ERR_ARG, "%s: NULL out", who);
  if (!aligned(a.out, 16)) return set_error(AQUA_ERR_ARG, "%s: out must be 16-byte aligned", who);
  return AQUA_OK;
}

int check_workspace(const aqua_cache* c, int Hq, const void* ws, size_t ws_bytes, const char* who) {
  if (ws == nullptr) return set_error(AQUA_ERR_ARG, "%s: NULL workspace", who);
  if (!aligned(ws, 256)) return set_error(AQUA_ERR_ARG, "%s: workspace must be 256-byte aligned", who);
  const size_t need = aqua::decode_workspace_bytes(c->B * c->Hkv, Hq / c->Hkv, c->dv_store > 0);
  if (ws_bytes < need) return set_error(AQUA_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", who, ws_bytes, need);
  return AQUA_OK;
}

}  // namespace

namespace aqua {
// Every argument check of aqua_decode_attn except the workspace; also used by
// aqua_decode_attn_static, so both reject the same calls with the same codes.
int check_decode_args(const aqua_cache* c, const DecodeArgs& a, const char* who) {
  int rc = validate_cache(c);
  if (rc == AQUA_OK) rc = check_heads(c, a.Hq, who);
  if (rc == AQUA_OK) rc = check_attend_args(a, who);
  if (rc == AQUA_OK) rc = check_select_args(c, a, who);
  return rc;
}
}  // namespace aqua

extern "C" {

const char* aqua_last_error(void) { return aqua::g_err; }

int aqua_version(void) { return 4; }

int aqua_status(const aqua_cache* cache, int* status_out, aqua_stream_t stream) {
  if (cache == nullptr || cache->ctrl == nullptr || status_out == nullptr)
    return set_error(AQUA_ERR_ARG, "aqua_status: NULL argument");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, cache->ctrl + aqua::kCtrlStatus, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return aqua::check_launch("aqua_status copy");
  if (v != 0) {
    if (cudaMemsetAsync(cache->ctrl + aqua::kCtrlStatus, 0, sizeof(int32_t), st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return aqua::check_launch("aqua_status clear");
  }
  *status_out = v;
  return AQUA_OK;
}

size_t aqua_calibrate_workspace_size(int n, int d) {
  if (n < 1 || d != aqua::kHeadDim) return 0;
  return aqua::calibrate_workspace_bytes(n, d);
}

int aqua_calibrate(const float* X, int n, int d, float* P_out, float* sigma_out, void* workspace,
                   size_t workspace_bytes, aqua_stream_t stream) {
  aqua::g_err[0] = '\0';
  if (X == nullptr || P_out == nullptr || sigma_out == nullptr || workspace == nullptr)
    return set_error(AQUA_ERR_ARG, "aqua_calibrate: NULL pointer");
  if (d != aqua::kHeadDim) return set_error(AQUA_ERR_UNSUPPORTED, "aqua_calibrate: d=%d (only 128)", d);
  if (n < 1) return set_error(AQUA_ERR_ARG, "aqua_calibrate: n=%d", n);
  if (!aligned(X, 16) || !aligned(workspace, 256))
    return set_error(AQUA_ERR_ARG, "aqua_calibrate: X 16-byte, workspace 256-byte alignment required");
  if (workspace_bytes < aqua::calibrate_workspace_bytes(n, d))
    return set_error(AQUA_ERR_WORKSPACE, "aqua_calibrate: workspace %zu < %zu bytes", workspace_bytes,
                     aqua::calibrate_workspace_bytes(n, d));
  return aqua::launch_calibrate(X, n, P_out, sigma_out, workspace, reinterpret_cast<cudaStream_t>(stream));
}

int aqua_project_keys(aqua_cache* cache, const void* k_new, const void* v_new, const float* P, int L,
                      aqua_stream_t stream) {
  aqua::g_err[0] = '\0';
  int rc = validate_cache(cache);
  if (rc != AQUA_OK) return rc;
  if (k_new == nullptr || v_new == nullptr || P == nullptr)
    return set_error(AQUA_ERR_ARG, "aqua_project_keys: NULL input");
  if (L < 1) return set_error(AQUA_ERR_ARG, "aqua_project_keys: L=%d", L);
  if ((long long)cache->max_len + L > cache->Tcap)
    return set_error(AQUA_ERR_ARG, "aqua_project_keys: max_len %d + L %d exceeds Tcap %d", cache->max_len, L,
                     cache->Tcap);
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(P, 16))
    return set_error(AQUA_ERR_ARG, "aqua_project_keys: inputs must be 16-byte aligned");
  rc = aqua::launch_project_keys(cache, k_new, v_new, P, L, reinterpret_cast<cudaStream_t>(stream));
  if (rc == AQUA_OK) cache->max_len += L;
  return rc;
}

size_t aqua_decode_workspace_size(const aqua_cache* cache, int Hq) {
  if (validate_cache(cache) != AQUA_OK || Hq < 1 || Hq % cache->Hkv != 0) return 0;
  return aqua::decode_workspace_bytes(cache->B * cache->Hkv, Hq / cache->Hkv, cache->dv_store > 0);
}

int aqua_decode_attn(aqua_cache* cache, const void* q, const void* k_new, const void* v_new, const float* P,
                     int Hq, int k, float scale, void* out, int out_dtype, int32_t* sel_out, float* qproj_out,
                     float* scores_out, float* lse_out, void* workspace, size_t workspace_bytes,
                     aqua_stream_t stream) {
  aqua::g_err[0] = '\0';
  aqua::DecodeArgs a;
  a.q = q; a.k_new = k_new; a.v_new = v_new; a.P = P; a.Hq = Hq; a.k = k; a.scale = scale;
  a.out = out; a.out_dtype = out_dtype; a.sel_out = sel_out; a.qproj_out = qproj_out;
  a.scores_out = scores_out; a.lse_out = lse_out; a.ws = workspace; a.appended = k_new != nullptr;
  int rc = aqua::check_decode_args(cache, a, "aqua_decode_attn");
  if (rc == AQUA_OK) rc = check_workspace(cache, Hq, workspace, workspace_bytes, "aqua_decode_attn");
  if (rc != AQUA_OK) return rc;
  if (!(a.scale > 0.f)) a.scale = 1.0f / std::sqrt((float)cache->d);
  rc = aqua::launch_decode(cache, a, aqua::kPhaseSelect | aqua::kPhaseAttend, reinterpret_cast<cudaStream_t>(stream));
  if (rc == AQUA_OK && k_new != nullptr) cache->max_len += 1;
  return rc;
}

int aqua_decode_select(aqua_cache* cache, const void* q, const void* k_new, const void* v_new, const float* P,
                       int Hq, int k, float scale, int32_t* sel_out, float* qproj_out, void* workspace,
                       size_t workspace_bytes, aqua_stream_t stream) {
  aqua::g_err[0] = '\0';
  aqua::DecodeArgs a;
  a.q = q; a.k_new = k_new; a.v_new = v_new; a.P = P; a.Hq = Hq; a.k = k; a.scale = scale;
  a.sel_out = sel_out; a.qproj_out = qproj_out; a.ws = workspace; a.appended = k_new != nullptr;
  int rc = validate_cache(cache);
  if (rc == AQUA_OK) rc = check_heads(cache, Hq, "aqua_decode_select");
  if (rc == AQUA_OK) rc = check_select_args(cache, a, "aqua_decode_select");
  if (rc == AQUA_OK) rc = check_workspace(cache, Hq, workspace, workspace_bytes, "aqua_decode_select");
  if (rc != AQUA_OK) return rc;
  if (!(a.scale > 0.f)) a.scale = 1.0f / std::sqrt((float)cache->d);
  rc = aqua::launch_decode(cache, a, aqua::kPhaseSelect, reinterpret_cast<cudaStream_t>(stream));
  if (rc == AQUA_OK && k_new != nullptr) cache->max_len += 1;
  return rc;
}

int aqua_decode_attend(aqua_cache* cache, const float* P, int Hq, int appended, void* out, int out_dtype,
                       float* scores_out, float* lse_out, void* workspace, size_t workspace_bytes,
                       aqua_stream_t stream) {
  aqua::g_err[0] = '\0';
  aqua::DecodeArgs a;
  a.P = P; a.Hq = Hq; a.out = out; a.out_dtype = out_dtype; a.scores_out = scores_out; a.lse_out = lse_out;
  a.ws = workspace; a.appended = appended;
  int rc = validate_cache(cache);
  if (rc == AQUA_OK) rc = check_heads(cache, Hq, "aqua_decode_attend");
  if (rc == AQUA_OK) rc = check_attend_args(a, "aqua_decode_attend");
  if (rc == AQUA_OK && appended != 0 && appended != 1)
    rc = set_error(AQUA_ERR_ARG, "aqua_decode_attend: appended=%d (0 or 1)", appended);
  if (rc == AQUA_OK && cache->dv_store > 0 && (P == nullptr || !aligned(P, 16)))
    rc = set_error(AQUA_ERR_ARG, "aqua_decode_attend: projected values (dv_store > 0) need a 16-byte aligned P");
  if (rc == AQUA_OK && appended && cache->max_len < 1)
    rc = set_error(AQUA_ERR_ARG, "aqua_decode_attend: appended=1 with max_len 0 (no selection appended a token)");
  if (rc == AQUA_OK) rc = check_workspace(cache, Hq, workspace, workspace_bytes, "aqua_decode_attend");
  if (rc != AQUA_OK) return rc;
  return aqua::launch_decode(cache, a, aqua::kPhaseAttend, reinterpret_cast<cudaStream_t>(stream));
}

size_t aqua_prefill_workspace_size(const aqua_cache* cache, int Hq, int L) {
  if (validate_cache(cache) != AQUA_OK || Hq < 1 || Hq % cache->Hkv != 0 || L < 1) return 0;
  return aqua::prefill_workspace_bytes(cache, Hq, L);
}

int aqua_prefill_attn(const aqua_cache* cache, const void* q, int pos0, int L, const float* P, int Hq, int k,
                      float scale, void* out, int out_dtype, int32_t* sel_out, float* qproj_out, void* workspace,
                      size_t workspace_bytes, aqua_stream_t stream) {
  aqua::g_err[0] = '\0';
  int rc = validate_cache(cache);
  if (rc != AQUA_OK) return rc;
  if ((rc = check_out_dtype(out_dtype)) != AQUA_OK) return rc;
  if (q == nullptr || P == nullptr || out == nullptr || workspace == nullptr)
    return set_error(AQUA_ERR_ARG, "aqua_prefill_attn: NULL q, P, out or workspace");
  if (cache->dtype != AQUA_BF16) return set_error(AQUA_ERR_UNSUPPORTED, "aqua_prefill_attn: bf16 cache only");
  if (cache->dv_store != 0)
    return set_error(AQUA_ERR_UNSUPPORTED, "aqua_prefill_attn: projected values (dv_store > 0) are decode-only");
  if (Hq < 1 || Hq % cache->Hkv != 0)
    return set_error(AQUA_ERR_ARG, "aqua_prefill_attn: Hq=%d not a multiple of Hkv=%d", Hq, cache->Hkv);
  if (k < 1 || k > cache->d_store)
    return set_error(AQUA_ERR_ARG, "aqua_prefill_attn: k=%d outside [1, d_store=%d]", k, cache->d_store);
  if (L < 1 || pos0 < 0 || (long long)pos0 + L > cache->Tcap)
    return set_error(AQUA_ERR_ARG, "aqua_prefill_attn: pos0=%d L=%d outside Tcap=%d", pos0, L, cache->Tcap);
  if (!aligned(q, 16) || !aligned(P, 16) || !aligned(out, 16) || !aligned(workspace, 256) ||
      !aligned(qproj_out, 16))
    return set_error(AQUA_ERR_ARG, "aqua_prefill_attn: q, P, out, qproj_out 16-byte and workspace 256-byte alignment required");
  const size_t need = aqua::prefill_workspace_bytes(cache, Hq, L);
  if (workspace_bytes < need)
    return set_error(AQUA_ERR_WORKSPACE, "aqua_prefill_attn: workspace %zu < %zu bytes", workspace_bytes, need);
  if (!(scale > 0.f)) scale = 1.0f / std::sqrt((float)cache->d);
  return aqua::launch_prefill(cache, q, pos0, L, P, Hq, k, scale, out, out_dtype, sel_out, qproj_out, workspace,
                              reinterpret_cast<cudaStream_t>(stream));
}

int aqua_h2o_update(aqua_cache* cache, const float* scores, const float* lse, int Hq, int budget, int recent,
                    int32_t* evicted_out, aqua_stream_t stream) {
  aqua::g_err[0] = '\0';
  int rc = validate_cache(cache);
  if (rc != AQUA_OK) return rc;
  if (cache->pos == nullptr || cache->score == nullptr || cache->n_abs == nullptr)
    return set_error(AQUA_ERR_ARG, "aqua_h2o_update: cache needs pos, score and n_abs");
  if (scores == nullptr || lse == nullptr) return set_error(AQUA_ERR_ARG, "aqua_h2o_update: NULL scores or lse");
  if (Hq < 1 || Hq % cache->Hkv != 0)
    return set_error(AQUA_ERR_ARG, "aqua_h2o_update: Hq=%d not a multiple of Hkv=%d", Hq, cache->Hkv);
  if (budget < 1 || recent < 0 || recent > budget)
    return set_error(AQUA_ERR_ARG, "aqua_h2o_update: need budget >= 1 and 0 <= recent <= budget (%d, %d)", budget,
                     recent);
  rc = aqua::launch_h2o_update(cache, scores, lse, Hq, budget, recent, evicted_out,
                               reinterpret_cast<cudaStream_t>(stream));
  if (rc == AQUA_OK && cache->max_len > budget) cache->max_len -= 1;
  return rc;
}

}  // extern "C"
