// Key projection + append: k~ = k P, stored dimension-major (one contiguous row
// per projected dimension over the tokens), values copied token-major.
//
// AQUA abstract / edgentiq "How AQUA Works", Online Inference: keys are
// projected with the offline matrix before attention; AQUA-Memory
// ("AQUA-Memory: Dual Savings") keeps only the leading d_store projected
// dimensions in the cache.
#include "aqua_internal.cuh"

namespace aqua {

namespace {

constexpr int D = kHeadDim;
constexpr int kWarps = 8;
constexpr int kTokPerWarp = 4;
constexpr int kTokPerCta = kWarps * kTokPerWarp;   // 32

template <typename T>
__device__ __forceinline__ void load4(const T* p, float (&f)[4]);
template <>
__device__ __forceinline__ void load4(const float* p, float (&f)[4]) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}
template <>
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&f)[4]) {
  const uint2 w = *reinterpret_cast<const uint2*>(p);
  f[0] = bf16lo(w.x); f[1] = bf16hi(w.x); f[2] = bf16lo(w.y); f[3] = bf16hi(w.y);
}

// four consecutive elements as one vector (16 bytes of f32, 8 of bf16)
template <typename T> struct Vec4;
template <> struct Vec4<float> { using type = float4; };
template <> struct Vec4<__nv_bfloat16> { using type = uint2; };

// four floats rounded to T (RNE for bf16) as one vector
__device__ __forceinline__ float4 to_vec4(const float (&y)[4], float*) { return make_float4(y[0], y[1], y[2], y[3]); }
__device__ __forceinline__ uint2 to_vec4(const float (&y)[4], __nv_bfloat16*) {
  return make_uint2(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]));
}

// grid (ceil(L/32), Hkv, B), block 256: P[g] is staged in shared memory by one
// bulk copy; warp w projects tokens blockIdx.x*32 + 4w .. 4w+3 of (b, g) with
// one pass over P, the projected keys are staged as a [dim][32 token] tile and
// written out as runs of 32 consecutive slots per dimension row (the cache is
// dimension-major), values are copied token-major.
//
// Launched as a programmatic dependent of the previous kernel: everything up to
// the projection reads only P and the new keys and values, so it runs while the
// previous kernel (an attention kernel of the previous chunk or step, which
// never writes them) finishes; the lengths are read, and the cache written,
// after the wait.  The slots written lie at or past the lengths, which no
// earlier kernel of the stream still reads.
template <typename T>
__global__ void __launch_bounds__(256) project_keys_kernel(const T* __restrict__ k_new,
                                                           const T* __restrict__ v_new,
                                                           const float* __restrict__ P,
                                                           T* __restrict__ kproj, T* __restrict__ vcache,
                                                           int32_t* len, int32_t* n_abs, int32_t* pos,
                                                           float* score, int32_t* ctrl, int B, int L,
                                                           int Hkv, int d_store, int Tcap, int dv) {
  using V4 = typename Vec4<T>::type;
  extern __shared__ __align__(128) float Ps[];              // [D][D], then (dv > 0) the value rows
  __shared__ __align__(16) float xs[kWarps][kTokPerWarp][D];  // the warp's key rows
  // the warp's value rows, projected too when dv > 0: [kWarps][kTokPerWarp][D] after P
  float (*xv)[kTokPerWarp][D] = reinterpret_cast<float (*)[kTokPerWarp][D]>(Ps + D * D);
  __shared__ T kt[D][kTokPerCta];                           // projected keys, dimension-major
  __shared__ __align__(8) uint64_t pbar;
  __shared__ int is_last;
  const int g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int l0 = blockIdx.x * kTokPerCta;
  const int ntok = min(kTokPerCta, L - l0);
  const size_t unit = (size_t)b * Hkv + g;
  if (threadIdx.x == 0) {
    mbar_init(&pbar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&pbar, D * D * 4);
    bulk_g2s_plain(Ps, P + (size_t)g * D * D, D * D * 4, &pbar);
  }
  // key rows of this warp's tokens (zeros past the chunk); value rows held in registers
  V4 vrow[kTokPerWarp];
#pragma unroll
  for (int t = 0; t < kTokPerWarp; ++t) {
    const int l = warp * kTokPerWarp + t;
    float kv[4] = {0.f, 0.f, 0.f, 0.f};
    if (l < ntok) {
      const size_t row = ((size_t)b * L + l0 + l) * Hkv + g;
      load4<T>(k_new + row * D + 4 * lane, kv);
      vrow[t] = *reinterpret_cast<const V4*>(v_new + row * D + 4 * lane);
    }
    *reinterpret_cast<float4*>(&xs[warp][t][4 * lane]) = make_float4(kv[0], kv[1], kv[2], kv[3]);
    if (dv > 0) {
      float vv[4] = {0.f, 0.f, 0.f, 0.f};
      if (l < ntok) load4<T>(reinterpret_cast<const T*>(&vrow[t]), vv);
      *reinterpret_cast<float4*>(&xv[warp][t][4 * lane]) = make_float4(vv[0], vv[1], vv[2], vv[3]);
    }
  }
  __syncwarp();
  const bool ok = mbar_wait_bounded(&pbar, 0);
  const bool bad = __syncthreads_or(!ok);
  if (bad && threadIdx.x == 0) record_status(ctrl, AQUA_ERR_TIMEOUT);
  if (!bad) {
    float y[kTokPerWarp][4];
    project_rows_smem<kTokPerWarp>(Ps, &xs[warp][0][0], lane, y);
#pragma unroll
    for (int t = 0; t < kTokPerWarp; ++t)
#pragma unroll
      for (int s = 0; s < 4; ++s) kt[4 * lane + s][warp * kTokPerWarp + t] = Elem<T>::from_f32(y[t][s]);
    if (dv > 0) {
      // projected values v~ = v P (AQUA-Memory on the values), rounded to the cache type in registers
      project_rows_smem<kTokPerWarp>(Ps, &xv[warp][0][0], lane, y);
#pragma unroll
      for (int t = 0; t < kTokPerWarp; ++t) vrow[t] = to_vec4(y[t], static_cast<T*>(nullptr));
    }
  }
  pdl_wait();
  // Lengths are read before this CTA takes its ticket below; the last CTA
  // advances them only after every CTA has taken one.
  const int base = __ldcg(len + b);
  const int abase = n_abs ? __ldcg(n_abs + b) : base;
  const bool in_range = base >= 0 && base + l0 + ntok <= Tcap;
  if (!in_range && threadIdx.x == 0) record_status(ctrl, AQUA_ERR_ARG);   // device length beyond capacity
  __syncthreads();                                          // kt complete
  if (!bad && in_range) {
#pragma unroll
    for (int t = 0; t < kTokPerWarp; ++t) {
      const int l = warp * kTokPerWarp + t;
      if (l < ntok) {
        const int slot = base + l0 + l;
        const int vcols = dv > 0 ? dv : D;                   // V row length
        if (4 * lane < vcols) *reinterpret_cast<V4*>(vcache + (unit * Tcap + slot) * vcols + 4 * lane) = vrow[t];
        if (pos != nullptr && lane == 0) {
          pos[unit * Tcap + slot] = abase + l0 + l;
          score[unit * Tcap + slot] = 0.f;
        }
      }
    }
    // dimension row jd, tokens 0..ntok-1 -> slots base+l0 .. : one warp per row, one lane per token
    T* kp = kproj + unit * d_store * (size_t)Tcap + base + l0;
    for (int jd = warp; jd < d_store; jd += kWarps)
      if (lane < ntok) kp[(size_t)jd * Tcap + lane] = kt[jd][lane];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int total = gridDim.x * gridDim.y * gridDim.z;
    is_last = (atomicAdd(ctrl + kCtrlAppendTicket, 1) == total - 1);
  }
  __syncthreads();
  if (is_last) {
    __threadfence();
    for (int bb = threadIdx.x; bb < B; bb += blockDim.x) {
      len[bb] += L;
      if (n_abs) n_abs[bb] += L;
    }
    if (threadIdx.x == 0) ctrl[kCtrlAppendTicket] = 0;
  }
}

}  // namespace

int launch_project_keys(aqua_cache* c, const void* k_new, const void* v_new, const float* P, int L,
                        cudaStream_t st) {
  dim3 grid((L + kTokPerCta - 1) / kTokPerCta, c->Hkv, c->B);
  const int smem = D * D * 4 + (c->dv_store > 0 ? kWarps * kTokPerWarp * D * 4 : 0);
  if (c->dtype == AQUA_BF16) {
    const int rc = set_smem_limit(project_keys_kernel<__nv_bfloat16>, smem, "project_keys_kernel");
    if (rc != AQUA_OK) return rc;
    const cudaError_t e = launch_pdl(
        project_keys_kernel<__nv_bfloat16>, grid, dim3(256), smem, st, static_cast<const __nv_bfloat16*>(k_new),
        static_cast<const __nv_bfloat16*>(v_new), P, static_cast<__nv_bfloat16*>(c->k_proj),
        static_cast<__nv_bfloat16*>(c->v), c->len, c->n_abs, c->pos, c->score, c->ctrl, c->B, L, c->Hkv, c->d_store,
        c->Tcap, c->dv_store);
    if (e != cudaSuccess) return set_error(AQUA_ERR_CUDA, "project_keys_kernel: %s", cudaGetErrorString(e));
  } else {
    const int rc = set_smem_limit(project_keys_kernel<float>, smem, "project_keys_kernel");
    if (rc != AQUA_OK) return rc;
    const cudaError_t e = launch_pdl(project_keys_kernel<float>, grid, dim3(256), smem, st,
                                     static_cast<const float*>(k_new), static_cast<const float*>(v_new), P,
                                     static_cast<float*>(c->k_proj), static_cast<float*>(c->v), c->len, c->n_abs,
                                     c->pos, c->score, c->ctrl, c->B, L, c->Hkv, c->d_store, c->Tcap,
                                     c->dv_store);
    if (e != cudaSuccess) return set_error(AQUA_ERR_CUDA, "project_keys_kernel: %s", cudaGetErrorString(e));
  }
  return check_launch("project_keys_kernel");
}

}  // namespace aqua
