// Internal helpers shared by the AQUA kernels: error plumbing, PTX wrappers for
// mbarriers and bulk asynchronous copies (sm_90+ / sm_100a), bounded waits.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <utility>

#include "aqua.h"

namespace aqua {

constexpr int kHeadDim = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// Device-side wait limit before a kernel gives up and records AQUA_ERR_TIMEOUT.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// control-word indices inside aqua_cache::ctrl
enum CtrlWord { kCtrlStatus = 0, kCtrlAppendTicket = 1, kCtrlH2OTicket = 2, kCtrlStepTicket = 3 };

// ---------------------------------------------------------------- host side errors
int set_error(int code, const char* fmt, ...);
void clear_error();   // empties the thread's last-error text (at the start of each entry point)
int check_launch(const char* what);
int device_sm_count();
// Raise a kernel's dynamic shared-memory limit to `bytes` on the CURRENT device.
// cudaFuncSetAttribute acts per device, so the library records, per (kernel,
// device), the limit already set (thread-safe); later calls cost one lookup.
int set_smem_limit(const void* kernel, int bytes, const char* name);
template <typename... KArgs>
int set_smem_limit(void (*kernel)(KArgs...), int bytes, const char* name) {
  return set_smem_limit(reinterpret_cast<const void*>(kernel), bytes, name);
}

// Arguments of a decode step (aqua_decode_attn, or its two phases
// aqua_decode_select / aqua_decode_attend; see include/aqua.h).
struct DecodeArgs {
  const void* q = nullptr;
  const void* k_new = nullptr;
  const void* v_new = nullptr;
  const float* P = nullptr;
  int Hq = 0, k = 0;
  float scale = 0.f;
  void* out = nullptr;
  int out_dtype = 0;
  int32_t* sel_out = nullptr;
  float* qproj_out = nullptr;
  float* scores_out = nullptr;
  float* lse_out = nullptr;
  void* ws = nullptr;
  int appended = 0;   // the step appends its token (k_new/v_new given to the selection phase)
};
enum DecodePhase { kPhaseSelect = 1, kPhaseAttend = 2 };
// scratch of a decode step; with projected values also the pre-projection outputs
size_t decode_workspace_bytes(int n_units, int G, bool projected_values);
// Every host-side argument check of a whole decode step except the workspace
// (AQUA_OK or the status, with the message set).
int check_decode_args(const aqua_cache* c, const DecodeArgs& a, const char* who);
int launch_decode(const aqua_cache* c, const DecodeArgs& a, int phases, cudaStream_t st);
// 2-D tiled tensor map over a row-major bf16 matrix [rows][cols] (cols contiguous,
// row stride in bytes), box [box_rows][box_cols]; swizzle128 selects the 128-byte
// shared-memory swizzle.  Returns AQUA_OK or AQUA_ERR_CUDA.
int encode_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                        uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows, bool swizzle128);
// 3-D tiled tensor map over a bf16 array with dims {d0 (contiguous), d1, d2},
// byte strides of d1 and d2, and box {b0, b1, b2} (written to shared memory
// with d0 fastest, then d1, then d2).
int encode_tmap_bf16_3d(CUtensorMap* map, const void* base, const uint64_t dims[3], const uint64_t strides_bytes[2],
                        const uint32_t box[3], bool swizzle128);

// Launch with programmatic stream serialization: the kernel may begin while
// the previous kernel in the stream is still running; it must call pdl_wait()
// before reading or writing anything that kernel may touch.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- element access
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float load(const float* p) { return *p; }
  static __device__ __forceinline__ float from_f32(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ __nv_bfloat16 from_f32(float x) { return __float2bfloat16_rn(x); }
};

// bf16 pair packed in a 32-bit word -> two exact floats (low half first)
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// y = x P for one row vector x (shared memory, kHeadDim floats, 16-byte aligned)
// and P in shared memory ([kHeadDim][kHeadDim], row i = input dim i); lane
// computes outputs 4*lane .. 4*lane+3.  Every projection in the library (keys
// appended by either entry point, queries) uses this one summation order.
__device__ __forceinline__ void project_row_smem(const float* Ps, const float* xs, int lane, float (&y)[4]) {
  float a[4] = {0.f, 0.f, 0.f, 0.f}, b[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
  for (int i = 0; i < kHeadDim; i += 4) {
    const float4 x4 = *reinterpret_cast<const float4*>(xs + i);
    const float4 p0 = reinterpret_cast<const float4*>(Ps + (i + 0) * kHeadDim)[lane];
    const float4 p1 = reinterpret_cast<const float4*>(Ps + (i + 1) * kHeadDim)[lane];
    const float4 p2 = reinterpret_cast<const float4*>(Ps + (i + 2) * kHeadDim)[lane];
    const float4 p3 = reinterpret_cast<const float4*>(Ps + (i + 3) * kHeadDim)[lane];
    a[0] = fmaf(x4.x, p0.x, a[0]); a[1] = fmaf(x4.x, p0.y, a[1]); a[2] = fmaf(x4.x, p0.z, a[2]); a[3] = fmaf(x4.x, p0.w, a[3]);
    b[0] = fmaf(x4.y, p1.x, b[0]); b[1] = fmaf(x4.y, p1.y, b[1]); b[2] = fmaf(x4.y, p1.z, b[2]); b[3] = fmaf(x4.y, p1.w, b[3]);
    a[0] = fmaf(x4.z, p2.x, a[0]); a[1] = fmaf(x4.z, p2.y, a[1]); a[2] = fmaf(x4.z, p2.z, a[2]); a[3] = fmaf(x4.z, p2.w, a[3]);
    b[0] = fmaf(x4.w, p3.x, b[0]); b[1] = fmaf(x4.w, p3.y, b[1]); b[2] = fmaf(x4.w, p3.z, b[2]); b[3] = fmaf(x4.w, p3.w, b[3]);
  }
#pragma unroll
  for (int s = 0; s < 4; ++s) y[s] = a[s] + b[s];
}

// project_row_smem for NR row vectors at once (xs: NR rows of kHeadDim floats,
// consecutive): every output element is summed in exactly the same order as
// project_row_smem, so the results are bit-identical; P is read once per NR rows.
template <int NR>
__device__ __forceinline__ void project_rows_smem(const float* Ps, const float* xs, int lane, float (&y)[NR][4]) {
  float a[NR][4], b[NR][4];
#pragma unroll
  for (int t = 0; t < NR; ++t)
#pragma unroll
    for (int s = 0; s < 4; ++s) a[t][s] = b[t][s] = 0.f;
#pragma unroll 4
  for (int i = 0; i < kHeadDim; i += 4) {
    const float4 p0 = reinterpret_cast<const float4*>(Ps + (i + 0) * kHeadDim)[lane];
    const float4 p1 = reinterpret_cast<const float4*>(Ps + (i + 1) * kHeadDim)[lane];
    const float4 p2 = reinterpret_cast<const float4*>(Ps + (i + 2) * kHeadDim)[lane];
    const float4 p3 = reinterpret_cast<const float4*>(Ps + (i + 3) * kHeadDim)[lane];
#pragma unroll
    for (int t = 0; t < NR; ++t) {
      const float4 x4 = *reinterpret_cast<const float4*>(xs + t * kHeadDim + i);
      a[t][0] = fmaf(x4.x, p0.x, a[t][0]); a[t][1] = fmaf(x4.x, p0.y, a[t][1]); a[t][2] = fmaf(x4.x, p0.z, a[t][2]); a[t][3] = fmaf(x4.x, p0.w, a[t][3]);
      b[t][0] = fmaf(x4.y, p1.x, b[t][0]); b[t][1] = fmaf(x4.y, p1.y, b[t][1]); b[t][2] = fmaf(x4.y, p1.z, b[t][2]); b[t][3] = fmaf(x4.y, p1.w, b[t][3]);
      a[t][0] = fmaf(x4.z, p2.x, a[t][0]); a[t][1] = fmaf(x4.z, p2.y, a[t][1]); a[t][2] = fmaf(x4.z, p2.z, a[t][2]); a[t][3] = fmaf(x4.z, p2.w, a[t][3]);
      b[t][0] = fmaf(x4.w, p3.x, b[t][0]); b[t][1] = fmaf(x4.w, p3.y, b[t][1]); b[t][2] = fmaf(x4.w, p3.z, b[t][2]); b[t][3] = fmaf(x4.w, p3.w, b[t][3]);
    }
  }
#pragma unroll
  for (int t = 0; t < NR; ++t)
#pragma unroll
    for (int s = 0; s < 4; ++s) y[t][s] = a[t][s] + b[t][s];
}

__device__ __forceinline__ void store_out(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_out(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase of `bar` with the given parity; false if it did not
// complete within limit_ns (every kernel uses kWaitLimitNs).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// Bulk (non-tensor) asynchronous copy global -> shared, completion counted in
// bytes on `bar`.  dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// same without an L2 cache hint
__device__ __forceinline__ void bulk_g2s_plain(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// 16-byte asynchronous copy global -> shared through L2 only (LDGSTS), with an L2 policy
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint64_t policy) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "l"(policy)
               : "memory");
}

// 4-, 8- or 16-byte asynchronous copy global -> shared (both addresses aligned to the size)
template <int N>
__device__ __forceinline__ void cp_async_small(void* dst, const void* src) {
  static_assert(N == 4 || N == 8 || N == 16, "cp.async copies 4, 8 or 16 bytes");
  if constexpr (N == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(smem_u32(dst)), "l"(src), "n"(N) : "memory");
}

// arrive on `bar` once every cp.async this thread issued so far has landed
// (the arrival is one of the barrier's expected arrivals)
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// 2-D tiled TMA load (no multicast) of the box at (x = inner, y = outer) into shared memory.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                           uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// GPU-scope fetch-and-add with acquire-release semantics (returns the old value)
__device__ __forceinline__ int atom_add_acq_rel_gpu(int32_t* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// bulk prefetch of [ptr, ptr + bytes) into L2 (16-byte aligned, bytes a multiple of 16)
__device__ __forceinline__ void prefetch_l2_bulk(const void* ptr, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(ptr)), "r"(bytes)
               : "memory");
}

// order this thread's generic-proxy shared-memory accesses before later async-proxy ones
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// four 8x8 b16 matrices, transposed on load; lane i supplies the row address
// of row (i & 7) of matrix (i >> 3)
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const void* addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(addr)));
}

// 8x8 b16 matrix held one row per four lanes (lane i: row i / 4, elements
// 2 (i % 4) and 2 (i % 4) + 1) -> its transpose in the same layout
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

// D = A (16x16 bf16, row) * B (16x8 bf16, col) + D, f32 accumulators
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// two floats -> packed bf16x2 (RNE), first argument in the low half
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// bf16 high part of x and the bf16 rounding of the remainder: x ~= hi + lo to ~16 bits
__device__ __forceinline__ void split_bf16(float x, float& hi, float& lo) {
  hi = __bfloat162float(__float2bfloat16_rn(x));
  lo = x - hi;
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// named barrier among `nthreads` threads (multiple of 32); id 0 is __syncthreads
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// named barrier that also counts the participating threads whose predicate is true
__device__ __forceinline__ int named_bar_popc(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.popc.u32 %0, %2, %3, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return (int)r;
}

// named barrier that also ORs a predicate over the participating threads
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// Programmatic dependent launch: let the next kernel in the stream start its
// prologue now / wait until every prerequisite grid has completed and its
// memory is visible.  Both are no-ops for kernels launched without the
// programmatic-serialization attribute.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void record_status(int32_t* ctrl, int code) {
  if (ctrl) atomicCAS(ctrl + kCtrlStatus, 0, code);
}

}  // namespace aqua
