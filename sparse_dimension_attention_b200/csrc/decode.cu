// AQUA decode step on sm_100a.
//
// qproj_topk_kernel -- one CTA per (sequence b, KV head g): four warps per
// query head of the group project row slices of every head and then rank the
// head's dimensions (P[g] staged in shared memory by bulk copies), plus one
// warp that appends the step's new key and value when the call carries them
// (k~ = k P rounded to the cache type, written at slot len[b]; the attention
// kernel's last CTA advances the lengths):
//   q~ = q P                                  (abstract: queries and keys projected by P)
//   S_h = k largest |q~_j|, ties to lower j  (edgentiq, Online Inference: the dimensions
//                                             where the projected query is largest in magnitude)
//   U_g = union of the group's S_h and the masked, pre-scaled query rows
//   qm[r][h] = (U_r in S_h) ? q~_h[U_r] * scale * log2(e) : 0.
//
// decode_attn_*_kernel -- persistent, one CTA per SM.  The cached tokens of all
// (b, g) units are cut into tiles of TT tokens and the flat tile sequence is
// split over the CTAs by a position model (see kTilePos).  Per tile the
// producer warps gather the |U_g| selected rows of the dimension-major K~
// cache (one union read per GQA group) and the V tile into shared memory with
// asynchronous copies, three stages deep.  Consumer warps compute the scores on the selected
// dimensions only, s_{h,t} = sum_r qm[r][h] K~[U_r][t], an online softmax, and
// o_h += p_{h,t} V_t over the unprojected values (AQUA abstract; edgentiq,
// "How AQUA Works").  A CTA that ends inside a unit writes (m, l, o) and takes
// a ticket; the unit's last CTA merges the partials (log-sum-exp).  No CTA
// ever waits for another.
//
// bf16 caches: the consumers use the tensor cores (mma.sync m16n8k16, bf16 in,
// f32 accumulate) on the transposed products S^T = K~^T qm^T and
// O^T += V^T P^T: each warp's 16 tokens of a tile are the 16 MMA rows, and
// the 8 columns are (head, part) pairs, q~ and p split into bf16 high and low
// parts, so the products keep ~16 significant bits.  Each warp keeps its own
// running max, merged at the end of a segment.  The K~ rows are gathered with
// 16-byte cp.async by four producer warps (many small bulk copies from one warp
// cannot keep HBM busy); the V tile arrives by a 128B-swizzled tensor copy.
// f32 caches: CUDA-core FMA consumers (exact f32 products).
#include <math.h>

#include <mutex>
#include <iterator>
#include <unordered_map>

#include "aqua_internal.cuh"

namespace aqua {

namespace {

constexpr int D = kHeadDim;
constexpr int NCW = 8;                 // consumer warps
constexpr int NCT = NCW * 32;          // consumer threads
constexpr int NTHREADS = NCT + 32;     // + one producer warp
constexpr int NSTAGE = 3;
constexpr int RMAX = D / NCW;          // union rows per consumer warp (f32 kernel)
constexpr int kMaxCtas = 1024;
constexpr int KROW_BF16 = 272;         // padded byte stride of a K~ row in shared memory (bf16 kernel)
constexpr float kLazyRescale = 8.0f;   // running max is raised only when exceeded by 2^8
constexpr int NPW_BF16 = 4;            // producer warps of the bf16 kernel (K~ gather by 16-byte cp.async)
constexpr int NTHREADS_BF16 = NCT + NPW_BF16 * 32;

struct DecodeParams {
  const void* q;
  const float* P;
  const int32_t* len;
  const void* kproj;
  const void* v;
  void* out;
  float* qm;          // [n_units][D][G] masked scaled q~ of the union rows, union order
  float* qmn;         // [n_units][D][G] the same in dimension order (0 for dims no head kept)
  int32_t* ulist;     // [n_units][D]
  int32_t* ucount;    // [n_units]
  int32_t* counters;  // [n_units]
  float* part_ml;     // [nseg_max][G][2]
  float* part_o;      // [nseg_max][G][D]
  int32_t* sel_out;
  float* qproj_out;
  float* scores_out;
  float* lse_out;
  int32_t* ctrl;
  // optional fused append of the step's new token (k_new == nullptr: none)
  const void* k_new;      // [B][Hkv][D] cache dtype
  const void* v_new;      // [B][Hkv][D]
  int32_t* len_w;         // == len, advanced by the attention kernel's last CTA
  int32_t* n_abs;
  int32_t* pos;
  float* score;
  int B, Hq, Hkv, d_store, Tcap, k;
  int dv;                 // 0: unprojected values of D dims; > 0: the first dv projected value dims
  float* ohat;            // dv > 0: [B][Hq][D] outputs over the projected value dims (workspace)
  int len_add;            // 1 with a fused append: the step attends len[b] + 1 tokens
  int n_late;             // attention CTAs (the last ones) expected to start after the projection kernel
  int early_select;       // the projection kernel selects before waiting for the previous kernel
  int out_bf16;
  float scale_log2;
};

// cached tokens of sequence b, clamped to the cache capacity (lengths are caller-owned device data)
__device__ __forceinline__ int seq_len(const int32_t* len, int b, int Tcap) { return min(max(len[b], 0), Tcap); }
// tokens the attention kernels attend for sequence b: the cached ones plus the
// token appended in this step.  len[b] itself is advanced only at the end of
// the attention kernel (step_done), so it is stable while both kernels run.
__device__ __forceinline__ int kv_len(const DecodeParams& p, int b) {
  return min(max(p.len[b], 0) + p.len_add, p.Tcap);
}

// Called once per attention CTA (thread 0) after all of its work: the last CTA
// of the grid advances the lengths of a step with a fused append.  The
// increments are atomic adds whose results nobody reads (reductions): the
// thread issues all of them back to back instead of waiting on a load before
// each store, which put B memory round trips at the end of every step.
__device__ __forceinline__ void step_done(const DecodeParams& p) {
  if (p.len_add == 0) return;
  if (atom_add_acq_rel_gpu(p.ctrl + kCtrlStepTicket, 1) == (int)(gridDim.x * gridDim.y * gridDim.z) - 1) {
    for (int bb = 0; bb < p.B; ++bb) {
      atomicAdd(p.len_w + bb, p.len_add);
      if (p.n_abs) atomicAdd(p.n_abs + bb, p.len_add);
    }
    p.ctrl[kCtrlStepTicket] = 0;
  }
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ void store_val(const DecodeParams& p, size_t idx, float v) {
  if (p.out_bf16)
    static_cast<__nv_bfloat16*>(p.out)[idx] = __float2bfloat16_rn(v);
  else
    static_cast<float*>(p.out)[idx] = v;
}

// A final output element.  With projected values (dv > 0) the result over the
// stored projected dimensions goes to the workspace; vproj_out_kernel then
// brings it back to the value space (o = o^ P[:, :dv]^T) and writes out.
__device__ __forceinline__ void store_result(const DecodeParams& p, size_t idx, float v) {
  if (p.dv > 0)
    p.ohat[idx] = v;
  else
    store_val(p, idx, v);
}

// Sequences with no tokens have no tiles: attention over zero tokens is the
// empty sum, output 0 and lse = -inf.  The attention CTAs share these units
// (unit u goes to CTA u mod grid).  Only steps without an append can meet one.
template <int G>
__device__ __forceinline__ void write_empty_units(const DecodeParams& p) {
  if (p.len_add != 0) return;
  const int n_units = p.B * p.Hkv;
  for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
    const int b = u / p.Hkv;
    if (seq_len(p.len, b, p.Tcap) > 0) continue;
    const size_t bhq0 = (size_t)b * p.Hq + (size_t)(u % p.Hkv) * G;
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) store_result(p, bhq0 * D + i, 0.f);
    if (p.lse_out != nullptr && threadIdx.x < G) p.lse_out[bhq0 + threadIdx.x] = -INFINITY;
  }
}

// ============================================================================
// query projection + magnitude top-k + group union
// ============================================================================
// Selection kernel geometry: NPW = 4 G warps first project row slices of all
// G query heads (each warp RW input dims, so P is read from shared memory once
// per CTA), then rank the dims, four warps per head (32 dims each); one more
// warp appends the step's key and value.
template <int G>
struct QprojCfg {
  static constexpr int NWQ = 4;                 // selection warps per head
  static constexpr int NPW = G * NWQ;           // projection and selection warps
  static constexpr int WARPS = NPW + 1;
};
constexpr int kPChunks = 4;   // P[g] staged as four 32-row chunks, each with its own barrier

// MINB = 2 caps the registers so that two CTAs share an SM (used when the
// units outnumber the SMs, which would otherwise run in two waves).
template <typename T, int G, int MINB>
__global__ void __launch_bounds__(QprojCfg<G>::WARPS * 32, MINB) qproj_topk_kernel(DecodeParams p) {
  constexpr int NWQ = QprojCfg<G>::NWQ, NPW = QprojCfg<G>::NPW;
  constexpr int NPT = NPW * 32;                 // threads of the projection/selection warps
  constexpr int RW = D / NPW;                   // input dims per projection warp
  constexpr int CROWS = D / kPChunks;           // rows per P chunk
  static_assert(NWQ * 32 == D, "four warps of 32 dims rank one head");
  static_assert(RW % 4 == 0 && CROWS % RW == 0, "projection slices vs P chunks");
  extern __shared__ __align__(128) float Ps[];   // P[g], [D][D]
  __shared__ __align__(16) float qs[G][D];       // q rows, later the kept scaled q~
  __shared__ __align__(16) float part[NPW][G][D];
  __shared__ __align__(16) float knew_s[D];
  __shared__ __align__(16) float vnew_s[D];     // the new value row (projected when dv > 0)
  __shared__ uint32_t masks[G][NWQ];
  __shared__ int neq[G][NWQ];
  __shared__ __align__(8) uint64_t pbars[kPChunks];
  __shared__ int s_abort;
  const int u = blockIdx.x;
  const int b = u / p.Hkv, g = u % p.Hkv;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = p.d_store;
  const bool append = p.k_new != nullptr;

  if (threadIdx.x == 0) {
    for (int c = 0; c < kPChunks; ++c) mbar_init(&pbars[c], 1);
    fence_barrier_init();
    // P is staged before the wait on the previous kernel: the kernels that may
    // still be running then (the attention kernels of a previous step or chunk,
    // the only ones that release their dependents early) never write it.
    for (int c = 0; c < kPChunks; ++c) {
      mbar_arrive_expect_tx(&pbars[c], CROWS * D * 4);
      bulk_g2s_plain(Ps + c * CROWS * D, p.P + (size_t)g * D * D + c * CROWS * D, CROWS * D * 4, &pbars[c]);
    }
  }
  // With early_select the projection and selection below run before the wait
  // on the previous kernel: they read only q and P and write only this call's
  // half of the workspace's selection buffers (calls alternate halves), so they
  // overlap the end of the previous kernel (the H2O update, or the previous
  // step's attention kernel, which reads the other half).  Used when the units
  // outnumber the SMs (this kernel then runs two CTAs per SM and takes several
  // microseconds); with fewer units its selection is shorter than the
  // attention kernel's own prologue, which it hides when it runs after the wait.
  // Either way every thread waits before the kernel releases its dependent (the
  // attention kernel reads the lengths, which the previous step's attention
  // kernel advances at its end, before its own wait), and before the append
  // reads the lengths and writes the cache.
  if (!p.early_select) {
    pdl_wait();
    pdl_launch_dependents();
  }
  if (threadIdx.x == 0) s_abort = 0;
  __syncthreads();

  if (w == NPW) {
    // ---- fused append of the new token of unit (b, g), in the key projection
    // order.  This warp takes no part in the selection below (which does not
    // depend on it), so the two run side by side.
    if (p.early_select) {
      pdl_wait();
      pdl_launch_dependents();
    }
    if (!append) return;
    const int slot = __ldcg(p.len + b);
    const int nabs = p.pos != nullptr ? __ldcg(p.n_abs + b) : 0;
    const T* kr = static_cast<const T*>(p.k_new) + (size_t)u * D;
    const T* vr = static_cast<const T*>(p.v_new) + (size_t)u * D;
    float kx[4];
    T vx[4];
#pragma unroll
    for (int s2 = 0; s2 < 4; ++s2) {
      kx[s2] = Elem<T>::load(kr + 4 * lane + s2);
      vx[s2] = vr[4 * lane + s2];
    }
    bool ok = true;
    for (int c = 0; c < kPChunks; ++c) ok = mbar_wait_bounded(&pbars[c], 0) && ok;
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) record_status(p.ctrl, AQUA_ERR_TIMEOUT);
      return;
    }
    if (slot < 0 || slot >= p.Tcap) {
      if (lane == 0) record_status(p.ctrl, AQUA_ERR_ARG);   // device length beyond capacity: write nothing
      return;
    }
#pragma unroll
    for (int s2 = 0; s2 < 4; ++s2) {
      knew_s[4 * lane + s2] = kx[s2];
      vnew_s[4 * lane + s2] = Elem<T>::load(&vx[s2]);
    }
    __syncwarp();
    float kt[4];
    project_row_smem(Ps, knew_s, lane, kt);
    T* kp = const_cast<T*>(static_cast<const T*>(p.kproj)) + (size_t)u * p.d_store * p.Tcap + slot;
#pragma unroll
    for (int s2 = 0; s2 < 4; ++s2) {
      const int jd = 4 * lane + s2;
      if (jd < p.d_store) kp[(size_t)jd * p.Tcap] = Elem<T>::from_f32(kt[s2]);
    }
    if (p.dv > 0) {
      // projected value v~ = v P, first dv dims (same projection routine and order as the key)
      float vt[4];
      project_row_smem(Ps, vnew_s, lane, vt);
      T* vp = const_cast<T*>(static_cast<const T*>(p.v)) + ((size_t)u * p.Tcap + slot) * p.dv;
      if (4 * lane < p.dv) {
#pragma unroll
        for (int s2 = 0; s2 < 4; ++s2) vp[4 * lane + s2] = Elem<T>::from_f32(vt[s2]);
      }
    } else {
      T* vp = const_cast<T*>(static_cast<const T*>(p.v)) + ((size_t)u * p.Tcap + slot) * D;
#pragma unroll
      for (int s2 = 0; s2 < 4; ++s2) vp[4 * lane + s2] = vx[s2];
    }
    if (p.pos != nullptr && lane == 0) {
      p.pos[(size_t)u * p.Tcap + slot] = nabs;
      p.score[(size_t)u * p.Tcap + slot] = 0.f;
    }
    return;
  }

  // ---- projection/selection warps (named barrier 1 over their NPT threads)
  if (w < G) {
    const T* qrow = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + g * G + w) * D;
#pragma unroll
    for (int s = 0; s < 4; ++s) qs[w][4 * lane + s] = Elem<T>::load(qrow + 4 * lane + s);
  }
  named_bar_sync(1, NPT);
  {
    // partial q~ of every head over input dims [w*RW, (w+1)*RW), outputs
    // 4*lane .. 4*lane+3: two chains per head (even / odd rows)
    const bool ok = mbar_wait_bounded(&pbars[w * RW / CROWS], 0);
    float a[G][4], c4[G][4];
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int s2 = 0; s2 < 4; ++s2) a[hh][s2] = c4[hh][s2] = 0.f;
#pragma unroll
    for (int r = 0; r < RW; r += 4) {
      const int i0 = w * RW + r;
      const float4 p0 = reinterpret_cast<const float4*>(Ps + (i0 + 0) * D)[lane];
      const float4 p1 = reinterpret_cast<const float4*>(Ps + (i0 + 1) * D)[lane];
      const float4 p2 = reinterpret_cast<const float4*>(Ps + (i0 + 2) * D)[lane];
      const float4 p3 = reinterpret_cast<const float4*>(Ps + (i0 + 3) * D)[lane];
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float4 x4 = *reinterpret_cast<const float4*>(&qs[hh][i0]);
        float* A = a[hh];
        float* C = c4[hh];
        A[0] = fmaf(x4.x, p0.x, A[0]); A[1] = fmaf(x4.x, p0.y, A[1]); A[2] = fmaf(x4.x, p0.z, A[2]); A[3] = fmaf(x4.x, p0.w, A[3]);
        C[0] = fmaf(x4.y, p1.x, C[0]); C[1] = fmaf(x4.y, p1.y, C[1]); C[2] = fmaf(x4.y, p1.z, C[2]); C[3] = fmaf(x4.y, p1.w, C[3]);
        A[0] = fmaf(x4.z, p2.x, A[0]); A[1] = fmaf(x4.z, p2.y, A[1]); A[2] = fmaf(x4.z, p2.z, A[2]); A[3] = fmaf(x4.z, p2.w, A[3]);
        C[0] = fmaf(x4.w, p3.x, C[0]); C[1] = fmaf(x4.w, p3.y, C[1]); C[2] = fmaf(x4.w, p3.z, C[2]); C[3] = fmaf(x4.w, p3.w, C[3]);
      }
    }
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
      *reinterpret_cast<float4*>(&part[w][hh][4 * lane]) =
          make_float4(a[hh][0] + c4[hh][0], a[hh][1] + c4[hh][1], a[hh][2] + c4[hh][2], a[hh][3] + c4[hh][3]);
    if (!ok) s_abort = 1;
  }
  named_bar_sync(1, NPT);
  if (s_abort) {
    if (threadIdx.x == 0) record_status(p.ctrl, AQUA_ERR_TIMEOUT);
    if (p.early_select) {
      pdl_wait();
      pdl_launch_dependents();
    }
    return;
  }

  // ---- selection: warp (hw, sl) ranks dims i = 32 sl + lane of head hw.
  // Keys: magnitude bits + 1 for candidate dims (i < m), 0 otherwise, so that
  // unsigned order equals |q~| order and non-candidates rank below every
  // candidate (NaN payloads are clamped to one key above inf).  rank_i = #{j : key_j > key_i} + #{j < i : key_j == key_i}
  // (ties to the lower index) and dim i is kept iff i < m and rank_i < k.
  const int hw = w / NWQ, sl = w % NWQ;
  const int h = g * G + hw;
  const size_t bh = (size_t)b * p.Hq + h;
  const int i = 32 * sl + lane;
  float qt = part[0][hw][i];                    // q~_i: the slices' partials added in slice order
#pragma unroll
  for (int x = 1; x < NPW; ++x) qt += part[x][hw][i];
  const uint32_t ki = i < m ? min(__float_as_uint(fabsf(qt)), 0x7F800001u) + 1u : 0u;   // NaN above inf
  // tau = the largest value with #{key >= tau} >= k over the head's 128 keys
  // (its four warps, one key per thread), one bit per round from the top (keys
  // are below 2^31), each count one barrier reduction over the four warps; the
  // search stops once exactly k keys are >= tau.
  const int hbar = 2 + hw;                      // named barrier of the head's warps
  uint32_t tau = 0;
  int cnt = D;
#pragma unroll 1
  for (int bit = 30; bit >= 0 && cnt != p.k; --bit) {   // cnt is uniform over the head's warps
    const uint32_t cand = tau | (1u << bit);
    const int c = named_bar_popc(hbar, NWQ * 32, ki >= cand);
    if (c >= p.k) {
      tau = cand;
      cnt = c;
    }
  }
  bool keep = i < m && ki >= tau;
  if (cnt > p.k) {
    // equal keys straddle the cut: every key above tau, then keys equal to tau
    // from the lowest index up
    const int ngt = named_bar_popc(hbar, NWQ * 32, ki > tau);
    const uint32_t eqb = __ballot_sync(0xffffffffu, ki == tau);
    if (lane == 0) neq[hw][sl] = __popc(eqb);
    named_bar_sync(hbar, NWQ * 32);
    int before = __popc(eqb & ((1u << lane) - 1u));
    for (int x = 0; x < sl; ++x) before += neq[hw][x];
    keep = i < m && (ki > tau || (ki == tau && before < p.k - ngt));
  }
  const uint32_t bal = __ballot_sync(0xffffffffu, keep);
  if (lane == 0) masks[hw][sl] = bal;
  if (p.qproj_out) p.qproj_out[bh * D + i] = qt;
  qs[hw][i] = keep ? qt * p.scale_log2 : 0.f;

  named_bar_sync(1, NPT);

  if (p.sel_out && keep) {                      // kept dims of the head in ascending order
    int pos = __popc(bal & ((1u << lane) - 1u));
    for (int x = 0; x < sl; ++x) pos += __popc(masks[hw][x]);
    p.sel_out[bh * p.k + pos] = i;
  }
  uint32_t um[4];
#pragma unroll
  for (int wd = 0; wd < 4; ++wd) {
    uint32_t x = 0;
#pragma unroll
    for (int hh = 0; hh < G; ++hh) x |= masks[hh][wd];
    um[wd] = x;
  }
  for (int j = threadIdx.x; j < D; j += NPT) {
    float* dn = p.qmn + ((size_t)u * D + j) * G;
#pragma unroll
    for (int hh = 0; hh < G; ++hh) dn[hh] = qs[hh][j];
    const int wd = j >> 5, bit = j & 31;
    // register selects instead of a run-time index into um[]
    const uint32_t word = wd == 0 ? um[0] : (wd == 1 ? um[1] : (wd == 2 ? um[2] : um[3]));
    if ((word >> bit) & 1u) {
      int r = __popc(word & ((1u << bit) - 1u));
      r += (wd > 0 ? __popc(um[0]) : 0) + (wd > 1 ? __popc(um[1]) : 0) + (wd > 2 ? __popc(um[2]) : 0);
      p.ulist[(size_t)u * D + r] = j;
      float* dst = p.qm + ((size_t)u * D + r) * G;
#pragma unroll
      for (int hh = 0; hh < G; ++hh) dst[hh] = qs[hh][j];
    }
  }
  if (threadIdx.x == 0) {
    p.ucount[u] = __popc(um[0]) + __popc(um[1]) + __popc(um[2]) + __popc(um[3]);
    p.counters[u] = 0;
  }
  if (p.early_select) {
    pdl_wait();
    pdl_launch_dependents();
  }
}

// ============================================================================
// shared pieces of the attention kernels
// ============================================================================
struct StageHdr {
  int u;       // unit b*Hkv + g
  int t0;      // first token of the tile
  int nvalid;  // valid tokens in the tile
  int nU;      // union rows
  int flags;   // kFirst | kLast
  int seg;     // partial slot, or -1 when the segment is the whole unit
  int nseg;    // segments of this unit
  int seg0;    // first partial slot of this unit (slots seg0 .. seg0+nseg-1)
};
constexpr int kFirst = 1, kLast = 2;

// The tiles of all (sequence, KV head) units form one flat sequence of
// positions in which every non-empty unit first occupies kBoundaryPos
// positions without work, then kTilePos positions per tile.  CTA c takes
// positions [floor(c NV / C), floor((c+1) NV / C)) and the tiles whose first
// position lies in that range (consecutive in the plain tile order).  A CTA
// whose range crosses into a new unit pays a second segment merge and a
// switch of the selection data, about 3.5 tiles' time at the Llama decode
// shape (fitted to per-CTA timings), and receives that many fewer tiles.
constexpr int kTilePos = 4;
constexpr int kBoundaryPos = 14;

// The split is in two parts.  The last n_late CTAs (by index) start only when
// the projection kernel's CTAs leave their SMs (measured ≈ 2.2 µs after the
// others at the Llama decode shape; a sweep of 0..14 positions was fastest at
// 10), so the first c0 = C - n_late CTAs share the first E positions,
// E = c0 (NV + n_late kLatePos) / C, and the late ones share the rest; within
// each part CTA c takes [floor(c N / C), floor((c+1) N / C)).
constexpr int kLatePos = 10;

struct Split {
  long long NV, E;   // positions in all, positions of the early part
  int C, c0;         // CTAs in all, early CTAs
};

__device__ __forceinline__ int cta_of_pos_even(long long p, long long N, int C) {
  const long long c = ((p + 1) * C + N - 1) / N - 1;
  return (int)(c < C - 1 ? c : C - 1);
}

// CTA whose range holds position p
__device__ __forceinline__ int cta_of_pos(long long p, const Split& sp) {
  return p < sp.E ? cta_of_pos_even(p, sp.E, sp.c0) : sp.c0 + cta_of_pos_even(p - sp.E, sp.NV - sp.E, sp.C - sp.c0);
}

// first position of CTA c's range (c = C gives NV)
__device__ __forceinline__ long long split_start(int c, const Split& sp) {
  return c <= sp.c0 ? (long long)c * sp.E / sp.c0
                    : sp.E + (long long)(c - sp.c0) * (sp.NV - sp.E) / (sp.C - sp.c0);
}

// Both parts keep at least kTilePos positions per CTA (every CTA between the
// first and last owner of a unit's tiles then owns one of them: the merge
// counts them); otherwise the split is even.
__device__ __forceinline__ Split make_split(long long NV, int grid, int n_late) {
  Split sp;
  sp.NV = NV;
  sp.C = (int)min((long long)grid, max(1LL, NV / kTilePos));
  sp.c0 = sp.C;
  sp.E = NV;
  if (n_late > 0 && n_late < sp.C) {
    const int c0 = sp.C - n_late;
    const long long E = (long long)c0 * (NV + (long long)n_late * kLatePos) / sp.C;
    if (E <= NV && E / c0 >= kTilePos && (NV - E) / n_late >= kTilePos) {
      sp.c0 = c0;
      sp.E = E;
    }
  }
  return sp;
}

// exclusive scans of two values over all NT threads of the block at once;
// tot[0], tot[1] receive the sums
template <int NT>
__device__ __forceinline__ void block_excl_scan2(long long v0, long long v1, long long* sh, long long (&excl)[2],
                                                 long long (&tot)[2]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int NW = NT / 32;
  static_assert(NW <= 32, "scan uses one warp for the warp totals");
  long long x0 = v0, x1 = v1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y0 = __shfl_up_sync(0xffffffffu, x0, o);
    const long long y1 = __shfl_up_sync(0xffffffffu, x1, o);
    if (lane >= o) {
      x0 += y0;
      x1 += y1;
    }
  }
  if (lane == 31) {
    sh[warp] = x0;
    sh[NW + warp] = x1;
  }
  __syncthreads();
  if (warp == 0) {
    long long y0 = lane < NW ? sh[lane] : 0, y1 = lane < NW ? sh[NW + lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long z0 = __shfl_up_sync(0xffffffffu, y0, o);
      const long long z1 = __shfl_up_sync(0xffffffffu, y1, o);
      if (lane >= o) {
        y0 += z0;
        y1 += z1;
      }
    }
    if (lane < NW) {
      sh[lane] = y0;
      sh[NW + lane] = y1;
    }
  }
  __syncthreads();
  excl[0] = (warp > 0 ? sh[warp - 1] : 0) + x0 - v0;
  excl[1] = (warp > 0 ? sh[NW + warp - 1] : 0) + x1 - v1;
  tot[0] = sh[NW - 1];
  tot[1] = sh[2 * NW - 1];
  __syncthreads();
}

struct Sched {
  long long N, NV;             // tiles, positions
  long long my_start, my_end;  // this CTA's tiles (plain tile order)
  const Split* sp;             // positions over CTAs (in shared memory; read at unit switches)
  int C;
  int u0;                      // unit of tile my_start
  long long ts0, sb0, vs0;     // its first tile, first partial slot and first position
};

template <int TT>
__device__ __forceinline__ long long unit_tiles(const DecodeParams& p, int u) {
  return (kv_len(p, u / p.Hkv) + TT - 1) / TT;
}

// Partial slots: the segment of unit u on CTA c uses slot u + c.  The CTAs
// covering a unit are consecutive and a later unit never starts on an earlier
// CTA, so slots are distinct, consecutive within a unit, and below
// n_units + C - 1 (no scan over the segment counts is needed).
//
// This CTA's tiles and first unit.  Returns false (for the whole CTA) when the
// CTA has no tile.  `scratch` needs 2 * NT / 32 long longs (sch + 8 .. sch + 31);
// sch[0..7] and the split (sch + 32) receive
// results.  All NT threads take part: one paired scan of the units' tile and
// position counts, then the thread whose units hold this CTA's first and last
// positions writes them to sch.
template <int TT, int NT>
__device__ bool make_schedule(const DecodeParams& p, long long* scratch, long long* sch, Sched& S) {
  const int tid = threadIdx.x;
  const int n_units = p.B * p.Hkv;
  const int c = blockIdx.x;
  const int chunk = (n_units + NT - 1) / NT;
  const int u_lo = min(n_units, tid * chunk), u_hi = min(n_units, u_lo + chunk);
  const long long nt_lo = u_lo < u_hi ? unit_tiles<TT>(p, u_lo) : 0;   // the usual case: one unit per thread
  long long my_tiles = 0, my_pos = 0;
  for (int u = u_lo; u < u_hi; ++u) {
    const long long nt = u == u_lo ? nt_lo : unit_tiles<TT>(p, u);
    my_tiles += nt;
    my_pos += nt > 0 ? nt * kTilePos + kBoundaryPos : 0;
  }
  long long excl[2], tot[2];
  block_excl_scan2<NT>(my_tiles, my_pos, scratch, excl, tot);
  const long long N = tot[0], NV = tot[1];
  const Split sp = make_split(NV, gridDim.x, p.n_late);
  Split* sp_s = reinterpret_cast<Split*>(sch + 32);
  if (tid == 0) *sp_s = sp;
  const int C = sp.C;
  if (c >= C) {
    // an idle CTA (the grid is sized from the host's length bound, the split
    // from the actual lengths): an empty schedule, never walked
    S.N = N;
    S.NV = NV;
    S.sp = sp_s;
    S.C = C;
    S.my_start = S.my_end = 0;
    S.u0 = 0;
    S.ts0 = S.sb0 = S.vs0 = 0;
    return false;
  }
  const long long a = split_start(c, sp), e = split_start(c + 1, sp);   // this CTA's positions
  if (tid == 0 && e == NV) sch[1] = N;    // the last CTA's tiles run to the end
  {
    long long ts = excl[0], vs = excl[1];
    for (int u = u_lo; u < u_hi; ++u) {
      const long long nt = u == u_lo ? nt_lo : unit_tiles<TT>(p, u);
      if (nt == 0) continue;
      const long long first = vs + kBoundaryPos, end = first + nt * kTilePos;   // unit's positions: [vs, end)
      if (vs <= a && a < end) {          // the range starts in this unit: its first tile starts at or after a
        sch[0] = ts + (a > first ? (a - first + kTilePos - 1) / kTilePos : 0);
        sch[2] = u;
        sch[3] = ts;
        sch[4] = u + cta_of_pos(first, sp);
        sch[5] = vs;
      }
      if (vs <= e && e < end) sch[1] = ts + (e > first ? (e - first + kTilePos - 1) / kTilePos : 0);
      ts += nt;
      vs = end;
    }
  }
  __syncthreads();
  S.N = N;
  S.NV = NV;
  S.sp = sp_s;
  S.C = C;
  S.my_start = sch[0];
  S.my_end = sch[1];
  S.u0 = (int)sch[2];
  S.ts0 = sch[3];
  S.sb0 = sch[4];
  S.vs0 = sch[5];
  return S.my_end > S.my_start;
}

// L2 prefetch of the first NSTAGE tiles this CTA most likely owns, issued
// while the schedule (which needs every length) is still being built, so the
// first tiles' copies find their data in L2.  The guess takes every sequence
// to have sequence 0's length, which makes it exact for equal lengths; a
// wrong guess only spends bandwidth.  Thread tid prefetches K~ row tid % D of
// guessed tile tid / D (the row's tokens of that tile), and row 0's thread
// also the tile's V rows.  Every address stays inside the unit's slots:
// u < B Hkv, r < d_store, t0 < T <= Tcap and t0 + ntok <= Tcap; the sizes
// are multiples of 32 bytes and the offsets of 32 bytes (Tcap, t0 and dv are
// multiples of 16 elements).
template <int TT, int NSTG>
__device__ __forceinline__ void prefetch_first_tiles_l2(const DecodeParams& p, int len0, int tid) {
  const int T = min(max(len0, 0) + p.len_add, p.Tcap);
  const int nt = (T + TT - 1) / TT;
  const int n_units = p.B * p.Hkv;
  const int j = tid / D, r = tid % D;                  // tile j of the first NSTG, K~ row r
  // only with no more units than SMs (n_late > 0): measured faster there (Llama
  // decode, long context) and slower with 256 units under H2O updates
  if (p.n_late == 0 || nt == 0 || j >= NSTG) return;
  const long long unitpos = (long long)nt * kTilePos + kBoundaryPos;   // positions of one unit
  const long long NV = (long long)n_units * unitpos;
  if (NV > 0x7fffffffLL) return;                      // 32-bit position arithmetic below
  const Split sp = make_split(NV, gridDim.x, p.n_late);
  if ((int)blockIdx.x >= sp.C) return;
  const int a = (int)split_start((int)blockIdx.x, sp);   // this CTA's first position
  const int u = a / (int)unitpos;
  if (u >= n_units) return;
  const int off = a - u * (int)unitpos;
  const int t = (off > kBoundaryPos ? (off - kBoundaryPos + kTilePos - 1) / kTilePos : 0) + j;
  if (t >= nt) return;
  const int t0 = t * TT;
  const int ntok = min(TT, p.Tcap - t0);
  const __nv_bfloat16* kp = static_cast<const __nv_bfloat16*>(p.kproj);
  if (r < p.d_store) prefetch_l2_bulk(kp + ((size_t)u * p.d_store + r) * p.Tcap + t0, (uint32_t)ntok * 2u);
  if (r == 0) {
    const int vcols = p.dv > 0 ? p.dv : D;
    const __nv_bfloat16* vp = static_cast<const __nv_bfloat16*>(p.v);
    prefetch_l2_bulk(vp + ((size_t)u * p.Tcap + t0) * vcols, (uint32_t)(ntok * vcols * 2));
  }
}

// Walks the units of this CTA's tile range; one instance per producer warp.
struct UnitWalker {
  int u = 0, b = 0, Tb = 0, nU = 0, nseg = 0, cf = 0;
  int nTb = 0, nnU = 0;                       // unit u + 1's length and union size, loaded on entering u
  long long ts = 0, te = 0, sb = 0, vs = 0;   // unit u: tiles [ts, te), first partial slot, first position
  __device__ void preload(const DecodeParams& p, bool with_nU) {
    if (u + 1 < p.B * p.Hkv) {
      nTb = kv_len(p, (u + 1) / p.Hkv);
      nnU = with_nU ? p.ucount[u + 1] : 0;
    }
  }
  template <int TT>
  __device__ void start(const DecodeParams& p, const Sched& S, bool with_nU = true) {
    u = S.u0;
    ts = S.ts0;
    sb = S.sb0;
    vs = S.vs0;
    b = u / p.Hkv;
    Tb = kv_len(p, b);
    te = ts + (Tb + TT - 1) / TT;
    cf = cta_of_pos(vs + kBoundaryPos, *S.sp);
    nseg = cta_of_pos(vs + kBoundaryPos + (te - ts - 1) * kTilePos, *S.sp) - cf + 1;
    nU = with_nU ? p.ucount[u] : 0;
    preload(p, with_nU);
  }
  // advance to the unit holding flat tile t; true when the unit changed
  template <int TT>
  __device__ bool seek(const DecodeParams& p, const Sched& S, long long t, bool with_nU = true) {
    bool changed = false;
    while (t >= te) {
      if (te > ts) vs += kBoundaryPos + (te - ts) * kTilePos;
      ++u;
      b = u / p.Hkv;
      Tb = nTb;                 // preloaded when the previous unit was entered
      const int nU1 = nnU;
      ts = te;
      te = ts + (Tb + TT - 1) / TT;
      preload(p, with_nU);
      if (te > ts) {
        cf = cta_of_pos(vs + kBoundaryPos, *S.sp);
        nseg = cta_of_pos(vs + kBoundaryPos + (te - ts - 1) * kTilePos, *S.sp) - cf + 1;
        sb = u + cf;
        nU = nU1;
      } else {
        nseg = 0;
      }
      changed = true;
    }
    return changed;
  }
  __device__ StageHdr header(const Sched& S, long long t, int TT) const {
    StageHdr hh;
    hh.u = u;
    hh.t0 = (int)(t - ts) * TT;
    hh.nvalid = min(TT, Tb - hh.t0);
    hh.nU = nU;
    hh.flags = ((t == S.my_start || t == ts) ? kFirst : 0) | ((t == S.my_end - 1 || t == te - 1) ? kLast : 0);
    hh.seg = nseg > 1 ? (int)(sb + (blockIdx.x - cf)) : -1;
    hh.nseg = nseg;
    hh.seg0 = (int)sb;
    return hh;
  }
};

// Segment result (M, L per head; O unnormalised, thread tid holding element
// idx = tid + NCT i of [G][D] in Ov[i]) -> output, or partial + ticket +
// merge by the unit's last CTA.  Called by all consumer threads; element idx
// is (h, dim) = (idx / D, idx % D).
template <int G>
__device__ void finish_segment(const DecodeParams& p, const StageHdr& hh, int tid, const float (&Mh)[G],
                               const float (&Lh)[G], const float (&Ov)[(G * D + NCT - 1) / NCT], int* s_last) {
  const int b = hh.u / p.Hkv, g = hh.u % p.Hkv;
  const size_t bhq0 = (size_t)b * p.Hq + g * G;
#pragma unroll
  for (int i = 0; i < (G * D + NCT - 1) / NCT; ++i) {
    const int idx = tid + NCT * i;
    if (idx < G * D) {
      const int h = idx / D, dim = idx % D;
      float lh = 0.f;
#pragma unroll
      for (int x = 0; x < G; ++x)
        if (x == h) lh = Lh[x];
      const float o = Ov[i];
      if (hh.seg < 0)
        store_result(p, (bhq0 + h) * D + dim, o / lh);
      else
        p.part_o[((size_t)hh.seg * G + h) * D + dim] = o;
    }
  }
  if (tid < G) {
#pragma unroll
    for (int h = 0; h < G; ++h)
      if (h == tid) {
        if (hh.seg < 0) {
          if (p.lse_out) p.lse_out[bhq0 + h] = (Mh[h] + log2f(Lh[h])) * kLn2;
        } else {
          p.part_ml[((size_t)hh.seg * G + h) * 2 + 0] = Mh[h];
          p.part_ml[((size_t)hh.seg * G + h) * 2 + 1] = Lh[h];
        }
      }
  }
  if (hh.seg < 0) return;
  // publish this partial and take a ticket; the unit's last arrival merges.
  // The barrier orders every thread's partial stores before thread 0's
  // GPU-scope fence (fences are cumulative), which precedes the ticket.
  // (the pattern of a barrier, then one thread's release, orders every
  // thread's partial stores before the ticket; the last arrival's acquire,
  // then a barrier, orders the other partials before every thread's loads)
  named_bar_sync(1, NCT);
  if (tid == 0) *s_last = (atom_add_acq_rel_gpu(p.counters + hh.u, 1) == hh.nseg - 1);
  named_bar_sync(1, NCT);
  if (!*s_last) return;
  constexpr int NI = (G * D + NCT - 1) / NCT;   // outputs per thread (2 at G = 4)
  constexpr int MB = 8 / NI;                    // partials per round: 8 loads x 3 in flight per thread
  // one pass over the unit's partials for all of this thread's outputs at once
  // (their loads in flight together): each round of MB partials raises the
  // running max and rescales what was summed before (nothing in the first)
  float M[NI], Lsum[NI], O[NI];
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    M[i] = -INFINITY;
    Lsum[i] = 0.f;
    O[i] = 0.f;
  }
#pragma unroll 1
  for (int s0 = 0; s0 < hh.nseg; s0 += MB) {
    float mv[NI][MB], lv[NI][MB], ov[NI][MB];
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const int idx = tid + NCT * i;
      const int h = idx / D, dim = idx % D;
#pragma unroll
      for (int j = 0; j < MB; ++j) {
        const bool in = idx < G * D && s0 + j < hh.nseg;
        const size_t slot = (size_t)(hh.seg0 + s0 + j) * G + h;
        mv[i][j] = in ? __ldcg(p.part_ml + slot * 2) : -INFINITY;
        lv[i][j] = in ? __ldcg(p.part_ml + slot * 2 + 1) : 0.f;
        ov[i][j] = in ? __ldcg(p.part_o + slot * D + dim) : 0.f;
      }
    }
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      float Mn = M[i];
#pragma unroll
      for (int j = 0; j < MB; ++j) Mn = fmaxf(Mn, mv[i][j]);
      if (s0 > 0) {
        const float c = exp2f(M[i] - Mn);
        Lsum[i] *= c;
        O[i] *= c;
      }
      M[i] = Mn;
#pragma unroll
      for (int j = 0; j < MB; ++j) {
        const float f = exp2f(mv[i][j] - M[i]);
        Lsum[i] = fmaf(f, lv[i][j], Lsum[i]);
        O[i] = fmaf(f, ov[i][j], O[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const int idx = tid + NCT * i;
    if (idx >= G * D) break;
    const int h = idx / D, dim = idx % D;
    store_result(p, (bhq0 + h) * D + dim, O[i] / Lsum[i]);
    if (dim == 0 && p.lse_out) p.lse_out[bhq0 + h] = (M[i] + log2f(Lsum[i])) * kLn2;
  }
  if (tid == 0) p.counters[hh.u] = 0;
}

// ============================================================================
// bf16 cache: tensor-core consumers
// ============================================================================
template <int G>
struct SmemBF16 {
  static constexpr int TT = 128;
  static constexpr int VHALF = TT * 128;                // [TT tokens][64 dims] bf16, 128B-swizzled
  static constexpr int KBYTES = D * KROW_BF16;          // [128 rows][272 B]
  static constexpr int STAGE = 2 * VHALF + KBYTES;      // multiple of 1024
  static constexpr int OFF_RED = NSTAGE * STAGE;        // [NCW][G][D] f32
  static constexpr int OFF_ML = OFF_RED + NCW * G * D * 4;   // [NCW][G][2] f32, [NCW][G] factors, [2][G]
  static constexpr int OFF_HDR = OFF_ML + (NCW * G * 3 + 2 * G) * 4;
  static constexpr int OFF_BAR = OFF_HDR + NSTAGE * (int)sizeof(StageHdr);
  static constexpr int OFF_SCH = OFF_BAR + 2 * NSTAGE * 8;
  static constexpr int OFF_MISC = OFF_SCH + 40 * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static_assert(STAGE % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
  static_assert(KROW_BF16 >= 2 * TT + G * 4, "a K~ row's padding holds the row's G masked queries");
};

// The V tile of TT = 128 tokens as two tensor copies of 64-dim halves,
// 128B-swizzled.  With projected values the tensor map's rows hold the dv
// stored dims and the copy fills the dims past them with zeros (a half that
// starts past dv is all zeros), so the PV products run over all 128 dims with
// no bound in the loop.
__device__ __forceinline__ void issue_v_tile(unsigned char* st, const CUtensorMap* tmap, int row, uint64_t* bar,
                                             uint64_t pol) {
  constexpr int VHALF = 128 * 128;
  mbar_arrive_expect_tx(bar, 2 * VHALF);
  tma_load_2d(st, tmap, 0, row, bar, pol);
  tma_load_2d(st + VHALF, tmap, 64, row, bar, pol);
}

// Scores S^T of a warp's 16 tokens (MMA rows) over NKS k-steps of 16 union
// rows: A = the K~ tile read transposed, B = the masked queries (qb); even
// k-steps accumulate into c, odd ones into d (two chains).
template <int NKS>
__device__ __forceinline__ void score_ksteps(const unsigned char* a0, const uint32_t (&qb)[8][2], float (&c)[4],
                                             float (&d)[4]) {
#pragma unroll
  for (int kk = 0; kk < NKS; ++kk) {
    uint32_t ka[4];
    ldsm_x4_trans(ka, a0 + kk * 16 * KROW_BF16);
    if (kk & 1)
      mma_bf16_16816(d, ka, qb[kk][0], qb[kk][1]);
    else
      mma_bf16_16816(c, ka, qb[kk][0], qb[kk][1]);
  }
}

template <int G>
__global__ void __launch_bounds__(NTHREADS_BF16, 1)
    decode_attn_bf16_kernel(const __grid_constant__ CUtensorMap tmap_v, DecodeParams p) {
  using S = SmemBF16<G>;
  constexpr int TT = S::TT;
  static_assert(G <= 8, "head rows 0..G-1 (high parts) and 8..8+G-1 (low parts)");
  extern __shared__ __align__(1024) unsigned char smem[];
  float* red = reinterpret_cast<float*>(smem + S::OFF_RED);
  float* mlb = reinterpret_cast<float*>(smem + S::OFF_ML);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR);
  uint64_t* empty = full + NSTAGE;
  long long* sch = reinterpret_cast<long long*>(smem + S::OFF_SCH);
  int* s_last = reinterpret_cast<int*>(smem + S::OFF_MISC);   // [0]: merge ticket, [1]: timeout flag

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  if (tid == 0) s_last[1] = 0;
  const int len0 = p.len[0];   // for the L2 prefetch below; the load overlaps the zeroing

  // the K~ rows of every stage start zeroed: union padding rows and never-copied
  // tokens must be finite (the V halves are rewritten whole by every tile copy)
  constexpr int KQ = S::KBYTES / 16;
  for (int i = tid; i < NSTAGE * KQ; i += NTHREADS_BF16) {
    const int s = i / KQ;
    reinterpret_cast<uint4*>(smem + (size_t)s * S::STAGE + 2 * S::VHALF)[i - s * KQ] = make_uint4(0, 0, 0, 0);
  }
  static_assert(NTHREADS_BF16 >= NSTAGE * D, "one thread per prefetched K~ row");
  prefetch_first_tiles_l2<TT, NSTAGE>(p, len0, tid);
  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      // arrivals: one cp.async arrival per producer thread + the V tensor-copy arrival
      mbar_init(&full[s], NPW_BF16 * 32 + 1);
      mbar_init(&empty[s], NCW);
    }
    fence_barrier_init();
  }
  if (tid == NCT) prefetch_tmap(&tmap_v);
  // The schedule depends only on the lengths, which the projection kernel does
  // not change (the lengths advance at the end of this kernel, and the
  // projection kernel releases this one only once its own predecessors are
  // complete): compute it while the projection kernel runs.  Loading tiles
  // early as well was measured to slow the step down (the copies compete with
  // the projection kernel's latency-bound loads).
  Sched Sd;
  const bool has_work = make_schedule<TT, NTHREADS_BF16>(p, sch + 8, sch, Sd);
  fence_proxy_async_smem();
  __syncthreads();
  const int n_tiles = has_work ? (int)(Sd.my_end - Sd.my_start) : 0;
  // The first n_nat tiles (at most NSTAGE, all in the CTA's first unit, none
  // its last tile, which holds this step's appended token) are loaded before
  // the wait: V, and every kept K~ row in dimension order (the union list that
  // picks rows is not known yet).  Nothing the projection kernel writes is in
  // them, and everything before it on the stream is complete once it has
  // released this kernel.  Their scores contract over all d_store dims with
  // the masked queries in dimension order (zero for dims no head kept), which
  // is the same sum as over the union rows.
  int n_nat = 0;
  if (has_work) {
    // (a CTA without work has no schedule: make_schedule leaves Sd unset for it)
    UnitWalker W0;
    W0.start<TT>(p, Sd, false);
    const int u_first = W0.u;
    for (int it = 0; it < NSTAGE && it < n_tiles; ++it) {
      const long long t = Sd.my_start + it;
      W0.seek<TT>(p, Sd, t, false);
      const int t0 = (int)(t - W0.ts) * TT;
      if (W0.u != u_first || t0 + TT >= W0.Tb) break;
      ++n_nat;
      if (warp < NCW) continue;
      const int pt = tid - NCT;
      const uint64_t pol = policy_evict_first();
      unsigned char* st = smem + (size_t)it * S::STAGE;
      if (pt == 0) issue_v_tile(st, &tmap_v, W0.u * p.Tcap + t0, &full[it], pol);
      const int chunk = pt & 15, r0 = pt >> 4;
      const __nv_bfloat16* kbase =
          static_cast<const __nv_bfloat16*>(p.kproj) + (size_t)W0.u * p.d_store * p.Tcap + t0 + chunk * 8;
      unsigned char* ks = st + 2 * S::VHALF + chunk * 16;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int r = r0 + 8 * j;
        if (r < p.d_store) cp_async16(ks + r * KROW_BF16, kbase + (size_t)r * p.Tcap, pol);
      }
      cp_async_arrive_noinc(&full[it]);
    }
  }
  pdl_launch_dependents();
  pdl_wait();   // the projection kernel (and its append) must be complete
  write_empty_units<G>(p);
  if (!has_work) {
    if (tid == 0) step_done(p);
    return;
  }

  if (warp >= NCW) {
    // ======================= producer warps =======================
    // Thread pt copies 16-byte chunk (pt & 15) of union rows (pt >> 4) + 8 j,
    // j = 0..15, of every tile; producer thread 0 also issues the V tile.
    const int pt = tid - NCT;
    const int chunk = pt & 15, r0 = pt >> 4;
    const uint64_t pol = policy_evict_first();
    UnitWalker W;
    W.start<TT>(p, Sd);
    if (pt == 0) {
      // the other V tiles of the first stages do not depend on the union
      // list either: issue them before the union rows are fetched
      UnitWalker W0 = W;
      for (int it = 0; it < NSTAGE && it < n_tiles; ++it) {
        const long long t = Sd.my_start + it;
        W0.seek<TT>(p, Sd, t);
        if (it < n_nat) continue;
        const StageHdr h0 = W0.header(Sd, t, TT);
        unsigned char* st = smem + (size_t)it * S::STAGE;
        issue_v_tile(st, &tmap_v, h0.u * p.Tcap + h0.t0, &full[it], pol);
      }
    }
    // union rows of the current unit and, loaded ahead, of the next one
    const int n_units = p.B * p.Hkv;
    int urow[16], unext[16];
    int unext_u = W.u + 1;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int r = r0 + 8 * j;
      urow[j] = r < W.nU ? p.ulist[(size_t)W.u * D + r] : 0;
      unext[j] = unext_u < n_units ? p.ulist[(size_t)unext_u * D + r] : 0;
    }
    for (int it = 0; it < n_tiles; ++it) {
      const long long t = Sd.my_start + it;
      if (W.seek<TT>(p, Sd, t)) {
        const bool ahead = W.u == unext_u;      // else empty units were skipped
#pragma unroll
        for (int j = 0; j < 16; ++j) urow[j] = ahead ? unext[j] : p.ulist[(size_t)W.u * D + r0 + 8 * j];
        unext_u = W.u + 1;
#pragma unroll
        for (int j = 0; j < 16; ++j) unext[j] = unext_u < n_units ? p.ulist[(size_t)unext_u * D + r0 + 8 * j] : 0;
      }
      if (it < n_nat) continue;                 // loaded before the wait
      const int s = it % NSTAGE;
      if (it >= NSTAGE) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait_bounded(&empty[s], ((it / NSTAGE) & 1) ^ 1);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) record_status(p.ctrl, AQUA_ERR_TIMEOUT);
          return;
        }
      }
      const StageHdr hh = W.header(Sd, t, TT);
      unsigned char* st = smem + (size_t)s * S::STAGE;
      if (pt == 0 && it >= NSTAGE) issue_v_tile(st, &tmap_v, hh.u * p.Tcap + hh.t0, &full[s], pol);
      const int nch = (hh.nvalid + 7) / 8;                  // 16-byte groups of 8 tokens
      if (chunk < nch) {
        const __nv_bfloat16* kbase =
            static_cast<const __nv_bfloat16*>(p.kproj) + (size_t)hh.u * p.d_store * p.Tcap + hh.t0 + chunk * 8;
        unsigned char* ks = st + 2 * S::VHALF + chunk * 16;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int r = r0 + 8 * j;
          if (r < hh.nU) cp_async16(ks + r * KROW_BF16, kbase + (size_t)urow[j] * p.Tcap, pol);
        }
      }
      if ((hh.flags & kFirst) || (it == n_nat && n_nat > 0)) {
        // the masked queries of union row r (G floats) ride in the padding
        // after the row's TT keys; the consumers read them on a unit's first
        // tile (and on the first tile after the dimension-order ones)
        const int r = r0 + 8 * chunk;
        if (r < hh.nU)
          cp_async_small<G * 4>(st + 2 * S::VHALF + r * KROW_BF16 + 2 * TT, p.qm + ((size_t)hh.u * D + r) * G);
      }
      cp_async_arrive_noinc(&full[s]);
    }
    return;
  }

  // ======================= consumer warps =======================
  // Transposed products: S^T = K~^T Q~m^T and O^T = V^T P^T, with the warp's
  // 16 tokens as the MMA rows (M = 16) and 8 columns of (head, part) pairs:
  // column 2h carries head h's bf16 high part, column 2h + 1 its low part.
  // The thread of fragment column pair q4 thus holds both parts of head q4
  // (and adds them itself); P's fragment, laid out as the scores' accumulator
  // (tokens x columns), becomes the B operand of the P V product by one 8x8
  // transpose per 8 tokens.
  const int grp = lane >> 2, q4 = lane & 3;    // mma fragment coordinates
  const int tb = 16 * warp;                     // this warp's tokens in every tile
  const bool head_ok = q4 < G;                 // head q4 exists
  uint32_t qb[8][2];                            // scores' B operand: column grp, union rows 16 kk + 2 q4 (+1, +8, +9)
  float o[8][4];                                // O^T: dims 16 j + grp (+ 8) x columns 2 q4, 2 q4 + 1
  float mu = -INFINITY;                         // running max of head q4 (the same in all its lanes)
  float ell = 0.f;                              // this thread's share of head q4's sum (reduced at segment ends)
  int cur_u = -1, nks = 0;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) qb[kk][0] = qb[kk][1] = 0u;
#pragma unroll
  for (int n = 0; n < 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  // Every consumer warp walks the schedule itself, so all warps agree on the
  // segment ends (where they synchronise) whatever happens to the data.  A
  // warp whose wait runs out records the error, stops computing and keeps
  // taking part in the segment-end barriers; the other warps follow it.
  UnitWalker W;
  W.start<TT>(p, Sd);
  volatile int* dead_flag = s_last + 1;
  bool dead = false;

  for (int it = 0; it < n_tiles; ++it) {
    const int s = it % NSTAGE;
    const long long t = Sd.my_start + it;
    W.seek<TT>(p, Sd, t);
    const StageHdr hh = W.header(Sd, t, TT);
    if (!dead) {
      const bool ok = mbar_wait_bounded(&full[s], (it / NSTAGE) & 1);
      const bool timed_out = __any_sync(0xffffffffu, !ok);     // warp-uniform decision
      if (timed_out && lane == 0) {
        *dead_flag = 1;
        record_status(p.ctrl, AQUA_ERR_TIMEOUT);
      }
      dead = timed_out || __any_sync(0xffffffffu, *dead_flag != 0);
    }
    unsigned char* st = smem + (size_t)s * S::STAGE;
    const unsigned char* ks_base = st + 2 * S::VHALF;

    // B operand: the masked queries of the unit in the order of the tile's K~
    // rows, dimension order on the tiles loaded before the wait, union order
    // (from the rows' padding) from the first tile after them on.  Column grp
    // is head grp >> 1, part grp & 1.
    const bool nat0 = it == 0 && n_nat > 0;
    const bool comp0 = it == n_nat && n_nat > 0;
    if (!dead && ((hh.flags & kFirst) || comp0)) {
      if (hh.u != cur_u || nat0 || comp0) {
        cur_u = hh.u;
        const int nrow = nat0 ? p.d_store : hh.nU;
        nks = (nrow + 15) / 16;
        const int qh = grp >> 1;
        const bool col_ok = qh < G, low = (grp & 1) != 0;
        // source of row r's query for head qh: dimension-order array or the row padding
        const float* qsrc = nat0 ? p.qmn + (size_t)hh.u * D * G + qh
                                 : reinterpret_cast<const float*>(ks_base + 2 * TT) + qh;
        const int qstride = nat0 ? G : KROW_BF16 / 4;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            float v2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int r = kk * 16 + half * 8 + 2 * q4 + e;
              const float x = (col_ok && r < nrow) ? qsrc[r * qstride] : 0.f;
              float hi, lo;
              split_bf16(x, hi, lo);
              v2[e] = low ? lo : hi;
            }
            qb[kk][half] = pack_bf16(v2[0], v2[1]);
          }
        }
      }
    }
    if (!dead && (hh.flags & kFirst)) {
      mu = -INFINITY;
      ell = 0.f;
#pragma unroll
      for (int n = 0; n < 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    }

    bool wrote_smem = false;
    if (!dead && tb < hh.nvalid) {
      if (tb + 16 > hh.nvalid) {
        // zero the V rows of this warp's tokens past the end (p = 0 there, V must be finite)
        for (int i = lane; i < 16 * 16; i += 32) {
          const int row = tb + (i >> 4), chunk = i & 15;
          if (row >= hh.nvalid)
            *reinterpret_cast<uint4*>(st + (chunk >> 3) * S::VHALF + row * 128 + (chunk & 7) * 16) =
                make_uint4(0, 0, 0, 0);
        }
        wrote_smem = true;
      }
      // ldmatrix, mma.sync and movmatrix below need the whole warp converged:
      // the query build above and the zeroing take lane-dependent paths (for
      // G < 4 the lanes of absent heads load nothing)
      __syncwarp();
      const int mtx = lane >> 3, r8 = lane & 7;
      // ---- S^T for this warp's 16 tokens
      float c[4] = {0.f, 0.f, 0.f, 0.f}, d[4] = {0.f, 0.f, 0.f, 0.f};
      {
        // matrices: (rows 0-7, tokens 0-7), (rows 0-7, tokens 8-15), (rows 8-15, tokens 0-7), (rows 8-15, tokens 8-15)
        const unsigned char* a0 = ks_base + ((mtx >> 1) * 8 + r8) * KROW_BF16 + (tb + (mtx & 1) * 8) * 2;
        // the k-steps as straight-line code for the union size (no test between the MMAs)
        switch (nks) {
          case 8: score_ksteps<8>(a0, qb, c, d); break;
          case 7: score_ksteps<7>(a0, qb, c, d); break;
          case 6: score_ksteps<6>(a0, qb, c, d); break;
          case 5: score_ksteps<5>(a0, qb, c, d); break;
          case 4: score_ksteps<4>(a0, qb, c, d); break;
          case 3: score_ksteps<3>(a0, qb, c, d); break;
          case 2: score_ksteps<2>(a0, qb, c, d); break;
          default: score_ksteps<1>(a0, qb, c, d); break;
        }
      }
      // A operand of P V: the V tile read transposed (dims x tokens), loaded
      // ahead of the softmax; matrices (tokens 0-7, dims 0-7), (tokens 0-7,
      // dims 8-15), (tokens 8-15, dims 0-7), (tokens 8-15, dims 8-15) of each
      // 16-dim block
      uint32_t va[8][4];
      {
        const int tok = tb + (mtx >> 1) * 8 + r8;
        const unsigned char* vrow = st + tok * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int dim0 = 16 * j + (mtx & 1) * 8;
          const int chunk = (dim0 & 63) >> 3;
          ldsm_x4_trans(va[j], vrow + (dim0 >> 6) * S::VHALF + ((chunk ^ (tok & 7)) << 4));
        }
      }
      // head q4 at tokens tb + grp and tb + grp + 8: high + low parts
      float sc[2] = {(c[0] + c[1]) + (d[0] + d[1]), (c[2] + c[3]) + (d[2] + d[3])};
      if (tb + grp >= hh.nvalid) sc[0] = -INFINITY;
      if (tb + grp + 8 >= hh.nvalid) sc[1] = -INFINITY;
      if (p.scores_out != nullptr && head_ok) {
        const int b = hh.u / p.Hkv, g = hh.u % p.Hkv;
        float* dst = p.scores_out + ((size_t)b * p.Hq + g * G + q4) * p.Tcap + hh.t0 + tb + grp;
        if (tb + grp < hh.nvalid) dst[0] = sc[0] * kLn2;
        if (tb + grp + 8 < hh.nvalid) dst[8] = sc[1] * kLn2;
      }
      // ---- online softmax: the running max is raised only when a score
      // exceeds it by 2^8 (exact; it avoids rescaling), and the warp's maximum
      // over its tokens is formed only then
      const bool over = head_ok && fmaxf(sc[0], sc[1]) > mu + kLazyRescale;
      if (__any_sync(0xffffffffu, over)) {
        float mx = fmaxf(sc[0], sc[1]);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        if (head_ok && mx > mu + kLazyRescale) {
          const float alpha = exp2f(mu - mx);
          mu = mx;
#pragma unroll
          for (int n = 0; n < 8; ++n) {
            o[n][0] *= alpha;
            o[n][1] *= alpha;
            o[n][2] *= alpha;
            o[n][3] *= alpha;
          }
          ell *= alpha;
        }
      }
      const float p0 = head_ok ? exp2f(sc[0] - mu) : 0.f;
      const float p1 = head_ok ? exp2f(sc[1] - mu) : 0.f;
      ell += p0 + p1;
      float h0, l0, h1, l1;
      split_bf16(p0, h0, l0);
      split_bf16(p1, h1, l1);
      // P as (tokens x columns) accumulator-layout fragments, transposed into
      // the B operand (tokens x columns, column-major); the lanes of absent
      // heads (G < 4) took other paths above
      __syncwarp();
      const uint32_t pb0 = movmatrix_trans(pack_bf16(h0, l0));
      const uint32_t pb1 = movmatrix_trans(pack_bf16(h1, l1));
      // ---- O^T += V^T P^T over 128 dims (zeros past dv with projected values)
#pragma unroll
      for (int j = 0; j < 8; ++j) mma_bf16_16816(o[j], va[j], pb0, pb1);
    }
    if (wrote_smem) fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);

    if (!(hh.flags & kLast)) continue;

    // ---- end of a segment: the warp's sum of head q4, then merge the warps'
    // (m, l, o) and output or partial
    ell += __shfl_xor_sync(0xffffffffu, ell, 4);
    ell += __shfl_xor_sync(0xffffffffu, ell, 8);
    ell += __shfl_xor_sync(0xffffffffu, ell, 16);
    if (head_ok) {
      float* rw = red + ((size_t)warp * G + q4) * D + grp;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        rw[16 * j] = o[j][0] + o[j][1];
        rw[16 * j + 8] = o[j][2] + o[j][3];
      }
      if (grp == 0) {
        mlb[(warp * G + q4) * 2 + 0] = mu;
        mlb[(warp * G + q4) * 2 + 1] = ell;
      }
    }
    named_bar_sync(1, NCT);
    // per-head running max over the warps and each warp's scale factor, once
    float* fac = mlb + NCW * G * 2;          // [NCW][G] scale factors, then [G] M and [G] L
    if (tid < G) {
      const int h = tid;
      float M = -INFINITY;
#pragma unroll
      for (int w2 = 0; w2 < NCW; ++w2) M = fmaxf(M, mlb[(w2 * G + h) * 2]);
      float L = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < NCW; ++w2) {
        const float f = exp2f(mlb[(w2 * G + h) * 2] - M);
        fac[w2 * G + h] = f;
        L = fmaf(f, mlb[(w2 * G + h) * 2 + 1], L);
      }
      fac[NCW * G + h] = M;
      fac[NCW * G + G + h] = L;
    }
    named_bar_sync(1, NCT);
    float Mh[G], Lh[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      Mh[h] = fac[NCW * G + h];
      Lh[h] = fac[NCW * G + G + h];
    }
    float merged[(G * D + NCT - 1) / NCT];
#pragma unroll
    for (int i = 0; i < (G * D + NCT - 1) / NCT; ++i) {
      const int idx = tid + NCT * i;
      merged[i] = 0.f;
      if (idx < G * D) {
        const int h = idx / D, dim = idx % D;
        float acc = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < NCW; ++w2) acc = fmaf(fac[w2 * G + h], red[((size_t)w2 * G + h) * D + dim], acc);
        merged[i] = acc;
      }
    }
    // each thread passes its own merged elements on; red is next written at the
    // following segment end, after the barrier below
    finish_segment<G>(p, hh, tid, Mh, Lh, merged, s_last);
    named_bar_sync(1, NCT);
  }
  named_bar_sync(1, NCT);               // every consumer warp is done with this CTA's work
  if (tid == 0) step_done(p);
}

// ============================================================================
// f32 cache: CUDA-core consumers
// ============================================================================
template <int G>
struct SmemF32 {
  static constexpr int TT = 64;
  static constexpr int KBYTES = D * TT * 4;
  static constexpr int VBYTES = TT * D * 4;
  static constexpr int STAGE = KBYTES + VBYTES;
  static constexpr int RW = D;
  static constexpr int SLOTS = (G * TT + NCT - 1) / NCT;
  static constexpr int OFF_RED = NSTAGE * STAGE;
  static constexpr int OFF_PSM = OFF_RED + NCW * G * RW * 4;
  static constexpr int OFF_WST = OFF_PSM + TT * G * 4;
  static constexpr int OFF_HDR = OFF_WST + 2 * SLOTS * NCW * 4;
  static constexpr int OFF_BAR = OFF_HDR + NSTAGE * (int)sizeof(StageHdr);
  static constexpr int OFF_SCH = OFF_BAR + 2 * NSTAGE * 8;
  static constexpr int OFF_MISC = OFF_SCH + 40 * 8;
  static constexpr int BYTES = OFF_MISC + 16;
};

template <int G>
__global__ void __launch_bounds__(NTHREADS, 1) decode_attn_f32_kernel(DecodeParams p) {
  using S = SmemF32<G>;
  constexpr int TT = S::TT;
  constexpr int TPL = TT / 32;        // tokens per lane in the score pass
  constexpr int TPW = TT / NCW;       // tokens per warp in the PV pass
  static_assert(TPL == 2, "score pass loads two f32 tokens per lane");

  extern __shared__ __align__(1024) unsigned char smem[];
  float* red = reinterpret_cast<float*>(smem + S::OFF_RED);
  float* psm = reinterpret_cast<float*>(smem + S::OFF_PSM);
  float* wmax = reinterpret_cast<float*>(smem + S::OFF_WST);
  float* wsum = wmax + S::SLOTS * NCW;
  StageHdr* hdr = reinterpret_cast<StageHdr*>(smem + S::OFF_HDR);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR);
  uint64_t* empty = full + NSTAGE;
  long long* sch = reinterpret_cast<long long*>(smem + S::OFF_SCH);
  int* s_last = reinterpret_cast<int*>(smem + S::OFF_MISC);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int vcols = p.dv > 0 ? p.dv : D;       // stored value dims (V row length)

  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCW);
    }
    fence_barrier_init();
  }
  pdl_launch_dependents();
  pdl_wait();
  write_empty_units<G>(p);
  Sched Sd;
  if (!make_schedule<TT, NTHREADS>(p, sch + 8, sch, Sd)) {
    if (tid == 0) step_done(p);
    return;
  }
  const int n_tiles = (int)(Sd.my_end - Sd.my_start);

  if (warp == NCW) {
    const uint64_t pol = policy_evict_first();
    UnitWalker W;
    W.start<TT>(p, Sd);
    int urow[D / 32];
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      const int r = lane + 32 * i;
      urow[i] = r < W.nU ? p.ulist[(size_t)W.u * D + r] : 0;
    }
    for (int it = 0; it < n_tiles; ++it) {
      const long long t = Sd.my_start + it;
      if (W.seek<TT>(p, Sd, t)) {
#pragma unroll
        for (int i = 0; i < D / 32; ++i) {
          const int r = lane + 32 * i;
          urow[i] = r < W.nU ? p.ulist[(size_t)W.u * D + r] : 0;
        }
      }
      const int s = it % NSTAGE;
      if (it >= NSTAGE) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait_bounded(&empty[s], ((it / NSTAGE) & 1) ^ 1);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) record_status(p.ctrl, AQUA_ERR_TIMEOUT);
          return;
        }
      }
      const StageHdr hh = W.header(Sd, t, TT);
      const uint32_t kbytes = (uint32_t)((hh.nvalid + 3) / 4 * 16);
      const uint32_t vbytes = (uint32_t)hh.nvalid * vcols * 4;
      unsigned char* st = smem + (size_t)s * S::STAGE;
      if (lane == 0) {
        hdr[s] = hh;
        mbar_arrive_expect_tx(&full[s], kbytes * hh.nU + vbytes);
      }
      __syncwarp();
      const float* kbase = static_cast<const float*>(p.kproj) + (size_t)hh.u * p.d_store * p.Tcap + hh.t0;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        const int r = lane + 32 * i;
        if (r < hh.nU) bulk_g2s(st + (size_t)r * TT * 4, kbase + (size_t)urow[i] * p.Tcap, kbytes, &full[s], pol);
      }
      if (lane == 0) {
        const float* vsrc = static_cast<const float*>(p.v) + ((size_t)hh.u * p.Tcap + hh.t0) * vcols;
        bulk_g2s(st + S::KBYTES, vsrc, vbytes, &full[s], pol);
      }
    }
    return;
  }

  float qreg[RMAX][G];
  float oacc[G][4];
  float m_run[G], l_run[G];
  int cur_u = -1;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m_run[h] = -INFINITY;
    l_run[h] = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) oacc[h][e] = 0.f;
  }
#pragma unroll
  for (int i = 0; i < RMAX; ++i)
#pragma unroll
    for (int h = 0; h < G; ++h) qreg[i][h] = 0.f;

  for (int it = 0; it < n_tiles; ++it) {
    const int s = it % NSTAGE;
    const bool ok = mbar_wait_bounded(&full[s], (it / NSTAGE) & 1);
    const StageHdr hh = hdr[s];
    const unsigned char* st = smem + (size_t)s * S::STAGE;
    const float* Ks = reinterpret_cast<const float*>(st);
    const float* Vs = reinterpret_cast<const float*>(st + S::KBYTES);
    const int b = hh.u / p.Hkv, g = hh.u % p.Hkv;

    if (ok && (hh.flags & kFirst)) {
      if (hh.u != cur_u) {
        cur_u = hh.u;
        const float* qmu = p.qm + (size_t)hh.u * D * G;
#pragma unroll
        for (int i = 0; i < RMAX; ++i) {
          const int r = warp + NCW * i;
#pragma unroll
          for (int h = 0; h < G; ++h) qreg[i][h] = r < hh.nU ? __ldg(qmu + (size_t)r * G + h) : 0.f;
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m_run[h] = -INFINITY;
        l_run[h] = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[h][e] = 0.f;
      }
    }

    if (ok) {
      float sacc[G][TPL];
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < TPL; ++e) sacc[h][e] = 0.f;
#pragma unroll
      for (int i = 0; i < RMAX; ++i) {
        const int r = warp + NCW * i;
        if (r < hh.nU) {
          const float2 kf = *reinterpret_cast<const float2*>(Ks + (size_t)r * TT + TPL * lane);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            sacc[h][0] = fmaf(qreg[i][h], kf.x, sacc[h][0]);
            sacc[h][1] = fmaf(qreg[i][h], kf.y, sacc[h][1]);
          }
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < TPL; ++e) red[((size_t)warp * G + h) * S::RW + TPL * lane + e] = sacc[h][e];
    }
    if (named_bar_or(1, NCT, !ok)) {
      if (tid == 0) record_status(p.ctrl, AQUA_ERR_TIMEOUT);
      return;
    }

    float sv[S::SLOTS];
#pragma unroll
    for (int i = 0; i < S::SLOTS; ++i) {
      const int idx = tid + NCT * i;
      sv[i] = -INFINITY;
      if (idx < G * TT) {
        const int h = idx / TT, tok = idx % TT;
        float sacc = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < NCW; ++w2) sacc += red[((size_t)w2 * G + h) * S::RW + tok];
        sv[i] = tok < hh.nvalid ? sacc : -INFINITY;
        const float mx = warp_max(sv[i]);
        if (lane == 0) wmax[i * NCW + warp] = mx;
      }
    }
    named_bar_sync(1, NCT);
    float mnew[G], alpha[G];
#pragma unroll
    for (int h = 0; h < G; ++h) mnew[h] = m_run[h];
#pragma unroll
    for (int i = 0; i < S::SLOTS; ++i)
#pragma unroll
      for (int w2 = 0; w2 < NCW; ++w2) {
        const int idx = NCT * i + 32 * w2;
        if (idx < G * TT) {
          const int h = idx / TT;
#pragma unroll
          for (int x = 0; x < G; ++x)
            if (x == h) mnew[x] = fmaxf(mnew[x], wmax[i * NCW + w2]);
        }
      }
#pragma unroll
    for (int h = 0; h < G; ++h) alpha[h] = exp2f(m_run[h] - mnew[h]);
#pragma unroll
    for (int i = 0; i < S::SLOTS; ++i) {
      const int idx = tid + NCT * i;
      if (idx < G * TT) {
        const int h = idx / TT, tok = idx % TT;
        float mh = 0.f;
#pragma unroll
        for (int x = 0; x < G; ++x)
          if (x == h) mh = mnew[x];
        const float pr = exp2f(sv[i] - mh);
        psm[tok * G + h] = pr;
        const float sm = warp_sum(pr);
        if (lane == 0) wsum[i * NCW + warp] = sm;
        if (p.scores_out != nullptr && tok < hh.nvalid)
          p.scores_out[((size_t)b * p.Hq + g * G + h) * p.Tcap + hh.t0 + tok] = sv[i] * kLn2;
      }
    }
    named_bar_sync(1, NCT);
#pragma unroll
    for (int h = 0; h < G; ++h) l_run[h] *= alpha[h];
#pragma unroll
    for (int i = 0; i < S::SLOTS; ++i)
#pragma unroll
      for (int w2 = 0; w2 < NCW; ++w2) {
        const int idx = NCT * i + 32 * w2;
        if (idx < G * TT) {
          const int h = idx / TT;
#pragma unroll
          for (int x = 0; x < G; ++x)
            if (x == h) l_run[x] += wsum[i * NCW + w2];
        }
      }
#pragma unroll
    for (int h = 0; h < G; ++h) m_run[h] = mnew[h];

#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < 4; ++e) oacc[h][e] *= alpha[h];
#pragma unroll 4
    for (int j = 0; j < TPW; ++j) {
      const int tok = warp * TPW + j;
      if (tok < hh.nvalid && 4 * lane < vcols) {   // V rows hold vcols dims ([TT][vcols] in the stage)
        const float4 vf = *reinterpret_cast<const float4*>(Vs + (size_t)tok * vcols + 4 * lane);
        float pv[G];
#pragma unroll
        for (int h = 0; h < G; ++h) pv[h] = psm[tok * G + h];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          oacc[h][0] = fmaf(pv[h], vf.x, oacc[h][0]);
          oacc[h][1] = fmaf(pv[h], vf.y, oacc[h][1]);
          oacc[h][2] = fmaf(pv[h], vf.z, oacc[h][2]);
          oacc[h][3] = fmaf(pv[h], vf.w, oacc[h][3]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);

    if (!(hh.flags & kLast)) continue;

#pragma unroll
    for (int h = 0; h < G; ++h)
      *reinterpret_cast<float4*>(red + ((size_t)warp * G + h) * S::RW + 4 * lane) =
          make_float4(oacc[h][0], oacc[h][1], oacc[h][2], oacc[h][3]);
    named_bar_sync(1, NCT);
    float merged[(G * D + NCT - 1) / NCT];
#pragma unroll
    for (int i = 0; i < (G * D + NCT - 1) / NCT; ++i) {
      const int idx = tid + NCT * i;
      merged[i] = 0.f;
      if (idx < G * D) {
        const int h = idx / D, dim = idx % D;
        float acc = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < NCW; ++w2) acc += red[((size_t)w2 * G + h) * S::RW + dim];
        merged[i] = acc;
      }
    }
    finish_segment<G>(p, hh, tid, m_run, l_run, merged, s_last);
    named_bar_sync(1, NCT);
  }
  named_bar_sync(1, NCT);               // every consumer warp is done with this CTA's work
  if (tid == 0) step_done(p);
}

// ============================================================================
// projected values: back to the value space
// ============================================================================
// With projected values (AQUA-Memory on the values) the attention kernels
// leave, per query head, o^ over the dv stored projected value dims in the
// workspace; the output is o[i] = sum_{j < dv} o^[j] P[g][i][j] (o^ times the
// transpose of P's first dv columns).  One CTA of 128 threads per (b, g) unit:
// the first dv columns of P[g] are staged in shared memory by coalesced loads
// before the dependency wait (rows padded to dv + 1 floats, so that thread i
// reading row i is free of bank conflicts), then thread i computes output dim
// i of the G heads.  Launched as a programmatic dependent of the attention
// kernel.
constexpr int kVprojThreads = 128;
__host__ __device__ constexpr int vproj_smem_bytes(int dv) { return D * (dv + 1) * 4; }

template <int G>
__global__ void __launch_bounds__(kVprojThreads) vproj_out_kernel(DecodeParams p) {
  extern __shared__ float Pm[];                 // [D][dv + 1]: P[g][i][j], j < dv
  __shared__ float oh[G][D];
  const int u = blockIdx.x;
  const int b = u / p.Hkv, g = u % p.Hkv;
  const int dv = p.dv, ld = dv + 1;
  const size_t bhq0 = (size_t)b * p.Hq + (size_t)g * G;
  const float* Pg = p.P + (size_t)g * D * D;
  // P does not depend on the attention kernel: stage it before the wait
  const int q4 = dv / 4;                        // float4 per row (dv is a multiple of 16)
  for (int idx = threadIdx.x; idx < D * q4; idx += kVprojThreads) {
    const int i = idx / q4, c = idx - i * q4;
    const float4 x = __ldg(reinterpret_cast<const float4*>(Pg + (size_t)i * D) + c);
    float* dst = Pm + i * ld + 4 * c;
    dst[0] = x.x; dst[1] = x.y; dst[2] = x.z; dst[3] = x.w;
  }
  pdl_wait();   // the attention kernel's o^ must be complete
  for (int idx = threadIdx.x; idx < G * D; idx += kVprojThreads) oh[idx / D][idx % D] = __ldcg(p.ohat + bhq0 * D + idx);
  __syncthreads();
  const int i = threadIdx.x;                    // output dim
  float acc[G];
#pragma unroll
  for (int h = 0; h < G; ++h) acc[h] = 0.f;
  const float* prow = Pm + i * ld;
#pragma unroll 8
  for (int j = 0; j < dv; ++j) {
    const float pij = prow[j];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = fmaf(oh[h][j], pij, acc[h]);
  }
#pragma unroll
  for (int h = 0; h < G; ++h) store_val(p, (bhq0 + h) * D + i, acc[h]);
}

// ============================================================================
// host launch
// ============================================================================
template <typename T, int G, int MINB>
int launch_qproj_variant(const DecodeParams& p, int n_units, int smem, cudaStream_t st) {
  const int rc = set_smem_limit(qproj_topk_kernel<T, G, MINB>, smem, "qproj_topk_kernel");
  if (rc != AQUA_OK) return rc;
  const cudaError_t e =
      launch_pdl(qproj_topk_kernel<T, G, MINB>, dim3(n_units), dim3(QprojCfg<G>::WARPS * 32), smem, st, p);
  if (e != cudaSuccess) return set_error(AQUA_ERR_CUDA, "qproj_topk_kernel: %s", cudaGetErrorString(e));
  return check_launch("qproj_topk_kernel");
}

template <typename T, int G>
int launch_qproj(const DecodeParams& p, int n_units, cudaStream_t st) {
  // With no more units than SMs, the dynamic shared memory request is raised
  // above half an SM's so that every CTA gets an SM of its own: the kernel is
  // latency-bound, and CTAs sharing an SM were measured to take twice as long.
  // With more units, two CTAs share each SM (registers capped to fit), rather
  // than a second wave.
  constexpr int kOwnSm = 116 * 1024;
  return n_units <= device_sm_count() ? launch_qproj_variant<T, G, 1>(p, n_units, kOwnSm, st)
                                      : launch_qproj_variant<T, G, 2>(p, n_units, D * D * 4, st);
}

template <int G>
int launch_attn_bf16(const aqua_cache* c, const DecodeParams& p, int C, cudaStream_t st) {
  using S = SmemBF16<G>;
  auto kernel = decode_attn_bf16_kernel<G>;
  int rc = set_smem_limit(kernel, S::BYTES, "decode_attn_bf16_kernel");
  if (rc != AQUA_OK) return rc;
  // The tensor map depends only on the V buffer and its row count; reuse the
  // last encoding while they are unchanged (encoding costs host time every step).
  static thread_local const void* last_base = nullptr;
  static thread_local uint64_t last_rows = 0;
  static thread_local CUtensorMap tmap;
  static thread_local uint64_t last_cols = 0;
  const uint64_t rows = (uint64_t)c->B * c->Hkv * c->Tcap;
  const uint64_t cols = c->dv_store > 0 ? (uint64_t)c->dv_store : (uint64_t)D;   // V row length
  if (last_base != c->v || last_rows != rows || last_cols != cols) {
    if ((rc = encode_tmap_bf16_2d(&tmap, c->v, cols, rows, cols * 2, 64, S::TT, true)) != AQUA_OK) return rc;
    last_base = c->v;
    last_rows = rows;
    last_cols = cols;
  }
  const cudaError_t e = launch_pdl(kernel, dim3(C), dim3(NTHREADS_BF16), S::BYTES, st, tmap, p);
  if (e != cudaSuccess) return set_error(AQUA_ERR_CUDA, "decode_attn_bf16_kernel: %s", cudaGetErrorString(e));
  return check_launch("decode_attn_bf16_kernel");
}

template <int G>
int launch_attn_f32(const DecodeParams& p, int C, cudaStream_t st) {
  using S = SmemF32<G>;
  const int rc = set_smem_limit(decode_attn_f32_kernel<G>, S::BYTES, "decode_attn_f32_kernel");
  if (rc != AQUA_OK) return rc;
  const cudaError_t e = launch_pdl(decode_attn_f32_kernel<G>, dim3(C), dim3(NTHREADS), S::BYTES, st, p);
  if (e != cudaSuccess) return set_error(AQUA_ERR_CUDA, "decode_attn_f32_kernel: %s", cudaGetErrorString(e));
  return check_launch("decode_attn_f32_kernel");
}

template <int G>
int launch_phases(const aqua_cache* c, const DecodeParams& p, int n_units, int C, int phases, cudaStream_t st) {
  const bool bf = c->dtype == AQUA_BF16;
  int rc = AQUA_OK;
  if (phases & kPhaseSelect)
    rc = bf ? launch_qproj<__nv_bfloat16, G>(p, n_units, st) : launch_qproj<float, G>(p, n_units, st);
  if (rc == AQUA_OK && (phases & kPhaseAttend))
    rc = bf ? launch_attn_bf16<G>(c, p, C, st) : launch_attn_f32<G>(p, C, st);
  if (rc == AQUA_OK && (phases & kPhaseAttend) && p.dv > 0) {
    const int smem = vproj_smem_bytes(p.dv);
    if ((rc = set_smem_limit(vproj_out_kernel<G>, smem, "vproj_out_kernel")) != AQUA_OK) return rc;
    const cudaError_t e = launch_pdl(vproj_out_kernel<G>, dim3(n_units), dim3(kVprojThreads), smem, st, p);
    if (e != cudaSuccess) return set_error(AQUA_ERR_CUDA, "vproj_out_kernel: %s", cudaGetErrorString(e));
    rc = check_launch("vproj_out_kernel");
  }
  return rc;
}

}  // namespace

size_t decode_workspace_bytes(int n_units, int G, bool projected_values) {
  size_t off = 0;
  auto take = [&](size_t bytes) { off += (bytes + 255) & ~size_t(255); };
  const size_t nseg = (size_t)n_units + kMaxCtas;
  for (int half = 0; half < 2; ++half) {   // selection buffers, alternating between calls
    take((size_t)n_units * D * G * 4);  // qm
    take((size_t)n_units * D * G * 4);  // qmn
    take((size_t)n_units * D * 4);      // ulist
    take((size_t)n_units * 4);          // ucount
    take((size_t)n_units * 4);          // counters
  }
  take(nseg * G * 2 * 4);             // part_ml
  take(nseg * G * D * 4);             // part_o
  if (projected_values) take((size_t)n_units * G * D * 4);   // ohat
  return off;
}

// Half of a workspace's selection buffers for a call: calls that select flip
// the workspace's half, so that a step's selection never writes the half the
// previous step's attention kernel may still be reading; a call that only
// attends keeps the half.  Kept per workspace address (thread-safe).  The
// record stays bounded however many workspaces a process uses: once it holds
// more than kMaxTracked addresses, those not used in the last kMaxTracked / 2
// calls are dropped (their kernels completed long ago, so they may start again
// from half 0).
int workspace_half(const void* ws, bool flip) {
  constexpr size_t kMaxTracked = 4096;
  struct Entry {
    int half;
    unsigned long long last;   // call count at the latest use
  };
  static std::mutex mu;
  static std::unordered_map<const void*, Entry> halves;
  static unsigned long long calls = 0;
  std::lock_guard<std::mutex> lock(mu);
  ++calls;
  Entry& e = halves[ws];   // a new address starts at half 0
  e.last = calls;
  if (flip) e.half ^= 1;
  const int h = e.half;
  if (halves.size() > kMaxTracked) {
    for (auto it = halves.begin(); it != halves.end();)
      it = (calls - it->second.last >= kMaxTracked / 2) ? halves.erase(it) : std::next(it);
  }
  return h;
}

// One decode step, or one of its phases: kPhaseSelect launches the projection
// and selection kernel (with the fused append when a.k_new is given),
// kPhaseAttend the attention kernel over the selection in the workspace.
int launch_decode(const aqua_cache* c, const DecodeArgs& a, int phases, cudaStream_t st) {
  const int G = a.Hq / c->Hkv;
  const int n_units = c->B * c->Hkv;
  DecodeParams p;
  unsigned char* base = static_cast<unsigned char*>(a.ws);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    void* ptr = base + off;
    off += (bytes + 255) & ~size_t(255);
    return ptr;
  };
  const size_t nseg = (size_t)n_units + kMaxCtas;
  // this call's half of the selection buffers: a call with the selection phase
  // takes the other half than the previous call on this workspace; the
  // attention phase alone uses the half its selection phase wrote
  const int half = workspace_half(a.ws, (phases & kPhaseSelect) != 0);
  for (int h = 0; h < 2; ++h) {
    float* qm = static_cast<float*>(take((size_t)n_units * D * G * 4));
    float* qmn = static_cast<float*>(take((size_t)n_units * D * G * 4));
    int32_t* ulist = static_cast<int32_t*>(take((size_t)n_units * D * 4));
    int32_t* ucount = static_cast<int32_t*>(take((size_t)n_units * 4));
    int32_t* counters = static_cast<int32_t*>(take((size_t)n_units * 4));
    if (h == half) {
      p.qm = qm;
      p.qmn = qmn;
      p.ulist = ulist;
      p.ucount = ucount;
      p.counters = counters;
    }
  }
  p.part_ml = static_cast<float*>(take(nseg * G * 2 * 4));
  p.part_o = static_cast<float*>(take(nseg * G * D * 4));
  p.dv = c->dv_store;
  p.ohat = c->dv_store > 0 ? static_cast<float*>(take((size_t)n_units * G * D * 4)) : nullptr;
  p.q = a.q;
  p.P = a.P;
  p.len = c->len;
  p.kproj = c->k_proj;
  p.v = c->v;
  p.out = a.out;
  p.sel_out = a.sel_out;
  p.qproj_out = a.qproj_out;
  p.scores_out = a.scores_out;
  p.lse_out = a.lse_out;
  p.ctrl = c->ctrl;
  p.k_new = (phases & kPhaseSelect) ? a.k_new : nullptr;
  p.v_new = (phases & kPhaseSelect) ? a.v_new : nullptr;
  p.len_w = c->len;
  p.len_add = a.appended ? 1 : 0;
  // the projection kernel gives each of its CTAs an SM of its own when there
  // are no more units than SMs; that many attention CTAs then start late
  p.n_late = n_units <= device_sm_count() ? n_units : 0;
  p.early_select = n_units > device_sm_count() ? 1 : 0;
  p.n_abs = c->n_abs;
  p.pos = c->pos;
  p.score = c->score;
  p.B = c->B;
  p.Hq = a.Hq;
  p.Hkv = c->Hkv;
  p.d_store = c->d_store;
  p.Tcap = c->Tcap;
  p.k = a.k;
  p.out_bf16 = a.out_dtype == AQUA_BF16;
  p.scale_log2 = a.scale * kLog2e;
  const bool bf = c->dtype == AQUA_BF16;
  const int TT = bf ? SmemBF16<1>::TT : SmemF32<1>::TT;
  // host bound of the tokens attended: the selection phase has not yet counted
  // the token it appends in cache->max_len, the attention phase alone has
  const int max_len = c->max_len + ((phases & kPhaseSelect) && a.appended ? 1 : 0);
  const long long tiles_ub = (long long)n_units * ((max_len + TT - 1) / TT);
  long long C = device_sm_count();
  if (C > tiles_ub) C = tiles_ub;
  if (C < 1) C = 1;
  if (C > kMaxCtas) C = kMaxCtas;
  switch (G) {
    case 1: return launch_phases<1>(c, p, n_units, (int)C, phases, st);
    case 2: return launch_phases<2>(c, p, n_units, (int)C, phases, st);
    case 4: return launch_phases<4>(c, p, n_units, (int)C, phases, st);
    default: return set_error(AQUA_ERR_UNSUPPORTED, "decode: Hq/Hkv = %d not in {1,2,4}", G);
  }
}

}  // namespace aqua
