// H2O heavy-hitter update on top of AQUA decode.
//
// The AQUA abstract names H2O (AQUA combines with token eviction methods such
// as H2O and speeds them up) without giving its rule; the reading taken:
// every cached token of a (sequence, KV head) carries a cumulative score, the
// sum over the group's query heads and over the decode steps it has seen of
// its AQUA softmax probability; after a step that leaves more than `budget`
// tokens, the lowest-scored token outside the `recent` newest positions is
// evicted (ties to the older position) and its slot is reused.
#include <math.h>

#include "aqua_internal.cuh"

namespace aqua {

namespace {

constexpr int D = kHeadDim;
constexpr int kThreads = 256;

struct Cand {
  float score;
  int pos;
  int slot;
};

__device__ __forceinline__ bool better(const Cand& a, const Cand& b) {
  if (a.slot < 0) return false;
  if (b.slot < 0) return true;
  return a.score < b.score || (a.score == b.score && a.pos < b.pos);
}

constexpr int kTokPerThread = 9;   // tokens whose loads one thread issues together (2304 per pass)

template <typename T, int G>
__global__ void __launch_bounds__(kThreads) h2o_update_kernel(T* __restrict__ kproj, T* __restrict__ vcache,
                                                              int32_t* len, const int32_t* __restrict__ n_abs,
                                                              int32_t* __restrict__ pos, float* __restrict__ score,
                                                              int32_t* ctrl, const float* __restrict__ scores,
                                                              const float* __restrict__ lse, int32_t* evicted_out,
                                                              int B, int Hq, int Hkv, int d_store, int Tcap,
                                                              int budget, int recent, int vcols) {
  __shared__ Cand wbest[kThreads / 32];
  __shared__ int s_victim, s_vpos, is_last;
  const int u = blockIdx.x;
  const int b = u / Hkv, g = u % Hkv;
  // launched as a dependent of the decode step: every input below is its output
  pdl_wait();
  // the next kernel may start now: a decode step's projection kernel reads only
  // q and P and writes its own workspace half before it waits for this kernel
  pdl_launch_dependents();
  const int n = min(max(__ldcg(len + b), 0), Tcap);   // read before the ticket below
  const int newest = __ldcg(n_abs + b) - 1;
  const size_t ub = (size_t)u * Tcap;
  const size_t bh0 = (size_t)b * Hq + (size_t)g * G;   // first query head of the group
  float lse_h[G];
#pragma unroll
  for (int x = 0; x < G; ++x) lse_h[x] = lse[bh0 + x];

  // Per slot t: score[t] += sum over the group's heads (in head order) of
  // exp(scores - lse); candidates are the slots outside the recent window.
  // A thread issues the loads of kTokPerThread slots before using any of
  // them: the kernel is bound by memory latency, not bandwidth.
  // the last slot's key column and value row, read ahead of the arg-min:
  // they move into the victim's slot if one is evicted
  const int last = n - 1;
  T* kp = kproj + (size_t)u * d_store * Tcap;
  T* vp = vcache + ub * vcols;                        // V rows of vcols elements (projected values: dv)
  T klast = T(0.f), vlast = T(0.f);
  if (n > budget) {
    if (threadIdx.x < d_store) klast = kp[(size_t)threadIdx.x * Tcap + last];
    if (threadIdx.x < vcols) vlast = vp[(size_t)last * vcols + threadIdx.x];
  }
  Cand best{INFINITY, 0, -1};
  for (int tb = threadIdx.x; tb < n; tb += kThreads * kTokPerThread) {
    float sv[kTokPerThread][G], scv[kTokPerThread];
    int psv[kTokPerThread];
#pragma unroll
    for (int r = 0; r < kTokPerThread; ++r) {
      const int t = tb + r * kThreads;
      if (t < n) {
#pragma unroll
        for (int x = 0; x < G; ++x) sv[r][x] = scores[(bh0 + x) * Tcap + t];
        scv[r] = score[ub + t];
        psv[r] = pos[ub + t];
      }
    }
#pragma unroll
    for (int r = 0; r < kTokPerThread; ++r) {
      const int t = tb + r * kThreads;
      if (t < n) {
        float acc = 0.f;
#pragma unroll
        for (int x = 0; x < G; ++x) acc += expf(sv[r][x] - lse_h[x]);
        const float sc = scv[r] + acc;
        score[ub + t] = sc;
        if (psv[r] <= newest - recent) {
          const Cand cnd{sc, psv[r], t};
          if (better(cnd, best)) best = cnd;
        }
      }
    }
  }
  // block arg-min
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Cand other;
    other.score = __shfl_xor_sync(0xffffffffu, best.score, o);
    other.pos = __shfl_xor_sync(0xffffffffu, best.pos, o);
    other.slot = __shfl_xor_sync(0xffffffffu, best.slot, o);
    if (better(other, best)) best = other;
  }
  if ((threadIdx.x & 31) == 0) wbest[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    Cand bb = wbest[0];
    for (int w = 1; w < kThreads / 32; ++w)
      if (better(wbest[w], bb)) bb = wbest[w];
    const bool evict = n > budget && bb.slot >= 0;
    s_victim = evict ? bb.slot : -1;
    s_vpos = evict ? bb.pos : -1;
    if (evicted_out) evicted_out[u] = s_vpos;
  }
  __syncthreads();
  const int v = s_victim;
  if (v >= 0 && v != last) {
    // move the last slot into the evicted one
    static_assert(kThreads >= D, "one thread per key dimension and value element");
    if (threadIdx.x < d_store) kp[(size_t)threadIdx.x * Tcap + v] = klast;
    if (threadIdx.x < vcols) vp[(size_t)v * vcols + threadIdx.x] = vlast;
    if (threadIdx.x == 0) {
      pos[ub + v] = pos[ub + last];
      score[ub + v] = score[ub + last];
    }
  }
  // the last CTA shortens the sequences that evicted (all KV heads of a
  // sequence evict together: they hold the same number of tokens and the same
  // recent window)
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    is_last = (atomicAdd(ctrl + kCtrlH2OTicket, 1) == (int)gridDim.x - 1);
  }
  __syncthreads();
  if (is_last) {
    __threadfence();
    for (int bb = threadIdx.x; bb < B; bb += kThreads) {
      const int nb = len[bb];
      // eviction happened iff the sequence was over budget and some slot lay
      // outside the recent window (the recent positions are always present)
      if (nb > budget && nb - min(recent, n_abs[bb]) > 0) len[bb] = nb - 1;
    }
    if (threadIdx.x == 0) ctrl[kCtrlH2OTicket] = 0;
  }
}

template <int G>
int launch_h2o_g(aqua_cache* c, const float* scores, const float* lse, int Hq, int budget, int recent,
                  int32_t* evicted_out, int n_units, cudaStream_t st) {
  // programmatic dependent launch: the grid is resident as the decode step's
  // CTAs retire and starts the moment the step completes (it waits first)
  cudaError_t e;
  if (c->dtype == AQUA_BF16) {
    e = launch_pdl(h2o_update_kernel<__nv_bfloat16, G>, dim3(n_units), dim3(kThreads), 0, st,
                   static_cast<__nv_bfloat16*>(c->k_proj), static_cast<__nv_bfloat16*>(c->v), c->len,
                   (const int32_t*)c->n_abs, c->pos, c->score, c->ctrl, scores, lse, evicted_out, c->B, Hq,
                   c->Hkv, c->d_store, c->Tcap, budget, recent, c->dv_store > 0 ? c->dv_store : D);
  } else {
    e = launch_pdl(h2o_update_kernel<float, G>, dim3(n_units), dim3(kThreads), 0, st,
                   static_cast<float*>(c->k_proj), static_cast<float*>(c->v), c->len, (const int32_t*)c->n_abs,
                   c->pos, c->score, c->ctrl, scores, lse, evicted_out, c->B, Hq, c->Hkv, c->d_store, c->Tcap,
                   budget, recent, c->dv_store > 0 ? c->dv_store : D);
  }
  if (e != cudaSuccess) return set_error(AQUA_ERR_CUDA, "h2o_update_kernel: %s", cudaGetErrorString(e));
  return AQUA_OK;
}

}  // namespace

int launch_h2o_update(aqua_cache* c, const float* scores, const float* lse, int Hq, int budget, int recent,
                      int32_t* evicted_out, cudaStream_t st) {
  const int n_units = c->B * c->Hkv;
  int rc;
  switch (Hq / c->Hkv) {
    case 1: rc = launch_h2o_g<1>(c, scores, lse, Hq, budget, recent, evicted_out, n_units, st); break;
    case 2: rc = launch_h2o_g<2>(c, scores, lse, Hq, budget, recent, evicted_out, n_units, st); break;
    case 4: rc = launch_h2o_g<4>(c, scores, lse, Hq, budget, recent, evicted_out, n_units, st); break;
    default: return set_error(AQUA_ERR_UNSUPPORTED, "aqua_h2o_update: Hq/Hkv = %d not in {1,2,4}", Hq / c->Hkv);
  }
  if (rc != AQUA_OK) return rc;
  return check_launch("h2o_update_kernel");
}

}  // namespace aqua
