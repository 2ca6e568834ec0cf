// Chunked causal AQUA prefill on the tcgen05 tensor cores (sm_100a).
//
// For a chunk of L prompt tokens at absolute positions pos0 .. pos0+L-1 (their
// keys already appended), every (row i, query head h) projects its query,
// keeps its k largest |q~| dimensions (ties to the lower index), and attends
// causally to tokens 0 .. pos0+i with scores on those dimensions only
// (AQUA abstract; edgentiq, "How AQUA Works": project, select by query
// magnitude, attend on the selected dimensions; the per-query mask makes the
// score a dense contraction over a masked q~).
//
// prefill_select_kernel: one warp per (row, head): q~ = q P[g] (f32, shared
//   routine), radix select, masked q~ * scale * log2(e) split into bf16 high
//   and low parts, written row-major in (b, g, row, head) order.
// prefill_attn_kernel: one CTA per (b, g, block of 128/G rows), i.e. 128 query
//   rows of one GQA group that share every K~/V tile.  Warp roles:
//     warps 0-3  softmax (thread r <-> TMEM lane r <-> query row r)
//     warp 4     TMEM allocation and the single thread issuing tcgen05.mma
//     warp 5     TMA producer
//   Per 128-token KV tile: S = Qh K~ + Ql K~ (M=128, N=128, K=d_store) into
//   TMEM, causal mask, online softmax with a lazily raised running max,
//   P split into bf16 high/low parts in shared memory, O += Ph V + Pl V
//   (K=128 tokens, N=128 dims) into TMEM.  Operands are 128B-swizzled tiles:
//   Q~m and P K-major, the dimension-major K~ and token-major V MN-major.
#include <math.h>

#include "aqua_internal.cuh"

namespace aqua {

namespace {

constexpr int D = kHeadDim;
constexpr int PM = 128;          // query rows per CTA (TMEM lanes)
constexpr int PN = 128;          // tokens per KV tile
constexpr int kSelWarps = 8;     // selection kernel: warps per CTA
constexpr int kSelRows = 64;     // selection kernel: (row, head) pairs per CTA
constexpr int kAttnThreads = 192;
constexpr float kLazy = 8.0f;    // running max raised only when exceeded by 2^8

// ------------------------------------------------------------------ tcgen05 wrappers
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16 (bf16 in, f32 accumulate)
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
      : "memory");
}

// arrive on `bar` once all tcgen05.mma issued so far by this thread complete
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 32 consecutive f32 columns of this warp's 32 TMEM lanes
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
      "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
      "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
      "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
      "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
      "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
      "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
      "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle (sm100 layout: version 1,
// layout type 2).  lbo/sbo in bytes.
__device__ __forceinline__ uint64_t smem_desc_sw128(const void* p, uint32_t lbo, uint32_t sbo) {
  const uint64_t start = (smem_u32(p) >> 4) & 0x3FFF;
  return start | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) | ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) |
         (2ull << 61);
}

// kind::f16 instruction descriptor: bf16 A and B, f32 D, A K-major, B MN-major, M x N
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

struct PrefillParams {
  const void* q;             // [B][L][Hq][D] bf16
  const float* P;            // [Hkv][D][D]
  __nv_bfloat16* qm;         // [2][B*Hkv*L*G][D]: masked scaled q~, high part then low part
  void* out;                 // [B][L][Hq][D]
  int32_t* sel_out;          // nullable [B][L][Hq][k]
  int32_t* ctrl;
  int B, L, Hq, Hkv, d_store, Tcap, k, pos0;
  int out_bf16;
  float scale_log2;
};

// ============================================================================
// selection: q~ = q P, top-k by |q~|, masked pre-scaled rows as bf16 hi / lo
// ============================================================================
template <int G>
__global__ void __launch_bounds__(kSelWarps * 32) prefill_select_kernel(PrefillParams p) {
  extern __shared__ __align__(128) float Ps[];
  __shared__ __align__(16) float xs[kSelWarps][D];
  __shared__ __align__(8) uint64_t pbar;
  const int g = blockIdx.y, b = blockIdx.z;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t rows_total = (size_t)p.B * p.Hkv * p.L * G;
  if (threadIdx.x == 0) {
    mbar_init(&pbar, 1);
    fence_barrier_init();
  }
  pdl_launch_dependents();
  pdl_wait();
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&pbar, D * D * 4);
    bulk_g2s_plain(Ps, p.P + (size_t)g * D * D, D * D * 4, &pbar);
  }
  const bool ok = mbar_wait_bounded(&pbar, 0);
  if (__syncthreads_or(!ok)) {
    if (threadIdx.x == 0) record_status(p.ctrl, AQUA_ERR_TIMEOUT);
    return;
  }
  const int m = p.d_store;
  for (int i = w; i < kSelRows; i += kSelWarps) {
    const int pair = blockIdx.x * kSelRows + i;    // (row l, head hh) within this (b, g)
    const int l = pair / G, hh = pair % G;
    if (l >= p.L) break;
    const int h = g * G + hh;
    const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(p.q) + (((size_t)b * p.L + l) * p.Hq + h) * D;
#pragma unroll
    for (int s = 0; s < 4; ++s) xs[w][4 * lane + s] = __bfloat162float(qrow[4 * lane + s]);
    __syncwarp();
    float qt[4];
    project_row_smem(Ps, xs[w], lane, qt);
    __syncwarp();
    uint32_t key[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int j = 4 * lane + s;
      key[s] = (j < m) ? (__float_as_uint(fabsf(qt[s])) + 1u) : 0u;
    }
    uint32_t tau = 0;
#pragma unroll 4
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = tau | (1u << bit);
      const int c = __popc(__ballot_sync(0xffffffffu, key[0] >= cand)) +
                    __popc(__ballot_sync(0xffffffffu, key[1] >= cand)) +
                    __popc(__ballot_sync(0xffffffffu, key[2] >= cand)) +
                    __popc(__ballot_sync(0xffffffffu, key[3] >= cand));
      if (c >= p.k) tau = cand;
    }
    int ngt = 0, neq = 0;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      ngt += __popc(__ballot_sync(0xffffffffu, key[s] > tau));
      neq += (key[s] == tau);
    }
    const int need = p.k - ngt;
    int incl = neq;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int rank = incl - neq;
    bool sel[4];
    int nsel = 0;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      sel[s] = key[s] > tau;
      if (key[s] == tau) {
        sel[s] = rank < need;
        ++rank;
      }
      nsel += sel[s];
    }
    if (p.sel_out) {
      int pincl = nsel;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, pincl, o);
        if (lane >= o) pincl += y;
      }
      int opos = pincl - nsel;
      int32_t* so = p.sel_out + (((size_t)b * p.L + l) * p.Hq + h) * p.k;
#pragma unroll
      for (int s = 0; s < 4; ++s)
        if (sel[s]) so[opos++] = 4 * lane + s;
    }
    const size_t row = (((size_t)b * p.Hkv + g) * p.L + l) * G + hh;
    __nv_bfloat16* hi_row = p.qm + row * D;
    __nv_bfloat16* lo_row = p.qm + (rows_total + row) * D;
    float hv[4], lv[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) split_bf16(sel[s] ? qt[s] * p.scale_log2 : 0.f, hv[s], lv[s]);
    *reinterpret_cast<uint2*>(hi_row + 4 * lane) = make_uint2(pack_bf16(hv[0], hv[1]), pack_bf16(hv[2], hv[3]));
    *reinterpret_cast<uint2*>(lo_row + 4 * lane) = make_uint2(pack_bf16(lv[0], lv[1]), pack_bf16(lv[2], lv[3]));
  }
}

// ============================================================================
// causal attention on tcgen05
// ============================================================================
struct AttnSmem {
  static constexpr int TILE = PM * 128;              // 128 rows x 128 B = 16 KB (one 64-column half)
  static constexpr int OFF_QH = 0;                   // [2 halves][128 rows][128 B]
  static constexpr int OFF_QL = OFF_QH + 2 * TILE;
  static constexpr int OFF_K = OFF_QL + 2 * TILE;    // [2 token halves][<=128 dims][128 B]
  static constexpr int OFF_V = OFF_K + 2 * TILE;     // [2 dim halves][128 tokens][128 B]
  static constexpr int OFF_PH = OFF_V + 2 * TILE;    // [2 token halves][128 rows][128 B]
  static constexpr int OFF_PL = OFF_PH + 2 * TILE;
  static constexpr int OFF_BAR = OFF_PL + 2 * TILE;  // 8 mbarriers
  static constexpr int OFF_MISC = OFF_BAR + 8 * 8;
  static constexpr int USED = OFF_MISC + 64;
  static constexpr int BYTES = USED + 1024;          // + slack to align the base to the 1024-byte swizzle period
};
enum { BAR_Q = 0, BAR_K, BAR_V, BAR_S, BAR_P, BAR_O, BAR_DRAIN };

template <int G>
__global__ void __launch_bounds__(kAttnThreads, 1)
    prefill_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, PrefillParams p) {
  using S = AttnSmem;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // The 128B swizzle pattern (TMA, tcgen05 descriptors and the hand-written P
  // tiles) is a function of address bits 4-9: every tile starts on a 1024-byte boundary.
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::OFF_MISC + 4);

  constexpr int RPB = PM / G;                         // prompt rows (positions) per CTA
  const int qb = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int l0 = qb * RPB;
  const int l_end = min(p.L, l0 + RPB);
  const int kv_valid = p.pos0 + p.L;                  // keys present in the cache for this chunk
  const int kv_end = p.pos0 + l_end;                  // keys visible to some row of this CTA
  const int n_tiles = (kv_end + PN - 1) / PN;
  const int DS = p.d_store;                           // contraction length of Q K~^T (multiple of 16)
  const int unit = b * p.Hkv + g;

  if (tid == 0) {
    for (int i = 0; i <= BAR_DRAIN; ++i) mbar_init(&bars[i], i == BAR_P ? 128 : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, 256);                       // S: columns [0,128), O: [128,256)
    tmem_relinquish();
  }
  if (tid == 160) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  pdl_launch_dependents();
  pdl_wait();                                         // the selection kernel wrote q~m
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_S = tmem, tm_O = tmem + 128;

  if (warp == 5) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const int qrow = ((unit * p.L) + l0) * G;
      const int rows_total = p.B * p.Hkv * p.L * G;
      mbar_arrive_expect_tx(&bars[BAR_Q], 4 * S::TILE);
      tma_load_2d(smem + S::OFF_QH, &tm_q, 0, qrow, &bars[BAR_Q], pol);
      tma_load_2d(smem + S::OFF_QH + S::TILE, &tm_q, 64, qrow, &bars[BAR_Q], pol);
      tma_load_2d(smem + S::OFF_QL, &tm_q, 0, rows_total + qrow, &bars[BAR_Q], pol);
      tma_load_2d(smem + S::OFF_QL + S::TILE, &tm_q, 64, rows_total + qrow, &bars[BAR_Q], pol);
      const uint32_t kbytes = 2u * DS * 128u;
      int nk = 0, nv = 0;                             // K~ and V tiles issued
      for (int j = 0; j < n_tiles && !*abort_flag; ++j) {
        const int t0 = j * PN;
        if (j > 0 && !mbar_wait_bounded(&bars[BAR_S], (j - 1) & 1)) { *abort_flag = 1; break; }   // K~ buffer free
        mbar_arrive_expect_tx(&bars[BAR_K], kbytes);
        tma_load_2d(smem + S::OFF_K, &tm_k, t0, unit * DS, &bars[BAR_K], pol);
        tma_load_2d(smem + S::OFF_K + DS * 128, &tm_k, t0 + 64, unit * DS, &bars[BAR_K], pol);
        ++nk;
        if (j > 0 && !mbar_wait_bounded(&bars[BAR_O], (j - 1) & 1)) { *abort_flag = 1; break; }   // V buffer free
        mbar_arrive_expect_tx(&bars[BAR_V], 2 * S::TILE);
        tma_load_2d(smem + S::OFF_V, &tm_v, 0, unit * p.Tcap + t0, &bars[BAR_V], pol);
        tma_load_2d(smem + S::OFF_V + S::TILE, &tm_v, 64, unit * p.Tcap + t0, &bars[BAR_V], pol);
        ++nv;
      }
      // Before the CTA exits, every copy it issued must have landed (normally
      // they all have been consumed already; after an abort this is the drain).
      bool drained = mbar_wait_bounded(&bars[BAR_Q], 0);
      if (nk > 0) drained = mbar_wait_bounded(&bars[BAR_K], (nk - 1) & 1) && drained;
      if (nv > 0) drained = mbar_wait_bounded(&bars[BAR_V], (nv - 1) & 1) && drained;
      if (!drained) *abort_flag = 1;
    }
  } else if (warp == 4) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(PM, 128);
      bool ok = mbar_wait_bounded(&bars[BAR_Q], 0);
      for (int j = 0; j < n_tiles && ok; ++j) {
        ok = mbar_wait_bounded(&bars[BAR_K], j & 1);
        if (ok && j > 0) ok = mbar_wait_bounded(&bars[BAR_P], (j - 1) & 1);    // softmax done with S(j-1)
        if (!ok) break;
        tc_fence_after();
        // S = Qh K~ + Ql K~: A K-major (32 B per k-step inside a 64-column half), B MN-major
        int n = 0;
        for (int part = 0; part < 2; ++part) {
          const unsigned char* qa = smem + (part == 0 ? S::OFF_QH : S::OFF_QL);
          for (int ks = 0; ks < DS / 16; ++ks, ++n) {
            const uint64_t ad = smem_desc_sw128(qa + (ks >> 2) * S::TILE + (ks & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(smem + S::OFF_K + ks * 16 * 128, DS * 128, 1024);
            tc_mma(tm_S, ad, bd, idesc, n > 0);
          }
        }
        tc_commit(&bars[BAR_S]);
        ok = mbar_wait_bounded(&bars[BAR_V], j & 1) && mbar_wait_bounded(&bars[BAR_P], j & 1);
        if (!ok) break;
        tc_fence_after();
        // O += Ph V + Pl V
        for (int part = 0; part < 2; ++part) {
          const unsigned char* pa = smem + (part == 0 ? S::OFF_PH : S::OFF_PL);
          for (int ks = 0; ks < PN / 16; ++ks) {
            const uint64_t ad = smem_desc_sw128(pa + (ks >> 2) * S::TILE + (ks & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(smem + S::OFF_V + ks * 16 * 128, S::TILE, 1024);
            tc_mma(tm_O, ad, bd, idesc, j > 0 || part > 0 || ks > 0);
          }
        }
        tc_commit(&bars[BAR_O]);
      }
      if (!ok) *abort_flag = 1;
      // wait for every MMA this thread issued before TMEM may be released
      tc_commit(&bars[BAR_DRAIN]);
      if (!mbar_wait_bounded(&bars[BAR_DRAIN], 0)) *abort_flag = 1;
    }
  } else {
    // ======================= softmax warps (row r = tid) =======================
    const int r = tid;
    const int lr = l0 + r / G;                       // prompt row of this TMEM lane
    const int pos_r = p.pos0 + lr;                   // last visible token
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float mu = -INFINITY, ell = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles && ok; ++j) {
      const int t0 = j * PN;
      ok = mbar_wait_bounded(&bars[BAR_S], j & 1);
      if (!ok) break;
      tc_fence_after();
      float s[PN];
#pragma unroll
      for (int c = 0; c < PN; c += 32) tmem_ld32(tm_S + lane_base + c, *reinterpret_cast<float(*)[32]>(&s[c]));
      tmem_wait_ld();
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < PN; ++c) {
        if (t0 + c > pos_r) s[c] = -INFINITY;
        mx = fmaxf(mx, s[c]);
      }
      // the previous PV must be complete before O is rescaled or P is rewritten
      if (j > 0) {
        ok = mbar_wait_bounded(&bars[BAR_O], (j - 1) & 1);
        if (!ok) break;
        tc_fence_after();
      }
      if (mx > mu + kLazy) {
        const float alpha = exp2f(mu - mx);          // 0 on the first visible tile
        if (j > 0 && mu > -INFINITY) {
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            float o[32];
            tmem_ld32(tm_O + lane_base + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tm_O + lane_base + c, o);
          }
          tmem_wait_st();
        }
        ell *= alpha;
        mu = mx;
      }
      // P = exp2(s - mu), high and low bf16 parts, K-major 128B-swizzled rows
      unsigned char* ph = smem + S::OFF_PH;
      unsigned char* pl = smem + S::OFF_PL;
      float rs = 0.f;
#pragma unroll
      for (int c8 = 0; c8 < PN / 8; ++c8) {
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = (mu == -INFINITY) ? 0.f : exp2f(s[8 * c8 + 2 * e] - mu);
          const float p1 = (mu == -INFINITY) ? 0.f : exp2f(s[8 * c8 + 2 * e + 1] - mu);
          rs += p0 + p1;
          float h0, lo0, h1, lo1;
          split_bf16(p0, h0, lo0);
          split_bf16(p1, h1, lo1);
          hw[e] = pack_bf16(h0, h1);
          lw[e] = pack_bf16(lo0, lo1);
        }
        const int half = c8 >> 3, chunk = c8 & 7;
        const int off = half * S::TILE + r * 128 + ((chunk ^ (r & 7)) << 4);
        *reinterpret_cast<uint4*>(ph + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(pl + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      ell += rs;
      // tokens past the chunk's keys are not in the cache yet: their V rows must be finite
      if (t0 + PN > kv_valid) {
        ok = mbar_wait_bounded(&bars[BAR_V], j & 1);
        if (!ok) break;
        if (t0 + r >= kv_valid) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            *reinterpret_cast<uint4*>(smem + S::OFF_V + r * 128 + c * 16) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(smem + S::OFF_V + S::TILE + r * 128 + c * 16) = make_uint4(0, 0, 0, 0);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[BAR_P]);
    }
    // epilogue: O / l
    if (ok) ok = mbar_wait_bounded(&bars[BAR_O], (n_tiles - 1) & 1);
    if (ok) {
      tc_fence_after();
      const bool live = lr < l_end;
      const int h = g * G + (r % G);
      const size_t obase = (((size_t)b * p.L + lr) * p.Hq + h) * D;
      const float inv = 1.f / ell;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        float o[32];
        tmem_ld32(tm_O + lane_base + c, o);
        tmem_wait_ld();
        if (live) {
          if (p.out_bf16) {
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + obase + c;
#pragma unroll
            for (int i = 0; i < 32; i += 8)
              *reinterpret_cast<uint4*>(dst + i) =
                  make_uint4(pack_bf16(o[i] * inv, o[i + 1] * inv), pack_bf16(o[i + 2] * inv, o[i + 3] * inv),
                             pack_bf16(o[i + 4] * inv, o[i + 5] * inv), pack_bf16(o[i + 6] * inv, o[i + 7] * inv));
          } else {
            float* dst = static_cast<float*>(p.out) + obase + c;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(dst + i) = make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv);
          }
        }
      }
    }
    if (!ok) *abort_flag = 1;
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && tid == 0) record_status(p.ctrl, AQUA_ERR_TIMEOUT);
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int G>
int launch_prefill_g(const aqua_cache* c, const PrefillParams& p, cudaStream_t st) {
  static bool configured = false;
  if (!configured) {
    if (cudaFuncSetAttribute(prefill_select_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, D * D * 4) !=
            cudaSuccess ||
        cudaFuncSetAttribute(prefill_attn_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, AttnSmem::BYTES) !=
            cudaSuccess)
      return check_launch("cudaFuncSetAttribute(prefill)");
    configured = true;
  }
  const uint64_t rows_total = (uint64_t)p.B * p.Hkv * p.L * G;
  CUtensorMap tq, tk, tv;
  int rc = encode_tmap_bf16_2d(&tq, p.qm, D, 2 * rows_total, D * 2, 64, PM, true);
  if (rc == AQUA_OK)
    rc = encode_tmap_bf16_2d(&tk, c->k_proj, (uint64_t)c->Tcap, (uint64_t)c->B * c->Hkv * c->d_store,
                             (uint64_t)c->Tcap * 2, 64, (uint32_t)c->d_store, true);
  if (rc == AQUA_OK)
    rc = encode_tmap_bf16_2d(&tv, c->v, D, (uint64_t)c->B * c->Hkv * c->Tcap, D * 2, 64, PN, true);
  if (rc != AQUA_OK) return rc;
  dim3 gsel((p.L * G + kSelRows - 1) / kSelRows, p.Hkv, p.B);
  cudaError_t e = launch_pdl(prefill_select_kernel<G>, gsel, dim3(kSelWarps * 32), D * D * 4, st, p);
  if (e != cudaSuccess) return set_error(AQUA_ERR_CUDA, "prefill_select_kernel: %s", cudaGetErrorString(e));
  if ((rc = check_launch("prefill_select_kernel")) != AQUA_OK) return rc;
  dim3 gattn((p.L + PM / G - 1) / (PM / G), p.Hkv, p.B);
  e = launch_pdl(prefill_attn_kernel<G>, gattn, dim3(kAttnThreads), AttnSmem::BYTES, st, tq, tk, tv, p);
  if (e != cudaSuccess) return set_error(AQUA_ERR_CUDA, "prefill_attn_kernel: %s", cudaGetErrorString(e));
  return check_launch("prefill_attn_kernel");
}

}  // namespace

size_t prefill_workspace_bytes(const aqua_cache* c, int Hq, int L) {
  return 2ull * (size_t)c->B * L * Hq * D * 2 + 256;   // q~m high and low parts
}

int launch_prefill(const aqua_cache* c, const void* q, int pos0, int L, const float* P, int Hq, int k, float scale,
                   void* out, int out_dtype, int32_t* sel_out, void* ws, cudaStream_t st) {
  if (c->d_store % 16 != 0)
    return set_error(AQUA_ERR_UNSUPPORTED, "aqua_prefill_attn: d_store %d must be a multiple of 16", c->d_store);
  PrefillParams p;
  p.q = q;
  p.P = P;
  p.qm = static_cast<__nv_bfloat16*>(ws);
  p.out = out;
  p.sel_out = sel_out;
  p.ctrl = c->ctrl;
  p.B = c->B;
  p.L = L;
  p.Hq = Hq;
  p.Hkv = c->Hkv;
  p.d_store = c->d_store;
  p.Tcap = c->Tcap;
  p.k = k;
  p.pos0 = pos0;
  p.out_bf16 = out_dtype == AQUA_BF16;
  p.scale_log2 = scale * kLog2e;
  switch (Hq / c->Hkv) {
    case 1: return launch_prefill_g<1>(c, p, st);
    case 2: return launch_prefill_g<2>(c, p, st);
    case 4: return launch_prefill_g<4>(c, p, st);
    default: return set_error(AQUA_ERR_UNSUPPORTED, "aqua_prefill_attn: Hq/Hkv = %d not in {1,2,4}", Hq / c->Hkv);
  }
}

}  // namespace aqua
