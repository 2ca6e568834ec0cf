// Chunked causal AQUA prefill on the tcgen05 tensor cores (sm_100a).
//
// For a chunk of L prompt tokens at absolute positions pos0 .. pos0+L-1 (their
// keys already appended), every (row i, query head h) projects its query,
// keeps its k largest |q~| dimensions (ties to the lower index), and attends
// causally to tokens 0 .. pos0+i with scores on those dimensions only
// (AQUA abstract; edgentiq, "How AQUA Works": project, select by query
// magnitude, attend on the selected dimensions).  The per-row mask turns the
// score into a dense contraction over a masked q~, which runs on tcgen05.
//
// One kernel, one CTA per (sequence b, KV head g, block of 128/G prompt rows):
// the 128 TMEM lanes are the 128 (row, head) query rows of one GQA group, which
// share every K~/V tile.  Warp roles (320 threads):
//   warps 0-3  softmax warpgroup 0: S columns 0-63 / O columns 0-63, and the
//              per-row top-k selection in the prologue
//   warps 4-7  softmax warpgroup 1: S columns 64-127 / O columns 64-127
//   warp 8     TMEM allocation and the single thread issuing tcgen05.mma
//   warp 9     TMA producer
// Prologue: q~ = q P on the tensor cores (P split into three bf16 parts, f32
// accumulation, so q~ carries ~24 bits), selection per row from TMEM, masked
// q~ * scale * log2(e) written to TMEM as bf16 high and low parts.
// Per 128-token KV tile j: S = Qh K~ + Ql K~ (M=128, N=128, K=d_store; A from
// TMEM, B from shared memory) into TMEM; the softmax warps copy S to registers
// and release it, so S(j+1) is
// computed while tile j's softmax runs (K~ and V tiles double-buffered); causal
// mask on diagonal tiles, online softmax with a lazily raised running max, P
// split into bf16 high/low parts written to tensor memory, O += Ph V + Pl V with
// the A operand read from tensor memory (P never goes through shared memory).
// The softmax warpgroups' per-tile work, not the MMAs, sets the tile time.
#include <math.h>

#include "aqua_internal.cuh"

namespace aqua {

namespace {

constexpr int D = kHeadDim;
constexpr int PM = 128;          // query rows per CTA (TMEM lanes)
constexpr int PN = 128;          // tokens per KV tile
constexpr int kAttnThreads = 320;
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

// D[tmem] (+)= A[tmem] * B[smem desc]: A (M rows x K) read from tensor memory,
// row i in lane i, 16-bit elements packed two per 32-bit column (K-major)
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
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
  const float* P;            // [Hkv][D][D]
  void* out;                 // [B][L][Hq][D]
  int32_t* sel_out;          // nullable [B][L][Hq][k]
  float* qproj_out;          // nullable [B][L][Hq][D]: the q~ the selection used
  int32_t* ctrl;
  int B, L, Hq, Hkv, d_store, Tcap, k, pos0;
  int out_bf16;
  float scale_log2;
};

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 2^x on the SFU; results below the normal range flush to zero (they are
// softmax weights at least 2^-126 below the row's running maximum).
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// x ~= hi + lo, both bf16 by truncation: hi = x with the low 16 bits cleared,
// lo = (x - hi) likewise (x - hi is exact in f32).  |x - hi - lo| < 2^-14 |x|.
// Returns hi and lo as f32 bit patterns with zero low halves; integer and
// logic instructions only.
__device__ __forceinline__ void split_trunc(float x, uint32_t& hi, uint32_t& lo) {
  hi = __float_as_uint(x) & 0xffff0000u;
  lo = __float_as_uint(x - __uint_as_float(hi)) & 0xffff0000u;
}
// two bf16 values held as f32 bit patterns with zero low halves -> one packed word (first in the low half)
__device__ __forceinline__ uint32_t pack_hi_halves(uint32_t a, uint32_t b) { return __byte_perm(a, b, 0x7632); }

struct AttnSmem {
  static constexpr int TILE = 128 * 128;             // 128 rows x 128 B = 16 KB (one 64-column half)
  static constexpr int OFF_QH = 0;                   // prologue: P part 3 ([2 halves][128 rows][128 B])
  static constexpr int OFF_QL = OFF_QH + 2 * TILE;   // prologue: the raw query rows
  static constexpr int OFF_K0 = OFF_QL + 2 * TILE;   // K~ buffer 0: [2 token halves][d_store rows][128 B];
                                                     // prologue: P[g] in f32 (64 KB over K0 and K1)
  static constexpr int OFF_K1 = OFF_K0 + 2 * TILE;   // K~ buffer 1
  static constexpr int OFF_V0 = OFF_K1 + 2 * TILE;   // V buffer 0: [2 dim halves][128 tokens][128 B]
  static constexpr int OFF_V1 = OFF_V0 + 2 * TILE;   // V buffer 1; prologue: P part 1
  static constexpr int OFF_PP = OFF_V1 + 2 * TILE;   // prologue: P part 2
  static constexpr int OFF_RED = OFF_PP + 2 * TILE;  // float [2][128]: row max / row sum exchange
  static constexpr int OFF_BAR = OFF_RED + 2 * 128 * 4;
  static constexpr int N_BAR = 24;
  static constexpr int OFF_MISC = OFF_BAR + N_BAR * 8;
  static constexpr int USED = OFF_MISC + 64;
  static constexpr int BYTES = USED + 1024;          // + slack to align the base to the 1024-byte swizzle period
};
enum {
  BAR_Q = 0,     // raw query rows landed (TMA)
  BAR_PF,        // P[g] in f32 landed in the K~ buffers (bulk copies)
  BAR_PS,        // P parts written, the K~ buffers free again (256 softmax threads)
  BAR_QT,        // q~ = q P complete in TMEM (commit)
  BAR_QM,        // masked q~ high/low parts written (both softmax warpgroups, 256 threads)
  BAR_KF0,       // K~ buffer 0 / 1 full (TMA)
  BAR_KF1,
  BAR_KE0,       // K~ buffer 0 / 1 free (commit after the QK MMAs reading it)
  BAR_KE1,
  BAR_VF0,       // V buffer 0 / 1 full (TMA)
  BAR_VF1,
  BAR_VE0,       // V buffer 0 / 1 free (commit after the P V MMAs reading it)
  BAR_VE1,
  BAR_S,         // S complete in TMEM (commit)
  BAR_SF,        // S copied to registers by all 256 softmax threads
  BAR_P,         // P written to TMEM, V tail zeroed (256 softmax threads)
  BAR_O,         // O += P V complete (commit)
  BAR_DRAIN,     // every MMA issued so far complete (commit)
  BAR_COUNT
};
static_assert(BAR_COUNT <= AttnSmem::N_BAR, "barrier slots");
static_assert(AttnSmem::BYTES <= 232448, "shared memory per CTA");
constexpr int kSoftThreads = 256;
constexpr int kMmaWarp = 8, kTmaWarp = 9;

// Bounded wait that also gives up once another role raised the abort flag.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag || globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// S(j) = Qh K~(j) + Ql K~(j) into TMEM over NKS k-steps of 16 dims (NKS =
// d_store / 16), the masked query parts (A) read from tensor memory, K~(j) (B)
// from shared memory; then commits: K~ buffer j&1 free, S ready.  Keeping A in
// tensor memory halves the shared-memory operand reads of these MMAs (the
// tile loop's shared memory also takes the TMA writes of every K~ and V tile).
// The contraction length is a template parameter so that the 2 NKS MMAs are
// issued back to back with nothing between them: a run-time test between two
// tcgen05.mma issues was measured to slow the tensor pipe from 64 to ~107
// cycles per 128 x 128 x 16 MMA.
template <int NKS>
__device__ __forceinline__ void issue_qk_n(unsigned char* smem, uint32_t tm_S, uint32_t tm_Q, int DS, int j,
                                           uint64_t* bars, uint32_t idesc) {
  using S = AttnSmem;
  const int kb = (j & 1) ? S::OFF_K1 : S::OFF_K0;
  // B descriptor of the first k-step, built once; a later k-step adds its byte
  // offset / 16 to the start-address field (every offset is a multiple of 16 and
  // every address stays below 2^18, so the field never carries).
  const uint64_t bd0 = smem_desc_sw128(smem + kb, DS * 128, 1024);
#pragma unroll
  for (int part = 0; part < 2; ++part)
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks)
      tc_mma_ts(tm_S, tm_Q + part * 64 + ks * 8, bd0 + (uint64_t)((ks * 16 * 128) >> 4), idesc, part > 0 || ks > 0);
  tc_commit(&bars[BAR_KE0 + (j & 1)]);
  tc_commit(&bars[BAR_S]);
}

__device__ __forceinline__ void issue_qk(unsigned char* smem, uint32_t tm_S, uint32_t tm_Q, int DS, int j,
                                         uint64_t* bars, uint32_t idesc) {
  switch (DS / 16) {
    case 1: issue_qk_n<1>(smem, tm_S, tm_Q, DS, j, bars, idesc); break;
    case 2: issue_qk_n<2>(smem, tm_S, tm_Q, DS, j, bars, idesc); break;
    case 3: issue_qk_n<3>(smem, tm_S, tm_Q, DS, j, bars, idesc); break;
    case 4: issue_qk_n<4>(smem, tm_S, tm_Q, DS, j, bars, idesc); break;
    case 5: issue_qk_n<5>(smem, tm_S, tm_Q, DS, j, bars, idesc); break;
    case 6: issue_qk_n<6>(smem, tm_S, tm_Q, DS, j, bars, idesc); break;
    case 7: issue_qk_n<7>(smem, tm_S, tm_Q, DS, j, bars, idesc); break;
    default: issue_qk_n<8>(smem, tm_S, tm_Q, DS, j, bars, idesc); break;
  }
}

template <int G>
__global__ void __launch_bounds__(kAttnThreads, 1)
    prefill_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, PrefillParams p) {
  using S = AttnSmem;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // The 128B swizzle pattern (TMA, tcgen05 descriptors and the hand-written
  // tiles) is a function of address bits 4-9: every tile starts on a 1024-byte boundary.
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR);
  float* red = reinterpret_cast<float*>(smem + S::OFF_RED);
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
    for (int i = 0; i < BAR_COUNT; ++i) {
      const int cnt = (i == BAR_PS || i == BAR_SF || i == BAR_P || i == BAR_QM) ? kSoftThreads : 1;
      mbar_init(&bars[i], cnt);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);                       // S [0,128), P high/low [128,256), O (q~ first) [256,384),
                                                      // masked q~ high/low [384,512)
    tmem_relinquish();
  }
  if (tid == kTmaWarp * 32) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  pdl_launch_dependents();
  pdl_wait();                                         // the previous kernel's appends are visible
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_S = tmem, tm_P = tmem + 128, tm_O = tmem + 256, tm_Q = tmem + 384;
  constexpr uint32_t idesc = idesc_bf16(PM, 128);

  if (warp == kTmaWarp) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      const uint64_t pol_q = policy_evict_first();
      const uint64_t pol_kv = policy_evict_normal();  // every row block of this (b, g) re-reads the tiles
      mbar_arrive_expect_tx(&bars[BAR_Q], 2 * S::TILE);
      tma_load_3d(smem + S::OFF_QL, &tm_q, 0, g * G, b * p.L + l0, &bars[BAR_Q], pol_q);
      tma_load_3d(smem + S::OFF_QL + S::TILE, &tm_q, 64, g * G, b * p.L + l0, &bars[BAR_Q], pol_q);
      // P[g] (f32, 64 KB) into the K~ buffers, converted there by the softmax threads
      mbar_arrive_expect_tx(&bars[BAR_PF], D * D * 4);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        bulk_g2s_plain(smem + S::OFF_K0 + c * (D * D), p.P + (size_t)g * D * D + c * (D * D / 4), D * D, &bars[BAR_PF]);
      const uint32_t kbytes = 2u * DS * 128u;
      int jk = 0, jv = 0;                             // next K~ / V tile to load
      unsigned long long t_last = globaltimer_ns();
      while ((jk < n_tiles || jv < n_tiles) && !*abort_flag) {
        bool progress = false;
        // K~(jk) into buffer jk&1 once the QK MMAs of tile jk-2 are done with it (the
        // first two once P's conversion no longer reads the buffers)
        if (jk < n_tiles && (jk < 2 ? mbar_try_wait(&bars[BAR_PS], 0)
                                    : mbar_try_wait(&bars[BAR_KE0 + (jk & 1)], ((jk - 2) >> 1) & 1))) {
          unsigned char* kb = smem + ((jk & 1) ? S::OFF_K1 : S::OFF_K0);
          uint64_t* kf = &bars[BAR_KF0 + (jk & 1)];
          mbar_arrive_expect_tx(kf, kbytes);
          tma_load_2d(kb, &tm_k, jk * PN, unit * DS, kf, pol_kv);
          tma_load_2d(kb + DS * 128, &tm_k, jk * PN + 64, unit * DS, kf, pol_kv);
          ++jk;
          progress = true;
        }
        // V(jv) into buffer jv&1 once the P V MMAs of tile jv-2 are done with it (buffer 1
        // holds a P part of the prologue until the projection MMAs have completed)
        if (jv < n_tiles &&
            (jv == 0 || (jv == 1 ? mbar_try_wait(&bars[BAR_QT], 0)
                                 : mbar_try_wait(&bars[BAR_VE0 + (jv & 1)], ((jv - 2) >> 1) & 1)))) {
          unsigned char* vb = smem + ((jv & 1) ? S::OFF_V1 : S::OFF_V0);
          uint64_t* vf = &bars[BAR_VF0 + (jv & 1)];
          mbar_arrive_expect_tx(vf, 2 * S::TILE);
          tma_load_2d(vb, &tm_v, 0, unit * p.Tcap + jv * PN, vf, pol_kv);
          tma_load_2d(vb + S::TILE, &tm_v, 64, unit * p.Tcap + jv * PN, vf, pol_kv);
          ++jv;
          progress = true;
        }
        const unsigned long long now = globaltimer_ns();
        if (progress) t_last = now;
        else if (now - t_last > kWaitLimitNs) *abort_flag = 1;
      }
      // every copy issued must have landed before the CTA exits
      bool drained = mbar_wait_bounded(&bars[BAR_Q], 0) && mbar_wait_bounded(&bars[BAR_PF], 0);
      for (int t = max(0, jk - 2); t < jk; ++t)
        drained = mbar_wait_bounded(&bars[BAR_KF0 + (t & 1)], (t >> 1) & 1) && drained;
      for (int t = max(0, jv - 2); t < jv; ++t)
        drained = mbar_wait_bounded(&bars[BAR_VF0 + (t & 1)], (t >> 1) & 1) && drained;
      if (!drained) *abort_flag = 1;
    }
  } else if (warp == kMmaWarp) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      bool ok = wait_or_abort(&bars[BAR_Q], 0, abort_flag) && wait_or_abort(&bars[BAR_PS], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        // q~ = q (P1 + P2 + P3): A = raw q rows (K-major), B = P parts (MN-major: input dim x output dim)
        const uint64_t aq0 = smem_desc_sw128(smem + S::OFF_QL, 16, 1024);
#pragma unroll
        for (int part = 0; part < 3; ++part) {
          const int part_off = part == 0 ? S::OFF_V1 : (part == 1 ? S::OFF_PP : S::OFF_QH);
          const uint64_t bp0 = smem_desc_sw128(smem + part_off, S::TILE, 1024);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            tc_mma(tm_O, aq0 + (uint64_t)(((ks >> 2) * S::TILE + (ks & 3) * 32) >> 4),
                   bp0 + (uint64_t)((ks * 16 * 128) >> 4), idesc, part > 0 || ks > 0);
        }
        tc_commit(&bars[BAR_QT]);
        ok = wait_or_abort(&bars[BAR_QM], 0, abort_flag);
      }
      if (ok) ok = wait_or_abort(&bars[BAR_KF0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_qk(smem, tm_S, tm_Q, DS, 0, bars, idesc);
      }
      for (int j = 0; j < n_tiles && ok; ++j) {
        if (j + 1 < n_tiles) {
          // S is free once every softmax thread holds tile j's scores in registers
          ok = wait_or_abort(&bars[BAR_SF], j & 1, abort_flag) &&
               wait_or_abort(&bars[BAR_KF0 + ((j + 1) & 1)], ((j + 1) >> 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          issue_qk(smem, tm_S, tm_Q, DS, j + 1, bars, idesc);
        }
        ok = wait_or_abort(&bars[BAR_VF0 + (j & 1)], (j >> 1) & 1, abort_flag) &&
             wait_or_abort(&bars[BAR_P], j & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        // O += Ph V + Pl V, P (128 rows x 128 tokens, two tokens per column) from tensor memory
        const int vb = (j & 1) ? S::OFF_V1 : S::OFF_V0;
        const uint64_t bv0 = smem_desc_sw128(smem + vb, S::TILE, 1024);   // k-step ks adds ks * 2048 B / 16
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int ks = 0; ks < PN / 16; ++ks)
            tc_mma_ts(tm_O, tm_P + part * 64 + ks * 8, bv0 + (uint64_t)((ks * 16 * 128) >> 4), idesc,
                      j > 0 || part > 0 || ks > 0);
        tc_commit(&bars[BAR_VE0 + (j & 1)]);
        tc_commit(&bars[BAR_O]);
      }
      if (!ok) *abort_flag = 1;
      // every MMA this thread issued must be complete before TMEM is released
      tc_commit(&bars[BAR_DRAIN]);
      if (!mbar_wait_bounded(&bars[BAR_DRAIN], 0)) *abort_flag = 1;
    }
  } else {
    // ======================= softmax warpgroups =======================
    const int wg = tid >> 7;                          // column half of S and O
    const int r = tid & 127;                          // TMEM lane = query row of the tile
    const int lr = l0 + r / G;                        // prompt row of this lane
    const int pos_r = p.pos0 + lr;                    // last visible token
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    bool ok = true;

    // ---- prologue 1: P[g] (f32, landed in the K~ buffers) -> three bf16 parts,
    // MN-major 128B-swizzled tiles.  16-byte chunk `ch` holds input dim i =
    // ch / 32, output dims 4 (ch % 32) .. +3: a warp converts one row of P per
    // round (conflict-free loads), each part as one 8-byte store.
    {
      const bool landed = wait_or_abort(&bars[BAR_PF], 0, abort_flag);
      if (landed) {
        const unsigned char* pf = smem + S::OFF_K0;
#pragma unroll 4
        for (int it = 0; it < D * D / 4 / kSoftThreads; ++it) {
          const int ch = it * kSoftThreads + tid;
          const int i = ch >> 5, j0 = 4 * (ch & 31);
          const float4 x4 = *reinterpret_cast<const float4*>(pf + (size_t)ch * 16);
          const float x[4] = {x4.x, x4.y, x4.z, x4.w};
          uint32_t w1[2], w2[2], w3[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            float r0 = x[2 * e], r1 = x[2 * e + 1];
            const __nv_bfloat162 a = __floats2bfloat162_rn(r0, r1);
            r0 -= __low2float(a);
            r1 -= __high2float(a);
            const __nv_bfloat162 bb = __floats2bfloat162_rn(r0, r1);
            r0 -= __low2float(bb);
            r1 -= __high2float(bb);
            const __nv_bfloat162 cc = __floats2bfloat162_rn(r0, r1);
            w1[e] = *reinterpret_cast<const uint32_t*>(&a);
            w2[e] = *reinterpret_cast<const uint32_t*>(&bb);
            w3[e] = *reinterpret_cast<const uint32_t*>(&cc);
          }
          const int jj = j0 & 63;
          const int off = (j0 >> 6) * S::TILE + i * 128 + ((((jj >> 3) ^ (i & 7))) << 4) + (jj & 7) * 2;
          *reinterpret_cast<uint2*>(smem + S::OFF_V1 + off) = make_uint2(w1[0], w1[1]);
          *reinterpret_cast<uint2*>(smem + S::OFF_PP + off) = make_uint2(w2[0], w2[1]);
          *reinterpret_cast<uint2*>(smem + S::OFF_QH + off) = make_uint2(w3[0], w3[1]);
        }
      }
      if (!landed) *abort_flag = 1;
      fence_proxy_async_smem();
      mbar_arrive(&bars[BAR_PS]);
    }

    // ---- prologue 2: top-k of |q~| for row r, masked scaled q~ high/low parts.
    // Warpgroup wg holds dims 64 wg .. 64 wg + 63 of the row; the row's two
    // threads (warps w and w + 4 share TMEM lanes) exchange counts through
    // shared memory (the P part-2 area, free once q~ is complete) at a barrier
    // of their two warps.  Both take every round and exchange whatever their
    // waits returned, so neither is ever left alone at the barrier.
    {
      ok = wait_or_abort(&bars[BAR_QT], 0, abort_flag);
      int* xcnt = reinterpret_cast<int*>(smem + S::OFF_PP);   // [2 rounds][2 halves][128 rows]
      const int pair_bar = 2 + (warp & 3);
      const int m = p.d_store;
      const int d0 = 64 * wg;
      uint32_t key[64];                             // |q~| bits + 1 for dims < m (0 otherwise): order-preserving
      if (ok) {
        tc_fence_after();
        tmem_ld32(tm_O + lane_base + d0, *reinterpret_cast<float(*)[32]>(&key[0]));
        tmem_ld32(tm_O + lane_base + d0 + 32, *reinterpret_cast<float(*)[32]>(&key[32]));
        tmem_wait_ld();
      }
#pragma unroll
      for (int j = 0; j < 64; ++j)   // NaN payloads clamp to one key above inf, so every key is below 2^31
        key[j] = (ok && d0 + j < m) ? (min(key[j] & 0x7fffffffu, 0x7F800001u) + 1u) : 0u;
      // largest tau with #{key >= tau} >= k, bit by bit; stop early once exactly k keys are >= tau
      uint32_t tau = 0;
      int cnt_tau = D;
      int round = 0;
#pragma unroll 1
      for (int bit = 30; bit >= 0; --bit, ++round) {
        const uint32_t cand = tau | (1u << bit);
        // keys below cand: key - cand wraps past 2^31 (both are below 2^31)
        uint32_t cp[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
        for (int j = 0; j < 64; ++j) cp[j & 7] += (key[j] - cand) >> 31;
        const int ch = 64 - (int)(((cp[0] + cp[1]) + (cp[2] + cp[3])) + ((cp[4] + cp[5]) + (cp[6] + cp[7])));
        int* xr = xcnt + (round & 1) * 256;
        xr[wg * 128 + r] = ch;
        named_bar_sync(pair_bar, 64);
        const int c = ch + xr[(wg ^ 1) * 128 + r];
        if (c >= p.k) {
          tau = cand;
          cnt_tau = c;
        }
        if (__all_sync(0xffffffffu, cnt_tau == p.k)) break;   // same decision in the partner warp
      }
      // selected: every key above tau, then keys equal to tau from the lowest index up
      uint32_t selm[2], eqm[2];
      int ngt = 0, neq = 0;
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        uint32_t gt = 0u, eq = 0u;
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          gt |= (uint32_t)(key[32 * w + t] > tau) << t;
          eq |= (uint32_t)(key[32 * w + t] == tau) << t;
        }
        selm[w] = gt;
        eqm[w] = eq;
        ngt += __popc(gt);
        neq += __popc(eq);
      }
      int* xg = xcnt + 512;                         // [2 halves][128 rows]: above-tau count | equal count << 16
      xg[wg * 128 + r] = ngt | (neq << 16);
      named_bar_sync(pair_bar, 64);
      const int other = xg[(wg ^ 1) * 128 + r];
      const int ngt_lo = wg == 0 ? ngt : (other & 0xffff), neq_lo = wg == 0 ? neq : (other >> 16);
      int need = p.k - ngt - (other & 0xffff);      // ties to keep, taken from the lower half first
      const int ties_lo = min(need, neq_lo);
      if (wg == 1) need -= ties_lo;
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const int ne = __popc(eqm[w]);
        if (ne <= need) {
          selm[w] |= eqm[w];
          need -= ne;
        } else if (need > 0) {
          const uint32_t last = __fns(eqm[w], 0, need);   // position of the need-th tie in this word
          selm[w] |= eqm[w] & (last >= 31 ? 0xffffffffu : ((2u << last) - 1u));
          need = 0;
        }
      }
      const bool live = lr < l_end;
      if (ok && p.sel_out != nullptr && live) {
        int32_t* so = p.sel_out + (((size_t)b * p.L + lr) * p.Hq + g * G + (r % G)) * p.k;
        int n = wg == 0 ? 0 : ngt_lo + ties_lo;      // the lower half's kept dims come first
#pragma unroll
        for (int w = 0; w < 2; ++w)
          for (uint32_t word = selm[w]; word != 0u; word &= word - 1u) so[n++] = d0 + 32 * w + (__ffs(word) - 1);
      }
      if (ok) {
        // second pass over this half of q~ (still in TMEM): masked, scaled, split into
        // bf16 high and low parts and stored to tensor memory as the A operand of
        // the QK MMAs (K-major, two dims per column, the lower dim in the low half):
        // high parts in columns [tm_Q, tm_Q + 64), low parts in [tm_Q + 64, tm_Q + 128)
        float* qpo = (p.qproj_out != nullptr && live)
                         ? p.qproj_out + (((size_t)b * p.L + lr) * p.Hq + g * G + (r % G)) * D + d0
                         : nullptr;
        uint32_t hq[32], lq[32];
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 32) {
          float v[32];
          tmem_ld32(tm_O + lane_base + d0 + c0, v);
          tmem_wait_ld();
          if (qpo != nullptr) {                       // the exact f32 values the keys above came from
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(qpo + c0 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
          }
          const uint32_t word = selm[c0 >> 5];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int jj = 2 * e;
            const float x0 = ((word >> jj) & 1u) ? v[jj] * p.scale_log2 : 0.f;
            const float x1 = ((word >> (jj + 1)) & 1u) ? v[jj + 1] * p.scale_log2 : 0.f;
            // high part truncated, low part rounded: |x - hi - lo| <= 2^-16 |x|, unbiased
            const uint32_t h0 = __float_as_uint(x0) & 0xffff0000u, h1 = __float_as_uint(x1) & 0xffff0000u;
            hq[(c0 >> 1) + e] = pack_hi_halves(h0, h1);
            lq[(c0 >> 1) + e] = pack_bf16(x0 - __uint_as_float(h0), x1 - __uint_as_float(h1));
          }
        }
        tmem_st32(tm_Q + lane_base + (d0 >> 1), *reinterpret_cast<const float(*)[32]>(hq));
        tmem_st32(tm_Q + 64 + lane_base + (d0 >> 1), *reinterpret_cast<const float(*)[32]>(lq));
        tmem_wait_st();
        tc_fence_before();
      }
      mbar_arrive(&bars[BAR_QM]);
    }

    // ---- main loop: this warpgroup's 64 columns of every S tile.  Every softmax
    // thread runs all n_tiles iterations and reaches the named barrier in each,
    // also after a failed wait (then it only raises the abort flag and skips the
    // work), so a timeout never leaves a partner blocked at the barrier.
    float mu = -INFINITY, ell = 0.f;
    const int cbase = wg * 64;
    const int pair_bar = 2 + (warp & 3);            // the row's two threads: warps w and w + 4
    // the row maximum exchange of every tile, [tile parity][2 halves][128 rows]:
    // in the P part-2 area (free after the prologue), past the selection's counts
    float* xmax = reinterpret_cast<float*>(smem + S::OFF_PP + 4096);
    if (!ok) *abort_flag = 1;
    for (int j = 0; j < n_tiles; ++j) {
      const int t0 = j * PN;
      float s[64];
      float mx = -INFINITY;
      if (ok) ok = wait_or_abort(&bars[BAR_S], j & 1, abort_flag);
      if (ok) {
        tc_fence_after();
        tmem_ld32(tm_S + lane_base + cbase, *reinterpret_cast<float(*)[32]>(&s[0]));
        tmem_ld32(tm_S + lane_base + cbase + 32, *reinterpret_cast<float(*)[32]>(&s[32]));
        tmem_wait_ld();
        const int tc0 = t0 + cbase;                   // token of s[0]
        if (tc0 + 63 > pos_r) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (tc0 + c > pos_r) s[c] = -INFINITY;
        }
        float m8[8];                                // eight independent chains
#pragma unroll
        for (int c = 0; c < 8; ++c) m8[c] = s[c];
#pragma unroll
        for (int c = 8; c < 64; ++c) m8[c & 7] = fmaxf(m8[c & 7], s[c]);
        mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      }
      // row maximum over both column halves (the buffer alternates by tile, so a
      // value is never overwritten before the partner has read it)
      float* xm = xmax + (j & 1) * 256;
      xm[wg * 128 + r] = mx;
      named_bar_sync(pair_bar, 64);
      mx = fmaxf(mx, xm[(wg ^ 1) * 128 + r]);
      if (!ok) {
        *abort_flag = 1;
        continue;
      }
      // S may now be overwritten by the next tile's QK (the partner has read this tile's maximum)
      tc_fence_before();
      mbar_arrive(&bars[BAR_SF]);
      // running maximum: raised (and O, ell rescaled below) only when exceeded by 2^kLazy
      const bool raise = mx > mu + kLazy;
      const float mu_new = raise ? mx : mu;
      // P = 2^(s - mu) as bf16 high + low parts, computed while the previous P V may still run;
      // the row sum takes the values exactly as the tensor cores will see them
      uint32_t hw[32], lw[32];
      float rs[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};   // eight independent chains
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const float p0 = ex2_ftz(s[c] - mu_new);
        const float p1 = ex2_ftz(s[c + 1] - mu_new);
        uint32_t h0, l0, h1, l1;
        split_trunc(p0, h0, l0);
        split_trunc(p1, h1, l1);
        rs[(c >> 1) & 7] += (__uint_as_float(h0) + __uint_as_float(l0)) + (__uint_as_float(h1) + __uint_as_float(l1));
        hw[c >> 1] = pack_hi_halves(h0, h1);
        lw[c >> 1] = pack_hi_halves(l0, l1);
      }
      const float rs0 = (rs[0] + rs[1]) + (rs[2] + rs[3]), rs1 = (rs[4] + rs[5]) + (rs[6] + rs[7]);
      // the previous P V must be complete before O is rescaled or P is rewritten
      if (j > 0) {
        ok = wait_or_abort(&bars[BAR_O], (j - 1) & 1, abort_flag);
        if (!ok) {
          *abort_flag = 1;
          continue;
        }
        tc_fence_after();
      }
      // P into tensor memory: this lane's row, tokens 64*wg .. 64*wg+63 as 32 packed columns
      tmem_st32(tm_P + lane_base + 32 * wg, *reinterpret_cast<const float(*)[32]>(hw));
      tmem_st32(tm_P + 64 + lane_base + 32 * wg, *reinterpret_cast<const float(*)[32]>(lw));
      if (raise) {
        const float alpha = ex2_ftz(mu - mu_new);     // 0 on the first tile
        if (j > 0) {
#pragma unroll
          for (int c = 0; c < 64; c += 32) {
            float o[32];
            tmem_ld32(tm_O + lane_base + cbase + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tm_O + lane_base + cbase + c, o);
          }
          tmem_wait_st();
        }
        ell *= alpha;
        mu = mu_new;
      }
      ell += rs0 + rs1;
      tmem_wait_st();
      // tokens past the chunk's keys are not in the cache yet: their V rows must be finite
      if (t0 + PN > kv_valid) {
        ok = wait_or_abort(&bars[BAR_VF0 + (j & 1)], (j >> 1) & 1, abort_flag);
        if (!ok) {
          *abort_flag = 1;
          continue;
        }
        if (t0 + r >= kv_valid) {
          unsigned char* vrow = smem + ((j & 1) ? S::OFF_V1 : S::OFF_V0) + wg * S::TILE + r * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(vrow + c * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[BAR_P]);
    }
    // epilogue: O / (sum over both halves)
    if (ok) ok = wait_or_abort(&bars[BAR_O], (n_tiles - 1) & 1, abort_flag);
    red[wg * 128 + r] = ell;
    named_bar_sync(1, kSoftThreads);                 // reached by every softmax thread
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / (ell + red[(wg ^ 1) * 128 + r]);
      const bool live = lr < l_end;
      const size_t obase = (((size_t)b * p.L + lr) * p.Hq + g * G + (r % G)) * D + cbase;
#pragma unroll
      for (int c = 0; c < 64; c += 32) {
        float o[32];
        tmem_ld32(tm_O + lane_base + cbase + c, o);
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
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int G>
int launch_prefill_g(const aqua_cache* c, const PrefillParams& p, const void* q, cudaStream_t st) {
  int rc = set_smem_limit(prefill_attn_kernel<G>, AttnSmem::BYTES, "prefill_attn_kernel");
  if (rc != AQUA_OK) return rc;
  CUtensorMap tq, tk, tv;
  // q [B*L][Hq][D]: box {64 dims, G heads, 128/G positions} = the CTA's 128 rows in (position, head) order
  const uint64_t qdims[3] = {(uint64_t)D, (uint64_t)p.Hq, (uint64_t)p.B * p.L};
  const uint64_t qstr[2] = {(uint64_t)D * 2, (uint64_t)p.Hq * D * 2};
  const uint32_t qbox[3] = {64u, (uint32_t)G, (uint32_t)(PM / G)};
  rc = encode_tmap_bf16_3d(&tq, q, qdims, qstr, qbox, true);
  if (rc == AQUA_OK)
    rc = encode_tmap_bf16_2d(&tk, c->k_proj, (uint64_t)c->Tcap, (uint64_t)c->B * c->Hkv * c->d_store,
                             (uint64_t)c->Tcap * 2, 64, (uint32_t)c->d_store, true);
  if (rc == AQUA_OK)
    rc = encode_tmap_bf16_2d(&tv, c->v, D, (uint64_t)c->B * c->Hkv * c->Tcap, D * 2, 64, PN, true);
  if (rc != AQUA_OK) return rc;
  dim3 grid((p.L + PM / G - 1) / (PM / G), p.Hkv, p.B);
  const cudaError_t e = launch_pdl(prefill_attn_kernel<G>, grid, dim3(kAttnThreads), AttnSmem::BYTES, st, tq, tk, tv, p);
  if (e != cudaSuccess) return set_error(AQUA_ERR_CUDA, "prefill_attn_kernel: %s", cudaGetErrorString(e));
  return check_launch("prefill_attn_kernel");
}

}  // namespace

size_t prefill_workspace_bytes(const aqua_cache*, int, int) {
  return 256;   // reserved; the kernel keeps all its intermediates on chip
}

int launch_prefill(const aqua_cache* c, const void* q, int pos0, int L, const float* P, int Hq, int k, float scale,
                   void* out, int out_dtype, int32_t* sel_out, float* qproj_out, void*, cudaStream_t st) {
  if (c->d_store % 16 != 0)
    return set_error(AQUA_ERR_UNSUPPORTED, "aqua_prefill_attn: d_store %d must be a multiple of 16", c->d_store);
  PrefillParams p;
  p.P = P;
  p.out = out;
  p.sel_out = sel_out;
  p.qproj_out = qproj_out;
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
    case 1: return launch_prefill_g<1>(c, p, q, st);
    case 2: return launch_prefill_g<2>(c, p, q, st);
    case 4: return launch_prefill_g<4>(c, p, q, st);
    default: return set_error(AQUA_ERR_UNSUPPORTED, "aqua_prefill_attn: Hq/Hkv = %d not in {1,2,4}", Hq / c->Hkv);
  }
}

}  // namespace aqua
