// AQUA decode step on sm_100a.
//
// Kernel 1 (qproj_topk_kernel), one CTA per (sequence b, KV head g), one warp
// per query head of the group:
//   q~ = q P                                  (abstract: "project query ... vectors")
//   S_h = k largest |q~_j|, ties to lower j  (edgentiq, Online Inference: "highest
//                                             'magnitude' in the projected query")
//   U_g = union of the group's S_h, and the masked, pre-scaled query rows
//   qm[r][h] = (j_r in S_h) ? q~_h[j_r] * scale * log2(e) : 0 for j_r = U_g[r].
//
// Kernel 2 (decode_attn_kernel), persistent, one CTA per SM.  The cached
// tokens of all (b, g) units are cut into tiles of TT tokens and the flat tile
// sequence is split evenly over the CTAs.  Per tile a producer warp gathers the
// |U_g| selected rows of the dimension-major K~ cache and the V tile into shared
// memory with bulk asynchronous copies (one union read per GQA group), three
// stages deep; eight consumer warps compute
//   s_{h,t} = sum_{r} qm[r][h] K~[U_r][t]       (scores on the selected dims only)
// followed by an online softmax and o_h += p_{h,t} V_t (unprojected V).  A CTA
// that finishes a partial unit writes (m, l, o) and takes a ticket; the last
// CTA of a unit merges the partials (log-sum-exp) and writes the output.  No
// CTA ever waits for another.
#include <math.h>

#include "aqua_internal.cuh"

namespace aqua {

namespace {

constexpr int D = kHeadDim;
constexpr int NCW = 8;                 // consumer warps
constexpr int NCT = NCW * 32;          // consumer threads
constexpr int NTHREADS = NCT + 32;     // + one producer warp
constexpr int NSTAGE = 3;
constexpr int RMAX = D / NCW;          // union rows per consumer warp
constexpr int kMaxCtas = 1024;

struct DecodeParams {
  const void* q;
  const float* P;
  const int32_t* len;
  const void* kproj;
  const void* v;
  void* out;
  float* qm;          // [n_units][D][G]
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
  int B, Hq, Hkv, d_store, Tcap, k;
  int out_bf16;
  float scale_log2;
};

template <typename T> struct Tile;
template <> struct Tile<__nv_bfloat16> { static constexpr int TT = 128; };
template <> struct Tile<float> { static constexpr int TT = 64; };

// ------------------------------------------------------------------ small loads
template <typename T, int N>
__device__ __forceinline__ void load_row(const T* p, float (&f)[N]);
template <>
__device__ __forceinline__ void load_row<__nv_bfloat16, 4>(const __nv_bfloat16* p, float (&f)[4]) {
  const uint2 w = *reinterpret_cast<const uint2*>(p);
  f[0] = bf16lo(w.x); f[1] = bf16hi(w.x); f[2] = bf16lo(w.y); f[3] = bf16hi(w.y);
}
template <>
__device__ __forceinline__ void load_row<float, 4>(const float* p, float (&f)[4]) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}
template <>
__device__ __forceinline__ void load_row<float, 2>(const float* p, float (&f)[2]) {
  const float2 v = *reinterpret_cast<const float2*>(p);
  f[0] = v.x; f[1] = v.y;
}

// cached tokens of sequence b, clamped to the cache capacity (lengths are caller-owned device data)
__device__ __forceinline__ int seq_len(const int32_t* len, int b, int Tcap) { return min(max(len[b], 0), Tcap); }

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

// ============================================================================
// Kernel 1: query projection + magnitude top-k + group union
// ============================================================================
template <typename T, int G>
__global__ void __launch_bounds__(G * 32) qproj_topk_kernel(DecodeParams p) {
  __shared__ float qs[G][D];
  __shared__ uint32_t masks[G][4];
  const int u = blockIdx.x;
  const int b = u / p.Hkv, g = u % p.Hkv;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = g * G + w;
  const int m = p.d_store;

  const T* qrow = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + h) * D;
  float qv[4];
#pragma unroll
  for (int s = 0; s < 4; ++s) qv[s] = Elem<T>::load(qrow + 4 * lane + s);

  // q~_j for j = 4*lane + s
  float qt[4] = {0.f, 0.f, 0.f, 0.f};
  const float* Pg = p.P + (size_t)g * D * D;
#pragma unroll 8
  for (int i = 0; i < D; ++i) {
    const float qi = __shfl_sync(0xffffffffu, qv[i & 3], i >> 2);
    const float4 pr = __ldg(reinterpret_cast<const float4*>(Pg + (size_t)i * D) + lane);
    qt[0] = fmaf(qi, pr.x, qt[0]);
    qt[1] = fmaf(qi, pr.y, qt[1]);
    qt[2] = fmaf(qi, pr.z, qt[2]);
    qt[3] = fmaf(qi, pr.w, qt[3]);
  }

  // Keys: magnitude bits + 1 for candidate dims (j < m), 0 otherwise, so that
  // unsigned order equals |q~| order and non-candidates rank below everything.
  uint32_t key[4];
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const int j = 4 * lane + s;
    key[s] = (j < m) ? (__float_as_uint(fabsf(qt[s])) + 1u) : 0u;
  }
  // Radix select of the k-th largest key: the largest tau with #{key >= tau} >= k.
  uint32_t tau = 0;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = tau | (1u << bit);
    int c = 0;
#pragma unroll
    for (int s = 0; s < 4; ++s) c += (key[s] >= cand);
    c = __reduce_add_sync(0xffffffffu, c);
    if (c >= p.k) tau = cand;
  }
  int ngt = 0, neq = 0;
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    ngt += (key[s] > tau);
    neq += (key[s] == tau);
  }
  const int need = p.k - __reduce_add_sync(0xffffffffu, ngt);  // ties to take, lowest index first
  // exclusive prefix of equal-key counts over lanes (index order = lane-major)
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
  // ascending output position of each selected dim
  int pincl = nsel;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, pincl, o);
    if (lane >= o) pincl += y;
  }
  int opos = pincl - nsel;
  const size_t bh = (size_t)b * p.Hq + h;
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const int j = 4 * lane + s;
    if (sel[s]) {
      if (p.sel_out) p.sel_out[bh * p.k + opos] = j;
      ++opos;
    }
    if (p.qproj_out) p.qproj_out[bh * D + j] = qt[s];
    qs[w][j] = sel[s] ? qt[s] * p.scale_log2 : 0.f;
  }
  // 128-bit selection mask of this head
  const uint32_t nib = (uint32_t)sel[0] | ((uint32_t)sel[1] << 1) | ((uint32_t)sel[2] << 2) |
                       ((uint32_t)sel[3] << 3);
  const uint32_t shifted = nib << (4 * (lane & 7));
#pragma unroll
  for (int wd = 0; wd < 4; ++wd) {
    const uint32_t word = __reduce_or_sync(0xffffffffu, (lane >> 3) == wd ? shifted : 0u);
    if (lane == 0) masks[w][wd] = word;
  }

  // sequences with no tokens: zero output, lse = -inf
  const int T_b = seq_len(p.len, b, p.Tcap);
  if (T_b <= 0) {
    for (int j = lane; j < D; j += 32) {
      if (p.out_bf16)
        static_cast<__nv_bfloat16*>(p.out)[bh * D + j] = __float2bfloat16_rn(0.f);
      else
        static_cast<float*>(p.out)[bh * D + j] = 0.f;
    }
    if (p.lse_out && lane == 0) p.lse_out[bh] = -INFINITY;
  }
  __syncthreads();

  // group union U_g (ascending) and the masked query rows over it
  uint32_t um[4];
#pragma unroll
  for (int wd = 0; wd < 4; ++wd) {
    uint32_t x = 0;
#pragma unroll
    for (int hh = 0; hh < G; ++hh) x |= masks[hh][wd];
    um[wd] = x;
  }
  for (int j = threadIdx.x; j < D; j += G * 32) {
    const int wd = j >> 5, bit = j & 31;
    if ((um[wd] >> bit) & 1u) {
      int r = __popc(um[wd] & ((1u << bit) - 1u));
      for (int x = 0; x < wd; ++x) r += __popc(um[x]);
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
}

// ============================================================================
// Kernel 2: persistent split-K sparse-dimension attention
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

// CTA that owns flat tile t when N tiles are split over C CTAs as [floor(c N / C), floor((c+1) N / C))
__device__ __forceinline__ int cta_of_tile(long long t, long long N, int C) {
  long long c = ((t + 1) * C + N - 1) / N - 1;
  return (int)(c < C - 1 ? c : C - 1);
}

// exclusive scan over all NTHREADS threads; *total receives the sum
__device__ __forceinline__ long long block_excl_scan(long long v, long long* sh, long long* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int NW = NTHREADS / 32;
  long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    long long y = lane < NW ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long z = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) y += z;
    }
    if (lane < NW) sh[lane] = y;
  }
  __syncthreads();
  const long long base = warp > 0 ? sh[warp - 1] : 0;
  *total = sh[NW - 1];
  const long long excl = base + x - v;
  __syncthreads();
  return excl;
}

template <typename T, int G>
struct DecodeSmem {
  static constexpr int TT = Tile<T>::TT;
  static constexpr int KBYTES = D * TT * (int)sizeof(T);
  static constexpr int VBYTES = TT * D * (int)sizeof(T);
  static constexpr int STAGE = KBYTES + VBYTES;
  static constexpr int RW = TT > D ? TT : D;
  static constexpr int SLOTS = (G * TT + NCT - 1) / NCT;
  static constexpr int OFF_RED = NSTAGE * STAGE;
  static constexpr int OFF_PSM = OFF_RED + NCW * G * RW * 4;
  static constexpr int OFF_WST = OFF_PSM + TT * G * 4;
  static constexpr int OFF_HDR = OFF_WST + 2 * SLOTS * NCW * 4;
  static constexpr int OFF_BAR = OFF_HDR + NSTAGE * (int)sizeof(StageHdr);
  static constexpr int OFF_SCH = OFF_BAR + 2 * NSTAGE * 8;
  static constexpr int BYTES = OFF_SCH + 16 * 8;
};

template <typename T, int G>
__global__ void __launch_bounds__(NTHREADS, 1) decode_attn_kernel(DecodeParams p) {
  using S = DecodeSmem<T, G>;
  constexpr int TT = S::TT;
  constexpr int TPL = TT / 32;        // tokens per lane in the score pass
  constexpr int TPW = TT / NCW;       // tokens per warp in the PV pass
  constexpr int EPV = 16 / (int)sizeof(T);   // elements per 16-byte vector

  extern __shared__ __align__(1024) unsigned char smem[];
  float* red = reinterpret_cast<float*>(smem + S::OFF_RED);
  float* psm = reinterpret_cast<float*>(smem + S::OFF_PSM);
  float* wmax = reinterpret_cast<float*>(smem + S::OFF_WST);
  float* wsum = wmax + S::SLOTS * NCW;
  StageHdr* hdr = reinterpret_cast<StageHdr*>(smem + S::OFF_HDR);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR);
  uint64_t* empty = full + NSTAGE;
  long long* sch = reinterpret_cast<long long*>(smem + S::OFF_SCH);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int n_units = p.B * p.Hkv;
  const int C = gridDim.x, c = blockIdx.x;

  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCW);
    }
    fence_barrier_init();
  }

  // ---------------- schedule: flat tile range of this CTA and its first unit
  long long* scan_sh = reinterpret_cast<long long*>(smem);  // stage memory is free until the producer starts
  const int chunk = (n_units + NTHREADS - 1) / NTHREADS;
  const int u_lo = min(n_units, tid * chunk), u_hi = min(n_units, u_lo + chunk);
  long long my_tiles = 0;
  for (int u = u_lo; u < u_hi; ++u) my_tiles += (seq_len(p.len, u / p.Hkv, p.Tcap) + TT - 1) / TT;
  long long N;
  const long long t_excl = block_excl_scan(my_tiles, scan_sh, &N);
  const long long my_start = (long long)c * N / C, my_end = (long long)(c + 1) * N / C;
  long long my_segs = 0;
  {
    long long ts = t_excl;
    for (int u = u_lo; u < u_hi; ++u) {
      const long long nt = (seq_len(p.len, u / p.Hkv, p.Tcap) + TT - 1) / TT;
      if (nt > 0) my_segs += cta_of_tile(ts + nt - 1, N, C) - cta_of_tile(ts, N, C) + 1;
      ts += nt;
    }
  }
  long long NS;
  const long long s_excl = block_excl_scan(my_segs, scan_sh, &NS);
  {
    long long ts = t_excl, sb = s_excl;
    for (int u = u_lo; u < u_hi; ++u) {
      const long long nt = (seq_len(p.len, u / p.Hkv, p.Tcap) + TT - 1) / TT;
      if (nt > 0 && ts <= my_start && my_start < ts + nt) {
        sch[0] = u;
        sch[1] = ts;
        sch[2] = sb;
      }
      if (nt > 0) sb += cta_of_tile(ts + nt - 1, N, C) - cta_of_tile(ts, N, C) + 1;
      ts += nt;
    }
  }
  __syncthreads();
  if (my_start >= my_end) return;
  const int n_tiles = (int)(my_end - my_start);

  if (warp == NCW) {
    // ======================= producer warp =======================
    const uint64_t pol = policy_evict_first();
    int u = (int)sch[0];
    long long ts = sch[1], sb = sch[2];
    int b = u / p.Hkv;
    int Tb = seq_len(p.len, b, p.Tcap);
    long long te = ts + (Tb + TT - 1) / TT;
    int cf = cta_of_tile(ts, N, C);
    int nseg = cta_of_tile(te - 1, N, C) - cf + 1;
    int nU = p.ucount[u];
    int urow[D / 32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = lane + 32 * i;
      urow[i] = r < nU ? p.ulist[(size_t)u * D + r] : 0;
    }
    for (int it = 0; it < n_tiles; ++it) {
      const long long t = my_start + it;
      while (t >= te) {  // next non-empty unit
        sb += nseg;
        ++u;
        b = u / p.Hkv;
        Tb = seq_len(p.len, b, p.Tcap);
        ts = te;
        te = ts + (Tb + TT - 1) / TT;
        if (te > ts) {
          cf = cta_of_tile(ts, N, C);
          nseg = cta_of_tile(te - 1, N, C) - cf + 1;
        } else {
          nseg = 0;
        }
        if (te > ts) {
          nU = p.ucount[u];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = lane + 32 * i;
            urow[i] = r < nU ? p.ulist[(size_t)u * D + r] : 0;
          }
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
      const int t0 = (int)(t - ts) * TT;
      const int nvalid = min(TT, Tb - t0);
      const int kvec = (nvalid + EPV - 1) / EPV * EPV;          // row copy in 16-byte units
      const uint32_t kbytes = (uint32_t)kvec * sizeof(T);
      const uint32_t vbytes = (uint32_t)nvalid * D * sizeof(T);
      unsigned char* st = smem + (size_t)s * S::STAGE;
      if (lane == 0) {
        StageHdr hh;
        hh.u = u;
        hh.t0 = t0;
        hh.nvalid = nvalid;
        hh.nU = nU;
        hh.flags = ((t == my_start || t == ts) ? kFirst : 0) | ((t == my_end - 1 || t == te - 1) ? kLast : 0);
        hh.seg = nseg > 1 ? (int)(sb + (c - cf)) : -1;
        hh.nseg = nseg;
        hh.seg0 = (int)sb;
        hdr[s] = hh;
        mbar_arrive_expect_tx(&full[s], kbytes * nU + vbytes);
      }
      __syncwarp();
      const T* kbase = static_cast<const T*>(p.kproj) + (size_t)u * p.d_store * p.Tcap + t0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = lane + 32 * i;
        if (r < nU)
          bulk_g2s(st + (size_t)r * TT * sizeof(T), kbase + (size_t)urow[i] * p.Tcap, kbytes, &full[s], pol);
      }
      if (lane == 0) {
        const T* vsrc = static_cast<const T*>(p.v) + ((size_t)u * p.Tcap + t0) * D;
        bulk_g2s(st + S::KBYTES, vsrc, vbytes, &full[s], pol);
      }
    }
    return;
  }

  // ======================= consumer warps =======================
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

  __shared__ int s_last;
  for (int it = 0; it < n_tiles; ++it) {
    const int s = it % NSTAGE;
    const bool ok = mbar_wait_bounded(&full[s], (it / NSTAGE) & 1);
    const StageHdr hh = hdr[s];
    const unsigned char* st = smem + (size_t)s * S::STAGE;
    const T* Ks = reinterpret_cast<const T*>(st);
    const T* Vs = reinterpret_cast<const T*>(st + S::KBYTES);
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

    // ---- partial scores over this warp's union rows
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
          float kf[TPL];
          load_row<T, TPL>(Ks + (size_t)r * TT + TPL * lane, kf);
#pragma unroll
          for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < TPL; ++e) sacc[h][e] = fmaf(qreg[i][h], kf[e], sacc[h][e]);
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

    // ---- reduce over warps, mask, tile maxima
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
          for (int hh2 = 0; hh2 < G; ++hh2)
            if (hh2 == h) mnew[hh2] = fmaxf(mnew[hh2], wmax[i * NCW + w2]);
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
        for (int hh2 = 0; hh2 < G; ++hh2)
          if (hh2 == h) mh = mnew[hh2];
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
          for (int hh2 = 0; hh2 < G; ++hh2)
            if (hh2 == h) l_run[hh2] += wsum[i * NCW + w2];
        }
      }
#pragma unroll
    for (int h = 0; h < G; ++h) m_run[h] = mnew[h];

    // ---- o += p V over this warp's tokens
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < 4; ++e) oacc[h][e] *= alpha[h];
#pragma unroll 4
    for (int j = 0; j < TPW; ++j) {
      const int tok = warp * TPW + j;
      if (tok < hh.nvalid) {
        float vf[4];
        load_row<T, 4>(Vs + (size_t)tok * D + 4 * lane, vf);
        float pv[G];
#pragma unroll
        for (int h = 0; h < G; ++h) pv[h] = psm[tok * G + h];
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int e = 0; e < 4; ++e) oacc[h][e] = fmaf(pv[h], vf[e], oacc[h][e]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);

    if (!(hh.flags & kLast)) continue;

    // ---- end of a segment: reduce o over warps, then output or partial
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < 4; ++e) red[((size_t)warp * G + h) * S::RW + 4 * lane + e] = oacc[h][e];
    named_bar_sync(1, NCT);
    const size_t bhq0 = (size_t)b * p.Hq + g * G;
#pragma unroll
    for (int i = 0; i < (G * D + NCT - 1) / NCT; ++i) {
      const int idx = tid + NCT * i;
      if (idx < G * D) {
        const int h = idx / D, dim = idx % D;
        float o = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < NCW; ++w2) o += red[((size_t)w2 * G + h) * S::RW + dim];
        float lh = 0.f;
#pragma unroll
        for (int hh2 = 0; hh2 < G; ++hh2)
          if (hh2 == h) lh = l_run[hh2];
        if (hh.seg < 0) {
          const float val = o / lh;
          if (p.out_bf16)
            static_cast<__nv_bfloat16*>(p.out)[(bhq0 + h) * D + dim] = __float2bfloat16_rn(val);
          else
            static_cast<float*>(p.out)[(bhq0 + h) * D + dim] = val;
        } else {
          p.part_o[((size_t)hh.seg * G + h) * D + dim] = o;
        }
      }
    }
    if (tid < G) {
#pragma unroll
      for (int h = 0; h < G; ++h)
        if (h == tid) {
          if (hh.seg < 0) {
            if (p.lse_out) p.lse_out[bhq0 + h] = (m_run[h] + log2f(l_run[h])) * kLn2;
          } else {
            p.part_ml[((size_t)hh.seg * G + h) * 2 + 0] = m_run[h];
            p.part_ml[((size_t)hh.seg * G + h) * 2 + 1] = l_run[h];
          }
        }
    }
    if (hh.seg >= 0) {
      // publish this partial, take a ticket; the unit's last arrival merges
      __threadfence();
      named_bar_sync(1, NCT);
      if (tid == 0) s_last = (atomicAdd(p.counters + hh.u, 1) == hh.nseg - 1);
      named_bar_sync(1, NCT);
      if (s_last) {
        __threadfence();
#pragma unroll 1
        for (int i = 0; i < (G * D + NCT - 1) / NCT; ++i) {
          const int idx = tid + NCT * i;
          if (idx >= G * D) break;
          const int h = idx / D, dim = idx % D;
          float M = -INFINITY;
#pragma unroll 1
          for (int sg = 0; sg < hh.nseg; ++sg)
            M = fmaxf(M, __ldcg(p.part_ml + ((size_t)(hh.seg0 + sg) * G + h) * 2));
          float Lsum = 0.f, O = 0.f;
#pragma unroll 1
          for (int sg = 0; sg < hh.nseg; ++sg) {
            const size_t slot = (size_t)(hh.seg0 + sg) * G + h;
            const float f = exp2f(__ldcg(p.part_ml + slot * 2) - M);
            Lsum = fmaf(f, __ldcg(p.part_ml + slot * 2 + 1), Lsum);
            O = fmaf(f, __ldcg(p.part_o + slot * D + dim), O);
          }
          const float val = O / Lsum;
          if (p.out_bf16)
            static_cast<__nv_bfloat16*>(p.out)[(bhq0 + h) * D + dim] = __float2bfloat16_rn(val);
          else
            static_cast<float*>(p.out)[(bhq0 + h) * D + dim] = val;
          if (dim == 0 && p.lse_out) p.lse_out[bhq0 + h] = (M + log2f(Lsum)) * kLn2;
        }
        if (tid == 0) p.counters[hh.u] = 0;
      }
    }
    named_bar_sync(1, NCT);
  }
}

template <typename T, int G>
int launch_decode_t(const DecodeParams& p, int n_units, int C, cudaStream_t st) {
  using S = DecodeSmem<T, G>;
  static bool configured = false;
  if (!configured) {
    if (cudaFuncSetAttribute(decode_attn_kernel<T, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             S::BYTES) != cudaSuccess)
      return check_launch("cudaFuncSetAttribute(decode_attn_kernel)");
    configured = true;
  }
  qproj_topk_kernel<T, G><<<n_units, G * 32, 0, st>>>(p);
  int rc = check_launch("qproj_topk_kernel");
  if (rc != AQUA_OK) return rc;
  decode_attn_kernel<T, G><<<C, NTHREADS, S::BYTES, st>>>(p);
  return check_launch("decode_attn_kernel");
}

}  // namespace

size_t decode_workspace_bytes(int n_units, int G) {
  size_t off = 0;
  auto take = [&](size_t bytes) { off += (bytes + 255) & ~size_t(255); };
  const size_t nseg = (size_t)n_units + kMaxCtas;
  take((size_t)n_units * D * G * 4);  // qm
  take((size_t)n_units * D * 4);      // ulist
  take((size_t)n_units * 4);          // ucount
  take((size_t)n_units * 4);          // counters
  take(nseg * G * 2 * 4);             // part_ml
  take(nseg * G * D * 4);             // part_o
  return off;
}

int launch_decode(const aqua_cache* c, const void* q, const float* P, int Hq, int k, float scale,
                  void* out, int out_dtype, int32_t* sel_out, float* qproj_out, float* scores_out,
                  float* lse_out, void* ws, cudaStream_t st) {
  const int G = Hq / c->Hkv;
  const int n_units = c->B * c->Hkv;
  DecodeParams p;
  unsigned char* base = static_cast<unsigned char*>(ws);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    void* ptr = base + off;
    off += (bytes + 255) & ~size_t(255);
    return ptr;
  };
  const size_t nseg = (size_t)n_units + kMaxCtas;
  p.qm = static_cast<float*>(take((size_t)n_units * D * G * 4));
  p.ulist = static_cast<int32_t*>(take((size_t)n_units * D * 4));
  p.ucount = static_cast<int32_t*>(take((size_t)n_units * 4));
  p.counters = static_cast<int32_t*>(take((size_t)n_units * 4));
  p.part_ml = static_cast<float*>(take(nseg * G * 2 * 4));
  p.part_o = static_cast<float*>(take(nseg * G * D * 4));
  p.q = q;
  p.P = P;
  p.len = c->len;
  p.kproj = c->k_proj;
  p.v = c->v;
  p.out = out;
  p.sel_out = sel_out;
  p.qproj_out = qproj_out;
  p.scores_out = scores_out;
  p.lse_out = lse_out;
  p.ctrl = c->ctrl;
  p.B = c->B;
  p.Hq = Hq;
  p.Hkv = c->Hkv;
  p.d_store = c->d_store;
  p.Tcap = c->Tcap;
  p.k = k;
  p.out_bf16 = out_dtype == AQUA_BF16;
  p.scale_log2 = scale * kLog2e;
  const int TT = c->dtype == AQUA_BF16 ? Tile<__nv_bfloat16>::TT : Tile<float>::TT;
  const long long tiles_ub = (long long)n_units * ((c->max_len + TT - 1) / TT);
  long long C = device_sm_count();
  if (C > tiles_ub) C = tiles_ub;
  if (C < 1) C = 1;
  if (C > kMaxCtas) C = kMaxCtas;
  const bool bf = c->dtype == AQUA_BF16;
  switch (G) {
    case 1: return bf ? launch_decode_t<__nv_bfloat16, 1>(p, n_units, (int)C, st)
                      : launch_decode_t<float, 1>(p, n_units, (int)C, st);
    case 2: return bf ? launch_decode_t<__nv_bfloat16, 2>(p, n_units, (int)C, st)
                      : launch_decode_t<float, 2>(p, n_units, (int)C, st);
    case 4: return bf ? launch_decode_t<__nv_bfloat16, 4>(p, n_units, (int)C, st)
                      : launch_decode_t<float, 4>(p, n_units, (int)C, st);
    default: return set_error(AQUA_ERR_UNSUPPORTED, "decode: Hq/Hkv = %d not in {1,2,4}", G);
  }
}

}  // namespace aqua
