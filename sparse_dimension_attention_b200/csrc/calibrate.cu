// Offline calibration on the GPU: P = right singular vectors of X (columns by
// descending singular value), computed as the eigenvectors of the Gram matrix
// X^T X in float64 with cyclic Jacobi rotations.
//
// AQUA abstract (one projection matrix, computed offline once by an SVD of
// calibration data and shared across languages);
// edgentiq, "Offline Projection Computation".  The right singular vectors of X
// are the eigenvectors of X^T X and sigma_j = sqrt(lambda_j).
#include <math.h>

#include "aqua_internal.cuh"

namespace aqua {

namespace {

constexpr int D = kHeadDim;
constexpr int kGramThreads = 256;    // 16 x 16 threads, each an 8 x 8 block of the Gram matrix
constexpr int kGramRowsChunk = 32;
constexpr int kMaxGramBlocks = 128;
constexpr int kJacobiThreads = 1024;
constexpr int kMaxSweeps = 40;
constexpr int LDA = D + 1;           // padded row stride of the shared copy of A

int gram_blocks(int n) {
  int nb = (n + 255) / 256;
  return nb < 1 ? 1 : (nb > kMaxGramBlocks ? kMaxGramBlocks : nb);
}

// partial Gram matrices: block k sums rows [k*R, min(n, (k+1)*R)) in float64
__global__ void __launch_bounds__(kGramThreads) gram_partial_kernel(const float* __restrict__ X, int n, int rows_per_blk,
                                                                    double* __restrict__ part) {
  __shared__ float xs[kGramRowsChunk][D];
  const int ti = threadIdx.x / 16, tj = threadIdx.x % 16;
  double acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[a][c] = 0.0;
  const int r0 = blockIdx.x * rows_per_blk;
  const int r1 = min(n, r0 + rows_per_blk);
  for (int rc = r0; rc < r1; rc += kGramRowsChunk) {
    const int nr = min(kGramRowsChunk, r1 - rc);
    __syncthreads();
    for (int e = threadIdx.x; e < kGramRowsChunk * D; e += kGramThreads) {
      const int rr = e / D, cc = e % D;
      xs[rr][cc] = rr < nr ? X[(size_t)(rc + rr) * D + cc] : 0.f;
    }
    __syncthreads();
    for (int rr = 0; rr < nr; ++rr) {
      double a[8], c8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        a[e] = (double)xs[rr][8 * ti + e];
        c8[e] = (double)xs[rr][8 * tj + e];
      }
#pragma unroll
      for (int x = 0; x < 8; ++x)
#pragma unroll
        for (int y = 0; y < 8; ++y) acc[x][y] = fma(a[x], c8[y], acc[x][y]);
    }
  }
  double* dst = part + (size_t)blockIdx.x * D * D;
#pragma unroll
  for (int x = 0; x < 8; ++x)
#pragma unroll
    for (int y = 0; y < 8; ++y) dst[(size_t)(8 * ti + x) * D + 8 * tj + y] = acc[x][y];
}

// deterministic sum of the partial Gram matrices (fixed order)
__global__ void gram_sum_kernel(const double* __restrict__ part, int nblk, double* __restrict__ A) {
  const int i = blockIdx.x, j = threadIdx.x;
  double s = 0.0;
  for (int k = 0; k < nblk; ++k) s += part[((size_t)k * D + i) * D + j];
  A[(size_t)i * D + j] = s;
}

__device__ __forceinline__ void pair_of(int round, int i, int& p, int& q) {
  // round-robin tournament on D players: player D-1 is fixed, the others rotate
  int a, b;
  if (i == 0) {
    a = D - 1;
    b = round;
  } else {
    a = (round + i) % (D - 1);
    b = (round - i + (D - 1)) % (D - 1);
  }
  p = min(a, b);
  q = max(a, b);
}

// one CTA: Jacobi eigen-decomposition of the symmetric A (float64), V in global memory
__global__ void __launch_bounds__(kJacobiThreads) jacobi_kernel(const double* __restrict__ Ain, double* __restrict__ V,
                                                                float* __restrict__ P_out, float* __restrict__ sigma_out) {
  extern __shared__ double A[];  // [D][LDA]
  __shared__ double cs[D / 2][2];
  __shared__ int pq[D / 2][2];
  __shared__ double red[2][kJacobiThreads / 32];
  __shared__ int s_done;
  const int tid = threadIdx.x;
  for (int e = tid; e < D * D; e += kJacobiThreads) {
    const int i = e / D, j = e % D;
    A[i * LDA + j] = Ain[e];
    V[e] = (i == j) ? 1.0 : 0.0;
  }
  __syncthreads();
  for (int sweep = 0; sweep < kMaxSweeps; ++sweep) {
    // convergence test: off-diagonal mass relative to the diagonal
    double off = 0.0, dia = 0.0;
    for (int e = tid; e < D * D; e += kJacobiThreads) {
      const int i = e / D, j = e % D;
      const double x = A[i * LDA + j];
      if (i == j) dia += x * x; else off += x * x;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      off += __shfl_xor_sync(0xffffffffu, off, o);
      dia += __shfl_xor_sync(0xffffffffu, dia, o);
    }
    if ((tid & 31) == 0) {
      red[0][tid >> 5] = off;
      red[1][tid >> 5] = dia;
    }
    __syncthreads();
    if (tid == 0) {
      double o2 = 0.0, d2 = 0.0;
      for (int w = 0; w < kJacobiThreads / 32; ++w) {
        o2 += red[0][w];
        d2 += red[1][w];
      }
      s_done = (o2 <= 1e-30 * d2) ? 1 : 0;
    }
    __syncthreads();
    if (s_done) break;
    for (int round = 0; round < D - 1; ++round) {
      if (tid < D / 2) {
        int p, q;
        pair_of(round, tid, p, q);
        const double app = A[p * LDA + p], aqq = A[q * LDA + q], apq = A[p * LDA + q];
        double c = 1.0, s = 0.0;
        if (apq != 0.0) {
          const double tau = (aqq - app) / (2.0 * apq);
          double t;
          if (fabs(tau) > 1e100) {
            t = 0.5 / tau;
          } else {
            t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
          }
          c = 1.0 / sqrt(1.0 + t * t);
          s = t * c;
        }
        cs[tid][0] = c;
        cs[tid][1] = s;
        pq[tid][0] = p;
        pq[tid][1] = q;
      }
      __syncthreads();
      // rows: A <- J^T A
      for (int e = tid; e < (D / 2) * D; e += kJacobiThreads) {
        const int pr = e / D, col = e % D;
        const int p = pq[pr][0], q = pq[pr][1];
        const double c = cs[pr][0], s = cs[pr][1];
        const double ap = A[p * LDA + col], aq = A[q * LDA + col];
        A[p * LDA + col] = c * ap - s * aq;
        A[q * LDA + col] = s * ap + c * aq;
      }
      __syncthreads();
      // columns: A <- A J, V <- V J
      for (int e = tid; e < (D / 2) * D; e += kJacobiThreads) {
        const int pr = e / D, row = e % D;
        const int p = pq[pr][0], q = pq[pr][1];
        const double c = cs[pr][0], s = cs[pr][1];
        const double ap = A[row * LDA + p], aq = A[row * LDA + q];
        A[row * LDA + p] = c * ap - s * aq;
        A[row * LDA + q] = s * ap + c * aq;
        const double vp = V[(size_t)row * D + p], vq = V[(size_t)row * D + q];
        V[(size_t)row * D + p] = c * vp - s * vq;
        V[(size_t)row * D + q] = s * vp + c * vq;
      }
      __syncthreads();
    }
  }
  // order by descending eigenvalue (ties by index), fix each column's sign
  if (tid < D) {
    const int j = tid;
    const double lj = A[j * LDA + j];
    int rank = 0;
    for (int i = 0; i < D; ++i) {
      const double li = A[i * LDA + i];
      rank += (li > lj) || (li == lj && i < j);
    }
    int imax = 0;
    double vmax = -1.0;
    for (int i = 0; i < D; ++i) {
      const double a = fabs(V[(size_t)i * D + j]);
      if (a > vmax) {
        vmax = a;
        imax = i;
      }
    }
    const double sg = V[(size_t)imax * D + j] < 0.0 ? -1.0 : 1.0;
    for (int i = 0; i < D; ++i) P_out[(size_t)i * D + rank] = (float)(sg * V[(size_t)i * D + j]);
    sigma_out[rank] = (float)sqrt(lj > 0.0 ? lj : 0.0);
  }
}

}  // namespace

size_t calibrate_workspace_bytes(int n, int /*d*/) {
  const size_t nb = (size_t)gram_blocks(n);
  return (nb * D * D + 2 * (size_t)D * D) * sizeof(double);
}

int launch_calibrate(const float* X, int n, float* P_out, float* sigma_out, void* ws, cudaStream_t st) {
  const int nb = gram_blocks(n);
  const int rows = (n + nb - 1) / nb;
  double* part = static_cast<double*>(ws);
  double* A = part + (size_t)nb * D * D;
  double* V = A + (size_t)D * D;
  gram_partial_kernel<<<nb, kGramThreads, 0, st>>>(X, n, rows, part);
  int rc = check_launch("gram_partial_kernel");
  if (rc != AQUA_OK) return rc;
  gram_sum_kernel<<<D, D, 0, st>>>(part, nb, A);
  if ((rc = check_launch("gram_sum_kernel")) != AQUA_OK) return rc;
  const int smem = D * LDA * (int)sizeof(double);
  if ((rc = set_smem_limit(jacobi_kernel, smem, "jacobi_kernel")) != AQUA_OK) return rc;
  jacobi_kernel<<<1, kJacobiThreads, smem, st>>>(A, V, P_out, sigma_out);
  return check_launch("jacobi_kernel");
}

}  // namespace aqua
