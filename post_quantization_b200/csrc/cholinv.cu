// Damped inverse Cholesky factor K (upper, K^T K = (H + lambda I)^-1).
//
// KronQ (hyper.ai summary), Method, OBS update: the rows "[H_X^-1]_p,p+1:" that the column
// update subtracts are the rows of K. Route: reverse-order (UL) Cholesky H + lambda I = R R^T
// with R upper, and K = R^-1 (by uniqueness of the Cholesky factorization, K is the upper
// Cholesky factor of the damped inverse). lambda = damp_rel * mean(diag H).
//
// Recursive blocked algorithm on a diagonal block A = [[A11, A12], [A12^T, A22]] (upper triangle
// stored, lower triangle zero), which it overwrites with K:
//   K22 = chol_inv(A22)
//   R12 = A12 K22^T                 (A12 = R12 R22^T)
//   A11 <- A11 - R12 R12^T          (upper triangle)
//   K11 = chol_inv(A11)
//   K12 = -K11 R12 K22              ([[R11, R12], [0, R22]]^-1)
// Leaves of at most 64 columns are factored and inverted in shared memory by one CTA. The four
// products per level are large square fp32 GEMMs that skip the zero triangles of K.
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace kq {

namespace {

constexpr int NB = 64;

// lambda = damp_rel * mean(diag A); info = -1.
__global__ void damping_kernel(const float* __restrict__ a, int d, float damp_rel,
                               float* __restrict__ lam, int32_t* __restrict__ info) {
  __shared__ double red[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) s += a[static_cast<int64_t>(i) * d + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) {
      *lam = static_cast<float>(static_cast<double>(damp_rel) * v / d);
      *info = -1;
    }
  }
}

// A_ii += lambda, strict lower triangle := 0 (only the upper triangle is used from here on).
__global__ void prep_kernel(float* __restrict__ a, int d, const float* __restrict__ lam) {
  const int i = blockIdx.y;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j <= i && j < d; j += gridDim.x * blockDim.x) {
    float* p = a + static_cast<int64_t>(i) * d + j;
    if (j < i)
      *p = 0.f;
    else
      *p += *lam;
  }
}

// Leaf: factor the nb x nb diagonal block at a (ld) as A = R R^T (R upper) and overwrite its
// upper triangle with K = R^-1. One CTA of 256 threads.
__global__ void __launch_bounds__(256) leaf_kernel(float* __restrict__ a, int64_t ld, int nb,
                                                   int j0, int32_t* __restrict__ info) {
  __shared__ float S[NB][NB + 1];   // running block (upper triangle), then the inverse K
  __shared__ float R[NB][NB + 1];   // factor R
  if (*info >= 0) return;
  const int tid = threadIdx.x;
  for (int e = tid; e < NB * NB; e += blockDim.x) {
    const int i = e / NB, k = e % NB;
    S[i][k] = (i < nb && k < nb && k >= i) ? a[i * ld + k] : 0.f;
    R[i][k] = 0.f;
  }
  __syncthreads();
  // UL factorization, column c from the last to the first; one barrier per column.
  const int kc = tid & (NB - 1);   // this thread's column in the update
  const int i0 = tid >> 6;         // and its first row (rows i0, i0 + 4, ...)
  for (int c = nb - 1; c >= 0; --c) {
    const float piv = S[c][c];
    if (!(piv > 0.f) || !isfinite(piv)) {
      if (tid == 0) *info = j0 + c;
      return;                       // uniform: every thread read the same pivot
    }
    const float inv = 1.f / piv;
    if (tid < c) R[tid][c] = S[tid][c] * rsqrtf(piv);
    if (tid == c) R[c][c] = sqrtf(piv);
    if (kc < c) {
      const float s_kc = S[kc][c] * inv;
      for (int i = i0; i <= kc; i += 4) S[i][kc] -= S[i][c] * s_kc;
    }
    __syncthreads();
  }
  // K = R^-1 row by row from the bottom: K_ij = (delta_ij - sum_{i<l<=j} R_il K_lj) / R_ii.
  // Four threads share one column's dot product. K reuses the storage of S.
  float(*Kt)[NB + 1] = S;
  for (int e = tid; e < NB * NB; e += blockDim.x) Kt[e / NB][e % NB] = 0.f;
  __syncthreads();
  const int j = tid >> 2, part = tid & 3;
  for (int i = nb - 1; i >= 0; --i) {
    float s = 0.f;
    if (j < nb && j > i)
      for (int l = i + 1 + part; l <= j; l += 4) s += R[i][l] * Kt[l][j];
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    if (part == 0 && j < nb && j >= i) Kt[i][j] = ((i == j ? 1.f : 0.f) - s) / R[i][i];
    __syncthreads();
  }
  for (int e = tid; e < nb * nb; e += blockDim.x) {
    const int i = e / nb, k = e % nb;
    a[i * ld + k] = (k >= i) ? Kt[i][k] : 0.f;
  }
}

// Copy a rows x cols panel (row strides lds / ldd).
__global__ void copy_panel_kernel(const float* __restrict__ src, int64_t lds, float* __restrict__ dst,
                                  int64_t ldd, int rows, int cols) {
  const int64_t total = static_cast<int64_t>(rows) * cols;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = e / cols, c = e - r * cols;
    dst[r * ldd + c] = src[r * lds + c];
  }
}

struct Ctx {
  int64_t ld;
  float* ws;        // at least (n/2)^2 floats
  int32_t* info;
  cudaStream_t stream;
};

// Overwrite the n x n diagonal block at a (global index j0) with K.
kronq_status chol_inv_rec(const Ctx& c, float* a, int n, int j0) {
  if (n <= NB) {
    leaf_kernel<<<1, 256, 0, c.stream>>>(a, c.ld, n, j0, c.info);
    return check_launch("leaf_kernel");
  }
  // bottom-right part: a multiple of NB columns, about half
  int n2 = ((n / 2 + NB - 1) / NB) * NB;
  if (n2 >= n) n2 = n - NB;
  const int n1 = n - n2;
  float* a11 = a;
  float* a12 = a + n1;
  float* a22 = a + static_cast<int64_t>(n1) * c.ld + n1;
  const int64_t ld = c.ld;
  KQ_TRY(chol_inv_rec(c, a22, n2, j0 + n1));                                    // K22
  KQ_TRY(sgemm(false, true, n1, n2, n2, 1.f, a12, ld, a22, ld, 0.f, c.ws, n2, false, c.info,
               c.stream, GEMM_B_LOWER));                                        // R12 = A12 K22^T
  {
    int64_t blocks = (static_cast<int64_t>(n1) * n2 + 255) / 256;
    if (blocks > 8192) blocks = 8192;
    copy_panel_kernel<<<static_cast<int>(blocks), 256, 0, c.stream>>>(c.ws, n2, a12, ld, n1, n2);
    KQ_TRY(check_launch("copy_panel_kernel"));
  }
  KQ_TRY(sgemm(false, true, n1, n1, n2, -1.f, a12, ld, a12, ld, 1.f, a11, ld, true, c.info,
               c.stream));                                                      // A11 -= R12 R12^T
  KQ_TRY(chol_inv_rec(c, a11, n1, j0));                                         // K11
  KQ_TRY(sgemm(false, false, n1, n2, n2, 1.f, a12, ld, a22, ld, 0.f, c.ws, n2, false, c.info,
               c.stream, GEMM_B_UPPER));                                        // T = R12 K22
  KQ_TRY(sgemm(false, false, n1, n2, n1, -1.f, a11, ld, c.ws, n2, 0.f, a12, ld, false, c.info,
               c.stream, GEMM_A_UPPER));                                        // K12 = -K11 T
  return KRONQ_OK;
}

size_t ws_floats(int d) {
  const size_t h = static_cast<size_t>(d / 2 + NB);
  return h * h;
}

}  // namespace

size_t cholinv_workspace_bytes(int d) { return align256(sizeof(float) * ws_floats(d)) + 256; }

kronq_status run_cholinv(float* a, int d, float damp_rel, int32_t* info, void* ws,
                         cudaStream_t stream) {
  float* scratch = static_cast<float*>(ws);
  float* lam = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                        align256(sizeof(float) * ws_floats(d)));
  damping_kernel<<<1, 1024, 0, stream>>>(a, d, damp_rel, lam, info);
  KQ_TRY(check_launch("damping_kernel"));
  {
    dim3 grid((d + 255) / 256, d);
    prep_kernel<<<grid, 256, 0, stream>>>(a, d, lam);
    KQ_TRY(check_launch("prep_kernel"));
  }
  Ctx c{d, scratch, info, stream};
  return chol_inv_rec(c, a, d, 0);
}

}  // namespace kq
