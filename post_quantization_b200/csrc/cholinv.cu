// Damped inverse Cholesky factor K (upper, K^T K = (H + lambda I)^-1).
//
// KronQ (hyper.ai summary), Method, OBS update: the rows "[H_X^-1]_p,p+1:" that the column
// update subtracts are the rows of K. Route: reverse-order (UL) Cholesky H + lambda I = R R^T
// with R upper, blocked from the bottom-right corner, then the blocked triangular inverse
// K = R^-1 (by uniqueness of the Cholesky factorization, K is the upper Cholesky factor of the
// damped inverse). lambda = damp_rel * mean(diag H).
//
// Per 64-wide block (from the last one up):
//   diag    one CTA factors the block (A22 = R22 R22^T) and inverts it (K22 = R22^-1) in smem
//   panel   R12 = A12 K22^T                       (fp32 GEMM)
//   update  A11 -= R12 R12^T, upper triangle only (fp32 GEMM)
// then, per block row from the bottom:  K_i,>i = -K_ii (R_i,>i K_>i,>i).
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

// Factor the nb x nb diagonal block at (j0, j0): A22 = R R^T (R upper), write K22 = R^-1.
__global__ void __launch_bounds__(256) ul_diag_kernel(float* __restrict__ a, int d, int j0, int nb,
                                                      int32_t* __restrict__ info) {
  __shared__ float S[NB][NB + 1];
  __shared__ float Kt[NB][NB + 1];
  __shared__ int failed;
  if (*info >= 0) return;
  const int tid = threadIdx.x;
  if (tid == 0) failed = 0;
  for (int e = tid; e < NB * NB; e += blockDim.x) {
    const int i = e / NB, k = e % NB;
    float v = 0.f;
    if (i < nb && k < nb && k >= i) v = a[static_cast<int64_t>(j0 + i) * d + j0 + k];
    if (i >= nb || k >= nb) v = (i == k) ? 1.f : 0.f;
    S[i][k] = v;
    Kt[i][k] = 0.f;
  }
  __syncthreads();
  // column c from the last to the first
  const int col = tid & (NB - 1);   // thread's column in the trailing update
  const int half = tid / NB;        // 0..3: strided rows
  for (int c = nb - 1; c >= 0; --c) {
    if (tid == 0) {
      const float piv = S[c][c];
      if (!(piv > 0.f) || !isfinite(piv)) {
        failed = 1;
        *info = j0 + c;
      } else {
        S[c][c] = sqrtf(piv);
      }
    }
    __syncthreads();
    if (failed) return;
    const float r = S[c][c];
    for (int i = tid; i < c; i += blockDim.x) S[i][c] = S[i][c] / r;
    __syncthreads();
    if (col < c) {
      const float rk = S[col][c];
      for (int i = half; i <= col; i += 4) S[i][col] -= S[i][c] * rk;
    }
    __syncthreads();
  }
  // K = R^-1, one row of K per step from the bottom: K_ij = (delta_ij - sum_{l>i} R_il K_lj) / R_ii
  for (int i = nb - 1; i >= 0; --i) {
    for (int j = tid; j < nb; j += blockDim.x) {
      if (j < i) continue;
      float s = (i == j) ? 1.f : 0.f;
      for (int l = i + 1; l <= j; ++l) s -= S[i][l] * Kt[l][j];
      Kt[i][j] = s / S[i][i];
    }
    __syncthreads();
  }
  for (int e = tid; e < nb * nb; e += blockDim.x) {
    const int i = e / nb, k = e % nb;
    a[static_cast<int64_t>(j0 + i) * d + j0 + k] = (k >= i) ? Kt[i][k] : 0.f;
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

}  // namespace

size_t cholinv_workspace_bytes(int d) {
  return align256(sizeof(float) * static_cast<size_t>(d) * NB) + 256;
}

kronq_status run_cholinv(float* a, int d, float damp_rel, int32_t* info, void* ws,
                         cudaStream_t stream) {
  float* panel = static_cast<float*>(ws);   // up to d x NB
  float* lam = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                        align256(sizeof(float) * static_cast<size_t>(d) * NB));
  damping_kernel<<<1, 1024, 0, stream>>>(a, d, damp_rel, lam, info);
  KQ_TRY(check_launch("damping_kernel"));
  {
    dim3 grid((d + 255) / 256, d);
    prep_kernel<<<grid, 256, 0, stream>>>(a, d, lam);
    KQ_TRY(check_launch("prep_kernel"));
  }
  // factorization, blocks from the bottom-right corner
  for (int j1 = d; j1 > 0; j1 -= NB) {
    const int j0 = j1 > NB ? j1 - NB : 0;
    const int nb = j1 - j0;
    ul_diag_kernel<<<1, 256, 0, stream>>>(a, d, j0, nb, info);
    KQ_TRY(check_launch("ul_diag_kernel"));
    if (j0 == 0) break;
    // R12 = A12 K22^T  -> panel (j0 x nb), then back into A12
    KQ_TRY(sgemm(false, true, j0, nb, nb, 1.f, a + j0, d, a + static_cast<int64_t>(j0) * d + j0,
                 d, 0.f, panel, nb, false, info, stream));
    {
      int64_t blocks = (static_cast<int64_t>(j0) * nb + 255) / 256;
      if (blocks > 4096) blocks = 4096;
      copy_panel_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(panel, nb, a + j0, d, j0, nb);
      KQ_TRY(check_launch("copy_panel_kernel"));
    }
    // A11 -= R12 R12^T (upper triangle)
    KQ_TRY(sgemm(false, true, j0, j0, nb, -1.f, panel, nb, panel, nb, 1.f, a, d, true, info,
                 stream));
  }
  // inversion, block rows from the bottom: K_i,>i = -K_ii (R_i,>i K_>i,>i)
  for (int i1 = d; i1 > 0;) {
    const int i0 = i1 > NB ? i1 - NB : 0;   // same block boundaries as the factorization
    const int nbi = i1 - i0;
    const int m = d - i1;
    if (m > 0) {
      // T = R_i,>i K_>i,>i  (nbi x m)
      KQ_TRY(sgemm(false, false, nbi, m, m, 1.f, a + static_cast<int64_t>(i0) * d + i1, d,
                   a + static_cast<int64_t>(i1) * d + i1, d, 0.f, panel, m, false, info, stream));
      // K_i,>i = -K_ii T
      KQ_TRY(sgemm(false, false, nbi, m, nbi, -1.f, a + static_cast<int64_t>(i0) * d + i0, d,
                   panel, m, 0.f, a + static_cast<int64_t>(i0) * d + i1, d, false, info, stream));
    }
    i1 = i0;
  }
  return KRONQ_OK;
}

}  // namespace kq
