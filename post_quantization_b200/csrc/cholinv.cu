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
// Leaves of at most 128 columns are factored and inverted in shared memory by one CTA. The four
// products per level are large square GEMMs on the tensor cores (operands split into three bf16
// pieces, fp32-accurate) that skip the zero triangles of K.
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace kq {

namespace {

constexpr int NB = 128;   // leaf size

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
// upper triangle with K = R^-1. One CTA of 512 threads; thread t keeps the 4 x 8 block
// rows 4*(t/16) .. +3, columns 8*(t%16) .. +7 in registers. Both sweeps are right-looking with
// one barrier per column; the column (row) that drives a step is published in shared memory by
// the threads that own it:
//   factor   c = nb-1 .. 0:  u = S_:c;  R_:c = u / sqrt(u_c);  S_ik -= u_i u_k / u_c  (i <= k < c)
//   inverse  i = nb-1 .. 0:  K_ij = (delta_ij - acc_ij) / R_ii (j >= i);  acc_rj += R_ri K_ij (r < i)
constexpr int LEAF_THREADS = 512;
constexpr int LD_R = NB + 1;
constexpr size_t LEAF_SMEM = sizeof(float) * (NB * LD_R + 4 * NB);

__global__ void __launch_bounds__(LEAF_THREADS, 1) leaf_kernel(float* __restrict__ a, int64_t ld,
                                                            int nb, int j0,
                                                            int32_t* __restrict__ info) {
  extern __shared__ float leaf_smem[];
  float* R = leaf_smem;                 // NB x LD_R: the factor R
  float* pub = leaf_smem + NB * LD_R;   // 2 x NB double-buffered published column / row
  if (*info >= 0) return;
  const int tid = threadIdx.x;
  const int r0 = 4 * (tid >> 4);        // first owned row
  const int c0 = 8 * (tid & 15);        // first owned column
  float s[4][8];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = r0 + r, k = c0 + j;
      s[r][j] = (i < nb && k < nb && k >= i) ? a[i * ld + k] : 0.f;
    }
  for (int e = tid; e < NB * LD_R; e += blockDim.x) R[e] = 0.f;
  __syncthreads();

  for (int c = nb - 1; c >= 0; --c) {
    float* u = pub + (c & 1) * NB;
    if ((c >> 3) == (tid & 15)) {            // owners of column c publish it
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        // pick s[r][c % 8] with masks (an indexed read would move s to local memory)
        int vi = 0;
        const int cj = c & 7;
#pragma unroll
        for (int j = 0; j < 8; ++j) vi |= __float_as_int(s[r][j]) & -static_cast<int>(j == cj);
        u[r0 + r] = __int_as_float(vi);
      }
    }
    __syncthreads();
    const float piv = u[c];
    if (!(piv > 0.f) || !isfinite(piv)) {
      if (tid == 0) *info = j0 + c;
      return;                                // uniform: every thread read the same pivot
    }
    const float inv = 1.f / piv;
    if (tid < c) R[tid * LD_R + c] = u[tid] * rsqrtf(piv);
    if (tid == c) R[c * LD_R + c] = sqrtf(piv);
    // only blocks that meet the shrinking triangle i <= k < c have work
    if (c0 < c && r0 <= c0 + 7) {
      float ui[4], uk[8];
#pragma unroll
      for (int r = 0; r < 4; ++r) ui[r] = u[r0 + r] * inv;
#pragma unroll
      for (int j = 0; j < 8; ++j) uk[j] = u[c0 + j];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i = r0 + r, k = c0 + j;
          if (k < c && i <= k) s[r][j] -= ui[r] * uk[j];
        }
    }
  }
  __syncthreads();   // R complete

  // inverse: the registers now accumulate, and end up holding K
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int j = 0; j < 8; ++j) s[r][j] = 0.f;
  for (int i = nb - 1; i >= 0; --i) {
    float* kr = pub + (i & 1) * NB;
    if ((i >> 2) == (tid >> 4)) {            // owners of row i finish it and publish it
      const float rinv = 1.f / R[i * LD_R + i];
      const int ir = i & 3;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int k = c0 + j;
        float acc = s[0][j];
        acc = ir == 1 ? s[1][j] : acc;
        acc = ir == 2 ? s[2][j] : acc;
        acc = ir == 3 ? s[3][j] : acc;
        const float v = (k >= i && k < nb) ? ((k == i ? 1.f : 0.f) - acc) * rinv : 0.f;
        s[0][j] = ir == 0 ? v : s[0][j];
        s[1][j] = ir == 1 ? v : s[1][j];
        s[2][j] = ir == 2 ? v : s[2][j];
        s[3][j] = ir == 3 ? v : s[3][j];
        kr[k] = v;
      }
    }
    __syncthreads();
    // rows above i, columns from i on
    if (r0 < i && c0 + 7 >= i) {
      float rri[4], kij[8];
#pragma unroll
      for (int r = 0; r < 4; ++r) rri[r] = R[(r0 + r) * LD_R + i];
#pragma unroll
      for (int j = 0; j < 8; ++j) kij[j] = kr[c0 + j];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (r0 + r < i) s[r][j] += rri[r] * kij[j];
    }
  }
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = r0 + r, k = c0 + j;
      if (i < nb && k < nb) a[i * ld + k] = (k >= i) ? s[r][j] : 0.f;
    }
}

struct Ctx {
  int64_t ld;
  float* t;          // n1 x n2 product T of the top level (largest)
  uint8_t* splits;   // split operands of one GEMM at a time
  int32_t* info;
  cudaStream_t stream;
};

// Overwrite the n x n diagonal block at a (global index j0) with K.
kronq_status chol_inv_rec(const Ctx& c, float* a, int n, int j0) {
  if (n <= NB) {
    leaf_kernel<<<1, LEAF_THREADS, LEAF_SMEM, c.stream>>>(a, c.ld, n, j0, c.info);
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
  cudaStream_t st = c.stream;

  KQ_TRY(chol_inv_rec(c, a22, n2, j0 + n1));                               // K22
  {
    // R12 = A12 K22^T, written over A12 (the GEMM reads split copies)
    Carve cv{c.splits};
    Split3 s12 = cv.split(n1, n2), s22 = cv.split(n2, n2);
    KQ_TRY(split_bf16x3_2(a12, ld, n1, n2, s12, a22, ld, n2, n2, s22, st));
    KQ_TRY(tgemm(n1, n2, n2, 1.f, s12, s22, false, 0.f, a12, ld, false, GEMM_B_LOWER, c.info, st));
  }
  {
    // A11 -= R12 R12^T (upper triangle)
    Carve cv{c.splits};
    Split3 r12 = cv.split(n1, n2);
    KQ_TRY(split_bf16x3(a12, ld, n1, n2, r12, st));
    KQ_TRY(tgemm(n1, n1, n2, -1.f, r12, r12, false, 1.f, a11, ld, true, 0, c.info, st));
  }
  KQ_TRY(chol_inv_rec(c, a11, n1, j0));                                    // K11
  {
    // T = R12 K22
    Carve cv{c.splits};
    Split3 r12 = cv.split(n1, n2), s22 = cv.split(n2, n2);
    KQ_TRY(split_bf16x3_2(a12, ld, n1, n2, r12, a22, ld, n2, n2, s22, st));
    KQ_TRY(tgemm(n1, n2, n2, 1.f, r12, s22, true, 0.f, c.t, n2, false, GEMM_B_UPPER, c.info, st));
  }
  {
    // K12 = -K11 T
    Carve cv{c.splits};
    Split3 s11 = cv.split(n1, n1), tt = cv.split(n1, n2);
    KQ_TRY(split_bf16x3_2(a11, ld, n1, n1, s11, c.t, n2, n1, n2, tt, st));
    KQ_TRY(tgemm(n1, n2, n1, -1.f, s11, tt, true, 0.f, a12, ld, false, GEMM_A_UPPER, c.info, st));
  }
  return KRONQ_OK;
}

// Sizes of the top level (the largest of every level).
void top_split(int d, int& n1, int& n2) {
  if (d <= NB) {
    n1 = n2 = 0;
    return;
  }
  n2 = ((d / 2 + NB - 1) / NB) * NB;
  if (n2 >= d) n2 = d - NB;
  n1 = d - n2;
}

size_t t_bytes(int d) {
  int n1, n2;
  top_split(d, n1, n2);
  return align256(sizeof(float) * static_cast<size_t>(n1 > 0 ? n1 : 1) * (n2 > 0 ? n2 : 1));
}

size_t split_area_bytes(int d) {
  int n1, n2;
  top_split(d, n1, n2);
  if (n1 == 0) return 0;
  // the largest GEMM operand pair of any level is at the top level
  const size_t a = split_bytes(n1, n2) + split_bytes(n2, n2);
  const size_t b = split_bytes(n1, n1) + split_bytes(n1, n2);
  return a > b ? a : b;
}

}  // namespace

size_t cholinv_workspace_bytes(int d) { return 256 + t_bytes(d) + split_area_bytes(d); }

kronq_status run_cholinv(float* a, int d, float damp_rel, int32_t* info, void* ws,
                         cudaStream_t stream) {
  uint8_t* p = static_cast<uint8_t*>(ws);
  float* lam = reinterpret_cast<float*>(p);
  p += 256;
  float* t = reinterpret_cast<float*>(p);
  p += t_bytes(d);
  damping_kernel<<<1, 1024, 0, stream>>>(a, d, damp_rel, lam, info);
  KQ_TRY(check_launch("damping_kernel"));
  {
    dim3 grid((d + 255) / 256, d);
    prep_kernel<<<grid, 256, 0, stream>>>(a, d, lam);
    KQ_TRY(check_launch("prep_kernel"));
  }
  static bool attr = false;
  if (!attr) {
    KQ_CUDA_TRY(cudaFuncSetAttribute(leaf_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(LEAF_SMEM)));
    attr = true;
  }
  Ctx c{d, t, p, info, stream};
  return chol_inv_rec(c, a, d, 0);
}

}  // namespace kq
