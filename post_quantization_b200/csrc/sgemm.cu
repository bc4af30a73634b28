// fp32 GEMM on CUDA cores: C = alpha * op(A) op(B) + beta * C.
//
// Used where the quantizer needs full fp32 products (the blocked Cholesky/inverse, the GPTAQ
// pre-shift and the lazy trailing update of the column solve): bf16/tf32 tensor-core products
// would perturb the error feedback enough to flip quantized codes.
// 128 x 128 output tile per CTA, 256 threads, 8 x 8 outputs per thread, K step 8, operands
// staged k-major in shared memory.
#include "common.cuh"
#include "internal.h"

namespace kq {

namespace {

constexpr int TM = 128, TN = 128, TK = 8;

template <bool TA, bool TB>
__global__ void __launch_bounds__(256) sgemm_kernel(int M, int N, int K, float alpha,
                                                    const float* __restrict__ A, int64_t lda,
                                                    const float* __restrict__ B, int64_t ldb,
                                                    float beta, float* __restrict__ C, int64_t ldc,
                                                    int upper_only, int tri,
                                                    const int32_t* skip) {
  if (skip && *skip >= 0) return;
  const int bm = blockIdx.y * TM, bn = blockIdx.x * TN;
  if (upper_only && bm > bn + TN - 1) return;
  // K range that can be non-zero for this tile when an operand is triangular
  int k_lo = 0, k_hi = K;
  if (tri & GEMM_A_UPPER) k_lo = max(k_lo, bm);
  if (tri & GEMM_B_LOWER) k_lo = max(k_lo, bn);
  if (tri & GEMM_B_UPPER) k_hi = min(k_hi, bn + TN);
  k_lo = (k_lo / TK) * TK;
  __shared__ __align__(16) float As[TK][TM + 4];
  __shared__ __align__(16) float Bs[TK][TN + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  for (int k0 = k_lo; k0 < k_hi; k0 += TK) {
    // ---- stage op(A)[bm:bm+128, k0:k0+8] as As[k][m]
    if (!TA) {
      const int m = tid >> 1, kq = (tid & 1) * 4;
      const int gm = bm + m;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int gk = k0 + kq + e;
        As[kq + e][m] = (gm < M && gk < K) ? A[static_cast<int64_t>(gm) * lda + gk] : 0.f;
      }
    } else {
      const int k = tid >> 5, mq = (tid & 31) * 4;
      const int gk = k0 + k;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int gm = bm + mq + e;
        As[k][mq + e] = (gm < M && gk < K) ? A[static_cast<int64_t>(gk) * lda + gm] : 0.f;
      }
    }
    // ---- stage op(B)[k0:k0+8, bn:bn+128] as Bs[k][n]
    if (!TB) {
      const int k = tid >> 5, nq = (tid & 31) * 4;
      const int gk = k0 + k;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int gn = bn + nq + e;
        Bs[k][nq + e] = (gn < N && gk < K) ? B[static_cast<int64_t>(gk) * ldb + gn] : 0.f;
      }
    } else {
      const int n = tid >> 1, kq = (tid & 1) * 4;
      const int gn = bn + n;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int gk = k0 + kq + e;
        Bs[kq + e][n] = (gn < N && gk < K) ? B[static_cast<int64_t>(gn) * ldb + gk] : 0.f;
      }
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[kk][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[kk][64 + tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int gm = bm + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int gn = bn + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (gn >= N) continue;
      if (upper_only && gn < gm) continue;
      float* cp = C + static_cast<int64_t>(gm) * ldc + gn;
      float v = alpha * acc[i][j];
      if (beta != 0.f) v = fmaf(beta, *cp, v);
      *cp = v;
    }
  }
}

}  // namespace

kronq_status sgemm(bool ta, bool tb, int m, int n, int k, float alpha, const float* a,
                   int64_t lda, const float* b, int64_t ldb, float beta, float* c, int64_t ldc,
                   bool upper_only, const int32_t* skip, cudaStream_t stream, int tri) {
  if (m <= 0 || n <= 0) return KRONQ_OK;
  dim3 grid((n + TN - 1) / TN, (m + TM - 1) / TM);
  const int up = upper_only ? 1 : 0;
  if (!ta && !tb)
    sgemm_kernel<false, false><<<grid, 256, 0, stream>>>(m, n, k, alpha, a, lda, b, ldb, beta, c,
                                                         ldc, up, tri, skip);
  else if (!ta && tb)
    sgemm_kernel<false, true><<<grid, 256, 0, stream>>>(m, n, k, alpha, a, lda, b, ldb, beta, c,
                                                        ldc, up, tri, skip);
  else if (ta && !tb)
    sgemm_kernel<true, false><<<grid, 256, 0, stream>>>(m, n, k, alpha, a, lda, b, ldb, beta, c,
                                                        ldc, up, tri, skip);
  else
    sgemm_kernel<true, true><<<grid, 256, 0, stream>>>(m, n, k, alpha, a, lda, b, ldb, beta, c,
                                                       ldc, up, tri, skip);
  return check_launch("sgemm_kernel");
}

}  // namespace kq
