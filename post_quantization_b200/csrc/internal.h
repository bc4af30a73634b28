// Internal launchers shared between the kernel files and the C ABI layer.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kronq.h"

namespace kq {

// accumulate.cu
kronq_status launch_accumulate_tc(const void* a, int64_t ld_a, const void* b, int64_t ld_b,
                                  int64_t k, int m, int n, float* c, int64_t ldc, bool symmetric,
                                  cudaStream_t stream);
kronq_status launch_mirror_upper(float* c, int64_t ldc, int d, cudaStream_t stream);
kronq_status launch_drift_split(const void* xfp, int64_t ld_xfp, const void* xq, int64_t ld_xq,
                                int64_t rows, int cols, void* hi, void* lo, int64_t ld_out,
                                cudaStream_t stream);

// biip.cu
struct BiipArgs {
  const void* w;
  int w_dtype;
  float* w_out;
  float* hx;
  float* hg;
  float* dxx;
  double inv_n;
  const int8_t* sign_in;
  const int8_t* sign_out;
  int d_out, d_in;
  uint32_t flags;
  float* s_x;
  float* s_g;
  double* tr_hx;
  double* tr_hg;
};
size_t biip_workspace_bytes(int d_out, int d_in);
kronq_status run_biip(const BiipArgs& a, void* ws, cudaStream_t stream);

// cholinv.cu
size_t cholinv_workspace_bytes(int d);
kronq_status run_cholinv(float* a, int d, float damp_rel, int32_t* info, void* ws,
                         cudaStream_t stream);

// quantize.cu
size_t quantize_workspace_bytes(int d_out, int d_in, int block, bool with_dxx);
kronq_status run_quantize(const float* w, const float* k, const float* dxx, int d_out, int d_in,
                          int bits, int block, uint8_t* codes, float* scale, float* zero,
                          float* w_hat, void* ws, cudaStream_t stream);

// sgemm.cu: C = alpha * op(A) op(B) + beta * C, fp32 on CUDA cores.
//   op(A) is M x K: A stored M x K (lda) or, when ta, K x M.
//   op(B) is K x N: B stored K x N (ldb) or, when tb, N x K.
//   upper_only: only elements with col >= row are written (tiles fully below are skipped).
//   tri: zero structure of the operands (the zeros must be stored), used to skip K ranges:
//     GEMM_A_UPPER  op(A)[m][k] = 0 for k < m
//     GEMM_B_UPPER  op(B)[k][n] = 0 for k > n
//     GEMM_B_LOWER  op(B)[k][n] = 0 for k < n
//   skip_if_nonneg: device int; the kernel does nothing when it holds a value >= 0.
enum { GEMM_A_UPPER = 1, GEMM_B_UPPER = 2, GEMM_B_LOWER = 4 };
kronq_status sgemm(bool ta, bool tb, int m, int n, int k, float alpha, const float* a,
                   int64_t lda, const float* b, int64_t ldb, float beta, float* c, int64_t ldc,
                   bool upper_only, const int32_t* skip_if_nonneg, cudaStream_t stream,
                   int tri = 0);

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace kq
