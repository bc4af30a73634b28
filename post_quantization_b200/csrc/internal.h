// Internal launchers shared between the kernel files and the C ABI layer.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kronq.h"

namespace kq {

// accumulate.cu
// C (m x n, fp32, ldc) += A^T B with A: k x m, B: k x n, token-major (ld_a, ld_b elements),
// bf16 (f16 false) or fp16 (f16 true). amax (device, 2 floats, may be NULL): the operands were
// scaled by powers of two taken from these magnitudes (launch_drift_fp16); the epilogue divides
// the products by the same powers.
kronq_status launch_accumulate_tc(const void* a, int64_t ld_a, const void* b, int64_t ld_b,
                                  int64_t k, int m, int n, float* c, int64_t ldc, bool symmetric,
                                  cudaStream_t stream, bool f16 = false,
                                  const float* amax = nullptr);
kronq_status launch_mirror_upper(float* c, int64_t ldc, int d, cudaStream_t stream);
// amax[0] = max |xfp - xq|, amax[1] = max |xq| over rows x cols bf16 (amax zeroed first)
kronq_status launch_drift_amax(const void* xfp, int64_t ld_xfp, const void* xq, int64_t ld_xq,
                               int64_t rows, int cols, float* amax, cudaStream_t stream);
// da = fp16((xfp - xq) 2^ea), xb = fp16(xq 2^eb), rows x cols, row stride ld_out elements
kronq_status launch_drift_fp16(const void* xfp, int64_t ld_xfp, const void* xq, int64_t ld_xq,
                               int64_t rows, int cols, const float* amax, void* da, void* xb,
                               int64_t ld_out, cudaStream_t stream);
size_t accumulate_diag_workspace_bytes(int64_t n, int d);
// tokens one kronq_accumulate_diag call takes: 2048 per block row of the grid, 65535 rows
constexpr int64_t kMaxDiagTokens = 65535LL * 2048;
// SM count of the current device (queried per call; 148 if the query fails)
int device_sms();
kronq_status launch_accumulate_diag(const void* g, int64_t ld, int64_t n, int d, float* diag_sum,
                                    void* ws, cudaStream_t stream);

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
                          int bits, int block, int group, uint8_t* codes, float* scale,
                          float* zero, float* w_hat, void* ws, cudaStream_t stream);

// quantize.cu: rounding with feedback on both sides (comparison variant, not KronQ)
size_t twosided_workspace_bytes(int d_out, int d_in);
kronq_status run_twosided(const float* w, const float* k_in, const float* k_out, int d_out,
                          int d_in, int bits, uint8_t* codes, float* scale, float* zero,
                          float* w_hat, int32_t* iterations, void* ws, cudaStream_t stream);

// qlinear.cu: the quantized layer at inference (packed codes, input/output transforms).
struct QlinearArgs {
  const void* x;
  int x_dtype;
  int64_t ld_x;
  int n_tok;
  const void* packed;
  const void* grid;
  int group;
  const float* s_x;
  const float* s_g;
  const int8_t* sign_in;
  const int8_t* sign_out;
  uint32_t flags;
  int d_out, d_in, bits;
  float* y;
  int64_t ld_y;
};
size_t packed_code_bytes(int d_out, int d_in, int bits);
kronq_status run_pack_codes(const uint8_t* codes, int d_out, int d_in, int bits, void* packed,
                            cudaStream_t stream);
size_t packed_grid_bytes(int d_out, int d_in, int group);
kronq_status run_pack_grid(const float* scale, const float* zero, int d_out, int d_in, int group,
                           void* packed, cudaStream_t stream);
size_t qlinear_workspace_bytes(int d_out, int d_in, int n_tok);
kronq_status run_qlinear(const QlinearArgs& q, void* ws, cudaStream_t stream);

// Zero structure of GEMM operands (the zeros must be stored), used to skip K ranges:
//   GEMM_A_UPPER  A[m][k] = 0 for k < m
//   GEMM_B_UPPER  op(B)[k][n] = 0 for k > n
//   GEMM_B_LOWER  op(B)[k][n] = 0 for k < n
//   GEMM_A_LOWER  A[m][k] = 0 for k > m
enum { GEMM_A_UPPER = 1, GEMM_B_UPPER = 2, GEMM_B_LOWER = 4, GEMM_A_LOWER = 8 };

// tgemm.cu: fp32-accurate GEMM on tcgen05 tensor cores (bf16 x3 split, six products).
//   An fp32 operand x is first split (split_bf16x3) into three bf16 pieces x0 + x1 + x2 that
//   carry its 24 significant bits, each stored row-major with stride ld (a multiple of 8
//   elements, 16-byte aligned base).
//   C = alpha * A B + beta * C with A: m x k (k contiguous); B: n x k (k contiguous) or, when
//   b_mn_major, k x n (n contiguous). upper_only / tri / skip as for the zero-structure flags.
struct Split3 {
  uint16_t* part[3];
  int64_t ld;
};
kronq_status split_bf16x3(const float* src, int64_t lds, int rows, int cols, Split3 dst,
                          cudaStream_t stream);
// two matrices in one launch
kronq_status split_bf16x3_2(const float* src0, int64_t lds0, int rows0, int cols0, Split3 dst0,
                            const float* src1, int64_t lds1, int rows1, int cols1, Split3 dst1,
                            cudaStream_t stream);
// products: 6 (fp32-accurate: every term down to 2^-16 relative) or 3 (a0 b0 + a0 b1 + a1 b0,
// ~2^-16 relative; the third pieces are not read).
kronq_status tgemm(int m, int n, int k, float alpha, Split3 a, Split3 b, bool b_mn_major,
                   float beta, float* c, int64_t ldc, bool upper_only, int tri,
                   const int32_t* skip, cudaStream_t stream, int products = 6);
// the sub-matrix of a split operand starting at (row, col)
inline Split3 offset(Split3 s, int64_t row, int64_t col) {
  for (int i = 0; i < 3; ++i) s.part[i] += row * s.ld + col;
  return s;
}

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
inline int64_t pad8(int64_t x) { return (x + 7) & ~static_cast<int64_t>(7); }

// Bump allocator over a workspace region (256-byte aligned pieces).
struct Carve {
  uint8_t* p;
  float* floats(size_t n) {
    float* r = reinterpret_cast<float*>(p);
    p += align256(n * sizeof(float));
    return r;
  }
  Split3 split(int rows, int cols) {
    Split3 s;
    s.ld = pad8(cols);
    for (int i = 0; i < 3; ++i) {
      s.part[i] = reinterpret_cast<uint16_t*>(p);
      p += align256(static_cast<size_t>(rows) * s.ld * sizeof(uint16_t));
    }
    return s;
  }
};
inline size_t split_bytes(int rows, int cols) {
  return 3 * align256(static_cast<size_t>(rows) * pad8(cols) * sizeof(uint16_t));
}

}  // namespace kq
