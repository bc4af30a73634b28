// Bidirectional incoherence processing (BiIP) of one sublayer.
//
// KronQ (hyper.ai summary), Method, BiIP equations:
//   W <- S_G W S_X,  S_X = diag(H_X,jj / |W_:,j|^2)^(1/4),  S_G = diag(H_G,ii / |W_i,:|^2)^(1/4)
//   W <- U W V^T,  H_X <- V H_X V^T,  H_G <- U H_G U^T,  dXX^T <- V dXX^T V^T
// with U, V = (1/sqrt(b)) (I (x) H_b) diag(random signs), H_b Sylvester, b = largest power of
// two dividing the dimension. The Hessians follow the scaling as S^-1 H S^-1.
//
// Passes (all bandwidth-bound):
//   norms   one read of W: |W_:,j|^2 and |W_i,:|^2 (fp64 sums)
//   scales  S_X, S_G, the per-row / per-column factors of the passes below, traces
//   rows    for every row: multiply by row and column factors, FWHT along the row in b-blocks
//   cols    for every b-row block of every column: FWHT along the column (in place; one pass
//           for b <= 256, two for larger b)
// The passes work in registers (16-point butterflies per thread) with a shared-memory exchange
// between groups of four stages; b outside [16, 16384] takes plain shared-memory kernels.
// W' = rows(W) then cols; H_X and dXX^T = rows then cols (in place); H_G likewise if asked.
#include <cuda_bf16.h>

#include <cmath>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace kq {

namespace {

constexpr int kNormRows = 64;
constexpr int kNormCols = 256;

template <typename T>
__device__ __forceinline__ float load_as_float(const T* p, int64_t i);
template <>
__device__ __forceinline__ float load_as_float<float>(const float* p, int64_t i) {
  return p[i];
}
template <>
__device__ __forceinline__ float load_as_float<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}

// Partial squared column and row norms of a 64 x 256 tile, added into fp64 accumulators.
template <typename T>
__global__ void __launch_bounds__(256) colrow_norms_kernel(const T* __restrict__ w, int rows,
                                                           int cols, double* __restrict__ col_sq,
                                                           double* __restrict__ row_sq) {
  __shared__ float part[8][kNormRows];
  const int c = blockIdx.x * kNormCols + threadIdx.x;
  const int r0 = blockIdx.y * kNormRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float colacc = 0.f;
  for (int r = 0; r < kNormRows; ++r) {
    const int row = r0 + r;
    float v = 0.f;
    if (row < rows && c < cols) v = load_as_float(w, static_cast<int64_t>(row) * cols + c);
    const float sq = v * v;
    colacc += sq;
    float rs = sq;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, o);
    if (lane == 0) part[warp][r] = rs;
  }
  if (c < cols) atomicAdd(&col_sq[c], static_cast<double>(colacc));
  __syncthreads();
  if (threadIdx.x < kNormRows) {
    const int row = r0 + threadIdx.x;
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) s += part[k][threadIdx.x];
    if (row < rows) atomicAdd(&row_sq[row], static_cast<double>(s));
  }
}

// (diag * inv_n / norm_sq)^(1/4), or 1 where either is not positive.
__device__ __forceinline__ double biip_scale(double diag_raw, double inv_n, double norm_sq) {
  const double dg = diag_raw * inv_n;
  if (!(dg > 0.0) || !(norm_sq > 0.0)) return 1.0;
  return sqrt(sqrt(dg / norm_sq));
}

// Scales and factor vectors for one side (d entries).
//   s        = S (fp32 output)
//   fw       = S * sign            (factor on W)
//   fh       = sign / S            (factor on the Hessian, both sides)
__global__ void side_scales_kernel(int d, const float* __restrict__ h, const double* __restrict__ nsq,
                                   double inv_n, int do_scale, const int8_t* __restrict__ sign,
                                   float* __restrict__ s_out, float* __restrict__ fw,
                                   float* __restrict__ fh) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= d) return;
  double s = 1.0;
  if (do_scale) s = biip_scale(h[static_cast<int64_t>(i) * d + i], inv_n, nsq[i]);
  const double sg = sign ? static_cast<double>(sign[i]) : 1.0;
  s_out[i] = static_cast<float>(s);
  fw[i] = static_cast<float>(s * sg);
  fh[i] = static_cast<float>(sg / s);
}

// tr(S^-1 (inv_n H) S^-1) = sum_i inv_n H_ii / s_i^2, in fp64 (one block).
__global__ void side_trace_kernel(int d, const float* __restrict__ h, const double* __restrict__ nsq,
                                  double inv_n, int do_scale, double* __restrict__ tr) {
  __shared__ double red[32];
  double acc = 0.0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    const double hii = static_cast<double>(h[static_cast<int64_t>(i) * d + i]) * inv_n;
    double s = 1.0;
    if (do_scale) s = biip_scale(h[static_cast<int64_t>(i) * d + i], inv_n, nsq[i]);
    acc += hii / (s * s);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) *tr = v;
  }
}

// Row pass over a rows x cols matrix seen as a flat array of b-blocks (b divides cols):
// dst = FWHT_b(src * row_factor[r] * col_factor[c] * scalar) / sqrt(b), one chunk per CTA.
template <typename T>
__global__ void __launch_bounds__(256) fwht_rows_kernel(const T* src, float* dst, int64_t rows,
                                                        int64_t cols, const float* __restrict__ row_f,
                                                        const float* __restrict__ col_f, float scalar,
                                                        int log2b, int chunk, float out_scale) {
  extern __shared__ float sbuf[];
  const int64_t total = rows * cols;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * chunk;
  for (int e = threadIdx.x; e < chunk; e += blockDim.x) {
    const int64_t f = base + e;
    float v = 0.f;
    if (f < total) {
      const int64_t r = f / cols;
      const int64_t c = f - r * cols;
      v = load_as_float(src, f) * scalar;
      if (row_f) v *= row_f[r];
      if (col_f) v *= col_f[c];
    }
    sbuf[e] = v;
  }
  __syncthreads();
  const int half = chunk >> 1;
  for (int h = 0; h < log2b; ++h) {
    const int lowmask = (1 << h) - 1;
    for (int p = threadIdx.x; p < half; p += blockDim.x) {
      const int i = ((p >> h) << (h + 1)) | (p & lowmask);
      const int j = i | (1 << h);
      const float a = sbuf[i], b = sbuf[j];
      sbuf[i] = a + b;
      sbuf[j] = a - b;
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < chunk; e += blockDim.x) {
    const int64_t f = base + e;
    if (f < total) dst[f] = sbuf[e] * out_scale;
  }
}

// Column pass, in place: for each column, FWHT along rows in blocks of b; tile = b x cw.
__global__ void __launch_bounds__(256) fwht_cols_kernel(float* m, int64_t rows, int64_t cols,
                                                        int log2b, int cw, float out_scale) {
  extern __shared__ float sbuf[];
  const int b = 1 << log2b;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * cw;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * b;
  const int n = b * cw;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const int r = e / cw, c = e - r * cw;
    float v = 0.f;
    if (c0 + c < cols) v = m[(r0 + r) * cols + c0 + c];
    sbuf[e] = v;
  }
  __syncthreads();
  const int pairs = (b >> 1) * cw;
  for (int h = 0; h < log2b; ++h) {
    const int lowmask = (1 << h) - 1;
    for (int q = threadIdx.x; q < pairs; q += blockDim.x) {
      const int c = q % cw, p = q / cw;
      const int i = ((p >> h) << (h + 1)) | (p & lowmask);
      const int j = i | (1 << h);
      const float a = sbuf[i * cw + c], bb = sbuf[j * cw + c];
      sbuf[i * cw + c] = a + bb;
      sbuf[j * cw + c] = a - bb;
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const int r = e / cw, c = e - r * cw;
    if (c0 + c < cols) m[(r0 + r) * cols + c0 + c] = sbuf[e] * out_scale;
  }
}

// ---- register-radix passes (16 <= b <= 16384) ----
//
// Row pass: one CTA per chunk of C = max(b, 4096) consecutive elements (whole b-blocks),
// C / 16 threads. Round 0 takes 16 consecutive elements per thread straight from global
// memory and transforms index bits 0-3 in registers; round R takes the 16 elements whose index
// differs in bits 4R..4R+3 (stride 16^R) from shared memory. The last round writes to global
// memory, coalesced. log2(b) stages cost ceil(log2(b) / 4) - 1 shared-memory round trips.
//
// Column pass: a P-point transform along rows r_base + rs * j (j < P) of a tile of 32
// columns, P in [16, 256]. b <= 256 is one pass (P = b, rs = 1); larger b is two passes,
// 64-point over consecutive rows, then (b / 64)-point at row stride 64
// (H_b = (H_{b/64} (x) I_64)(I_{b/64} (x) H_64)). Every global access is a 128-byte row segment.

// 16-point Walsh-Hadamard butterflies on register-index bits [h0, h0 + nbits).
__device__ __forceinline__ void fwht16(float (&x)[16], int nbits, int h0 = 0) {
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    if (h >= h0 && h < h0 + nbits) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (j & (1 << h)) continue;
        const float a = x[j], b = x[j | (1 << h)];
        x[j] = a + b;
        x[j | (1 << h)] = a - b;
      }
    }
  }
}

__device__ __forceinline__ int pad16(int i) { return i + (i >> 4); }

__device__ __forceinline__ void load16(const float* p, bool vec, float (&x)[16]) {
  if (vec) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = reinterpret_cast<const float4*>(p)[q];
      x[4 * q] = v.x; x[4 * q + 1] = v.y; x[4 * q + 2] = v.z; x[4 * q + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k) x[k] = p[k];
  }
}

__device__ __forceinline__ void load16(const __nv_bfloat16* p, bool vec, float (&x)[16]) {
  if (vec) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint4 v = reinterpret_cast<const uint4*>(p)[q];
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[8 * q + 2 * e] = __uint_as_float(u[e] << 16);
        x[8 * q + 2 * e + 1] = __uint_as_float(u[e] & 0xFFFF0000u);
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k) x[k] = __bfloat162float(p[k]);
  }
}

// src may equal dst (every element is read before the chunk's first write).
template <typename T>
__global__ void __launch_bounds__(1024) fwht_rows_reg_kernel(
    const T* src, float* dst, int64_t total, int64_t cols, const float* __restrict__ row_f,
    const float* __restrict__ col_f, float scalar, int log2b, int chunk, float out_scale,
    int vec) {
  extern __shared__ float sb[];
  const int t = threadIdx.x;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * chunk;
  const int rounds = (log2b + 3) >> 2;
  float x[16];
  const int64_t f0 = base + 16 * t;
  if (f0 < total) {   // total is a multiple of b >= 16, so a group is all in or all out
    load16(src + f0, vec != 0, x);
    const int64_t r = f0 / cols;
    const int64_t c0 = f0 - r * cols;
    const float rf = row_f ? scalar * row_f[r] : scalar;
#pragma unroll
    for (int k = 0; k < 16; ++k) x[k] *= col_f ? rf * col_f[c0 + k] : rf;
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k) x[k] = 0.f;
  }
  fwht16(x, log2b < 4 ? log2b : 4);
  if (rounds == 1) {
    if (f0 < total) {
#pragma unroll
      for (int k = 0; k < 16; ++k) dst[f0 + k] = x[k] * out_scale;
    }
    return;
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) sb[pad16(16 * t + k)] = x[k];
  // log2 of the chunk: every round's 16-element window must stay inside it
  const int log2c = 31 - __clz(chunk);
  for (int R = 1; R < rounds; ++R) {
    __syncthreads();
    // round R transforms index bits [4R, min(4R + 4, log2b)); its window of 4 index bits starts
    // at 4R, or lower when that would leave the chunk (the last round of b > 4096), in which
    // case the bits below 4R ride along untouched
    const int nbits = log2b - 4 * R < 4 ? log2b - 4 * R : 4;
    const int sh = 4 * R + 4 <= log2c ? 4 * R : log2c - 4;
    const int s = 1 << sh;
    const int lo = (t & (s - 1)) + ((t >> sh) << (sh + 4));
#pragma unroll
    for (int k = 0; k < 16; ++k) x[k] = sb[pad16(lo + s * k)];
    fwht16(x, nbits, 4 * R - sh);
    if (R == rounds - 1) {
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int64_t f = base + lo + static_cast<int64_t>(s) * k;
        if (f < total) dst[f] = x[k] * out_scale;
      }
    } else {
#pragma unroll
      for (int k = 0; k < 16; ++k) sb[pad16(lo + s * k)] = x[k];
    }
  }
}

// P-point transform along rows r_base + rs * j of 32 columns, in place; 2P threads.
constexpr int kColTile = 32;
__global__ void __launch_bounds__(512) fwht_cols_reg_kernel(float* m, int64_t rows, int64_t cols,
                                                            int log2p, int rs, float out_scale) {
  extern __shared__ float sb[];
  const int P = 1 << log2p;
  const int t = threadIdx.x;
  const int c = t & (kColTile - 1);
  const int64_t col = static_cast<int64_t>(blockIdx.x) * kColTile + c;
  const bool cin = col < cols;
  const int y = blockIdx.y;
  const int64_t r_base = static_cast<int64_t>(y / rs) * P * rs + (y % rs);
  constexpr int LDT = kColTile + 1;
  float x[16];
  {
    const int jg = t / kColTile;   // round 0: rows 16 jg .. 16 jg + 15
#pragma unroll
    for (int k = 0; k < 16; ++k)
      x[k] = cin ? m[(r_base + static_cast<int64_t>(rs) * (16 * jg + k)) * cols + col] : 0.f;
    fwht16(x, 4);
    if (log2p == 4) {
      if (cin) {
#pragma unroll
        for (int k = 0; k < 16; ++k)
          m[(r_base + static_cast<int64_t>(rs) * (16 * jg + k)) * cols + col] = x[k] * out_scale;
      }
      return;
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) sb[(16 * jg + k) * LDT + c] = x[k];
  }
  __syncthreads();
  // round 1: bits 4.. of j; groups (c, jl), jl in [0, 16), P / 16 elements each
  const int M = P >> 4, per = 256 / P, q = t / kColTile;
  for (int u = 0; u < per; ++u) {
    const int jl = q * per + u;
#pragma unroll
    for (int mm = 0; mm < 16; ++mm) x[mm] = mm < M ? sb[(jl + 16 * mm) * LDT + c] : 0.f;
    fwht16(x, log2p - 4);
    if (cin) {
#pragma unroll
      for (int mm = 0; mm < 16; ++mm)
        if (mm < M)
          m[(r_base + static_cast<int64_t>(rs) * (jl + 16 * mm)) * cols + col] = x[mm] * out_scale;
    }
  }
}

int ilog2_pow2(int b) {
  int l = 0;
  while ((1 << l) < b) ++l;
  return l;
}

int largest_pow2_divisor(int d) { return d & (-d); }

template <typename T>
kronq_status row_pass(const T* src, float* dst, int64_t rows, int64_t cols, const float* row_f,
                      const float* col_f, float scalar, int b, cudaStream_t stream) {
  const int chunk = b > 4096 ? b : 4096;
  const int64_t total = rows * cols;
  const int64_t blocks = (total + chunk - 1) / chunk;
  const float out_scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(b)));
  if (b >= 16 && b <= 16384) {
    const int threads = chunk / 16;
    const size_t smem = static_cast<size_t>(chunk + chunk / 16) * sizeof(float);
    if (smem > 48 * 1024)
      KQ_CUDA_TRY(cudaFuncSetAttribute(fwht_rows_reg_kernel<T>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    const int vec = (reinterpret_cast<uintptr_t>(src) & 15u) == 0 &&
                    (reinterpret_cast<uintptr_t>(dst) & 15u) == 0;
    fwht_rows_reg_kernel<T><<<static_cast<unsigned>(blocks), threads, smem, stream>>>(
        src, dst, total, cols, row_f, col_f, scalar, ilog2_pow2(b), chunk, out_scale, vec);
    return check_launch("fwht_rows_reg_kernel");
  }
  const size_t smem = static_cast<size_t>(chunk) * sizeof(float);
  if (smem > 48 * 1024)
    KQ_CUDA_TRY(cudaFuncSetAttribute(fwht_rows_kernel<T>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  fwht_rows_kernel<T><<<static_cast<unsigned>(blocks), 256, smem, stream>>>(
      src, dst, rows, cols, row_f, col_f, scalar, ilog2_pow2(b), chunk, out_scale);
  return check_launch("fwht_rows_kernel");
}

// One P-point column pass (P in [16, 256]) at row stride rs.
kronq_status col_pass_reg(float* m, int64_t rows, int64_t cols, int log2p, int rs, float out_scale,
                          cudaStream_t stream) {
  const int P = 1 << log2p;
  const size_t smem = static_cast<size_t>(P) * (kColTile + 1) * sizeof(float);
  dim3 grid(static_cast<unsigned>((cols + kColTile - 1) / kColTile),
            static_cast<unsigned>(rows / P));
  fwht_cols_reg_kernel<<<grid, 2 * P, smem, stream>>>(m, rows, cols, log2p, rs, out_scale);
  return check_launch("fwht_cols_reg_kernel");
}

kronq_status col_pass(float* m, int64_t rows, int64_t cols, int b, cudaStream_t stream) {
  if (b <= 1) return KRONQ_OK;
  const float out_scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(b)));
  if (b >= 16 && b <= 16384) {
    const int L = ilog2_pow2(b);
    if (L <= 8) return col_pass_reg(m, rows, cols, L, 1, out_scale, stream);
    const int l1 = (L + 1) / 2, l2 = L / 2;   // H_b = (H_P2 (x) I_P1)(I_P2 (x) H_P1)
    KQ_TRY(col_pass_reg(m, rows, cols, l1, 1, 1.0f, stream));
    return col_pass_reg(m, rows, cols, l2, 1 << l1, out_scale, stream);
  }
  int cw = 32768 / b;
  if (cw > 64) cw = 64;
  if (cw < 1) cw = 1;
  const size_t smem = static_cast<size_t>(b) * cw * sizeof(float);
  if (smem > 48 * 1024)
    KQ_CUDA_TRY(cudaFuncSetAttribute(fwht_cols_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  dim3 grid(static_cast<unsigned>((cols + cw - 1) / cw), static_cast<unsigned>(rows / b));
  fwht_cols_kernel<<<grid, 256, smem, stream>>>(m, rows, cols, ilog2_pow2(b), cw, out_scale);
  return check_launch("fwht_cols_kernel");
}

struct BiipWs {
  double* col_sq;   // d_in
  double* row_sq;   // d_out
  float* fw_in;     // d_in   S_X * sign_in
  float* fh_in;     // d_in   sign_in / S_X
  float* fw_out;    // d_out  S_G * sign_out
  float* fh_out;    // d_out  sign_out / S_G
};

BiipWs carve(void* ws, int d_out, int d_in) {
  uint8_t* p = static_cast<uint8_t*>(ws);
  BiipWs w;
  w.col_sq = reinterpret_cast<double*>(p);
  p += align256(sizeof(double) * d_in);
  w.row_sq = reinterpret_cast<double*>(p);
  p += align256(sizeof(double) * d_out);
  w.fw_in = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * d_in);
  w.fh_in = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * d_in);
  w.fw_out = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * d_out);
  w.fh_out = reinterpret_cast<float*>(p);
  return w;
}

}  // namespace

size_t biip_workspace_bytes(int d_out, int d_in) {
  return align256(sizeof(double) * d_in) + align256(sizeof(double) * d_out) +
         2 * align256(sizeof(float) * d_in) + 2 * align256(sizeof(float) * d_out);
}

kronq_status run_biip(const BiipArgs& a, void* ws_raw, cudaStream_t stream) {
  const BiipWs ws = carve(ws_raw, a.d_out, a.d_in);
  const bool scale_in = a.flags & KRONQ_BIIP_SCALE_IN;
  const bool scale_out = a.flags & KRONQ_BIIP_SCALE_OUT;
  const bool rot_in = a.flags & KRONQ_BIIP_ROTATE_IN;
  const bool rot_out = a.flags & KRONQ_BIIP_ROTATE_OUT;
  const bool write_hg = (a.flags & KRONQ_BIIP_WRITE_HG) && a.hg;
  const int b_in = rot_in ? largest_pow2_divisor(a.d_in) : 1;
  const int b_out = rot_out ? largest_pow2_divisor(a.d_out) : 1;

  // 1. squared column / row norms of the original W
  KQ_CUDA_TRY(cudaMemsetAsync(ws.col_sq, 0, sizeof(double) * a.d_in, stream));
  KQ_CUDA_TRY(cudaMemsetAsync(ws.row_sq, 0, sizeof(double) * a.d_out, stream));
  {
    dim3 grid((a.d_in + kNormCols - 1) / kNormCols, (a.d_out + kNormRows - 1) / kNormRows);
    if (a.w_dtype == KRONQ_DTYPE_BF16)
      colrow_norms_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(a.w), a.d_out, a.d_in, ws.col_sq, ws.row_sq);
    else
      colrow_norms_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float*>(a.w),
                                                           a.d_out, a.d_in, ws.col_sq, ws.row_sq);
    KQ_TRY(check_launch("colrow_norms_kernel"));
  }

  // 2. scales, factors and traces (from the un-transformed diagonals)
  side_scales_kernel<<<(a.d_in + 255) / 256, 256, 0, stream>>>(
      a.d_in, a.hx, ws.col_sq, a.inv_n, scale_in, rot_in ? a.sign_in : nullptr, a.s_x, ws.fw_in,
      ws.fh_in);
  KQ_TRY(check_launch("side_scales_kernel(in)"));
  side_trace_kernel<<<1, 1024, 0, stream>>>(a.d_in, a.hx, ws.col_sq, a.inv_n, scale_in, a.tr_hx);
  KQ_TRY(check_launch("side_trace_kernel(in)"));
  side_scales_kernel<<<(a.d_out + 255) / 256, 256, 0, stream>>>(
      a.d_out, a.hg, ws.row_sq, a.inv_n, scale_out, rot_out ? a.sign_out : nullptr, a.s_g,
      ws.fw_out, ws.fh_out);
  KQ_TRY(check_launch("side_scales_kernel(out)"));
  if (a.hg && a.tr_hg) {
    side_trace_kernel<<<1, 1024, 0, stream>>>(a.d_out, a.hg, ws.row_sq, a.inv_n, scale_out,
                                              a.tr_hg);
    KQ_TRY(check_launch("side_trace_kernel(out)"));
  }

  // 3. W' = U S_G W S_X V^T: row pass (scales, output signs, input-side FWHT), column pass
  if (a.w_dtype == KRONQ_DTYPE_BF16)
    KQ_TRY(row_pass(static_cast<const __nv_bfloat16*>(a.w), a.w_out, a.d_out, a.d_in, ws.fw_out,
                    ws.fw_in, 1.0f, b_in, stream));
  else
    KQ_TRY(row_pass(static_cast<const float*>(a.w), a.w_out, a.d_out, a.d_in, ws.fw_out, ws.fw_in,
                    1.0f, b_in, stream));
  KQ_TRY(col_pass(a.w_out, a.d_out, a.d_in, b_out, stream));

  // 4. H_X <- V S_X^-1 (inv_n H_X) S_X^-1 V^T, same for dXX^T; H_G if asked
  const float inv_n = static_cast<float>(a.inv_n);
  KQ_TRY(row_pass(static_cast<const float*>(a.hx), a.hx, a.d_in, a.d_in, ws.fh_in, ws.fh_in, inv_n,
                  b_in, stream));
  KQ_TRY(col_pass(a.hx, a.d_in, a.d_in, b_in, stream));
  if (a.dxx) {
    KQ_TRY(row_pass(static_cast<const float*>(a.dxx), a.dxx, a.d_in, a.d_in, ws.fh_in, ws.fh_in,
                    inv_n, b_in, stream));
    KQ_TRY(col_pass(a.dxx, a.d_in, a.d_in, b_in, stream));
  }
  if (write_hg) {
    KQ_TRY(row_pass(static_cast<const float*>(a.hg), a.hg, a.d_out, a.d_out, ws.fh_out, ws.fh_out,
                    inv_n, b_out, stream));
    KQ_TRY(col_pass(a.hg, a.d_out, a.d_out, b_out, stream));
  }
  return KRONQ_OK;
}

}  // namespace kq

// ---------------------------------------------------------------------------------------------
// Variant of kronq_biip that allocates nothing: its scratch is a fixed array in device memory
// that every GPU holds from the moment this library is loaded until the process exits.
// ---------------------------------------------------------------------------------------------
namespace {
constexpr size_t kBiipStaticScratchBytes = size_t(1) << 20;   // 1 MiB
__device__ __align__(256) unsigned char g_biip_static_scratch[kBiipStaticScratchBytes];
constexpr int kMaxScratchDevices = 64;
void* g_biip_static_ptr[kMaxScratchDevices] = {nullptr};
std::mutex g_biip_static_mu;
}  // namespace

extern "C" kronq_status kronq_biip_noalloc(const void* w, int32_t w_dtype, float* w_out, float* hx,
                                           float* hg, float* dxx, double inv_n,
                                           const int8_t* sign_in, const int8_t* sign_out,
                                           int32_t d_out, int32_t d_in, uint32_t flags,
                                           float* s_x, float* s_g, double* tr_hx, double* tr_hg,
                                           kronq_stream_t stream) {
  if (d_out <= 0 || d_in <= 0)
    return kq::fail(KRONQ_ERR_SHAPE, "d_out and d_in must be positive");
  const size_t need = kq::biip_workspace_bytes(d_out, d_in);
  if (need > kBiipStaticScratchBytes)
    return kq::fail(KRONQ_ERR_UNSUPPORTED,
                    "kronq_biip_noalloc: d_out + d_in too large for the %zu-byte static scratch "
                    "(%zu bytes needed); use kronq_biip with a workspace",
                    kBiipStaticScratchBytes, need);
  int dev = 0;
  KQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxScratchDevices)
    return kq::fail(KRONQ_ERR_UNSUPPORTED, "device index %d out of range", dev);
  void* scratch = nullptr;
  {
    // first call on this device: look up the device address of the static array
    std::lock_guard<std::mutex> lock(g_biip_static_mu);
    if (!g_biip_static_ptr[dev]) {
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_biip_static_scratch);
      if (e != cudaSuccess || !p)
        return kq::fail(KRONQ_ERR_CUDA, "cudaGetSymbolAddress(static scratch): %s",
                        cudaGetErrorString(e));
      g_biip_static_ptr[dev] = p;
    }
    scratch = g_biip_static_ptr[dev];
  }
  return kronq_biip(w, w_dtype, w_out, hx, hg, dxx, inv_n, sign_in, sign_out, d_out, d_in, flags,
                    s_x, s_g, tr_hx, tr_hg, scratch, kBiipStaticScratchBytes, stream);
}

