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
// The row and column passes stream TMA-loaded chunks through shared memory: 32-point
// butterflies along 128-byte tile rows in registers, the higher index bits in vectorised rounds
// down the tile columns (fwht_rows_tma_kernel, fwht_cols_tma_kernel). b = 16 or 16384,
// unaligned operands and matrices narrower than 32 columns take register/shuffle kernels
// (fwht_rows_reg_kernel, fwht_cols_reg_kernel); b outside [16, 16384] plain shared-memory ones.
// W' = rows(W) then cols; H_X and dXX^T = rows then cols (in place); H_G likewise if asked.
#include <cuda_bf16.h>

#include <cmath>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace kq {

namespace {


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

// Squared column and row norms of a contiguous rows x cols W, added into fp64 accumulators. A CTA
// takes a panel of 32 V columns (V elements = one 16-byte load per lane) and chunk_rows rows (the
// host sizes the chunks so that the grid is one wave of resident CTAs); warp w takes rows w,
// w + 8, .. of it. Per row the warp sums its lanes' squares with five shuffles
// and one lane adds the row's panel sum; per column the lanes keep running sums, which the 8
// warps combine in shared memory at the end, one addition per column and CTA.
template <typename T>
__global__ void __launch_bounds__(256, 3) colrow_norms_kernel(const T* __restrict__ w, int rows,
                                                           int cols, int vec, int chunk_rows,
                                                           double* __restrict__ col_sq,
                                                           double* __restrict__ row_sq) {
  constexpr int V = 16 / sizeof(T);
  constexpr int PW = 32 * V;   // panel width
  __shared__ float part[8][PW];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c0 = blockIdx.x * PW + lane * V;
  const int r0 = blockIdx.y * chunk_rows;
  const int r1 = rows - r0 < chunk_rows ? rows : r0 + chunk_rows;
  const bool whole = vec && c0 + V <= cols;   // one aligned 16-byte load
  float colacc[V];
#pragma unroll
  for (int e = 0; e < V; ++e) colacc[e] = 0.f;
  // batches of 8 rows per warp, their loads issued together
  for (int rb = r0 + warp; rb < r1; rb += 64) {
    uint4 u[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int r = rb + 8 * j;
      if (whole && r < r1)
        u[j] = *reinterpret_cast<const uint4*>(w + static_cast<int64_t>(r) * cols + c0);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int r = rb + 8 * j;
      if (r >= r1) break;
      float v[V];
      if (whole) {
        const uint32_t q[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if constexpr (V == 8) {
            v[2 * e] = __uint_as_float(q[e] << 16);
            v[2 * e + 1] = __uint_as_float(q[e] & 0xFFFF0000u);
          } else {
            v[e] = __uint_as_float(q[e]);
          }
        }
      } else {
        const T* p = w + static_cast<int64_t>(r) * cols + c0;
#pragma unroll
        for (int e = 0; e < V; ++e) v[e] = c0 + e < cols ? load_as_float(p, e) : 0.f;
      }
      float sq = 0.f;
#pragma unroll
      for (int e = 0; e < V; ++e) {
        colacc[e] = fmaf(v[e], v[e], colacc[e]);
        sq = fmaf(v[e], v[e], sq);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
      if (lane == 0) atomicAdd(&row_sq[r], static_cast<double>(sq));
    }
  }
#pragma unroll
  for (int e = 0; e < V; ++e) part[warp][lane * V + e] = colacc[e];
  __syncthreads();
  for (int c = threadIdx.x; c < PW; c += blockDim.x) {
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) sum += part[k][c];
    const int col = blockIdx.x * PW + c;
    if (col < cols) atomicAdd(&col_sq[col], static_cast<double>(sum));
  }
}

// (diag * inv_n / norm_sq)^(1/4), or 1 where either is not positive.
__device__ __forceinline__ double biip_scale(double diag_raw, double inv_n, double norm_sq) {
  const double dg = diag_raw * inv_n;
  if (!(dg > 0.0) || !(norm_sq > 0.0)) return 1.0;
  return sqrt(sqrt(dg / norm_sq));
}

// Scales and factor vectors for one side (d entries), 256 threads per block.
//   s        = S (fp32 output)
//   fw       = S * sign            (factor on W)
//   fh       = sign / S            (factor on the Hessian, both sides)
//   tr_part  (if given) this block's share of tr(S^-1 (inv_n H) S^-1) = sum_i inv_n H_ii / s_i^2
// H_ii is h[i * hstep]: hstep = d + 1 for the full matrix, 1 for a vector of its diagonal.
__global__ void __launch_bounds__(256) side_scales_kernel(int d, const float* __restrict__ h,
                                                          int64_t hstep,
                                                          const double* __restrict__ nsq,
                                                          double inv_n, int do_scale,
                                                          const int8_t* __restrict__ sign,
                                                          float* __restrict__ s_out,
                                                          float* __restrict__ fw,
                                                          float* __restrict__ fh,
                                                          double* __restrict__ tr_part) {
  __shared__ double red[8];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  double contrib = 0.0;
  if (i < d) {
    double s = 1.0;
    if (do_scale) s = biip_scale(h[i * hstep], inv_n, nsq[i]);
    const double sg = sign ? static_cast<double>(sign[i]) : 1.0;
    s_out[i] = static_cast<float>(s);
    fw[i] = static_cast<float>(s * sg);
    fh[i] = static_cast<float>(sg / s);
    if (tr_part) contrib = static_cast<double>(h[i * hstep]) * inv_n / (s * s);
  }
  if (!tr_part) return;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) contrib += __shfl_xor_sync(0xffffffffu, contrib, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = contrib;
  __syncthreads();
  if (threadIdx.x == 0) {
    double v = 0.0;
    for (int k = 0; k < 8; ++k) v += red[k];
    tr_part[blockIdx.x] = v;
  }
}

// tr = sum of the n block shares, in a fixed order (one warp).
__global__ void trace_sum_kernel(const double* __restrict__ part, int n, double* __restrict__ tr) {
  double v = 0.0;
  for (int k = threadIdx.x; k < n; k += 32) v += part[k];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (threadIdx.x == 0) *tr = v;
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
// Row pass: chunks of C = max(b, 4096) consecutive elements (whole b-blocks), C / 16 threads per
// CTA, each CTA walking chunks. A thread takes 16 consecutive elements (streamed in with
// cp.async one chunk ahead) and transforms index bits 0-3 in registers, bits 4-8 with warp
// shuffles, and bits 9 and up through shared memory in 4-bit windows; it stores its 16 elements
// back as 16-byte vectors.
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

// src may equal dst: a chunk is read (the prefetch one iteration earlier) only by the CTA that
// writes it, before it writes it. A CTA walks chunks grid-stride with two staging buffers: the
// next chunk streams in (cp.async, no registers) while the current one is transformed and stored.
// vec = 0 (unaligned operands) takes plain loads instead.
template <typename T, int NT>
__global__ void __launch_bounds__(NT) fwht_rows_reg_kernel(
    const T* src, float* dst, int64_t total, int64_t cols, const float* __restrict__ row_f,
    const float* __restrict__ col_f, float scalar, int log2b, int chunk, float out_scale,
    int vec) {
  extern __shared__ __align__(16) float sb[];
  float* work = sb;                                                   // padded, chunk + chunk/16
  T* stage = reinterpret_cast<T*>(sb + chunk + chunk / 16);           // 2 x chunk elements
  constexpr int PIECES = 16 * sizeof(T) / 16;                         // 16-byte pieces per thread
  const int t = threadIdx.x;
  // log2 of the chunk: every shared-memory window must stay inside it
  const int log2c = 31 - __clz(chunk);
  const int64_t nchunks = (total + chunk - 1) / chunk;
  auto fetch = [&](int64_t c, T* buf) {
    const int64_t f = c * chunk + 16 * t;
    if (f < total) {   // total is a multiple of b >= 16: a group of 16 is all in or all out
#pragma unroll
      for (int q = 0; q < PIECES; ++q) {
        const uint32_t d = static_cast<uint32_t>(
            __cvta_generic_to_shared(reinterpret_cast<uint8_t*>(buf + 16 * t) + 16 * q));
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d),
                     "l"(reinterpret_cast<const uint8_t*>(src + f) + 16 * q)
                     : "memory");
      }
    }
  };
  int cur = 0;
  int64_t ch = blockIdx.x;
  if (vec && ch < nchunks) fetch(ch, stage);
  asm volatile("cp.async.commit_group;" ::: "memory");
  for (; ch < nchunks; ch += gridDim.x) {
    const int64_t f0 = ch * chunk + 16 * t;
    const bool in = f0 < total;
    float x[16];
    if (vec) {
      if (ch + gridDim.x < nchunks) fetch(ch + gridDim.x, stage + (cur ^ 1) * chunk);
      asm volatile("cp.async.commit_group;" ::: "memory");
      asm volatile("cp.async.wait_group 1;" ::: "memory");   // this thread's pieces landed
      if (in) {
        load16(stage + cur * chunk + 16 * t, true, x);
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) x[k] = 0.f;
      }
    } else if (in) {
      load16(src + f0, false, x);
    } else {
#pragma unroll
      for (int k = 0; k < 16; ++k) x[k] = 0.f;
    }
    if (in) {
      int64_t r;
      if (total < (int64_t(1) << 31))
        r = static_cast<uint32_t>(f0) / static_cast<uint32_t>(cols);
      else
        r = f0 / cols;
      const int64_t c0 = f0 - r * cols;
      const float rf = row_f ? scalar * row_f[r] : scalar;
      if (col_f) {
        float cf[16];
        load16(col_f + c0, true, cf);  // 16-byte aligned: workspace base, c0 a multiple of 16
#pragma unroll
        for (int k = 0; k < 16; ++k) x[k] *= rf * cf[k];
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) x[k] *= rf;
      }
    }
    // index bits 0-3: this thread's registers
    fwht16(x, log2b < 4 ? log2b : 4);
    // index bits 4-8: the lanes of the warp (lane = bits 4-8 of 16 t)
    const int lane = t & 31;
    for (int h = 4; h < log2b && h < 9; ++h) {
      const int o = 1 << (h - 4);
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float other = __shfl_xor_sync(0xffffffffu, x[k], o);
        x[k] = upper ? other - x[k] : x[k] + other;
      }
    }
    // index bits 9 and up: across warps, through shared memory in windows of four bits
    if (log2b > 9) {
#pragma unroll
      for (int k = 0; k < 16; ++k) work[pad16(16 * t + k)] = x[k];
      for (int hs = 9; hs < log2b; hs += 4) {
        __syncthreads();
        // the window of 4 index bits starts at hs, or lower when that would leave the chunk;
        // bits below hs ride along untouched
        const int nbits = log2b - hs < 4 ? log2b - hs : 4;
        const int sh = hs + 4 <= log2c ? hs : log2c - 4;
        const int s = 1 << sh;
        const int lo = (t & (s - 1)) + ((t >> sh) << (sh + 4));
#pragma unroll
        for (int k = 0; k < 16; ++k) x[k] = work[pad16(lo + s * k)];
        fwht16(x, nbits, hs - sh);
#pragma unroll
        for (int k = 0; k < 16; ++k) work[pad16(lo + s * k)] = x[k];
      }
      // back to the first layout: 16 consecutive elements per thread
      __syncthreads();
#pragma unroll
      for (int k = 0; k < 16; ++k) x[k] = work[pad16(16 * t + k)];
    }
    if (in) {
      if (vec) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          reinterpret_cast<float4*>(dst + f0)[q] =
              make_float4(x[4 * q] * out_scale, x[4 * q + 1] * out_scale,
                          x[4 * q + 2] * out_scale, x[4 * q + 3] * out_scale);
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) dst[f0 + k] = x[k] * out_scale;
      }
    }
    if (log2b > 9) __syncthreads();   // the next chunk overwrites the work buffer
    cur ^= 1;
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// P-point transform along rows r_base + rs * j of 32-column tiles, in place; 2P threads. The
// tiles move between global and shared memory in 16-byte pieces (8 per row, 128-byte row
// segments); the butterflies read and write them column by column in shared memory. A CTA walks
// tiles grid-stride with two tile buffers: the next tile streams in (cp.async, no registers)
// while the current one is transformed and stored, so HBM stays busy through the butterflies.
// vec = 0 (unaligned or ragged columns) takes plain loads into the current buffer instead.
constexpr int kColTile = 32;
constexpr int kColLd = kColTile + 4;   // 16-byte aligned rows

__device__ __forceinline__ void cp_async16(float* smem_dst, const float* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

template <int LOG2P>
__global__ void __launch_bounds__(2 << LOG2P) fwht_cols_reg_kernel(float* m, int64_t rows,
                                                                  int64_t cols, int rs,
                                                                  float out_scale, int vec) {
  extern __shared__ __align__(16) float sb[];
  constexpr int P = 1 << LOG2P;
  constexpr int nt = 2 * P;
  const int t = threadIdx.x;
  const int tiles_x = static_cast<int>((cols + kColTile - 1) / kColTile);
  const int num_tiles = tiles_x * static_cast<int>(rows / P);
  // top-left of a tile (its first row, r_base + rs * 0, and first column)
  auto origin = [&](int tile, int64_t& col0) {
    const int y = tile / tiles_x;
    col0 = static_cast<int64_t>(tile - y * tiles_x) * kColTile;
    const int64_t r_base = static_cast<int64_t>(y / rs) * P * rs + (y % rs);
    return m + r_base * cols + col0;
  };
  // piece u of this thread in a tile: e = t + nt * u, row j = e / 8, columns 4 (e % 8) ..
  const int64_t row_step = static_cast<int64_t>(rs) * cols;
  auto gaddr = [&](float* org, int64_t col0, int u, int64_t& gc) {
    const int e = t + nt * u, j = e >> 3, c4 = (e & 7) * 4;
    gc = col0 + c4;
    return org + j * row_step + c4;
  };
  auto soff = [&](int u) {
    const int e = t + nt * u;
    return (e >> 3) * kColLd + (e & 7) * 4;
  };
  auto fetch_async = [&](int tile, float* buf) {
    int64_t col0;
    float* org = origin(tile, col0);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      int64_t gc;
      const float* src = gaddr(org, col0, u, gc);
      cp_async16(buf + soff(u), src);
    }
  };
  auto fetch_plain = [&](int tile, float* buf) {
    int64_t col0;
    float* org = origin(tile, col0);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      int64_t gc;
      const float* src = gaddr(org, col0, u, gc);
      float* d = buf + soff(u);
      d[0] = gc < cols ? src[0] : 0.f;
      d[1] = gc + 1 < cols ? src[1] : 0.f;
      d[2] = gc + 2 < cols ? src[2] : 0.f;
      d[3] = gc + 3 < cols ? src[3] : 0.f;
    }
  };
  const int tile_floats = P * kColLd;
  int cur = 0;
  int tile = blockIdx.x;
  if (vec && tile < num_tiles) fetch_async(tile, sb);
  cp_async_commit();
  const int c = t & (kColTile - 1), jg = t / kColTile;
  for (; tile < num_tiles; tile += gridDim.x) {
    float* buf = sb + cur * tile_floats;
    if (vec) {
      if (tile + gridDim.x < num_tiles) fetch_async(tile + gridDim.x, sb + (cur ^ 1) * tile_floats);
      cp_async_commit();
      cp_async_wait1();            // this tile's group has landed (the next may be in flight)
    } else {
      fetch_plain(tile, buf);
    }
    __syncthreads();
    float x[16];
    // round 0: bits 0-3 of j (rows 16 jg .. 16 jg + 15 of column c)
#pragma unroll
    for (int k = 0; k < 16; ++k) x[k] = buf[(16 * jg + k) * kColLd + c];
    fwht16(x, 4);
#pragma unroll
    for (int k = 0; k < 16; ++k) buf[(16 * jg + k) * kColLd + c] = x[k];
    if constexpr (LOG2P > 4) {
      __syncthreads();
      // round 1: bits 4.. of j; groups (c, jl), jl in [0, 16), M = P / 16 elements each
      constexpr int M = P >> 4, per = 256 / P;
#pragma unroll
      for (int w = 0; w < per; ++w) {
        const int jl = jg * per + w;
        float y[M];
#pragma unroll
        for (int mm = 0; mm < M; ++mm) y[mm] = buf[(jl + 16 * mm) * kColLd + c];
#pragma unroll
        for (int h = 0; h < LOG2P - 4; ++h)
#pragma unroll
          for (int mm = 0; mm < M; ++mm) {
            if (mm & (1 << h)) continue;
            const float a = y[mm], b = y[mm | (1 << h)];
            y[mm] = a + b;
            y[mm | (1 << h)] = a - b;
          }
#pragma unroll
        for (int mm = 0; mm < M; ++mm) buf[(jl + 16 * mm) * kColLd + c] = y[mm];
      }
    }
    __syncthreads();
    int64_t col0;
    float* org = origin(tile, col0);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      int64_t gc;
      float* dst = gaddr(org, col0, u, gc);
      const float4 v = *reinterpret_cast<const float4*>(buf + soff(u));
      if (vec) {
        *reinterpret_cast<float4*>(dst) =
            make_float4(v.x * out_scale, v.y * out_scale, v.z * out_scale, v.w * out_scale);
      } else {
        if (gc < cols) dst[0] = v.x * out_scale;
        if (gc + 1 < cols) dst[1] = v.y * out_scale;
        if (gc + 2 < cols) dst[2] = v.z * out_scale;
        if (gc + 3 < cols) dst[3] = v.w * out_scale;
      }
    }
    __syncthreads();   // this buffer is the target of the prefetch two tiles on
    cur ^= 1;
  }
  cp_async_wait0();
}

// ---- tiled row pass (32 <= b <= 8192, 16-byte aligned operands) ----
//
// A chunk is RB = max(1, 4096 / b) matrix rows of one b-wide column band (one Hadamard block per
// row), C = RB b = max(4096, b) elements, seen as C / 32 tile rows of 32: tile row r is matrix
// row RB-row r / (b / 32), columns 32 (r % (b / 32)) .. + 31 of the band. Sylvester's H_b factors
// over index bits, H_b = H_{b/32} (x) H_32, so the transform is a 32-point butterfly along every
// tile row (index bits 0-4) and a (b/32)-point one down the tile columns inside each matrix row
// (bits 5 and up). C / 32 threads; each holds 32 elements in every step:
//   loads     TMA copies the chunk (a box of 32 x b/32 x RB) into one of several stages, up to
//             stages - 1 chunks ahead, completion on the stage's mbarrier; rows past the matrix
//             read as zeros
//   row step  a thread takes one tile row: the scaling (row factor x column factors x scalar x
//             1/sqrt(b); first, as the column factors differ inside a block), the five row bits
//             in registers, then into the fp32 tile (in place for fp32 sources)
//   rounds    a thread takes 2^m tile rows r0 + k 2^h0 (k < 2^m) of 32 / 2^m adjacent columns,
//             so the lanes of a warp cover whole tile rows; butterflies on the low n bits of k.
//             The last round stores to global memory, each tile row one 128-byte segment.
// The CTAs take contiguous ranges of chunks ordered band by band, so a thread's 32 columns stay
// the same from chunk to chunk and their factors stay in registers.
// Shared layouts are XOR-swizzled so that eight lanes reading eight tile rows at one offset and
// lanes reading along one tile row are both free of bank conflicts: 16-byte piece q of 128-byte
// fp32 tile row r sits at q ^ (r % 8) (TMA's 128-byte swizzle), piece q of a 64-byte bf16 row at
// q ^ ((r / 2) % 4) (TMA's 64-byte swizzle).
template <int LOG2B, bool F32>
struct RowTma {
  static constexpr int kLog2S = LOG2B - 5;                        // log2 tile rows per matrix row
  static constexpr int kSegs = 1 << kLog2S;
  static constexpr int kRB = LOG2B >= 12 ? 1 : 1 << (12 - LOG2B);  // matrix rows per chunk
  static constexpr int kLog2C = LOG2B > 12 ? LOG2B : 12;
  static constexpr int kC = 1 << kLog2C;
  static constexpr int kThreads = kC / 32;                         // = tile rows
  static constexpr int kStages = (!F32 && kLog2C == 12) ? 4 : 3;
  static constexpr int kStageBytes = kC * (F32 ? 4 : 2);
  static constexpr int kWorkBytes = F32 ? 0 : kC * 4;              // bf16: separate fp32 tile
  static constexpr int kMinBlocks = kLog2C == 12 ? 4 : 2;          // fits an SM's shared memory
  static constexpr size_t kSmem = 1024 + static_cast<size_t>(kStages) * kStageBytes + kWorkBytes + 64;
};

// Butterfly on two independent pairs at once with Blackwell's packed fp32 arithmetic:
// (a, b) <- (a + b, a - b) per component, rounded exactly as the scalar sum and difference (the
// difference is a fused b * -1 + a, whose product is exact).
__device__ __forceinline__ void bfly2(float2& a, float2& b) {
  const float2 s = __fadd2_rn(a, b);
  b = __ffma2_rn(b, make_float2(-1.f, -1.f), a);
  a = s;
}

// 32-point Walsh-Hadamard butterflies on x[2 i + c] = x2[i].c: index bit 0 inside each pair
// (scalar), bits 1-4 between pairs (packed).
__device__ __forceinline__ void fwht32(float2 (&x)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float a = x[i].x, b = x[i].y;
    x[i] = make_float2(a + b, a - b);
  }
#pragma unroll
  for (int h = 0; h < 4; ++h)
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i & (1 << h)) continue;
      bfly2(x[i], x[i | (1 << h)]);
    }
}

// float offset of 16-byte piece q of tile row r (128-byte rows, 128-byte swizzle)
__device__ __forceinline__ int tpos(int r, int q) { return r * 32 + 4 * (q ^ (r & 7)); }

// One round: tile rows r0 + (k << H0), k < 2^MLOG, butterflies on the low NB bits of k. The last
// round stores tile row r's W columns at out(r, column offset) (skipped where that is null),
// times `scale` if SCALE; the others write back to the tile.
template <int H0, int MLOG, int NB, bool LAST, bool SCALE, typename Out>
__device__ __forceinline__ void tile_round(float* work, int t, float scale, const Out& out) {
  constexpr int M = 1 << MLOG, W = 32 / M;
  const int g = t & (M - 1), s = t >> MLOG;
  const int r0 = (s & ((1 << H0) - 1)) | ((s >> H0) << (H0 + MLOG));
  // float offset of this lane's W columns in tile row r
  auto at = [&](int r) {
    if constexpr (W == 4) return tpos(r, g);
    else if constexpr (W == 2) return tpos(r, g >> 1) + 2 * (g & 1);
    else return tpos(r, g >> 2) + (g & 3);
  };
  if constexpr (W >= 2) {
    constexpr int Y = W / 2;   // column pairs per row, butterflied packed
    float2 y[M][Y];
#pragma unroll
    for (int k = 0; k < M; ++k) {
      const float* p = work + at(r0 + (k << H0));
      if constexpr (W == 4) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        y[k][0] = make_float2(v.x, v.y);
        y[k][Y - 1] = make_float2(v.z, v.w);
      } else {
        y[k][0] = *reinterpret_cast<const float2*>(p);
      }
    }
#pragma unroll
    for (int h = 0; h < NB; ++h)
#pragma unroll
      for (int k = 0; k < M; ++k) {
        if (k & (1 << h)) continue;
#pragma unroll
        for (int e = 0; e < Y; ++e) bfly2(y[k][e], y[k | (1 << h)][e]);
      }
#pragma unroll
    for (int k = 0; k < M; ++k) {
      const int r = r0 + (k << H0);
      float* p;
      if constexpr (LAST) {
        p = out(r, W * g);
        if (!p) continue;
        if constexpr (SCALE) {
#pragma unroll
          for (int e = 0; e < Y; ++e) y[k][e] = __fmul2_rn(y[k][e], make_float2(scale, scale));
        }
      } else {
        p = work + at(r);
      }
      if constexpr (W == 4)
        *reinterpret_cast<float4*>(p) = make_float4(y[k][0].x, y[k][0].y, y[k][Y - 1].x,
                                                    y[k][Y - 1].y);
      else
        *reinterpret_cast<float2*>(p) = y[k][0];
    }
  } else {
    float y[M];
#pragma unroll
    for (int k = 0; k < M; ++k) y[k] = work[at(r0 + (k << H0))];
#pragma unroll
    for (int h = 0; h < NB; ++h)
#pragma unroll
      for (int k = 0; k < M; ++k) {
        if (k & (1 << h)) continue;
        const float a = y[k], b = y[k | (1 << h)];
        y[k] = a + b;
        y[k | (1 << h)] = a - b;
      }
#pragma unroll
    for (int k = 0; k < M; ++k) {
      const int r = r0 + (k << H0);
      if constexpr (LAST) {
        float* p = out(r, g);
        if (!p) continue;
        *p = SCALE ? y[k] * scale : y[k];
      } else {
        work[at(r)] = y[k];
      }
    }
  }
}

// Butterflies on the low L bits of the tile-row index (L <= log2 of the tile rows, at least 7),
// in one or two rounds; a round of m bits starting at bit h0 needs h0 + m <= log2 tile rows.
template <int L, bool SCALE, typename Out>
__device__ __forceinline__ void tile_rounds(float* work, int t, float scale, const Out& out) {
  if constexpr (L == 0) {
    tile_round<0, 3, 0, true, SCALE>(work, t, scale, out);
  } else if constexpr (L <= 3) {
    tile_round<0, 3, L, true, SCALE>(work, t, scale, out);
  } else if constexpr (L == 4 || L == 5) {
    tile_round<0, L, L, true, SCALE>(work, t, scale, out);
  } else if constexpr (L == 6) {
    tile_round<0, 3, 3, false, SCALE>(work, t, scale, out);
    __syncthreads();
    tile_round<3, 3, 3, true, SCALE>(work, t, scale, out);
  } else if constexpr (L == 7) {
    tile_round<0, 3, 3, false, SCALE>(work, t, scale, out);
    __syncthreads();
    tile_round<3, 4, 4, true, SCALE>(work, t, scale, out);
  } else {
    static_assert(L == 8, "tile rounds cover up to 8 index bits");
    tile_round<0, 4, 4, false, SCALE>(work, t, scale, out);
    __syncthreads();
    tile_round<4, 4, 4, true, SCALE>(work, t, scale, out);
  }
}

// dst may be the source matrix itself (fp32): a chunk is loaded (by TMA, up to stages - 1 chunks
// ahead) and written only by the CTA that owns it, load before store.
template <typename T, int LOG2B>
__global__ void __launch_bounds__(RowTma<LOG2B, sizeof(T) == 4>::kThreads,
                                  RowTma<LOG2B, sizeof(T) == 4>::kMinBlocks)
    fwht_rows_tma_kernel(const __grid_constant__ CUtensorMap src_map, float* dst, int64_t rows,
                         int64_t cols, const float* __restrict__ row_f,
                         const float* __restrict__ col_f, float scalar, float out_scale,
                         int* err_word) {
  constexpr bool kF32 = sizeof(T) == 4;
  using S = RowTma<LOG2B, kF32>;
  constexpr int L = LOG2B - 5, LOG2S = S::kLog2S, NST = S::kStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* stages = sm;
  float* work_bf = reinterpret_cast<float*>(sm + NST * S::kStageBytes);   // bf16 sources only
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + NST * S::kStageBytes + S::kWorkBytes);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + NST);
  const int t = threadIdx.x;

  const int64_t nrg = (rows + S::kRB - 1) / S::kRB;        // row groups per band
  const int64_t nchunks = (cols >> LOG2B) * nrg;
  const int64_t k0 = nchunks * blockIdx.x / gridDim.x;
  const int64_t k1 = nchunks * (blockIdx.x + 1) / gridDim.x;
  const int n = static_cast<int>(k1 - k0);
  if (n <= 0) return;

  if (t == 0) {
    prefetch_tensormap(&src_map);
    for (int i = 0; i < NST; ++i) mbar_init(&full[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // chunk k0 + j: band, row group
  auto issue = [&](int j) {
    const int64_t k = k0 + j;
    const int64_t band = k / nrg, rg = k - band * nrg;
    uint64_t* bar = &full[j % NST];
    mbar_arrive_expect_tx(bar, S::kStageBytes);
    tma_load_3d(stages + (j % NST) * S::kStageBytes, &src_map, bar, 0,
                static_cast<int32_t>(band << LOG2S), static_cast<int32_t>(rg * S::kRB));
  };
  if (t == 0)
    for (int j = 0; j < NST - 1 && j < n; ++j) issue(j);

  const int rr = t >> LOG2S, seg = t & (S::kSegs - 1);    // row step: matrix row, segment
  int64_t band = k0 / nrg, rg = k0 - band * nrg;
  int64_t cf_band = -1;
  float2 cf[16];   // factors of this thread's 32 columns, in pairs
  bool aborted = false;
  int i = 0;
  for (; i < n; ++i) {
    const int st = i % NST;
    if (t == 0 && i + NST - 1 < n) issue(i + NST - 1);   // its stage was freed by chunk i - 1
    const int64_t row0 = rg * S::kRB, col0 = band << LOG2B;
    const int64_t row = row0 + rr;
    const float rf = (row_f && row < rows) ? row_f[row] : 1.f;
    if (band != cf_band) {   // column factors x scalar x 1/sqrt(b) of this thread's 32 columns
      const float sc = scalar * out_scale;
      if (col_f) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 v = *reinterpret_cast<const float4*>(col_f + col0 + 32 * seg + 4 * q);
          cf[2 * q] = make_float2(v.x * sc, v.y * sc);
          cf[2 * q + 1] = make_float2(v.z * sc, v.w * sc);
        }
      } else {
#pragma unroll
        for (int p = 0; p < 16; ++p) cf[p] = make_float2(sc, sc);
      }
      cf_band = band;
    }
    const bool ok = mbar_wait(&full[st], (i / NST) & 1, abort_flag, err_word, DEV_ERR_LOAD_WAIT);
    float* work = kF32 ? reinterpret_cast<float*>(stages + st * S::kStageBytes) : work_bf;
    if (ok) {
      float2 x[16];   // x[p] = elements 2 p, 2 p + 1 of tile row t
      if constexpr (kF32) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 v = *reinterpret_cast<const float4*>(work + tpos(t, q));
          x[2 * q] = make_float2(v.x, v.y);
          x[2 * q + 1] = make_float2(v.z, v.w);
        }
      } else {
        const T* sg = reinterpret_cast<const T*>(stages + st * S::kStageBytes) + 32 * t;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 v = *reinterpret_cast<const uint4*>(sg + 8 * (q ^ ((t >> 1) & 3)));
          const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            x[4 * q + e] = make_float2(__uint_as_float(u[e] << 16),
                                       __uint_as_float(u[e] & 0xFFFF0000u));
        }
      }
      if constexpr (S::kRB == 1) {   // one matrix row per chunk: its factor joins the store
#pragma unroll
        for (int p = 0; p < 16; ++p) x[p] = __fmul2_rn(x[p], cf[p]);
      } else {
        const float2 rf2 = make_float2(rf, rf);
#pragma unroll
        for (int p = 0; p < 16; ++p) x[p] = __fmul2_rn(x[p], __fmul2_rn(cf[p], rf2));
      }
      fwht32(x);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        *reinterpret_cast<float4*>(work + tpos(t, q)) =
            make_float4(x[2 * q].x, x[2 * q].y, x[2 * q + 1].x, x[2 * q + 1].y);
    }
    if (__syncthreads_or(!ok)) {
      aborted = true;
      break;
    }
    // the index bits above the tile row; the last round writes tile row r to matrix row
    // row0 + r / segs, columns col0 + 32 (r % segs) ..
    tile_rounds<L, S::kRB == 1>(work, t, rf, [&](int r, int c) -> float* {
      const int64_t row = row0 + (r >> LOG2S);
      return row < rows ? dst + row * cols + col0 + 32 * (r & (S::kSegs - 1)) + c : nullptr;
    });
    if constexpr (kF32) fence_proxy_async_smem();   // the stage was written in place; TMA refills it
    __syncthreads();
    if (++rg == nrg) {
      rg = 0;
      ++band;
    }
  }
  if (aborted && t == 0) {
    // let the loads already issued (chunks i .. i + stages - 1, one per stage) land before the
    // CTA exits
    for (int j = i; j < n && j < i + NST; ++j)
      mbar_drain(&full[j % NST], (j / NST) & 1, kWaitLimitNs);
  }
}

template <typename T>
kronq_status row_pass_tile(const T* src, float* dst, int64_t rows, int64_t cols,
                           const float* row_f, const float* col_f, float scalar, int log2b,
                           float out_scale, cudaStream_t stream) {
  constexpr bool kF32 = sizeof(T) == 4;
  CUtensorMap map;
  const uint64_t dims[3] = {32, static_cast<uint64_t>(cols / 32), static_cast<uint64_t>(rows)};
  const uint64_t strides[2] = {32 * sizeof(T), static_cast<uint64_t>(cols) * sizeof(T)};
  const int b = 1 << log2b;
  const uint32_t box[3] = {32, static_cast<uint32_t>(b / 32),
                           static_cast<uint32_t>(log2b >= 12 ? 1 : 4096 / b)};
  KQ_TRY(encode_tiled_map(&map, kF32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                          3, src, dims, strides, box,
                          kF32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B));
  int* err = device_error_word();
  const int64_t rb = log2b >= 12 ? 1 : 4096 / b;
  const int64_t nchunks = (cols / b) * ((rows + rb - 1) / rb);
  auto launch = [&](auto kern, int nt, size_t smem) -> kronq_status {
    KQ_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem)));
    int per_sm = 1;   // the CTAs that fit at once; each takes a contiguous range of chunks
    KQ_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, nt, smem));
    if (per_sm < 1) per_sm = 1;
    const int64_t cap = static_cast<int64_t>(sm_budget()) * per_sm;
    const unsigned grid = static_cast<unsigned>(nchunks < cap ? nchunks : cap);
    kern<<<grid, nt, smem, stream>>>(map, dst, rows, cols, row_f, col_f, scalar, out_scale, err);
    return check_launch("fwht_rows_tma_kernel");
  };
#define KQ_ROW_TMA(LB)                                                      \
  case LB:                                                                  \
    return launch(fwht_rows_tma_kernel<T, LB>, RowTma<LB, kF32>::kThreads, \
                  RowTma<LB, kF32>::kSmem);
  switch (log2b) {
    KQ_ROW_TMA(5) KQ_ROW_TMA(6) KQ_ROW_TMA(7) KQ_ROW_TMA(8) KQ_ROW_TMA(9)
    KQ_ROW_TMA(10) KQ_ROW_TMA(11) KQ_ROW_TMA(12) KQ_ROW_TMA(13)
    default: return fail(KRONQ_ERR_UNSUPPORTED, "tiled row pass: block size out of range");
  }
#undef KQ_ROW_TMA
}

// ---- tiled column pass (P = 16 .. 256 rows at stride rs, in place) ----
//
// A chunk is CT = max(1, 128 / P) adjacent 32-column tiles of the P rows r_base + rs j (j < P):
// CT TMA boxes of 32 x P from the view {cols, rs, rows / rs} of the matrix, stacked so that tile
// row ct P + j holds row j of column tile ct. The P-point butterflies run on the low log2 P bits
// of the tile-row index with the rounds of the row pass; the last one scales by out_scale and
// stores each tile row as one 128-byte segment. Columns past the matrix read as zeros and are not
// stored. Same pipeline as the row pass: CTAs take contiguous ranges of chunks (column groups of
// one row block, then the next row block), loads run up to stages - 1 chunks ahead.
template <int LP>
struct ColTma {
  static constexpr int kP = 1 << LP;
  static constexpr int kCT = LP >= 7 ? 1 : 1 << (7 - LP);   // column tiles per chunk
  static constexpr int kThreads = kCT * kP;                  // = tile rows
  static constexpr int kStages = 3;
  static constexpr int kStageBytes = kThreads * 128;
  static constexpr int kMinBlocks = LP == 8 ? 2 : 4;         // fits an SM's shared memory
  static constexpr size_t kSmem = 1024 + static_cast<size_t>(kStages) * kStageBytes + 64;
};

template <int LP>
__global__ void __launch_bounds__(ColTma<LP>::kThreads, ColTma<LP>::kMinBlocks)
    fwht_cols_tma_kernel(const __grid_constant__ CUtensorMap map, float* m, int64_t rows,
                         int64_t cols, int rs, float out_scale, int* err_word) {
  using S = ColTma<LP>;
  constexpr int P = S::kP, CT = S::kCT, NST = S::kStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* stages = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(stages + NST * S::kStageBytes);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + NST);
  const int t = threadIdx.x;

  const int ntiles = static_cast<int>((cols + 31) / 32);
  const int ncg = (ntiles + CT - 1) / CT;                  // column groups per row block
  const int64_t nchunks = (rows / P) * ncg;
  const int64_t k0 = nchunks * blockIdx.x / gridDim.x;
  const int64_t k1 = nchunks * (blockIdx.x + 1) / gridDim.x;
  const int n = static_cast<int>(k1 - k0);
  if (n <= 0) return;

  if (t == 0) {
    prefetch_tensormap(&map);
    for (int i = 0; i < NST; ++i) mbar_init(&full[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // chunk k0 + j: row block y (rows (y / rs) P rs + (y % rs) + rs j), column group cg
  auto issue = [&](int j) {
    const int64_t k = k0 + j;
    const int64_t y = k / ncg;
    const int cg = static_cast<int>(k - y * ncg);
    const int a = static_cast<int>(y % rs);
    const int z = static_cast<int>((y / rs) * P);
    const int nt = ntiles - cg * CT < CT ? ntiles - cg * CT : CT;
    uint64_t* bar = &full[j % NST];
    unsigned char* dst = stages + (j % NST) * S::kStageBytes;
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nt) * P * 128);
    for (int ct = 0; ct < nt; ++ct)
      tma_load_3d(dst + ct * P * 128, &map, bar, (cg * CT + ct) * 32, a, z);
  };
  if (t == 0)
    for (int j = 0; j < NST - 1 && j < n; ++j) issue(j);

  int64_t y = k0 / ncg;
  int cg = static_cast<int>(k0 - y * ncg);
  bool aborted = false;
  int i = 0;
  for (; i < n; ++i) {
    const int st = i % NST;
    if (t == 0 && i + NST - 1 < n) issue(i + NST - 1);   // its stage was freed by chunk i - 1
    const bool ok = mbar_wait(&full[st], (i / NST) & 1, abort_flag, err_word, DEV_ERR_LOAD_WAIT);
    if (__syncthreads_or(!ok)) {
      aborted = true;
      break;
    }
    float* work = reinterpret_cast<float*>(stages + st * S::kStageBytes);
    const int64_t rbase = (y / rs) * P * rs + (y % rs);
    const int64_t c0 = static_cast<int64_t>(cg) * CT * 32;
    auto out = [&](int r, int c) -> float* {
      const int64_t col = c0 + 32 * (r >> LP) + c;
      return col < cols ? m + (rbase + static_cast<int64_t>(rs) * (r & (P - 1))) * cols + col
                        : nullptr;
    };
    if (out_scale != 1.0f)
      tile_rounds<LP, true>(work, t, out_scale, out);
    else
      tile_rounds<LP, false>(work, t, 1.0f, out);
    fence_proxy_async_smem();   // the stage was written in place; TMA refills it
    __syncthreads();
    if (++cg == ncg) {
      cg = 0;
      ++y;
    }
  }
  if (aborted && t == 0) {
    // let the loads already issued (chunks i .. i + stages - 1) land before the CTA exits
    for (int j = i; j < n && j < i + NST; ++j)
      mbar_drain(&full[j % NST], (j / NST) & 1, kWaitLimitNs);
  }
}

kronq_status col_pass_tma(float* m, int64_t rows, int64_t cols, int log2p, int rs, float out_scale,
                          cudaStream_t stream) {
  CUtensorMap map;
  const uint64_t dims[3] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rs),
                            static_cast<uint64_t>(rows / rs)};
  const uint64_t strides[2] = {static_cast<uint64_t>(cols) * 4,
                               static_cast<uint64_t>(cols) * 4 * rs};
  const uint32_t box[3] = {32, 1, static_cast<uint32_t>(1 << log2p)};
  KQ_TRY(encode_tiled_map(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, m, dims, strides, box,
                          CU_TENSOR_MAP_SWIZZLE_128B));
  int* err = device_error_word();
  const int P = 1 << log2p;
  const int ct = log2p >= 7 ? 1 : 1 << (7 - log2p);
  const int64_t ncg = ((cols + 31) / 32 + ct - 1) / ct;
  const int64_t nchunks = (rows / P) * ncg;
  auto launch = [&](auto kern, int nt, size_t smem) -> kronq_status {
    KQ_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem)));
    int per_sm = 1;   // the CTAs that fit at once; each takes a contiguous range of chunks
    KQ_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, nt, smem));
    if (per_sm < 1) per_sm = 1;
    const int64_t cap = static_cast<int64_t>(sm_budget()) * per_sm;
    const unsigned grid = static_cast<unsigned>(nchunks < cap ? nchunks : cap);
    kern<<<grid, nt, smem, stream>>>(map, m, rows, cols, rs, out_scale, err);
    return check_launch("fwht_cols_tma_kernel");
  };
#define KQ_COL_TMA(LPV) \
  case LPV:             \
    return launch(fwht_cols_tma_kernel<LPV>, ColTma<LPV>::kThreads, ColTma<LPV>::kSmem);
  switch (log2p) {
    KQ_COL_TMA(4) KQ_COL_TMA(5) KQ_COL_TMA(6) KQ_COL_TMA(7) KQ_COL_TMA(8)
    default: return fail(KRONQ_ERR_UNSUPPORTED, "tiled column pass: block size out of range");
  }
#undef KQ_COL_TMA
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
  const bool aligned = (reinterpret_cast<uintptr_t>(src) & 15u) == 0 &&
                       (reinterpret_cast<uintptr_t>(dst) & 15u) == 0;
  if (aligned && b >= 32 && b <= 8192 && rows < (int64_t(1) << 31))
    return row_pass_tile(src, dst, rows, cols, row_f, col_f, scalar, ilog2_pow2(b), out_scale,
                         stream);
  if (b >= 16 && b <= 16384) {
    const int threads = chunk / 16;
    // padded work buffer + two staging buffers of the source type
    const size_t smem = static_cast<size_t>(chunk + chunk / 16) * sizeof(float) +
                        2 * static_cast<size_t>(chunk) * sizeof(T);
    const int vec = (reinterpret_cast<uintptr_t>(src) & 15u) == 0 &&
                    (reinterpret_cast<uintptr_t>(dst) & 15u) == 0;
    const int log2b = ilog2_pow2(b);
    // one instantiation per CTA size, so that each gets the register budget of its size; the
    // grid is the CTAs that fit at once (each walks chunks grid-stride)
    auto launch = [&](auto kern) -> kronq_status {
      if (smem > 48 * 1024)
        KQ_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem));
      int per_sm = 1;
      KQ_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem));
      if (per_sm < 1) per_sm = 1;
      const int64_t cap = static_cast<int64_t>(sm_budget()) * per_sm;
      const unsigned grid = static_cast<unsigned>(blocks < cap ? blocks : cap);
      kern<<<grid, threads, smem, stream>>>(src, dst, total, cols, row_f, col_f, scalar, log2b,
                                            chunk, out_scale, vec);
      return KRONQ_OK;
    };
    if (threads == 256)
      KQ_TRY(launch(fwht_rows_reg_kernel<T, 256>));
    else if (threads == 512)
      KQ_TRY(launch(fwht_rows_reg_kernel<T, 512>));
    else
      KQ_TRY(launch(fwht_rows_reg_kernel<T, 1024>));
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
  const size_t smem = 2 * static_cast<size_t>(P) * kColLd * sizeof(float);   // two tile buffers
  // 16-byte pieces need aligned rows and whole 32-column tiles
  const int vec = (reinterpret_cast<uintptr_t>(m) & 15u) == 0 && cols % kColTile == 0;
  const int64_t tiles = ((cols + kColTile - 1) / kColTile) * (rows / P);
  auto launch = [&](auto kern) -> kronq_status {
    if (smem > 48 * 1024)
      KQ_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem)));
    int per_sm = 1;   // the CTAs that fit at once; each walks tiles grid-stride
    KQ_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 2 * P, smem));
    if (per_sm < 1) per_sm = 1;
    const int64_t cap = static_cast<int64_t>(sm_budget()) * per_sm;
    const unsigned grid = static_cast<unsigned>(tiles < cap ? tiles : cap);
    kern<<<grid, 2 * P, smem, stream>>>(m, rows, cols, rs, out_scale, vec);
    return KRONQ_OK;
  };
  switch (log2p) {
    case 4: KQ_TRY(launch(fwht_cols_reg_kernel<4>)); break;
    case 5: KQ_TRY(launch(fwht_cols_reg_kernel<5>)); break;
    case 6: KQ_TRY(launch(fwht_cols_reg_kernel<6>)); break;
    case 7: KQ_TRY(launch(fwht_cols_reg_kernel<7>)); break;
    case 8: KQ_TRY(launch(fwht_cols_reg_kernel<8>)); break;
    default: return fail(KRONQ_ERR_UNSUPPORTED, "column pass of %d points", P);
  }
  return check_launch("fwht_cols_reg_kernel");
}

kronq_status col_pass(float* m, int64_t rows, int64_t cols, int b, cudaStream_t stream) {
  if (b <= 1) return KRONQ_OK;
  const float out_scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(b)));
  if (b >= 16 && b <= 16384) {
    const int L = ilog2_pow2(b);
    // TMA needs a 16-byte aligned base and row stride and row indices below 2^31; its boxes
    // are 32 columns wide
    const bool tma = (reinterpret_cast<uintptr_t>(m) & 15u) == 0 && cols % 4 == 0 &&
                     cols >= 32 && rows < (int64_t(1) << 31);
    auto pass = [&](int lp, int rs, float sc) {
      return tma ? col_pass_tma(m, rows, cols, lp, rs, sc, stream)
                 : col_pass_reg(m, rows, cols, lp, rs, sc, stream);
    };
    if (L <= 8) return pass(L, 1, out_scale);
    const int l1 = (L + 1) / 2, l2 = L / 2;   // H_b = (H_P2 (x) I_P1)(I_P2 (x) H_P1)
    KQ_TRY(pass(l1, 1, 1.0f));
    return pass(l2, 1 << l1, out_scale);
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
  double* tr_in;    // ceil(d_in / 256)   block shares of tr(H_X')
  double* tr_out;   // ceil(d_out / 256)  block shares of tr(H_G')
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
  p += align256(sizeof(float) * d_out);
  w.tr_in = reinterpret_cast<double*>(p);
  p += align256(sizeof(double) * ((d_in + 255) / 256));
  w.tr_out = reinterpret_cast<double*>(p);
  return w;
}

}  // namespace

size_t biip_workspace_bytes(int d_out, int d_in) {
  return align256(sizeof(double) * d_in) + align256(sizeof(double) * d_out) +
         2 * align256(sizeof(float) * d_in) + 2 * align256(sizeof(float) * d_out) +
         align256(sizeof(double) * ((d_in + 255) / 256)) +
         align256(sizeof(double) * ((d_out + 255) / 256));
}

kronq_status run_biip(const BiipArgs& a, void* ws_raw, cudaStream_t stream) {
  const BiipWs ws = carve(ws_raw, a.d_out, a.d_in);
  const bool scale_in = a.flags & KRONQ_BIIP_SCALE_IN;
  const bool scale_out = a.flags & KRONQ_BIIP_SCALE_OUT;
  const bool rot_in = a.flags & KRONQ_BIIP_ROTATE_IN;
  const bool rot_out = a.flags & KRONQ_BIIP_ROTATE_OUT;
  const bool hg_diag = a.flags & KRONQ_BIIP_HG_DIAG;   // hg holds the diagonal only
  const bool write_hg = (a.flags & KRONQ_BIIP_WRITE_HG) && a.hg && !hg_diag;
  const int b_in = rot_in ? largest_pow2_divisor(a.d_in) : 1;
  const int b_out = rot_out ? largest_pow2_divisor(a.d_out) : 1;

  // 1. squared column / row norms of the original W
  KQ_CUDA_TRY(cudaMemsetAsync(ws.col_sq, 0, sizeof(double) * a.d_in, stream));
  KQ_CUDA_TRY(cudaMemsetAsync(ws.row_sq, 0, sizeof(double) * a.d_out, stream));
  {
    const bool bf = a.w_dtype == KRONQ_DTYPE_BF16;
    const int esz = bf ? 2 : 4, pw = 32 * (16 / esz);
    const int vec = (reinterpret_cast<uintptr_t>(a.w) & 15u) == 0 && (a.d_in * esz) % 16 == 0;
    // row chunks (multiples of 64 rows) such that panels x chunks fills the 3 CTAs per SM once
    const int panels = (a.d_in + pw - 1) / pw;
    const int chunks = std::max(1, 3 * device_sms() / panels);
    int chunk_rows = (a.d_out + chunks - 1) / chunks;
    chunk_rows = std::max(64, (chunk_rows + 63) / 64 * 64);
    dim3 grid(panels, (a.d_out + chunk_rows - 1) / chunk_rows);
    if (bf)
      colrow_norms_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(a.w), a.d_out, a.d_in, vec, chunk_rows, ws.col_sq,
          ws.row_sq);
    else
      colrow_norms_kernel<float><<<grid, 256, 0, stream>>>(
          static_cast<const float*>(a.w), a.d_out, a.d_in, vec, chunk_rows, ws.col_sq, ws.row_sq);
    KQ_TRY(check_launch("colrow_norms_kernel"));
  }

  // 2. scales, factors and traces (from the un-transformed diagonals)
  const int nb_in = (a.d_in + 255) / 256, nb_out = (a.d_out + 255) / 256;
  side_scales_kernel<<<nb_in, 256, 0, stream>>>(
      a.d_in, a.hx, static_cast<int64_t>(a.d_in) + 1, ws.col_sq, a.inv_n, scale_in, rot_in ? a.sign_in : nullptr, a.s_x, ws.fw_in,
      ws.fh_in, a.tr_hx ? ws.tr_in : nullptr);
  KQ_TRY(check_launch("side_scales_kernel(in)"));
  if (a.tr_hx) {
    trace_sum_kernel<<<1, 32, 0, stream>>>(ws.tr_in, nb_in, a.tr_hx);
    KQ_TRY(check_launch("trace_sum_kernel(in)"));
  }
  const bool tr_g = a.hg && a.tr_hg;
  side_scales_kernel<<<nb_out, 256, 0, stream>>>(
      a.d_out, a.hg, hg_diag ? 1 : static_cast<int64_t>(a.d_out) + 1, ws.row_sq, a.inv_n, scale_out, rot_out ? a.sign_out : nullptr, a.s_g,
      ws.fw_out, ws.fh_out, tr_g ? ws.tr_out : nullptr);
  KQ_TRY(check_launch("side_scales_kernel(out)"));
  if (tr_g) {
    trace_sum_kernel<<<1, 32, 0, stream>>>(ws.tr_out, nb_out, a.tr_hg);
    KQ_TRY(check_launch("trace_sum_kernel(out)"));
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

