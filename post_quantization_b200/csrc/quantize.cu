// Column-wise OBS / GPTAQ solve onto a b-bit per-output-row asymmetric grid.
//
// KronQ (hyper.ai summary), Method, OBS update:
//     dW_:,p+1: = -delta_p [H_X^-1]_p,p+1: + W_:,p P_p,p+1:
// with delta_p = (w_p - deq(q(w_p))) / K_pp and K the upper factor of the damped inverse
// (H_G cancels from the update, Proposition 1, so the solve never sees H_G). P is the GPTAQ
// correction matrix, read as P = striu(D K^T) K. Its term uses the weights before any update,
// so its total contribution to column j, sum_{p<j} W_:,p P_p,j, is known in advance: the solve
// is GPTQ on W~ = W + W P, which this file forms up front with fp32 GEMMs.
//
// Solve: 128-column blocks. Inside a block every output row is independent given K, so one
// thread owns one row and walks the block's columns in order (quantize, error, update the
// remaining columns of the block). After the block the rest of every row is updated lazily with
// one GEMM: W~[:, e:] -= Delta_blk K[blk, e:].
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace kq {

namespace {

constexpr int QB = 128;        // column block
constexpr int QROWS = 128;     // rows (= threads) per CTA in the block solve
constexpr int QSUB = 32;       // columns per register-resident sub-block

// Per-row grid from W (before the solve), all decisions in fp32:
// scale = (hi - lo) / (2^b - 1) (1 if hi == lo), zero = rint(-lo / scale).
__global__ void grid_kernel(const float* __restrict__ w, int d_out, int d_in, float maxq,
                            float* __restrict__ scale, float* __restrict__ zero) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= d_out) return;
  const float* r = w + static_cast<int64_t>(row) * d_in;
  float lo = INFINITY, hi = -INFINITY;
  for (int j = lane; j < d_in; j += 32) {
    const float v = r[j];
    lo = fminf(lo, v);
    hi = fmaxf(hi, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    float s = __fdiv_rn(__fsub_rn(hi, lo), maxq);
    if (hi == lo) s = 1.f;
    scale[row] = s;
    zero[row] = rintf(__fdiv_rn(-lo, s));
  }
}

// Zero the diagonal and lower triangle (striu).
__global__ void striu_kernel(float* __restrict__ m, int d) {
  const int i = blockIdx.y;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j <= i && j < d; j += gridDim.x * blockDim.x)
    m[static_cast<int64_t>(i) * d + j] = 0.f;
}

// One 128-column block of the solve for QROWS rows (one thread per row).
// The block is walked in four 32-column sub-blocks: the current sub-block lives in registers
// (fully unrolled), the rest of the thread's row waits in shared memory and receives the
// sub-block's errors in one pass after it.
//   w_hat  d_out x d_in running weights (in: current values, out: dequantized for the block)
//   delta  d_out x QB errors scaled by 1/K_pp (input of the lazy trailing update)
__global__ void __launch_bounds__(QROWS) block_solve_kernel(
    float* __restrict__ w_hat, const float* __restrict__ k, int d_out, int d_in, int b0, int bw,
    const float* __restrict__ scale, const float* __restrict__ zero, float maxq,
    uint8_t* __restrict__ codes, float* __restrict__ delta) {
  extern __shared__ float sm[];
  float* Ks = sm;                              // QB x QB block of K (padding = identity)
  float* St = Ks + QB * QB;                    // QROWS x (QB + 1): running row values
  float* Dt = St + QROWS * (QB + 1);           // QROWS x (QB + 1): errors
  float* Rd = Dt + QROWS * (QB + 1);           // QB reciprocals of K's diagonal
  const int tid = threadIdx.x;
  const int row0 = blockIdx.x * QROWS;
  const int rows = min(QROWS, d_out - row0);

  // K block (rows/cols beyond bw become identity so that padding never feeds back) and the
  // rows' block of running weights, with 16-byte loads where the layout allows
  const bool vec = (d_in % 4 == 0) && bw == QB &&
                   ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(w_hat)) & 15u) == 0;
  if (vec) {
    for (int e = tid; e < QB * QB / 4; e += blockDim.x) {
      const int i = e / (QB / 4), j4 = (e % (QB / 4)) * 4;
      float4 v = *reinterpret_cast<const float4*>(k + static_cast<int64_t>(b0 + i) * d_in + b0 + j4);
      if (j4 + 0 < i) v.x = 0.f;
      if (j4 + 1 < i) v.y = 0.f;
      if (j4 + 2 < i) v.z = 0.f;
      if (j4 + 3 < i) v.w = 0.f;
      *reinterpret_cast<float4*>(Ks + i * QB + j4) = v;
    }
    for (int e = tid; e < QROWS * QB / 4; e += blockDim.x) {
      const int r = e / (QB / 4), c4 = (e % (QB / 4)) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < rows) v = *reinterpret_cast<const float4*>(w_hat + static_cast<int64_t>(row0 + r) * d_in + b0 + c4);
      float* dst = St + r * (QB + 1) + c4;
      dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
    }
  } else {
    for (int e = tid; e < QB * QB; e += blockDim.x) {
      const int i = e / QB, j = e % QB;
      float v;
      if (i < bw && j < bw)
        v = (j >= i) ? k[static_cast<int64_t>(b0 + i) * d_in + b0 + j] : 0.f;
      else
        v = (i == j) ? 1.f : 0.f;
      Ks[e] = v;
    }
    for (int e = tid; e < QROWS * QB; e += blockDim.x) {
      const int r = e / QB, c = e % QB;
      float v = 0.f;
      if (r < rows && c < bw) v = w_hat[static_cast<int64_t>(row0 + r) * d_in + b0 + c];
      St[r * (QB + 1) + c] = v;
    }
  }
  __syncthreads();
  if (tid < QB) Rd[tid] = 1.f / Ks[tid * QB + tid];
  __syncthreads();

  const int row = row0 + tid;
  const bool active = tid < rows;
  const float sc = active ? scale[row] : 1.f;
  const float zr = active ? zero[row] : 0.f;
  float* my = St + tid * (QB + 1);
  float* myd = Dt + tid * (QB + 1);
  uint32_t packed[QB / 4];

#pragma unroll 1
  for (int sb = 0; sb < QB; sb += QSUB) {
    float w[QSUB], err[QSUB];
#pragma unroll
    for (int c = 0; c < QSUB; ++c) w[c] = my[sb + c];
#pragma unroll
    for (int p = 0; p < QSUB; ++p) {
      const float t = __fdiv_rn(w[p], sc);
      float code = __fadd_rn(rintf(t), zr);
      code = fminf(fmaxf(code, 0.f), maxq);
      const float dq = __fmul_rn(sc, __fsub_rn(code, zr));
      const float* kr = Ks + (sb + p) * QB + sb;
      err[p] = __fsub_rn(w[p], dq) * Rd[sb + p];
#pragma unroll
      for (int j = p + 1; j < QSUB; ++j) w[j] = fmaf(-err[p], kr[j], w[j]);
      w[p] = dq;
      const int cc = sb + p;
      if ((p & 3) == 0) packed[cc >> 2] = 0u;
      packed[cc >> 2] |= (static_cast<uint32_t>(code) & 0xFFu) << (8 * (p & 3));
    }
#pragma unroll
    for (int c = 0; c < QSUB; ++c) {
      my[sb + c] = w[c];
      myd[sb + c] = err[c];
    }
    // the sub-block's errors reach the rest of the block
#pragma unroll 2
    for (int j = sb + QSUB; j < QB; ++j) {
      float acc = my[j];
#pragma unroll
      for (int p = 0; p < QSUB; ++p) acc = fmaf(-err[p], Ks[(sb + p) * QB + j], acc);
      my[j] = acc;
    }
  }
  __syncthreads();
  for (int e = tid; e < QROWS * QB; e += blockDim.x) {
    const int r = e / QB, c = e % QB;
    if (r < rows) {
      delta[static_cast<int64_t>(row0 + r) * QB + c] = (c < bw) ? Dt[r * (QB + 1) + c] : 0.f;
      if (c < bw) w_hat[static_cast<int64_t>(row0 + r) * d_in + b0 + c] = St[r * (QB + 1) + c];
    }
  }
  if (active) {
    uint8_t* cr = codes + static_cast<int64_t>(row) * d_in + b0;
    if (bw == QB && (reinterpret_cast<uintptr_t>(cr) & 15u) == 0) {
#pragma unroll
      for (int c = 0; c < QB / 16; ++c)
        reinterpret_cast<uint4*>(cr)[c] =
            make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
    } else {
      for (int c = 0; c < bw; ++c)
        cr[c] = static_cast<uint8_t>((packed[c >> 2] >> (8 * (c & 3))) & 0xFFu);
    }
  }
}

}  // namespace

size_t quantize_workspace_bytes(int d_out, int d_in, int block, bool with_dxx) {
  (void)block;
  size_t b = align256(sizeof(float) * static_cast<size_t>(d_out) * QB);   // delta
  if (with_dxx) {
    b += align256(sizeof(float) * static_cast<size_t>(d_in) * d_in);      // M = striu(D K^T)
    b += align256(sizeof(float) * static_cast<size_t>(d_out) * d_in);     // W striu(M)
  }
  return b;
}

kronq_status run_quantize(const float* w, const float* k, const float* dxx, int d_out, int d_in,
                          int bits, int block, uint8_t* codes, float* scale, float* zero,
                          float* w_hat, void* ws, cudaStream_t stream) {
  (void)block;
  const float maxq = static_cast<float>((1 << bits) - 1);
  uint8_t* p = static_cast<uint8_t*>(ws);
  float* delta = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * static_cast<size_t>(d_out) * QB);

  // grid from W before the solve
  grid_kernel<<<(d_out + 7) / 8, 256, 0, stream>>>(w, d_out, d_in, maxq, scale, zero);
  KQ_TRY(check_launch("grid_kernel"));

  KQ_CUDA_TRY(cudaMemcpyAsync(w_hat, w, sizeof(float) * static_cast<size_t>(d_out) * d_in,
                              cudaMemcpyDeviceToDevice, stream));
  if (dxx) {
    float* mm = reinterpret_cast<float*>(p);
    p += align256(sizeof(float) * static_cast<size_t>(d_in) * d_in);
    float* t1 = reinterpret_cast<float*>(p);
    // M = D K^T, striu(M)
    KQ_TRY(sgemm(false, true, d_in, d_in, d_in, 1.f, dxx, d_in, k, d_in, 0.f, mm, d_in, false,
                 nullptr, stream, GEMM_B_LOWER));
    {
      dim3 g((d_in + 255) / 256, d_in);
      striu_kernel<<<g, 256, 0, stream>>>(mm, d_in);
      KQ_TRY(check_launch("striu_kernel"));
    }
    // W~ = W + (W striu(M)) K
    KQ_TRY(sgemm(false, false, d_out, d_in, d_in, 1.f, w, d_in, mm, d_in, 0.f, t1, d_in, false,
                 nullptr, stream, GEMM_B_UPPER));
    KQ_TRY(sgemm(false, false, d_out, d_in, d_in, 1.f, t1, d_in, k, d_in, 1.f, w_hat, d_in, false,
                 nullptr, stream, GEMM_B_UPPER));
  }

  static bool attr = false;
  const size_t smem = sizeof(float) * (QB * QB + 2 * QROWS * (QB + 1) + QB);
  if (!attr) {
    KQ_CUDA_TRY(cudaFuncSetAttribute(block_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem));
    attr = true;
  }
  for (int b0 = 0; b0 < d_in; b0 += QB) {
    const int bw = d_in - b0 < QB ? d_in - b0 : QB;
    block_solve_kernel<<<(d_out + QROWS - 1) / QROWS, QROWS, smem, stream>>>(
        w_hat, k, d_out, d_in, b0, bw, scale, zero, maxq, codes, delta);
    KQ_TRY(check_launch("block_solve_kernel"));
    const int e = b0 + bw;
    if (e < d_in) {
      // W~[:, e:] -= Delta K[b0:e, e:]
      KQ_TRY(sgemm(false, false, d_out, d_in - e, bw, -1.f, delta, QB,
                   k + static_cast<int64_t>(b0) * d_in + e, d_in, 1.f, w_hat + e, d_in, false,
                   nullptr, stream));
    }
  }
  return KRONQ_OK;
}

}  // namespace kq
