// Column-wise OBS / GPTAQ solve onto a b-bit per-output-row asymmetric grid.
//
// KronQ (hyper.ai summary), Method, OBS update:
//     dW_:,p+1: = -delta_p [H_X^-1]_p,p+1: + W_:,p P_p,p+1:
// with delta_p = (w_p - deq(q(w_p))) / K_pp and K the upper factor of the damped inverse
// (H_G cancels from the update, Proposition 1, so the solve never sees H_G). P is the GPTAQ
// correction matrix, read as P = striu(D K^T) K. Its term uses the weights before any update,
// so its total contribution to column j, sum_{p<j} W_:,p P_p,j, is known in advance: the solve
// is GPTQ on W~ = W + W P, which this file forms up front (fp32-accurate tensor-core GEMMs).
//
// Solve: 128-column blocks. Inside a block every output row is independent given K; one lane
// per row walks the block's columns in order (quantize, error, update the remaining columns of
// the block), the four warps of a CTA each holding a quarter of the block's columns. The rest of
// every row is updated lazily with GEMMs, in two levels: after a block, the rest of its
// 1024-column super-block, W~[:, e:s1] -= Delta_blk K[blk, e:s1]; after a super-block, the rest
// of W, W~[:, s1:] -= Delta_sb K[sb, s1:].
#include <cuda_bf16.h>

#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace kq {

namespace {

constexpr int QB = 128;        // column block
constexpr int QSB = 1024;      // super-block: the rest of W is updated once per QSB columns
constexpr int RPL = 1;         // rows per lane in the block solve
constexpr int QROWS = 32 * RPL; // rows per CTA in the block solve
constexpr int QT = 4;          // warps per CTA: one column quarter each
constexpr int QW = QB / QT;    // columns per thread
constexpr int KS_LD = QB + 4;  // row of the K block in shared memory (16-byte aligned)
constexpr int E_LD = QB + 1;   // row of the error block (odd: one bank per lane)

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

// One 128-column block of the solve for QROWS = 32 * RPL rows: lane l of every warp owns rows
// blockIdx.x * QROWS + 32 r + l (r < RPL), and warp q owns the block's column quarter
// [32q, 32q + 32) of them, in registers. Quarter by quarter, its warp walks the 32 columns in order (quantize,
// scaled error, update its own columns to the right) with no exchange, parks the errors in
// shared memory, and after one barrier every later quarter subtracts those 32 errors times the
// matching K rows. K rows are read as broadcasts (every lane of a warp reads the same row) and
// serve all of a lane's rows. With RPL = 1 the solve is bound by the per-column dependency
// chain; RPL = 2 halves the CTAs but measured slower (the lane's instruction stream doubles).
//   w_hat  d_out x d_in running weights (in: current values, out: dequantized for the block)
//   delta  d_out x QB errors scaled by 1/K_pp (row stride ldd), written as three bf16 pieces
//          (the operand of the lazy trailing updates on the tensor cores)
__global__ void __launch_bounds__(32 * QT) block_solve_kernel(
    float* __restrict__ w_hat, const float* __restrict__ k, int d_out, int d_in, int b0, int bw,
    float* __restrict__ scale, float* __restrict__ zero, int grouped, int n_groups, float maxq,
    uint8_t* __restrict__ codes, uint16_t* __restrict__ delta0, uint16_t* __restrict__ delta1,
    uint16_t* __restrict__ delta2, int64_t ldd) {
  extern __shared__ __align__(16) float sm[];
  float* Ks = sm;                      // QB x KS_LD: the K block
  float* E = Ks + QB * KS_LD;          // QROWS x E_LD: scaled errors of the block
  float* Rd = E + QROWS * E_LD;        // QB reciprocals of K's diagonal
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int q = tid >> 5;              // column quarter of this warp

  // K block (rows/cols beyond bw become identity so that padding never feeds back)
  const bool kvec = (d_in % 4 == 0) && bw == QB && (reinterpret_cast<uintptr_t>(k) & 15u) == 0;
  if (kvec) {
    for (int e = tid; e < QB * QB / 4; e += blockDim.x) {
      const int i = e / (QB / 4), j4 = (e % (QB / 4)) * 4;
      const float4 v = *reinterpret_cast<const float4*>(k + static_cast<int64_t>(b0 + i) * d_in + b0 + j4);
      *reinterpret_cast<float4*>(Ks + i * KS_LD + j4) =
          make_float4(j4 >= i ? v.x : 0.f, j4 + 1 >= i ? v.y : 0.f, j4 + 2 >= i ? v.z : 0.f,
                      j4 + 3 >= i ? v.w : 0.f);
    }
  } else {
    for (int e = tid; e < QB * QB; e += blockDim.x) {
      const int i = e / QB, j = e % QB;
      float v;
      if (i < bw && j < bw)
        v = (j >= i) ? k[static_cast<int64_t>(b0 + i) * d_in + b0 + j] : 0.f;
      else
        v = (i == j) ? 1.f : 0.f;
      Ks[i * KS_LD + j] = v;
    }
  }
  __syncthreads();
  if (tid < QB) Rd[tid] = 1.f / Ks[tid * KS_LD + tid];

  // this lane's 32 columns of each of its rows
  float w[RPL][QW];
  float sc[RPL], zr[RPL];
  uint32_t packed[RPL][QW / 4];
#pragma unroll
  for (int r = 0; r < RPL; ++r) {
    const int row = blockIdx.x * QROWS + 32 * r + lane;
    const bool active = row < d_out;
    const float* wrow = w_hat + static_cast<int64_t>(row) * d_in + b0 + QW * q;
    const bool wvec = active && bw == QB && ((reinterpret_cast<uintptr_t>(wrow) & 15u) == 0);
    if (wvec) {
#pragma unroll
      for (int j = 0; j < QW; j += 4) {
        const float4 v = *reinterpret_cast<const float4*>(wrow + j);
        w[r][j] = v.x; w[r][j + 1] = v.y; w[r][j + 2] = v.z; w[r][j + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < QW; ++j) w[r][j] = (active && QW * q + j < bw) ? wrow[j] : 0.f;
    }
    if (!grouped) {
      sc[r] = active ? scale[row] : 1.f;
      zr[r] = active ? zero[row] : 0.f;
    } else {
      // this quarter's share of the row's lo / hi over the block's columns (E is free until
      // the solve starts)
      float lo = INFINITY, hi = -INFINITY;
#pragma unroll
      for (int j = 0; j < QW; ++j)
        if (QW * q + j < bw) {
          lo = fminf(lo, w[r][j]);
          hi = fmaxf(hi, w[r][j]);
        }
      E[q * QROWS + 32 * r + lane] = lo;
      E[(QT + q) * QROWS + 32 * r + lane] = hi;
    }
#pragma unroll
    for (int j = 0; j < QW / 4; ++j) packed[r][j] = 0u;
  }
  __syncthreads();   // Rd, and the quarters' lo / hi
  if (grouped) {
    // the group's grid, from the weights the solve is about to quantize (same formulas as the
    // per-row grid, decisions in fp32)
#pragma unroll
    for (int r = 0; r < RPL; ++r) {
      float lo = E[32 * r + lane], hi = E[QT * QROWS + 32 * r + lane];
#pragma unroll
      for (int qq = 1; qq < QT; ++qq) {
        lo = fminf(lo, E[qq * QROWS + 32 * r + lane]);
        hi = fmaxf(hi, E[(QT + qq) * QROWS + 32 * r + lane]);
      }
      float sv = __fdiv_rn(__fsub_rn(hi, lo), maxq);
      if (hi == lo) sv = 1.f;
      sc[r] = sv;
      zr[r] = rintf(__fdiv_rn(-lo, sv));
      const int row = blockIdx.x * QROWS + 32 * r + lane;
      if (q == 0 && row < d_out) {
        scale[static_cast<int64_t>(row) * n_groups + b0 / QB] = sc[r];
        zero[static_cast<int64_t>(row) * n_groups + b0 / QB] = zr[r];
      }
    }
    __syncthreads();   // every warp has its grid before the solve writes E
  }

  for (int qo = 0; qo < QT; ++qo) {
    if (q == qo) {
#pragma unroll
      for (int lp = 0; lp < QW; ++lp) {
        const int p = QW * qo + lp;
        float e[RPL];
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
          const float t = __fdiv_rn(w[r][lp], sc[r]);
          float code = __fadd_rn(rintf(t), zr[r]);
          code = fminf(fmaxf(code, 0.f), maxq);
          const float dq = __fmul_rn(sc[r], __fsub_rn(code, zr[r]));
          e[r] = __fsub_rn(w[r][lp], dq) * Rd[p];
          w[r][lp] = dq;
          E[(32 * r + lane) * E_LD + p] = e[r];
          packed[r][lp / 4] |= (static_cast<uint32_t>(code) & 0xFFu) << (8 * (lp % 4));
        }
        // own columns right of lp (a compile-time range)
        const float4* kr = reinterpret_cast<const float4*>(Ks + p * KS_LD + QW * qo);
#pragma unroll
        for (int j4 = 0; j4 < QW / 4; ++j4) {
          if (4 * j4 + 3 <= lp) continue;
          const float4 kv = kr[j4];
#pragma unroll
          for (int r = 0; r < RPL; ++r) {
            if (4 * j4 > lp) w[r][4 * j4] = fmaf(-e[r], kv.x, w[r][4 * j4]);
            if (4 * j4 + 1 > lp) w[r][4 * j4 + 1] = fmaf(-e[r], kv.y, w[r][4 * j4 + 1]);
            if (4 * j4 + 2 > lp) w[r][4 * j4 + 2] = fmaf(-e[r], kv.z, w[r][4 * j4 + 2]);
            if (4 * j4 + 3 > lp) w[r][4 * j4 + 3] = fmaf(-e[r], kv.w, w[r][4 * j4 + 3]);
          }
        }
      }
    }
    __syncthreads();
    if (q > qo) {
      // the finished quarter's 32 errors, applied to this warp's columns
#pragma unroll 2
      for (int p = QW * qo; p < QW * qo + QW; ++p) {
        float e[RPL];
#pragma unroll
        for (int r = 0; r < RPL; ++r) e[r] = E[(32 * r + lane) * E_LD + p];
        const float4* kr = reinterpret_cast<const float4*>(Ks + p * KS_LD + QW * q);
#pragma unroll
        for (int j4 = 0; j4 < QW / 4; ++j4) {
          const float4 kv = kr[j4];
#pragma unroll
          for (int r = 0; r < RPL; ++r) {
            w[r][4 * j4] = fmaf(-e[r], kv.x, w[r][4 * j4]);
            w[r][4 * j4 + 1] = fmaf(-e[r], kv.y, w[r][4 * j4 + 1]);
            w[r][4 * j4 + 2] = fmaf(-e[r], kv.z, w[r][4 * j4 + 2]);
            w[r][4 * j4 + 3] = fmaf(-e[r], kv.w, w[r][4 * j4 + 3]);
          }
        }
      }
    }
  }
  __syncthreads();   // every quarter's errors are in E

#pragma unroll
  for (int r = 0; r < RPL; ++r) {
    const int row = blockIdx.x * QROWS + 32 * r + lane;
    if (row >= d_out) continue;
    float* wrow = w_hat + static_cast<int64_t>(row) * d_in + b0 + QW * q;
    const bool wvec = bw == QB && ((reinterpret_cast<uintptr_t>(wrow) & 15u) == 0);
    if (wvec) {
#pragma unroll
      for (int j = 0; j < QW; j += 4)
        *reinterpret_cast<float4*>(wrow + j) =
            make_float4(w[r][j], w[r][j + 1], w[r][j + 2], w[r][j + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < QW; ++j)
        if (QW * q + j < bw) wrow[j] = w[r][j];
    }
    // the errors of this quarter, split into three bf16 pieces for the tensor-core trailing
    // update (8 columns per 16-byte store; the row's 32 columns start on a 64-byte boundary)
    const float* er = E + (32 * r + lane) * E_LD + QW * q;
    const int64_t o = static_cast<int64_t>(row) * ldd + QW * q;
#pragma unroll
    for (int j8 = 0; j8 < QW; j8 += 8) {
      uint32_t h0[4], h1[4], h2[4];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float dv = QW * q + j8 + u < bw ? er[j8 + u] : 0.f;
        const __nv_bfloat16 p0 = __float2bfloat16_rn(dv);
        const float r1 = dv - __bfloat162float(p0);
        const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
        const __nv_bfloat16 p2 = __float2bfloat16_rn(r1 - __bfloat162float(p1));
        const int sh = 16 * (u & 1);
        if ((u & 1) == 0) { h0[u >> 1] = 0u; h1[u >> 1] = 0u; h2[u >> 1] = 0u; }
        h0[u >> 1] |= static_cast<uint32_t>(__bfloat16_as_ushort(p0)) << sh;
        h1[u >> 1] |= static_cast<uint32_t>(__bfloat16_as_ushort(p1)) << sh;
        h2[u >> 1] |= static_cast<uint32_t>(__bfloat16_as_ushort(p2)) << sh;
      }
      *reinterpret_cast<uint4*>(delta0 + o + j8) = make_uint4(h0[0], h0[1], h0[2], h0[3]);
      *reinterpret_cast<uint4*>(delta1 + o + j8) = make_uint4(h1[0], h1[1], h1[2], h1[3]);
      *reinterpret_cast<uint4*>(delta2 + o + j8) = make_uint4(h2[0], h2[1], h2[2], h2[3]);
    }
    uint8_t* cr = codes + static_cast<int64_t>(row) * d_in + b0 + QW * q;
    if (bw == QB && (reinterpret_cast<uintptr_t>(cr) & 15u) == 0) {
      reinterpret_cast<uint4*>(cr)[0] =
          make_uint4(packed[r][0], packed[r][1], packed[r][2], packed[r][3]);
      reinterpret_cast<uint4*>(cr)[1] =
          make_uint4(packed[r][4], packed[r][5], packed[r][6], packed[r][7]);
    } else {
#pragma unroll
      for (int j = 0; j < QW; ++j)
        if (QW * q + j < bw)
          cr[j] = static_cast<uint8_t>((packed[r][j >> 2] >> (8 * (j & 3))) & 0xFFu);
    }
  }
}

}  // namespace

size_t quantize_workspace_bytes(int d_out, int d_in, int block, bool with_dxx) {
  (void)block;
  size_t b = split_bytes(d_in, d_in);        // K, split once per layer
  b += split_bytes(d_out, QSB);              // errors of one super-block
  if (with_dxx) {
    const size_t r1 = split_bytes(d_in, d_in) > split_bytes(d_out, d_in) ? split_bytes(d_in, d_in)
                                                                         : split_bytes(d_out, d_in);
    b += r1;                                                           // D / W / W striu(M) splits
    b += align256(sizeof(float) * static_cast<size_t>(d_in) * d_in);   // M = striu(D K^T)
    b += split_bytes(d_in, d_in);                                      // M split
    b += align256(sizeof(float) * static_cast<size_t>(d_out) * d_in); // W striu(M)
  }
  return b;
}

kronq_status run_quantize(const float* w, const float* k, const float* dxx, int d_out, int d_in,
                          int bits, int block, int group, uint8_t* codes, float* scale,
                          float* zero, float* w_hat, void* ws, cudaStream_t stream) {
  (void)block;
  const float maxq = static_cast<float>((1 << bits) - 1);
  Carve cv{static_cast<uint8_t*>(ws)};
  Split3 ks = cv.split(d_in, d_in);
  Split3 ds = cv.split(d_out, QSB);

  const int grouped = group > 0 ? 1 : 0;
  const int n_groups = grouped ? (d_in + QB - 1) / QB : 1;
  if (!grouped) {
    // grid from W before the solve (grouped grids are taken block by block in the solve)
    grid_kernel<<<(d_out + 7) / 8, 256, 0, stream>>>(w, d_out, d_in, maxq, scale, zero);
    KQ_TRY(check_launch("grid_kernel"));
  }
  KQ_TRY(split_bf16x3(k, d_in, d_in, d_in, ks, stream));

  KQ_CUDA_TRY(cudaMemcpyAsync(w_hat, w, sizeof(float) * static_cast<size_t>(d_out) * d_in,
                              cudaMemcpyDeviceToDevice, stream));
  if (dxx) {
    uint8_t* r1_base = cv.p;
    const size_t r1 = split_bytes(d_in, d_in) > split_bytes(d_out, d_in) ? split_bytes(d_in, d_in)
                                                                         : split_bytes(d_out, d_in);
    cv.p += r1;
    float* mm = cv.floats(static_cast<size_t>(d_in) * d_in);
    Split3 ms = cv.split(d_in, d_in);
    float* t1 = cv.floats(static_cast<size_t>(d_out) * d_in);
    // The pre-shift W (I + P) is W plus a correction of a few percent of W, computed from
    // products that keep the leading three bf16 terms (~2^-16 relative): its error is far below
    // fp32 rounding of W itself. Only the strict upper triangle of M = D K^T is formed (the
    // tiles below the diagonal are skipped, and K^T's zero triangle bounds each tile's K range).
    // M = D K^T, striu(M)
    {
      Carve r{r1_base};
      Split3 dsp = r.split(d_in, d_in);
      KQ_TRY(split_bf16x3(dxx, d_in, d_in, d_in, dsp, stream));
      KQ_TRY(tgemm(d_in, d_in, d_in, 1.f, dsp, ks, false, 0.f, mm, d_in, true, GEMM_B_LOWER,
                   nullptr, stream, 3));
    }
    {
      dim3 g((d_in + 255) / 256, d_in);
      striu_kernel<<<g, 256, 0, stream>>>(mm, d_in);
      KQ_TRY(check_launch("striu_kernel"));
    }
    KQ_TRY(split_bf16x3(mm, d_in, d_in, d_in, ms, stream));
    // T1 = W striu(M)
    {
      Carve r{r1_base};
      Split3 wsp = r.split(d_out, d_in);
      KQ_TRY(split_bf16x3(w, d_in, d_out, d_in, wsp, stream));
      KQ_TRY(tgemm(d_out, d_in, d_in, 1.f, wsp, ms, true, 0.f, t1, d_in, false, GEMM_B_UPPER,
                   nullptr, stream, 3));
    }
    // W~ = W + T1 K
    {
      Carve r{r1_base};
      Split3 tsp = r.split(d_out, d_in);
      KQ_TRY(split_bf16x3(t1, d_in, d_out, d_in, tsp, stream));
      KQ_TRY(tgemm(d_out, d_in, d_in, 1.f, tsp, ks, true, 1.f, w_hat, d_in, false, GEMM_B_UPPER,
                   nullptr, stream, 3));
    }
  }

  const size_t smem = sizeof(float) * (QB * KS_LD + QROWS * E_LD + QB);
  // per device and cheap on the host, so set on every call
  KQ_CUDA_TRY(cudaFuncSetAttribute(block_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)smem));
  // Two-level lazy updates: after a 128-column block only the rest of its super-block is
  // updated (K = 128); after a super-block, the rest of W at once (K = QSB), so the fp32 W is
  // read and written once per super-block instead of once per block.
  for (int s0 = 0; s0 < d_in; s0 += QSB) {
    const int s1 = d_in - s0 < QSB ? d_in : s0 + QSB;
    for (int b0 = s0; b0 < s1; b0 += QB) {
      const int bw = d_in - b0 < QB ? d_in - b0 : QB;
      const Split3 db = offset(ds, 0, b0 - s0);
      block_solve_kernel<<<(d_out + QROWS - 1) / QROWS, 32 * QT, smem, stream>>>(
          w_hat, k, d_out, d_in, b0, bw, scale, zero, grouped, n_groups, maxq, codes, db.part[0],
          db.part[1], db.part[2], db.ld);
      KQ_TRY(check_launch("block_solve_kernel"));
      const int e = b0 + bw;
      if (e < s1) {
        // W~[:, e:s1] -= Delta_blk K[b0:e, e:s1]
        KQ_TRY(tgemm(d_out, s1 - e, bw, -1.f, db, offset(ks, b0, e), true, 1.f, w_hat + e, d_in,
                     false, 0, nullptr, stream));
      }
    }
    if (s1 < d_in) {
      // W~[:, s1:] -= Delta_sb K[s0:s1, s1:]
      KQ_TRY(tgemm(d_out, d_in - s1, s1 - s0, -1.f, ds, offset(ks, s0, s1), true, 1.f,
                   w_hat + s1, d_in, false, 0, nullptr, stream));
    }
  }
  return KRONQ_OK;
}

// ---------------------------------------------------------------------------------------------
// Comparison variant (prior art, not KronQ): rounding with feedback on both sides.
//
// [YAQA notes], generalized LDLQ: for a Kronecker proxy H_O (x) H_I of the layer Hessian the
// quantized W^ is the fixed point of
//     W^ = Q(W + L_O'^T D L_I' + L_O'^T D + D L_I'),    D = W - W^,  L' = L - I,
// L the unit upper triangular factor of H (H = L diag L^T), reached within m + n - 1 updates of
// all elements at once, each update a pair of matrix products. Here H_I = H_X' and H_O = H_G'
// (damped), so L = U diag(U)^-1 with U U^T = H + lambda I, U upper; U = K^-1 for the inverse
// factor K of kronq_cholinv, and it is obtained with the same routine: by uniqueness of the
// factorization, the inverse factor of K K^T is K^-1.
// One update: P1 = D L_I', S = D + P1, P2 = L_O'^T S, T = W + P1 + P2, then codes = Q(T) per
// row and D = W - deq(codes). Both products read only the strictly triangular parts, and T
// reads P1 and P2 directly (not S - D, whose rounding would carry the element's own error), so
// an element's target reads only strictly earlier elements' errors: in floating point too, the
// iteration settles within d_out + d_in - 1 updates, and once no code changes the state is the
// fixed point (the test that ends the loop).

namespace {

// The strictly triangular unit factor L' of U (upper, d x d), split into three bf16 pieces:
// transpose 0: L'[i][j] = U[i][j] / U[j][j] for i < j, else 0;
// transpose 1: the transpose, L'^T[i][j] = U[j][i] / U[i][i] for j < i, else 0.
__global__ void unit_factor_split_kernel(const float* __restrict__ u, int d, int transpose,
                                         uint16_t* __restrict__ p0, uint16_t* __restrict__ p1,
                                         uint16_t* __restrict__ p2, int64_t ld) {
  __shared__ float tile[32][33];
  const int bx = blockIdx.x * 32, by = blockIdx.y * 32;   // output tile: rows by.., cols bx..
  const int tx = threadIdx.x, ty = threadIdx.y;            // 32 x 8
  if (transpose) {
    // read the mirrored tile U[bx.., by..] row by row (coalesced), write it transposed
    for (int r = ty; r < 32; r += 8) {
      const int i = bx + r, j = by + tx;
      tile[r][tx] = (i < d && j < d) ? u[static_cast<int64_t>(i) * d + j] : 0.f;
    }
    __syncthreads();
  }
  for (int r = ty; r < 32; r += 8) {
    const int i = by + r, j = bx + tx;   // output element (i, j)
    if (i >= d || j >= d) continue;
    float v = 0.f;
    if (!transpose) {
      if (i < j) v = __fdiv_rn(u[static_cast<int64_t>(i) * d + j], u[static_cast<int64_t>(j) * d + j]);
    } else {
      if (j < i) v = __fdiv_rn(tile[tx][r], u[static_cast<int64_t>(i) * d + i]);
    }
    const __nv_bfloat16 b0 = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(b0);
    const __nv_bfloat16 b1 = __float2bfloat16_rn(r1);
    const __nv_bfloat16 b2 = __float2bfloat16_rn(r1 - __bfloat162float(b1));
    const int64_t o = static_cast<int64_t>(i) * ld + j;
    p0[o] = __bfloat16_as_ushort(b0);
    p1[o] = __bfloat16_as_ushort(b1);
    p2[o] = __bfloat16_as_ushort(b2);
  }
}

// S = D + P1, elementwise.
__global__ void add_kernel(const float* __restrict__ a, const float* __restrict__ b,
                           float* __restrict__ out, int64_t total) {
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[e] = __fadd_rn(a[e], b[e]);
}

// One update of all elements (init: T = W). T = W + P1 + P2, code = Q(T) on the row's grid
// (decisions in fp32, like the column solve), D = W - deq(code); counts the codes that changed.
__global__ void twosided_step_kernel(const float* __restrict__ w, const float* __restrict__ p1,
                                     const float* __restrict__ p2, float* __restrict__ delta,
                                     uint8_t* __restrict__ codes, float* __restrict__ w_hat,
                                     const float* __restrict__ scale,
                                     const float* __restrict__ zero, int d_out, int d_in,
                                     float maxq, int init, unsigned int* __restrict__ changed) {
  const int64_t total = static_cast<int64_t>(d_out) * d_in;
  unsigned int local = 0;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int row = static_cast<int>(e / d_in);
    const float wv = w[e];
    float t = wv;
    if (!init) t = __fadd_rn(__fadd_rn(wv, p1[e]), p2[e]);
    const float sc = scale[row], zr = zero[row];
    float code = __fadd_rn(rintf(__fdiv_rn(t, sc)), zr);
    code = fminf(fmaxf(code, 0.f), maxq);
    const float dq = __fmul_rn(sc, __fsub_rn(code, zr));
    const uint8_t c8 = static_cast<uint8_t>(code);
    if (init || c8 != codes[e]) ++local;
    codes[e] = c8;
    w_hat[e] = dq;
    delta[e] = __fsub_rn(wv, dq);
  }
  local = __reduce_add_sync(0xffffffffu, local);
  if ((threadIdx.x & 31) == 0 && local) atomicAdd(changed, local);
}

}  // namespace

namespace {
struct TwoWs {
  float* u_in;       // d_in^2: K_in K_in^T, then its inverse factor U_in
  float* u_out;      // d_out^2
  Split3 kt;         // a split K (for K K^T), max(d_in, d_out)^2
  Split3 li;         // L_I' split, d_in^2
  Split3 lot;        // L_O'^T split, d_out^2
  float* delta;      // d_out x d_in
  float* p1;
  float* s;
  float* p2;
  Split3 ms;         // split of D, then of S (d_out x d_in)
  unsigned int* changed;
  uint8_t* chol_ws;
};

size_t two_chol_bytes(int d_out, int d_in) {
  const size_t a = cholinv_workspace_bytes(d_in), b = cholinv_workspace_bytes(d_out);
  return a > b ? a : b;
}

TwoWs two_carve(void* ws, int d_out, int d_in) {
  Carve cv{static_cast<uint8_t*>(ws)};
  TwoWs t;
  const int dm = d_in > d_out ? d_in : d_out;
  t.u_in = cv.floats(static_cast<size_t>(d_in) * d_in);
  t.u_out = cv.floats(static_cast<size_t>(d_out) * d_out);
  t.kt = cv.split(dm, dm);
  t.li = cv.split(d_in, d_in);
  t.lot = cv.split(d_out, d_out);
  t.delta = cv.floats(static_cast<size_t>(d_out) * d_in);
  t.p1 = cv.floats(static_cast<size_t>(d_out) * d_in);
  t.s = cv.floats(static_cast<size_t>(d_out) * d_in);
  t.p2 = cv.floats(static_cast<size_t>(d_out) * d_in);
  t.ms = cv.split(d_out, d_in);
  t.changed = reinterpret_cast<unsigned int*>(cv.floats(64));
  t.chol_ws = cv.p;
  return t;
}

// U with U U^T = H + lambda I (upper), from the inverse factor K of H: U = chol_inv(K K^T).
kronq_status inverse_of_factor(const float* k, int d, float* u, Split3 kt, void* chol_ws,
                               int32_t* info, cudaStream_t stream) {
  KQ_TRY(split_bf16x3(k, d, d, d, kt, stream));
  // K K^T: A = K (upper), B given K-major as K itself (op(B)[k][n] = K[n][k], zero for k < n)
  KQ_TRY(tgemm(d, d, d, 1.f, kt, kt, false, 0.f, u, d, false, GEMM_A_UPPER | GEMM_B_LOWER,
               nullptr, stream));
  KQ_TRY(run_cholinv(u, d, 0.f, info, chol_ws, stream));
  return KRONQ_OK;
}
}  // namespace

size_t twosided_workspace_bytes(int d_out, int d_in) {
  const int dm = d_in > d_out ? d_in : d_out;
  const size_t mn = static_cast<size_t>(d_out) * d_in;
  return align256(sizeof(float) * static_cast<size_t>(d_in) * d_in) +
         align256(sizeof(float) * static_cast<size_t>(d_out) * d_out) + split_bytes(dm, dm) +
         split_bytes(d_in, d_in) + split_bytes(d_out, d_out) + 4 * align256(sizeof(float) * mn) +
         split_bytes(d_out, d_in) + align256(sizeof(float) * 64) + two_chol_bytes(d_out, d_in);
}

kronq_status run_twosided(const float* w, const float* k_in, const float* k_out, int d_out,
                          int d_in, int bits, uint8_t* codes, float* scale, float* zero,
                          float* w_hat, int32_t* iterations, void* ws, cudaStream_t stream) {
  const float maxq = static_cast<float>((1 << bits) - 1);
  TwoWs t = two_carve(ws, d_out, d_in);
  int32_t* info = reinterpret_cast<int32_t*>(t.changed + 16);
  for (int side = 0; side < 2; ++side) {
    KQ_TRY(inverse_of_factor(side ? k_out : k_in, side ? d_out : d_in, side ? t.u_out : t.u_in,
                             t.kt, t.chol_ws, info, stream));
    int32_t bad = -1;
    KQ_CUDA_TRY(cudaMemcpyAsync(&bad, info, sizeof(bad), cudaMemcpyDeviceToHost, stream));
    KQ_CUDA_TRY(cudaStreamSynchronize(stream));
    if (bad >= 0)
      return fail(KRONQ_ERR_NOT_PD, "%s: K K^T has a non-positive pivot at %d (is it an inverse "
                  "factor from kronq_cholinv?)", side ? "k_out" : "k_in", bad);
  }
  {
    dim3 b(32, 8);
    unit_factor_split_kernel<<<dim3((d_in + 31) / 32, (d_in + 31) / 32), b, 0, stream>>>(
        t.u_in, d_in, 0, t.li.part[0], t.li.part[1], t.li.part[2], t.li.ld);
    KQ_TRY(check_launch("unit_factor_split_kernel"));
    unit_factor_split_kernel<<<dim3((d_out + 31) / 32, (d_out + 31) / 32), b, 0, stream>>>(
        t.u_out, d_out, 1, t.lot.part[0], t.lot.part[1], t.lot.part[2], t.lot.ld);
    KQ_TRY(check_launch("unit_factor_split_kernel"));
  }
  grid_kernel<<<(d_out + 7) / 8, 256, 0, stream>>>(w, d_out, d_in, maxq, scale, zero);
  KQ_TRY(check_launch("grid_kernel"));
  const int64_t total = static_cast<int64_t>(d_out) * d_in;
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(device_sms()) * 8;
  if (blocks > cap) blocks = cap;
  int it = 0;
  bool done = false;
  // init: codes = Q(W), D = W - deq; then updates until no code changes (at most m + n)
  for (; it <= d_out + d_in && !done; ++it) {
    if (it > 0) {
      // P1 = D L_I', S = D + P1
      KQ_TRY(split_bf16x3(t.delta, d_in, d_out, d_in, t.ms, stream));
      KQ_TRY(tgemm(d_out, d_in, d_in, 1.f, t.ms, t.li, true, 0.f, t.p1, d_in, false,
                   GEMM_B_UPPER, nullptr, stream));
      add_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(t.delta, t.p1, t.s, total);
      KQ_TRY(check_launch("add_kernel"));
      // P2 = L_O'^T S
      KQ_TRY(split_bf16x3(t.s, d_in, d_out, d_in, t.ms, stream));
      KQ_TRY(tgemm(d_out, d_in, d_out, 1.f, t.lot, t.ms, true, 0.f, t.p2, d_in, false,
                   GEMM_A_LOWER, nullptr, stream));
    }
    KQ_CUDA_TRY(cudaMemsetAsync(t.changed, 0, sizeof(unsigned int), stream));
    twosided_step_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(
        w, t.p1, t.p2, t.delta, codes, w_hat, scale, zero, d_out, d_in, maxq, it == 0 ? 1 : 0,
        t.changed);
    KQ_TRY(check_launch("twosided_step_kernel"));
    unsigned int host = 0;
    KQ_CUDA_TRY(cudaMemcpyAsync(&host, t.changed, sizeof(host), cudaMemcpyDeviceToHost, stream));
    KQ_CUDA_TRY(cudaStreamSynchronize(stream));
    if (it > 0 && host == 0) done = true;
  }
  if (iterations) *iterations = it - 1;   // update passes, the last one changing no code
  if (!done)
    return fail(KRONQ_ERR_CUDA, "two-sided rounding did not reach its fixed point in %d updates",
                d_out + d_in);
  return KRONQ_OK;
}

}  // namespace kq
