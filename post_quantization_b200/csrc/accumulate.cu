// Kronecker-factor accumulation on 5th-generation tensor cores.
//
// KronQ (hyper.ai summary), Method: H_X = E[x x^T] and H_G = E[g g^T] are the two Kronecker
// factors of the empirical Fisher; the GPTAQ asymmetric objective adds the drift term dX X^T.
// Over a chunk of tokens these are C += A^T B with A, B token-major (one token per row), i.e.
// both tensor-core operands are MN-major.
//
// Kernel: persistent, one CTA per SM, warp-specialised.
//   warp 0        TMA producer: loads 64-token x 64-column boxes (128-byte swizzle) of A and B
//                 into a 3-stage shared-memory ring (no multicast).
//   warp 1        TMEM allocator + MMA issuer: tcgen05.mma kind::f16, M=128, N=256, K=16,
//                 bf16 x bf16 -> fp32 in TMEM. An output tile is 256 x 256: two M=128 MMAs per
//                 K step share the stage's B operand, filling all 512 TMEM columns, so every
//                 operand byte staged from L2 feeds twice the tensor work of a 128-row tile and
//                 the ring holds more MMA time against the L2 latency.
//   warps 2..5    epilogue: tcgen05.ld the accumulator, add it into C with vector atomics (the
//                 call's contract is "+=", and split-K partial sums combine the same way). With
//                 TMEM full, the next unit's MMAs wait for the drain (a few percent of a unit).
// Work unit = (output tile, token chunk). For symmetric outputs only tiles touching the upper
// triangle are computed and a mirror kernel fills the strict lower triangle afterwards.
//
// The drift term D = (X - X~)^T X~ multiplies a difference of two bf16 tensors, which bf16 cannot
// hold to the 1e-3 the sums are held to (its rounding error is ~2^-9 per element). Both operands
// therefore go to the tensor cores as fp16 after a power-of-two rescale taken from their largest
// magnitude (drift_amax_kernel): X~ is exact in fp16 at that scale (bf16's 8 significant bits fit
// fp16's 11), and X - X~ is rounded once, to 2^-11 relative. One GEMM then does what two bf16
// GEMMs (a hi and a lo part of X - X~) would, and its epilogue undoes the rescale exactly.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "internal.h"

// Largest token chunk of a work unit (blocks of 64 tokens): 65536 tokens. Each unit ends in a
// read-modify-write of its fp32 output tile, so long units cut that traffic where the output has
// tiles enough to fill the GPU (measured on the 28672-wide symmetric sums: 168 ms against 178.5
// ms with 16384-token units); calls with few tiles split the tokens further.
#ifndef KQ_ACC_UNIT_KBLOCKS
#define KQ_ACC_UNIT_KBLOCKS 1024
#endif

namespace kq {

namespace acc {
constexpr int BM = 256;             // output rows per tile (two MMAs of M = 128)
constexpr int HM = 128;             // MMA M
constexpr int BN = 256;             // output cols per tile (MMA N)
constexpr int BK = 64;              // tokens per pipeline stage
constexpr int UK = 16;              // tokens per MMA instruction
constexpr int STAGES = 3;
constexpr int BOX = 64;             // columns per TMA box (128 bytes of bf16)
constexpr int BOX_BYTES = BOX * BK * 2;          // 8 KB
constexpr int A_BOXES = BM / BOX;                // 4
constexpr int B_BOXES = BN / BOX;                // 4
constexpr int STAGE_BYTES = (A_BOXES + B_BOXES) * BOX_BYTES;   // 64 KB
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 512;      // 2 M-halves x 256 fp32 columns
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
}  // namespace acc

struct AccParams {
  float* c;
  int64_t ldc;
  int m, n;               // output rows / cols
  int64_t k;              // tokens
  int tiles_m, tiles_n;
  int symmetric;          // 1: only tiles that touch the upper triangle
  int num_tiles;          // tiles actually computed
  int kblocks_per_unit;   // BK-blocks per token chunk
  int k_splits;
  int num_units;
  int fp16;               // operands are fp16 (else bf16)
  const float* amax;      // drift product: {max |A source|, max |B source|}; the epilogue scales
                          // by 2^-(fp16_shift(amax[0]) + fp16_shift(amax[1])). NULL: no scale
  int* err;
};

// Power-of-two exponent e with amax * 2^e in [2^14, 2^15), so that values scaled by 2^e stay
// below fp16's largest finite value (65504) and lose no precision to fp16's small-number range.
// 0 for a zero or non-finite amax; clamped to [-100, 100] (a tensor whose largest value is below
// 2^-85 is zero for every purpose here).
__device__ __forceinline__ int fp16_shift(float amax) {
  if (!(amax > 0.f) || !(amax <= 3.0e38f)) return 0;
  const int k = static_cast<int>((__float_as_uint(amax) >> 23) & 0xffu) - 126;  // amax in [2^(k-1), 2^k)
  return max(-100, min(100, 15 - k));
}
__device__ __forceinline__ float pow2f(int e) {   // 2^e for e in [-126, 127]
  return __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
}

// Map a computed-tile index to (tm, tn). Symmetric: row tm holds tiles tn >= tn_min(tm).
// Tiles are visited in groups of GROUP tile rows, column by column inside a group, so that the
// ~148 tiles in flight at any time cover a compact block of the output: they read GROUP row
// strips and ~148/GROUP column strips of the token chunk instead of every column, which keeps
// the chunk's DRAM re-reads down when the output has many more tiles than the GPU has SMs.
constexpr int GROUP = 8;

__device__ __forceinline__ int tn_min_of(const AccParams& p, int tm) {
  return p.symmetric ? (tm * acc::BM) / acc::BN : 0;
}

__device__ __forceinline__ void tile_coords(const AccParams& p, int t, int& tm, int& tn) {
  int g0 = 0;
  for (;;) {
    const int g1 = min(g0 + GROUP, p.tiles_m);
    int cnt = 0;
    for (int r = g0; r < g1; ++r) cnt += p.tiles_n - tn_min_of(p, r);
    if (t < cnt) break;
    t -= cnt;
    g0 = g1;
  }
  const int g1 = min(g0 + GROUP, p.tiles_m);
  for (int c = tn_min_of(p, g0);; ++c) {
    // rows of the group whose first tile is at or left of column c (tn_min grows with the row)
    int rows = 0;
    while (g0 + rows < g1 && tn_min_of(p, g0 + rows) <= c) ++rows;
    if (t < rows) {
      tm = g0 + t;
      tn = c;
      return;
    }
    t -= rows;
  }
}

__global__ void __launch_bounds__(acc::THREADS, 1)
    accumulate_tc_kernel(const __grid_constant__ CUtensorMap tma_a,
                         const __grid_constant__ CUtensorMap tma_b, const AccParams p) {
  using namespace acc;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* full = bars;                  // [STAGES]
  uint64_t* empty = bars + STAGES;        // [STAGES]
  uint64_t* tfull = bars + 2 * STAGES;    // [2]
  uint64_t* tempty = bars + 2 * STAGES + 2;   // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tma_a);
    prefetch_tensormap(&tma_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int kblocks_total = static_cast<int>((p.k + BK - 1) / BK);

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
        const int split = u / p.num_tiles;
        const int t = u % p.num_tiles;
        int tm, tn;
        tile_coords(p, t, tm, tn);
        const int kb0 = split * p.kblocks_per_unit;
        const int kb1 = min(kblocks_total, kb0 + p.kblocks_per_unit);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.err, DEV_ERR_TMA_WAIT)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          const int y = kb * BK;
#pragma unroll
          for (int b = 0; b < A_BOXES; ++b)
            tma_load_2d(st + b * BOX_BYTES, &tma_a, &full[s], tm * BM + b * BOX, y);
#pragma unroll
          for (int b = 0; b < B_BOXES; ++b)
            tma_load_2d(st + (A_BOXES + b) * BOX_BYTES, &tma_b, &full[s], tn * BN + b * BOX, y);
        }
      }
      if (!ok) {
        // aborted: let the copies still in flight land before the CTA exits
        for (uint32_t j = it > STAGES ? it - STAGES : 0; j < it; ++j)
          mbar_drain(&full[j % STAGES], (j / STAGES) & 1u, 1000000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = p.fp16 ? idesc_f16_f32_mn_mn(HM, BN) : idesc_bf16_f32_mn_mn(HM, BN);
      uint32_t it = 0;
      uint32_t ui = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x, ++ui) {
        const int split = u / p.num_tiles;
        const int kb0 = split * p.kblocks_per_unit;
        const int kb1 = min(kblocks_total, kb0 + p.kblocks_per_unit);
        int tm, tn;
        tile_coords(p, u % p.num_tiles, tm, tn);
        const bool half1 = tm * BM + HM < p.m;   // rows of the second M-half exist
        // TMEM holds one tile: wait until the epilogue has drained the previous one
        if (!mbar_wait(&tempty[0], (ui & 1u) ^ 1u, abort_flag, p.err, DEV_ERR_MMA_WAIT)) break;
        tc_fence_after();
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(&full[s], ph, abort_flag, p.err, DEV_ERR_MMA_WAIT)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t b_base = a_base + A_BOXES * BOX_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk) {
            // MN-major, 128B swizzle: 8 token rows of 128 bytes form one 1 KB atom (SBO);
            // successive 64-column boxes are one box apart (LBO). M-half h starts 2 boxes in.
            const uint32_t koff = kk * UK * 128;
            const uint32_t acc_flag = (kb > kb0 || kk > 0) ? 1u : 0u;
            const uint64_t bd = smem_desc_sw128(b_base + koff, BOX_BYTES, 1024);
            const uint64_t ad0 = smem_desc_sw128(a_base + koff, BOX_BYTES, 1024);
            umma_f16(tmem_base, ad0, bd, idesc, acc_flag);
            if (half1) {
              const uint64_t ad1 = smem_desc_sw128(a_base + 2 * BOX_BYTES + koff, BOX_BYTES, 1024);
              umma_f16(tmem_base + BN, ad1, bd, idesc, acc_flag);
            }
          }
          umma_commit(&empty[s]);   // frees the stage once these MMAs have read it
        }
        if (!ok) break;
        umma_commit(&tfull[0]);     // accumulator ready for the epilogue
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    // undo the operands' power-of-two rescale (two exact multiplications)
    float unscale_a = 1.f, unscale_b = 1.f;
    if (p.amax) {
      unscale_a = pow2f(-fp16_shift(p.amax[0]));
      unscale_b = pow2f(-fp16_shift(p.amax[1]));
    }
    uint32_t ui = 0;
    for (int u = blockIdx.x; u < p.num_units; u += gridDim.x, ++ui) {
      const int t = u % p.num_tiles;
      int tm, tn;
      tile_coords(p, t, tm, tn);
      // one lane waits, the warp follows its verdict (tcgen05.ld needs a converged warp)
      int ok = 1;
      if (lane == 0)
        ok = mbar_wait(&tfull[0], ui & 1u, abort_flag, p.err, DEV_ERR_EPI_WAIT) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      __syncwarp();
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const int row = tm * BM + h * HM + q * 32 + lane;
        if (tm * BM + h * HM >= p.m) break;              // uniform: the half has no rows
        const uint32_t taddr = tmem_base + ((q * 32u) << 16) + h * BN;
#pragma unroll 1
        for (int cb = 0; cb < BN / 32; ++cb) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + cb * 32, v);
          tmem_ld_wait();
          if (p.amax) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              v[j] = __float_as_uint(__uint_as_float(v[j]) * unscale_a * unscale_b);
          }
          const int col0 = tn * BN + cb * 32;
          if (row < p.m && col0 < p.n) {
            float* dst = p.c + static_cast<int64_t>(row) * p.ldc + col0;
            if (col0 + 32 <= p.n && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
#pragma unroll
              for (int j = 0; j < 32; j += 4) {
                float4 f = make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                       __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
                atomicAdd(reinterpret_cast<float4*>(dst + j), f);
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col0 + j < p.n) atomicAdd(dst + j, __uint_as_float(v[j]));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[0]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// Fill the strict lower triangle of a symmetric d x d matrix from its upper triangle.
__global__ void mirror_upper_kernel(float* c, int64_t ldc, int d) {
  __shared__ float tile[32][33];
  const int bi = blockIdx.y, bj = blockIdx.x;   // destination tile (row block bi, col block bj)
  if (bj > bi) return;
  const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
  // read source tile (bj, bi) from the upper triangle
  for (int r = ty; r < 32; r += 8) {
    const int i = bj * 32 + r, j = bi * 32 + tx;
    if (i < d && j < d) tile[r][tx] = c[static_cast<int64_t>(i) * ldc + j];
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int i = bi * 32 + r, j = bj * 32 + tx;
    if (i < d && j < d && i > j) c[static_cast<int64_t>(i) * ldc + j] = tile[tx][r];
  }
}

// Largest |X~| and |X - X~| over a token range (bf16 in): the scales of the fp16 drift operands.
// amax_bits[0] = max |x - x~|, amax_bits[1] = max |x~|, as fp32 bit patterns (non-negative
// floats order like their bits), combined with atomicMax: the result does not depend on order.
__global__ void drift_amax_kernel(const uint16_t* __restrict__ xfp, int64_t ld_xfp,
                                  const uint16_t* __restrict__ xq, int64_t ld_xq, int64_t rows,
                                  int cols, unsigned int* __restrict__ amax_bits) {
  const int groups = (cols + 7) / 8;
  const int64_t total = rows * groups;
  float md = 0.f, mq = 0.f;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / groups;
    const int c0 = static_cast<int>(i - r * groups) * 8;
    const uint16_t* pf = xfp + r * ld_xfp + c0;
    const uint16_t* pq = xq + r * ld_xq + c0;
    if (c0 + 8 <= cols) {
      const uint4 uf = *reinterpret_cast<const uint4*>(pf);
      const uint4 uq = *reinterpret_cast<const uint4*>(pq);
      const uint32_t f[4] = {uf.x, uf.y, uf.z, uf.w}, qv[4] = {uq.x, uq.y, uq.z, uq.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = __uint_as_float(f[e] << 16), x1 = __uint_as_float(f[e] & 0xFFFF0000u);
        const float q0 = __uint_as_float(qv[e] << 16), q1 = __uint_as_float(qv[e] & 0xFFFF0000u);
        md = fmaxf(md, fmaxf(fabsf(x0 - q0), fabsf(x1 - q1)));
        mq = fmaxf(mq, fmaxf(fabsf(q0), fabsf(q1)));
      }
    } else {
      for (int e = 0; c0 + e < cols; ++e) {
        const float x = __uint_as_float(static_cast<uint32_t>(pf[e]) << 16);
        const float q = __uint_as_float(static_cast<uint32_t>(pq[e]) << 16);
        md = fmaxf(md, fabsf(x - q));
        mq = fmaxf(mq, fabsf(q));
      }
    }
  }
  const unsigned bd = __reduce_max_sync(0xffffffffu, __float_as_uint(md));
  const unsigned bq = __reduce_max_sync(0xffffffffu, __float_as_uint(mq));
  if ((threadIdx.x & 31) == 0) {
    atomicMax(&amax_bits[0], bd);
    atomicMax(&amax_bits[1], bq);
  }
}

// The fp16 operands of the drift product over a token range: da = (x - x~) 2^ea and
// xb = x~ 2^eb, with ea, eb = fp16_shift of the amax pair; row stride ld_out (a multiple of 8).
__global__ void drift_fp16_kernel(const uint16_t* __restrict__ xfp, int64_t ld_xfp,
                                  const uint16_t* __restrict__ xq, int64_t ld_xq, int64_t rows,
                                  int cols, const float* __restrict__ amax,
                                  __half* __restrict__ da, __half* __restrict__ xb,
                                  int64_t ld_out) {
  const float sa = pow2f(fp16_shift(amax[0])), sb = pow2f(fp16_shift(amax[1]));
  const int groups = (cols + 7) / 8;
  const int64_t total = rows * groups;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / groups;
    const int c0 = static_cast<int>(i - r * groups) * 8;
    const uint16_t* pf = xfp + r * ld_xfp + c0;
    const uint16_t* pq = xq + r * ld_xq + c0;
    __half* oa = da + r * ld_out + c0;
    __half* ob = xb + r * ld_out + c0;
    if (c0 + 8 <= cols) {
      const uint4 uf = *reinterpret_cast<const uint4*>(pf);
      const uint4 uq = *reinterpret_cast<const uint4*>(pq);
      const uint32_t f[4] = {uf.x, uf.y, uf.z, uf.w}, qv[4] = {uq.x, uq.y, uq.z, uq.w};
      uint32_t ra[4], rb[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = __uint_as_float(f[e] << 16), x1 = __uint_as_float(f[e] & 0xFFFF0000u);
        const float q0 = __uint_as_float(qv[e] << 16), q1 = __uint_as_float(qv[e] & 0xFFFF0000u);
        const __half2 a2 = __floats2half2_rn((x0 - q0) * sa, (x1 - q1) * sa);
        const __half2 b2 = __floats2half2_rn(q0 * sb, q1 * sb);
        ra[e] = *reinterpret_cast<const uint32_t*>(&a2);
        rb[e] = *reinterpret_cast<const uint32_t*>(&b2);
      }
      *reinterpret_cast<uint4*>(oa) = make_uint4(ra[0], ra[1], ra[2], ra[3]);
      *reinterpret_cast<uint4*>(ob) = make_uint4(rb[0], rb[1], rb[2], rb[3]);
    } else {
      for (int e = 0; c0 + e < cols; ++e) {
        const float x = __uint_as_float(static_cast<uint32_t>(pf[e]) << 16);
        const float q = __uint_as_float(static_cast<uint32_t>(pq[e]) << 16);
        oa[e] = __float2half_rn((x - q) * sa);
        ob[e] = __float2half_rn(q * sb);
      }
    }
  }
}

// Column sums of squares of G (n x d bf16), the diagonal of G^T G. A block takes a panel of 256
// columns (8 per lane, one 16-byte load per token) and up to kDiagTokens tokens; warp w takes
// tokens w, w + 8, .. of them, eight loads in flight per lane. The 8 warps' sums meet in shared
// memory and the block writes its partial sums to part[split][column]; no atomics, so the result
// does not depend on the order blocks run in.
constexpr int kDiagTokens = 2048;

__global__ void __launch_bounds__(256, 3) diag_partial_kernel(const uint16_t* __restrict__ g,
                                                           int64_t ld, int64_t n, int d, int vec,
                                                           float* __restrict__ part) {
  __shared__ float red[8][256];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c0 = blockIdx.x * 256 + lane * 8;
  const int64_t t0 = static_cast<int64_t>(blockIdx.y) * kDiagTokens;
  const int64_t t1 = n - t0 < kDiagTokens ? n : t0 + kDiagTokens;
  const bool whole = vec && c0 + 8 <= d;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  for (int64_t tb = t0 + warp; tb < t1; tb += 64) {
    uint4 u[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t t = tb + 8 * j;
      if (whole && t < t1) u[j] = *reinterpret_cast<const uint4*>(g + t * ld + c0);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t t = tb + 8 * j;
      if (t >= t1) break;
      float v[8];
      if (whole) {
        const uint32_t q[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[2 * e] = __uint_as_float(q[e] << 16);
          v[2 * e + 1] = __uint_as_float(q[e] & 0xFFFF0000u);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          v[e] = c0 + e < d ? __uint_as_float(static_cast<uint32_t>(g[t * ld + c0 + e]) << 16) : 0.f;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = fmaf(v[e], v[e], acc[e]);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[warp][lane * 8 + e] = acc[e];
  __syncthreads();
  const int col = blockIdx.x * 256 + threadIdx.x;
  float sum = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) sum += red[k][threadIdx.x];
  if (col < d) part[static_cast<int64_t>(blockIdx.y) * d + col] = sum;
}

// diag_sum[j] += sum over splits of part[split][j], added in split order in fp64.
__global__ void diag_finalize_kernel(const float* __restrict__ part, int splits, int d,
                                     float* __restrict__ diag_sum) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= d) return;
  double s = 0.0;
  for (int k = 0; k < splits; ++k) s += part[static_cast<int64_t>(k) * d + j];
  diag_sum[j] = static_cast<float>(static_cast<double>(diag_sum[j]) + s);
}

// ---------------------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------------------
namespace {

// Tensor map over a rows x cols bf16 (or fp16) matrix (row stride ld elements), 64 x 64 boxes,
// 128B swizzle.
kronq_status make_map(CUtensorMap* map, const void* base, int64_t rows, int cols, int64_t ld,
                      bool f16) {
  const uint64_t dims[2] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(ld) * 2};
  const uint32_t box[2] = {static_cast<uint32_t>(acc::BOX), static_cast<uint32_t>(acc::BK)};
  return encode_tiled_map(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                          2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

// C (m x n, fp32, ldc) += A^T B with A: k x m bf16 (ld_a), B: k x n bf16 (ld_b).
kronq_status launch_accumulate_tc(const void* a, int64_t ld_a, const void* b, int64_t ld_b,
                                  int64_t k, int m, int n, float* c, int64_t ldc, bool symmetric,
                                  cudaStream_t stream, bool f16, const float* amax) {
  using namespace acc;
  if (k <= 0 || m <= 0 || n <= 0) return KRONQ_OK;
  CUtensorMap ma, mb;
  KQ_TRY(make_map(&ma, a, k, m, ld_a, f16));
  KQ_TRY(make_map(&mb, b, k, n, ld_b, f16));

  AccParams p{};
  p.c = c;
  p.ldc = ldc;
  p.m = m;
  p.n = n;
  p.k = k;
  p.tiles_m = (m + BM - 1) / BM;
  p.tiles_n = (n + BN - 1) / BN;
  p.symmetric = symmetric ? 1 : 0;
  if (symmetric) {
    int cnt = 0;
    for (int r = 0; r < p.tiles_m; ++r) cnt += p.tiles_n - (r * BM) / BN;
    p.num_tiles = cnt;
  } else {
    p.num_tiles = p.tiles_m * p.tiles_n;
  }
  const int sms = device_sms();
  const int kblocks = static_cast<int>((k + BK - 1) / BK);
  // Token chunk per unit: at most KQ_ACC_UNIT_KBLOCKS blocks of 64 tokens, fewer when there are
  // too few tiles to fill the GPU.
  int per = KQ_ACC_UNIT_KBLOCKS;
  while (per > 8 && static_cast<int64_t>(p.num_tiles) * ((kblocks + per - 1) / per) < 8 * sms)
    per >>= 1;
  if (per > kblocks) per = kblocks;
  p.kblocks_per_unit = per;
  p.k_splits = (kblocks + per - 1) / per;
  p.num_units = p.num_tiles * p.k_splits;
  p.fp16 = f16 ? 1 : 0;
  p.amax = amax;
  p.err = device_error_word();
  if (!p.err) return fail(KRONQ_ERR_CUDA, "device error word unavailable");

  // per device and cheap on the host, so set on every launch
  KQ_CUDA_TRY(cudaFuncSetAttribute(accumulate_tc_kernel,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES));
  const int budget = sm_budget();
  const int grid = p.num_units < budget ? p.num_units : budget;
  accumulate_tc_kernel<<<grid, THREADS, SMEM_BYTES, stream>>>(ma, mb, p);
  KQ_TRY(check_launch("accumulate_tc_kernel"));
  return KRONQ_OK;
}

kronq_status launch_mirror_upper(float* c, int64_t ldc, int d, cudaStream_t stream) {
  const int t = (d + 31) / 32;
  mirror_upper_kernel<<<dim3(t, t), dim3(32, 8), 0, stream>>>(c, ldc, d);
  return check_launch("mirror_upper_kernel");
}

kronq_status launch_drift_amax(const void* xfp, int64_t ld_xfp, const void* xq, int64_t ld_xq,
                               int64_t rows, int cols, float* amax, cudaStream_t stream) {
  KQ_CUDA_TRY(cudaMemsetAsync(amax, 0, 2 * sizeof(float), stream));
  const int64_t total = rows * ((cols + 7) / 8);
  if (total <= 0) return KRONQ_OK;
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(device_sms()) * 8;
  if (blocks > cap) blocks = cap;
  drift_amax_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(
      static_cast<const uint16_t*>(xfp), ld_xfp, static_cast<const uint16_t*>(xq), ld_xq, rows,
      cols, reinterpret_cast<unsigned int*>(amax));
  return check_launch("drift_amax_kernel");
}

kronq_status launch_drift_fp16(const void* xfp, int64_t ld_xfp, const void* xq, int64_t ld_xq,
                               int64_t rows, int cols, const float* amax, void* da, void* xb,
                               int64_t ld_out, cudaStream_t stream) {
  const int64_t total = rows * ((cols + 7) / 8);
  if (total <= 0) return KRONQ_OK;
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(device_sms()) * 8;
  if (blocks > cap) blocks = cap;
  drift_fp16_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(
      static_cast<const uint16_t*>(xfp), ld_xfp, static_cast<const uint16_t*>(xq), ld_xq, rows,
      cols, amax, static_cast<__half*>(da), static_cast<__half*>(xb), ld_out);
  return check_launch("drift_fp16_kernel");
}

size_t accumulate_diag_workspace_bytes(int64_t n, int d) {
  if (n <= 0 || d <= 0) return 0;
  const int64_t splits = (n + kDiagTokens - 1) / kDiagTokens;
  return static_cast<size_t>(splits) * d * sizeof(float);
}

kronq_status launch_accumulate_diag(const void* g, int64_t ld, int64_t n, int d, float* diag_sum,
                                    void* ws, cudaStream_t stream) {
  if (n <= 0) return KRONQ_OK;
  const int splits = static_cast<int>((n + kDiagTokens - 1) / kDiagTokens);
  const int vec = (reinterpret_cast<uintptr_t>(g) & 15u) == 0 && (ld * 2) % 16 == 0;
  float* part = static_cast<float*>(ws);
  diag_partial_kernel<<<dim3((d + 255) / 256, splits), 256, 0, stream>>>(
      static_cast<const uint16_t*>(g), ld, n, d, vec, part);
  KQ_TRY(check_launch("diag_partial_kernel"));
  diag_finalize_kernel<<<(d + 255) / 256, 256, 0, stream>>>(part, splits, d, diag_sum);
  return check_launch("diag_finalize_kernel");
}

}  // namespace kq
