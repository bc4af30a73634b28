// fp32-accurate GEMM on 5th-generation tensor cores: bf16 x3 split, six products.
//
//   C = alpha * A B + beta * C,   A: M x K (row-major, K contiguous), B: K x N given either as
//   an N x K row-major array (K-major) or a K x N row-major array (MN-major).
//
// Each fp32 operand x is split beforehand into three bf16 pieces x = x0 + x1 + x2 (each the
// bf16 rounding of what the previous pieces left), which carry its 24 significant bits. The
// product keeps every term down to 2^-16 relative, a0 b0 + a0 b1 + a1 b0 + a0 b2 + a1 b1 + a2 b0
// (a call may ask for the first three only, ~2^-16 relative, where the result is a small
// correction to a value held exactly elsewhere);
// bf16 x bf16 products are exact, the dropped terms are ~2^-24 relative, and the sums are the
// tensor core's fp32 accumulation (measured ~1e-5 relative at K = 1024, close to a CUDA-core
// fp32 GEMM). This is what the damped inverse factor and the trailing update of the column
// solve need: one bf16 or tf32 pass perturbs the error feedback enough to flip quantized codes.
// Six bf16 MMAs take the time of three tf32 ones and move 25% fewer operand bytes.
//
// Kernel: persistent, one CTA per SM. Warp 0 drives TMA (128-byte swizzle, 2-stage ring of the
// six operand pieces, no multicast), warp 1 owns TMEM and issues
// tcgen05.mma.cta_group::1.kind::f16 (M = N = 128, K = 16, bf16 in, fp32 accumulate), warps
// 2..5 run the epilogue (alpha * acc + beta * C, coalesced through a per-warp transpose tile)
// while the next tile accumulates in the other TMEM buffer.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <utility>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace kq {

namespace tg {
constexpr int BM = 128, UK = 16, THREADS = 192;

// Two tile shapes. A tcgen05 MMA takes about the same time for any N up to 256, so the 128 x 256
// tile runs the tensor pipe at twice the rate of the 128 x 128 one. Its operand pieces are
// K = 32 deep (64-byte rows, 64-byte swizzle) so that two pipeline stages of the six pieces still
// fit in shared memory; the 128 x 128 tile keeps K = 64 (128-byte rows, 128-byte swizzle).
// The 128 x 256 tile keeps three stages in flight: its epilogue stages 32 x 16 halves of each
// 32-column chunk (the 128 x 128 tile stages whole 32 x 32 chunks, with two stages).
template <int BN_>
struct Cfg {
  static constexpr int BN = BN_;
  static constexpr int STAGES = BN_ == 256 ? 3 : 2;
  static constexpr int EPI_COLS = BN_ == 256 ? 16 : 32;     // columns staged per pass
  static constexpr int EPI_LD = EPI_COLS + 1;
  static constexpr int EPI_BYTES = 4 * 32 * EPI_LD * 4;     // per warp: 32 rows x EPI_COLS
  static constexpr int BK = BN_ == 256 ? 32 : 64;
  static constexpr int ROW_BYTES = BK * 2;                  // one K-major row of a piece
  static constexpr uint32_t KSW = BN_ == 256 ? 4u : 2u;     // descriptor layout: 64B / 128B swizzle
  static constexpr uint32_t KSBO = 8 * ROW_BYTES;           // bytes per 8-row swizzle atom
  static constexpr int A_PIECE = BM * BK * 2;
  static constexpr int B_PIECE = BN_ * BK * 2;
  static constexpr int STAGE_BYTES = 3 * (A_PIECE + B_PIECE);   // A0, A1, A2, B0, B1, B2
  static constexpr int MN_BOX_BYTES = 64 * BK * 2;          // 64 columns x BK rows (MN-major B)
  static constexpr int TMEM_COLS = 2 * BN_;                 // two fp32 accumulators
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024 + 256;
};
static_assert(Cfg<256>::SMEM_BYTES <= 227 * 1024, "128 x 256 tile: shared memory");
}  // namespace tg

struct TgParams {
  float* c;
  int64_t ldc;
  int m, n, k;
  float alpha, beta;
  int tiles_m, tiles_n;
  int b_mn_major;
  int upper_only;
  int tri;
  int products;           // 6: every term down to 2^-16 relative; 3: a0 b0 + a0 b1 + a1 b0
  const int32_t* skip;
  int* err;
  // Tile schedule: slot j = blockIdx.x + i * gridDim.x holds the CTA's i-th tile; slot j is
  // tile j, unless the launch passes a table (TgOrder<true>).
  int n_slots;
};

// The table: order[j] is slot j's tile (kTgNoTile for none). A separate kernel parameter, so
// that launches without one keep a small parameter block.
template <bool SCHED>
struct TgOrder {
  uint16_t order[SCHED ? 1536 : 2];
};
constexpr uint16_t kTgNoTile = 0xFFFF;

template <bool SCHED>
__device__ __forceinline__ int slot_tile(const TgOrder<SCHED>& o, int j) {
  if constexpr (SCHED) return o.order[j] == kTgNoTile ? -1 : static_cast<int>(o.order[j]);
  return j;
}

__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n, bool b_mn) {
  return (1u << 4)                 // D: f32
         | (1u << 7)               // A: bf16
         | (1u << 10)              // B: bf16
         | (b_mn ? (1u << 16) : 0u)
         | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

// Tile order and K range of one output tile (identical in every role).
struct TileInfo {
  int tm, tn, kb0, kb1;   // K blocks [kb0, kb1) of BK
};

template <class C>
__device__ __forceinline__ bool tile_info(const TgParams& p, int t, TileInfo& ti) {
  ti.tm = t / p.tiles_n;
  ti.tn = t % p.tiles_n;
  const int bm = ti.tm * tg::BM, bn = ti.tn * C::BN;
  if (p.upper_only && bm > bn + C::BN - 1) return false;   // entirely below the diagonal
  int k_lo = 0, k_hi = p.k;
  if (p.tri & GEMM_A_UPPER) k_lo = max(k_lo, bm);
  if (p.tri & GEMM_A_LOWER) k_hi = min(k_hi, bm + tg::BM);
  if (p.tri & GEMM_B_LOWER) k_lo = max(k_lo, bn);
  if (p.tri & GEMM_B_UPPER) k_hi = min(k_hi, bn + C::BN);
  ti.kb0 = k_lo / C::BK;
  ti.kb1 = k_hi > k_lo ? (k_hi + C::BK - 1) / C::BK : ti.kb0;
  return true;
}

struct TgMaps {
  CUtensorMap a[3];
  CUtensorMap b[3];
};
static_assert(sizeof(TgMaps) + sizeof(TgParams) + sizeof(TgOrder<true>) <= 4096,
              "tgemm kernel parameters above 4 KB");

template <int BN_, bool SCHED>
__global__ void __launch_bounds__(tg::THREADS, 1)
    tgemm_kernel(const __grid_constant__ TgMaps maps, const TgParams p,
                 const __grid_constant__ TgOrder<SCHED> sched) {
  using namespace tg;
  using C = Cfg<BN_>;
  constexpr int BN = C::BN, BK = C::BK, STAGE_BYTES = C::STAGE_BYTES, TMEM_COLS = C::TMEM_COLS;
  constexpr int STAGES = C::STAGES, EPI_BYTES = C::EPI_BYTES, EPI_LD = C::EPI_LD;
  constexpr int A_PIECE = C::A_PIECE, B_PIECE = C::B_PIECE, MN_BOX_BYTES = C::MN_BOX_BYTES;
  if (p.skip && *p.skip >= 0) return;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* epi = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES + EPI_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = bars + 2 * STAGES + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

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
    for (int i = 0; i < 3; ++i) {
      prefetch_tensormap(&maps.a[i]);
      prefetch_tensormap(&maps.b[i]);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int j = blockIdx.x; j < p.n_slots && ok; j += gridDim.x) {
        const int t = slot_tile<SCHED>(sched, j);
        TileInfo ti;
        if (t < 0 || !tile_info<C>(p, t, ti)) continue;
        for (int kb = ti.kb0; kb < ti.kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.err, DEV_ERR_TMA_WAIT)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * STAGE_BYTES;
          // three products read only the first two pieces of each operand
          const int pieces = p.products == 3 ? 2 : 3;
          mbar_arrive_expect_tx(&full[s], pieces * (A_PIECE + B_PIECE));
          const int k0 = kb * BK;
#pragma unroll
          for (int i = 0; i < 3; ++i) {
            if (i >= pieces) break;
            tma_load_2d(st + i * A_PIECE, &maps.a[i], &full[s], k0, ti.tm * BM);
            uint8_t* bp = st + 3 * A_PIECE + i * B_PIECE;
            if (!p.b_mn_major) {
              tma_load_2d(bp, &maps.b[i], &full[s], k0, ti.tn * BN);
            } else {
#pragma unroll
              for (int bx = 0; bx < BN / 64; ++bx)
                tma_load_2d(bp + bx * MN_BOX_BYTES, &maps.b[i], &full[s], ti.tn * BN + 64 * bx, k0);
            }
          }
        }
      }
      if (!ok) {
        for (uint32_t j = it > STAGES ? it - STAGES : 0; j < it; ++j)
          mbar_drain(&full[j % STAGES], (j / STAGES) & 1u, 1000000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(BM, BN, p.b_mn_major != 0);
      uint32_t it = 0, ui = 0;
      bool ok = true;
      for (int j = blockIdx.x; j < p.n_slots && ok; j += gridDim.x) {
        const int t = slot_tile<SCHED>(sched, j);
        TileInfo ti;
        if (t < 0 || !tile_info<C>(p, t, ti)) continue;
        const uint32_t a = ui & 1u;
        const uint32_t aph = (ui >> 1) & 1u;
        ++ui;
        if (!mbar_wait(&tempty[a], aph ^ 1u, abort_flag, p.err, DEV_ERR_MMA_WAIT)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + a * BN;
        for (int kb = ti.kb0; kb < ti.kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(&full[s], ph, abort_flag, p.err, DEV_ERR_MMA_WAIT)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t base = smem_u32(smem + s * STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk) {
            uint64_t ad[3], bd[3];
#pragma unroll
            for (int i = 0; i < 3; ++i) {
              // A: K-major, 128 rows of BK elements, 8-row swizzle atoms; K step = 32 bytes.
              ad[i] = smem_desc(base + i * A_PIECE + kk * 32, 16, C::KSBO, C::KSW);
              const uint32_t bb = base + 3 * A_PIECE + i * B_PIECE;
              // B: K-major like A, or MN-major in 64-column boxes of 128-byte rows (LBO = box),
              // K step = 16 rows = 2 KB.
              bd[i] = p.b_mn_major ? smem_desc_sw128(bb + kk * 2048, MN_BOX_BYTES, 1024)
                                   : smem_desc(bb + kk * 32, 16, C::KSBO, C::KSW);
            }
            const uint32_t first = (kb == ti.kb0 && kk == 0) ? 0u : 1u;
            if (p.products == 3) {
              umma_f16(d_tmem, ad[1], bd[0], idesc, first);   // smallest terms first
              umma_f16(d_tmem, ad[0], bd[1], idesc, 1u);
              umma_f16(d_tmem, ad[0], bd[0], idesc, 1u);
            } else {
              umma_f16(d_tmem, ad[2], bd[0], idesc, first);
              umma_f16(d_tmem, ad[1], bd[1], idesc, 1u);
              umma_f16(d_tmem, ad[0], bd[2], idesc, 1u);
              umma_f16(d_tmem, ad[1], bd[0], idesc, 1u);
              umma_f16(d_tmem, ad[0], bd[1], idesc, 1u);
              umma_f16(d_tmem, ad[0], bd[0], idesc, 1u);
            }
          }
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&tfull[a]);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;
    uint32_t ui = 0;
    for (int j = blockIdx.x; j < p.n_slots; j += gridDim.x) {
      const int t = slot_tile<SCHED>(sched, j);
      TileInfo ti;
      if (t < 0 || !tile_info<C>(p, t, ti)) continue;
      const uint32_t a = ui & 1u;
      const uint32_t aph = (ui >> 1) & 1u;
      ++ui;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&tfull[a], aph, abort_flag, p.err, DEV_ERR_EPI_WAIT) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      __syncwarp();
      if (!ok) break;
      tc_fence_after();
      const bool has_k = ti.kb1 > ti.kb0;
      const int row0 = ti.tm * BM + q * 32;        // this warp's 32 rows
      const uint32_t taddr = tmem_base + ((q * 32u) << 16) + a * BN;
      float* tw = epi + q * (32 * EPI_LD);          // transpose tile of this warp
#pragma unroll 1
      for (int cb = 0; cb < BN / 32; ++cb) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + cb * 32, v);
        tmem_ld_wait();
        if constexpr (C::EPI_COLS == 32) {
          // lane = row: stage the 32 x 32 chunk, then lane = column for coalesced C traffic
#pragma unroll
          for (int j = 0; j < 32; ++j) tw[lane * EPI_LD + j] = has_k ? __uint_as_float(v[j]) : 0.f;
          __syncwarp();
          const int col = ti.tn * BN + cb * 32 + lane;
          float* cbase = p.c + static_cast<int64_t>(row0) * p.ldc + col;
          float old[32];
          // all 32 loads of C are issued before any is used
#pragma unroll
          for (int r = 0; r < 32; ++r) {
            const bool ok_rc = col < p.n && row0 + r < p.m && !(p.upper_only && col < row0 + r);
            old[r] = (ok_rc && p.beta != 0.f) ? cbase[static_cast<int64_t>(r) * p.ldc] : 0.f;
          }
#pragma unroll
          for (int r = 0; r < 32; ++r) {
            const bool ok_rc = col < p.n && row0 + r < p.m && !(p.upper_only && col < row0 + r);
            if (ok_rc)
              cbase[static_cast<int64_t>(r) * p.ldc] =
                  fmaf(p.beta, old[r], p.alpha * tw[r * EPI_LD + lane]);
          }
          __syncwarp();
        } else {
          // two 32 x 16 halves: lane = row to stage, then lanes 0..15 and 16..31 take the 16
          // columns of two rows at a time (two 64-byte segments per access)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              tw[lane * EPI_LD + j] = has_k ? __uint_as_float(v[16 * h + j]) : 0.f;
            __syncwarp();
            const int cl = lane & 15, rh = lane >> 4;
            const int col = ti.tn * BN + cb * 32 + 16 * h + cl;
            float* cbase = p.c + static_cast<int64_t>(row0 + rh) * p.ldc + col;
            float old[16];
#pragma unroll
            for (int it = 0; it < 16; ++it) {
              const int r = 2 * it + rh;
              const bool ok_rc = col < p.n && row0 + r < p.m && !(p.upper_only && col < row0 + r);
              old[it] = (ok_rc && p.beta != 0.f) ? cbase[static_cast<int64_t>(2 * it) * p.ldc] : 0.f;
            }
#pragma unroll
            for (int it = 0; it < 16; ++it) {
              const int r = 2 * it + rh;
              const bool ok_rc = col < p.n && row0 + r < p.m && !(p.upper_only && col < row0 + r);
              if (ok_rc)
                cbase[static_cast<int64_t>(2 * it) * p.ldc] =
                    fmaf(p.beta, old[it], p.alpha * tw[r * EPI_LD + cl]);
            }
            __syncwarp();
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[a]);
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

// x = x0 + x1 + x2 in bf16 (round to nearest even at each step; each residual is exact in fp32),
// rows x cols, any source stride, destination stride ld (a multiple of 8 elements).
// Up to two matrices per launch.
struct SplitJob {
  const float* src;
  int64_t lds;
  int rows, cols;
  uint16_t* part[3];
  int64_t ld;
};

// 8 consecutive columns of one row per thread (blockIdx.y = row, blockIdx.z = job): no index
// division, 16-byte stores of each piece (destination rows start on 16-byte boundaries: the
// stride is a multiple of 8 elements).
__global__ void __launch_bounds__(128) split_bf16x3_kernel(SplitJob j0, SplitJob j1) {
  const SplitJob& j = blockIdx.z ? j1 : j0;
  const int r = blockIdx.y;
  const int c8 = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (r >= j.rows || c8 >= j.cols) return;
  const float* src = j.src + static_cast<int64_t>(r) * j.lds + c8;
  float x[8];
  const bool vec = c8 + 8 <= j.cols && ((reinterpret_cast<uintptr_t>(src) & 15u) == 0);
  if (vec) {
    const float4 a = reinterpret_cast<const float4*>(src)[0];
    const float4 b = reinterpret_cast<const float4*>(src)[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  } else {
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = c8 + u < j.cols ? src[u] : 0.f;
  }
  uint32_t h[3][4];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const __nv_bfloat16 b0 = __float2bfloat16_rn(x[u]);
    const float r1 = x[u] - __bfloat162float(b0);
    const __nv_bfloat16 b1 = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(b1);
    const __nv_bfloat16 b2 = __float2bfloat16_rn(r2);
    const int sh = 16 * (u & 1);
    if ((u & 1) == 0) { h[0][u >> 1] = 0u; h[1][u >> 1] = 0u; h[2][u >> 1] = 0u; }
    h[0][u >> 1] |= static_cast<uint32_t>(__bfloat16_as_ushort(b0)) << sh;
    h[1][u >> 1] |= static_cast<uint32_t>(__bfloat16_as_ushort(b1)) << sh;
    h[2][u >> 1] |= static_cast<uint32_t>(__bfloat16_as_ushort(b2)) << sh;
  }
  const int64_t o = static_cast<int64_t>(r) * j.ld + c8;
  if (c8 + 8 <= j.cols) {
#pragma unroll
    for (int i = 0; i < 3; ++i)
      *reinterpret_cast<uint4*>(j.part[i] + o) = make_uint4(h[i][0], h[i][1], h[i][2], h[i][3]);
  } else {
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (c8 + u < j.cols) {
#pragma unroll
        for (int i = 0; i < 3; ++i)
          j.part[i][o + u] = static_cast<uint16_t>(h[i][u >> 1] >> (16 * (u & 1)));
      }
  }
}

namespace {

// bf16 tensor map: rows x cols (cols contiguous, row stride ld elements), box = box_cols x
// box_rows; the swizzle spans the box's row (64 or 128 bytes).
kronq_status map_bf16(CUtensorMap* map, const uint16_t* base, int64_t rows, int64_t cols,
                      int64_t ld, int box_cols, int box_rows) {
  if ((reinterpret_cast<uintptr_t>(base) & 15u) || (ld * 2) % 16)
    return fail(KRONQ_ERR_INVALID_ARG, "tensor-core GEMM operand not 16-byte aligned");
  const uint64_t dims[2] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(ld) * 2};
  const uint32_t box[2] = {static_cast<uint32_t>(box_cols), static_cast<uint32_t>(box_rows)};
  return encode_tiled_map(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
                          box_cols * 2 == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

// The 128 x 256 tile is the default; KRONQ_TGEMM_TILE=128 in the environment selects the
// 128 x 128 tile (same results to rounding order; kept to compare the two).
bool tgemm_wide_tiles() {
  const char* v = std::getenv("KRONQ_TGEMM_TILE");
  return !(v && std::strcmp(v, "128") == 0);
}

template <int BN_>
kronq_status launch_tgemm(const Split3& a, const Split3& b, TgParams p, bool b_mn_major,
                          cudaStream_t stream) {
  using C = tg::Cfg<BN_>;
  TgMaps maps;
  for (int i = 0; i < 3; ++i) {
    KQ_TRY(map_bf16(&maps.a[i], a.part[i], p.m, p.k, a.ld, C::BK, tg::BM));
    if (!b_mn_major)
      KQ_TRY(map_bf16(&maps.b[i], b.part[i], p.n, p.k, b.ld, C::BK, C::BN));
    else
      KQ_TRY(map_bf16(&maps.b[i], b.part[i], p.k, p.n, b.ld, 64, C::BK));
  }
  p.tiles_m = (p.m + tg::BM - 1) / tg::BM;
  p.tiles_n = (p.n + C::BN - 1) / C::BN;
  // per device and cheap on the host, so set on every launch
  KQ_CUDA_TRY(cudaFuncSetAttribute(tgemm_kernel<BN_, false>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
  KQ_CUDA_TRY(cudaFuncSetAttribute(tgemm_kernel<BN_, true>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
  // The tiles that have work, with their K lengths (the same rule as tile_info): triangular
  // operands make the lengths differ by up to the whole K.
  const int tiles = p.tiles_m * p.tiles_n;
  std::vector<std::pair<int, int>> work;   // (K blocks, tile)
  work.reserve(tiles);
  for (int t = 0; t < tiles; ++t) {
    const int tm = t / p.tiles_n, tn = t % p.tiles_n;
    const int bm = tm * tg::BM, bn = tn * C::BN;
    if (p.upper_only && bm > bn + C::BN - 1) continue;
    int k_lo = 0, k_hi = p.k;
    if (p.tri & GEMM_A_UPPER) k_lo = std::max(k_lo, bm);
    if (p.tri & GEMM_A_LOWER) k_hi = std::min(k_hi, bm + tg::BM);
    if (p.tri & GEMM_B_LOWER) k_lo = std::max(k_lo, bn);
    if (p.tri & GEMM_B_UPPER) k_hi = std::min(k_hi, bn + C::BN);
    const int kb = k_hi > k_lo ? (k_hi + C::BK - 1) / C::BK - k_lo / C::BK : 0;
    work.emplace_back(kb, t);
  }
  const int n_work = static_cast<int>(work.size());
  const int sms = sm_budget();
  bool uniform = true;
  for (const auto& w : work) uniform = uniform && w.first == work[0].first;
  TgOrder<true> order;
  constexpr int kMaxSlots = static_cast<int>(sizeof(order.order) / sizeof(order.order[0]));
  p.n_slots = tiles;
  int grid = 1;
  if ((!uniform || n_work < tiles) && n_work > 0 &&
      ((n_work + sms - 1) / sms) * std::min(sms, n_work) <= kMaxSlots) {
    // Tiles of different K lengths (triangular operands), or only some tiles with work (the
    // upper triangle): every SM takes part, and the tiles that have work, longest first, are
    // dealt to the CTAs in a snake (wave w forward when w is even, backward when odd), so that
    // each CTA gets a mix of long and short tiles and no CTA holds only the long ones. (In the
    // plain order a CTA's slots would fall on the skipped triangle unevenly.) The order travels
    // as a table in the kernel's parameters.
    grid = std::min(sms, n_work);
    const int waves = (n_work + grid - 1) / grid;
    std::stable_sort(work.begin(), work.end(),
                     [](const std::pair<int, int>& x, const std::pair<int, int>& y) {
                       return x.first > y.first;
                     });
    const int slots = waves * grid;
    for (int j = 0; j < slots; ++j) order.order[j] = kTgNoTile;
    for (int r = 0; r < n_work; ++r) {
      const int w = r / grid, i = r % grid;
      const int cta = (w & 1) ? grid - 1 - i : i;
      order.order[w * grid + cta] = static_cast<uint16_t>(work[r].second);
    }
    p.n_slots = slots;
    tgemm_kernel<BN_, true><<<grid, tg::THREADS, C::SMEM_BYTES, stream>>>(maps, p, order);
    return check_launch("tgemm_kernel");
  } else {
    // Equal tiles that all have work, or too many for the table (then enough per CTA for the
    // plain order to even out): as few CTAs as the minimal number of tile waves needs. Each CTA holds a whole SM
    // (shared memory), and SMs this GEMM does not need stay free for other streams' work.
    const int waves = (n_work + sms - 1) / sms;
    grid = waves > 0 ? (tiles + waves - 1) / waves : 1;
    grid = std::max(1, std::min(grid, sms));
  }
  tgemm_kernel<BN_, false><<<grid, tg::THREADS, C::SMEM_BYTES, stream>>>(maps, p,
                                                                          TgOrder<false>{});
  return check_launch("tgemm_kernel");
}


}  // namespace

kronq_status split_bf16x3(const float* src, int64_t lds, int rows, int cols, Split3 dst,
                          cudaStream_t stream) {
  return split_bf16x3_2(src, lds, rows, cols, dst, nullptr, 0, 0, 0, Split3{}, stream);
}

kronq_status split_bf16x3_2(const float* src0, int64_t lds0, int rows0, int cols0, Split3 dst0,
                            const float* src1, int64_t lds1, int rows1, int cols1, Split3 dst1,
                            cudaStream_t stream) {
  SplitJob j0{src0, lds0, cols0 > 0 ? rows0 : 0, cols0 > 0 ? cols0 : 1,
              {dst0.part[0], dst0.part[1], dst0.part[2]}, dst0.ld};
  SplitJob j1{src1, lds1, (src1 && cols1 > 0) ? rows1 : 0, cols1 > 0 ? cols1 : 1,
              {dst1.part[0], dst1.part[1], dst1.part[2]}, dst1.ld};
  const int rows = j0.rows > j1.rows ? j0.rows : j1.rows;
  const int cols = j0.cols > j1.cols ? j0.cols : j1.cols;
  if (rows <= 0) return KRONQ_OK;
  if (rows > 65535) return fail(KRONQ_ERR_SHAPE, "split: more than 65535 rows");
  dim3 grid(static_cast<unsigned>((cols + 8 * 128 - 1) / (8 * 128)), static_cast<unsigned>(rows),
            j1.rows > 0 ? 2u : 1u);
  split_bf16x3_kernel<<<grid, 128, 0, stream>>>(j0, j1);
  return check_launch("split_bf16x3_kernel");
}

kronq_status tgemm(int m, int n, int k, float alpha, Split3 a, Split3 b, bool b_mn_major,
                   float beta, float* c, int64_t ldc, bool upper_only, int tri,
                   const int32_t* skip, cudaStream_t stream, int products) {
  if (m <= 0 || n <= 0) return KRONQ_OK;
  if (k <= 0) return fail(KRONQ_ERR_SHAPE, "tensor-core GEMM needs k >= 1");
  if (products != 3 && products != 6) return fail(KRONQ_ERR_INVALID_ARG, "products must be 3 or 6");
  TgParams p{};
  p.c = c;
  p.ldc = ldc;
  p.m = m;
  p.n = n;
  p.k = k;
  p.alpha = alpha;
  p.beta = beta;
  p.b_mn_major = b_mn_major ? 1 : 0;
  p.upper_only = upper_only ? 1 : 0;
  p.tri = tri;
  p.products = products;
  p.skip = skip;
  p.err = device_error_word();
  if (!p.err) return fail(KRONQ_ERR_CUDA, "device error word unavailable");
  // 128 x 256 tiles where they still give every SM a tile (fewer, wider tiles halve the CTAs
  // of a small product, which then runs longer)
  const int64_t wide_tiles = static_cast<int64_t>((m + 127) / 128) * ((n + 255) / 256);
  if (n > 128 && wide_tiles >= sm_budget() && tgemm_wide_tiles())
    return launch_tgemm<256>(a, b, p, b_mn_major, stream);
  return launch_tgemm<128>(a, b, p, b_mn_major, stream);
}

}  // namespace kq
