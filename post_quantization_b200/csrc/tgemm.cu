// fp32-accurate GEMM on 5th-generation tensor cores: three tf32 passes.
//
//   C = alpha * A B + beta * C,   A: M x K (row-major, K contiguous), B: K x N given either as
//   an N x K row-major array (K-major) or a K x N row-major array (MN-major).
//
// Each fp32 operand x is split beforehand into hi = tf32(x) (round to nearest) and
// lo = x - hi (exact in fp32), and the product is hi*hi + hi*lo + lo*hi with fp32 accumulation
// in TMEM; the dropped lo*lo term and the tf32 rounding of lo are ~2^-22 relative, so the result
// is as accurate as an fp32 GEMM. This is what the damped inverse factor and the trailing update
// of the column solve need: a single tf32 pass would perturb the error feedback enough to flip
// quantized codes.
//
// Kernel: persistent, one CTA per SM. Warp 0 drives TMA (128-byte swizzle, 3-stage ring of
// A_hi, A_lo, B_hi, B_lo tiles, no multicast), warp 1 owns TMEM and issues
// tcgen05.mma.cta_group::1.kind::tf32 (M = N = 128, K = 8), warps 2..5 run the epilogue
// (alpha * acc + beta * C) while the next tile accumulates in the other TMEM buffer.
#include "common.cuh"
#include "internal.h"

namespace kq {

namespace tg {
constexpr int BM = 128, BN = 128, BK = 32, UK = 8, STAGES = 3;
constexpr int TILE_BYTES = 128 * BK * 4;          // 16 KB: one operand part of one stage
constexpr int STAGE_BYTES = 4 * TILE_BYTES;       // A_hi, A_lo, B_hi, B_lo
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 256;                    // two 128-column fp32 accumulators
constexpr int EPI_BYTES = 4 * 32 * 33 * 4;        // per epilogue warp: a 32 x 32 transpose tile
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024 + 256;
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
  const int32_t* skip;
  int* err;
};

__host__ __device__ constexpr uint32_t idesc_tf32_f32(int m, int n, bool b_mn) {
  return (1u << 4)                 // D: f32
         | (2u << 7)               // A: tf32
         | (2u << 10)              // B: tf32
         | (b_mn ? (1u << 16) : 0u)
         | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

__device__ __forceinline__ void umma_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Tile order and K range of one output tile (identical in every role).
struct TileInfo {
  int tm, tn, kb0, kb1;   // K blocks [kb0, kb1) of BK
};

__device__ __forceinline__ bool tile_info(const TgParams& p, int t, TileInfo& ti) {
  ti.tm = t / p.tiles_n;
  ti.tn = t % p.tiles_n;
  const int bm = ti.tm * tg::BM, bn = ti.tn * tg::BN;
  if (p.upper_only && bm > bn + tg::BN - 1) return false;   // entirely below the diagonal
  int k_lo = 0, k_hi = p.k;
  if (p.tri & GEMM_A_UPPER) k_lo = max(k_lo, bm);
  if (p.tri & GEMM_B_LOWER) k_lo = max(k_lo, bn);
  if (p.tri & GEMM_B_UPPER) k_hi = min(k_hi, bn + tg::BN);
  ti.kb0 = k_lo / tg::BK;
  ti.kb1 = k_hi > k_lo ? (k_hi + tg::BK - 1) / tg::BK : ti.kb0;
  return true;
}

__global__ void __launch_bounds__(tg::THREADS, 1)
    tgemm_kernel(const __grid_constant__ CUtensorMap ta_hi, const __grid_constant__ CUtensorMap ta_lo,
                 const __grid_constant__ CUtensorMap tb_hi, const __grid_constant__ CUtensorMap tb_lo,
                 const TgParams p) {
  using namespace tg;
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
  const int num_tiles = p.tiles_m * p.tiles_n;

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
    prefetch_tensormap(&ta_hi);
    prefetch_tensormap(&ta_lo);
    prefetch_tensormap(&tb_hi);
    prefetch_tensormap(&tb_lo);
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
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        TileInfo ti;
        if (!tile_info(p, t, ti)) continue;
        for (int kb = ti.kb0; kb < ti.kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.err, DEV_ERR_TMA_WAIT)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          const int k0 = kb * BK;
          tma_load_2d(st, &ta_hi, &full[s], k0, ti.tm * BM);
          tma_load_2d(st + TILE_BYTES, &ta_lo, &full[s], k0, ti.tm * BM);
          if (!p.b_mn_major) {
            tma_load_2d(st + 2 * TILE_BYTES, &tb_hi, &full[s], k0, ti.tn * BN);
            tma_load_2d(st + 3 * TILE_BYTES, &tb_lo, &full[s], k0, ti.tn * BN);
          } else {
#pragma unroll
            for (int j = 0; j < BN / 32; ++j) {
              tma_load_2d(st + 2 * TILE_BYTES + j * (TILE_BYTES / 4), &tb_hi, &full[s],
                          ti.tn * BN + 32 * j, k0);
              tma_load_2d(st + 3 * TILE_BYTES + j * (TILE_BYTES / 4), &tb_lo, &full[s],
                          ti.tn * BN + 32 * j, k0);
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
      const uint32_t idesc = idesc_tf32_f32(BM, BN, p.b_mn_major != 0);
      uint32_t it = 0, ui = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        TileInfo ti;
        if (!tile_info(p, t, ti)) continue;
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
            // A: K-major, 128 rows x 128 bytes, 8-row atoms of 1 KB; K step = 32 bytes.
            const uint64_t ah = smem_desc_sw128(base + kk * 32, 16, 1024);
            const uint64_t al = smem_desc_sw128(base + TILE_BYTES + kk * 32, 16, 1024);
            uint64_t bh, bl;
            if (!p.b_mn_major) {
              bh = smem_desc_sw128(base + 2 * TILE_BYTES + kk * 32, 16, 1024);
              bl = smem_desc_sw128(base + 3 * TILE_BYTES + kk * 32, 16, 1024);
            } else {
              // B: MN-major 32-bit operands use the 128-byte swizzle with 32-byte atoms (4-row
              // K groups of 512 bytes, SBO); boxes of 32 K-rows x 128 bytes, 4 along N
              // (LBO = 4 KB); K step = 8 rows = 1 KB.
              bh = smem_desc(base + 2 * TILE_BYTES + kk * 1024, TILE_BYTES / 4, 512, 1u);
              bl = smem_desc(base + 3 * TILE_BYTES + kk * 1024, TILE_BYTES / 4, 512, 1u);
            }
            const uint32_t first = (kb == ti.kb0 && kk == 0) ? 0u : 1u;
            umma_tf32(d_tmem, al, bh, idesc, first);   // lo * hi
            umma_tf32(d_tmem, ah, bl, idesc, 1u);      // hi * lo
            umma_tf32(d_tmem, ah, bh, idesc, 1u);      // hi * hi
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
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      TileInfo ti;
      if (!tile_info(p, t, ti)) continue;
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
      float* tw = epi + q * (32 * 33);              // transpose tile of this warp
#pragma unroll 1
      for (int cb = 0; cb < BN / 32; ++cb) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + cb * 32, v);
        tmem_ld_wait();
        // lane = row: stage the 32 x 32 chunk, then lane = column for coalesced C traffic
#pragma unroll
        for (int j = 0; j < 32; ++j) tw[lane * 33 + j] = has_k ? __uint_as_float(v[j]) : 0.f;
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
          if (ok_rc) cbase[static_cast<int64_t>(r) * p.ldc] = fmaf(p.beta, old[r], p.alpha * tw[r * 33 + lane]);
        }
        __syncwarp();
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

// hi = tf32(x) (round to nearest, ties away), lo = x - hi; rows x cols, any source stride,
// destination stride ld (a multiple of 4 floats). Up to two matrices per launch.
struct SplitJob {
  const float* src;
  int64_t lds;
  int rows, cols;
  float* hi;
  float* lo;
  int64_t ld;
};

__global__ void split_tf32_kernel(SplitJob j0, SplitJob j1) {
  const int64_t n0 = static_cast<int64_t>(j0.rows) * j0.cols;
  const int64_t total = n0 + static_cast<int64_t>(j1.rows) * j1.cols;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const bool second = e >= n0;
    const SplitJob& j = second ? j1 : j0;
    const int64_t f = second ? e - n0 : e;
    const int64_t r = f / j.cols, c = f - r * j.cols;
    const float x = j.src[r * j.lds + c];
    uint32_t h;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(x));
    const float hf = __uint_as_float(h);
    j.hi[r * j.ld + c] = hf;
    j.lo[r * j.ld + c] = x - hf;
  }
}

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// fp32 tensor map: rows x cols (cols contiguous, row stride ld floats), box = box_cols x box_rows,
// 128-byte swizzle with 16-byte (K-major operands) or 32-byte (MN-major operands) atoms.
kronq_status map_f32(CUtensorMap* map, const float* base, int64_t rows, int64_t cols, int64_t ld,
                     int box_cols, int box_rows, bool atom32 = false) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(KRONQ_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  if ((reinterpret_cast<uintptr_t>(base) & 15u) || (ld * 4) % 16)
    return fail(KRONQ_ERR_INVALID_ARG, "tensor-core GEMM operand not 16-byte aligned");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 4};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   atom32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KRONQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return KRONQ_OK;
}

int sm_count() {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}

}  // namespace

kronq_status split_tf32(const float* src, int64_t lds, int rows, int cols, SplitF32 dst,
                        cudaStream_t stream) {
  return split_tf32_2(src, lds, rows, cols, dst, nullptr, 0, 0, 0, SplitF32{}, stream);
}

kronq_status split_tf32_2(const float* src0, int64_t lds0, int rows0, int cols0, SplitF32 dst0,
                          const float* src1, int64_t lds1, int rows1, int cols1, SplitF32 dst1,
                          cudaStream_t stream) {
  SplitJob j0{src0, lds0, rows0, cols0 > 0 ? cols0 : 1, dst0.hi, dst0.lo, dst0.ld};
  SplitJob j1{src1, lds1, src1 ? rows1 : 0, cols1 > 0 ? cols1 : 1, dst1.hi, dst1.lo, dst1.ld};
  if (cols0 <= 0) j0.rows = 0;
  const int64_t total = static_cast<int64_t>(j0.rows) * j0.cols + static_cast<int64_t>(j1.rows) * j1.cols;
  if (total <= 0) return KRONQ_OK;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  split_tf32_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(j0, j1);
  return check_launch("split_tf32_kernel");
}

kronq_status tgemm(int m, int n, int k, float alpha, SplitF32 a, SplitF32 b, bool b_mn_major,
                   float beta, float* c, int64_t ldc, bool upper_only, int tri,
                   const int32_t* skip, cudaStream_t stream) {
  using namespace tg;
  if (m <= 0 || n <= 0) return KRONQ_OK;
  if (k <= 0) return fail(KRONQ_ERR_SHAPE, "tensor-core GEMM needs k >= 1");
  CUtensorMap mah, mal, mbh, mbl;
  const int kk = k;
  KQ_TRY(map_f32(&mah, a.hi, m, kk, a.ld, BK, BM));
  KQ_TRY(map_f32(&mal, a.lo, m, kk, a.ld, BK, BM));
  if (!b_mn_major) {
    KQ_TRY(map_f32(&mbh, b.hi, n, kk, b.ld, BK, BN));
    KQ_TRY(map_f32(&mbl, b.lo, n, kk, b.ld, BK, BN));
  } else {
    KQ_TRY(map_f32(&mbh, b.hi, kk, n, b.ld, 32, BK, true));
    KQ_TRY(map_f32(&mbl, b.lo, kk, n, b.ld, 32, BK, true));
  }
  TgParams p{};
  p.c = c;
  p.ldc = ldc;
  p.m = m;
  p.n = n;
  p.k = k;
  p.alpha = alpha;
  p.beta = beta;
  p.tiles_m = (m + BM - 1) / BM;
  p.tiles_n = (n + BN - 1) / BN;
  p.b_mn_major = b_mn_major ? 1 : 0;
  p.upper_only = upper_only ? 1 : 0;
  p.tri = tri;
  p.skip = skip;
  p.err = device_error_word();
  if (!p.err) return fail(KRONQ_ERR_CUDA, "device error word unavailable");
  static bool attr = false;
  if (!attr) {
    KQ_CUDA_TRY(cudaFuncSetAttribute(tgemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     SMEM_BYTES));
    attr = true;
  }
  const int tiles = p.tiles_m * p.tiles_n;
  const int sms = sm_count();
  tgemm_kernel<<<tiles < sms ? tiles : sms, THREADS, SMEM_BYTES, stream>>>(mah, mal, mbh, mbl, p);
  return check_launch("tgemm_kernel");
}

}  // namespace kq
