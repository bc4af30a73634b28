// The quantized layer at inference: packed 2/3/4-bit codes and
//     y = S_G^-1 U^T W^' V S_X^-1 x,   W^' = scale (codes - zero)
// ([KronQ-gist] Limitations: at inference the only overhead is the orthogonal transforms).
//
// Three kernels per pass of up to 32 tokens, chained with programmatic dependent launch so
// that each one's launch overlaps its predecessor:
//   qlin_in_kernel   x' = V S_X^-1 x (scale, sign, Hadamard blocks: radix-16 passes in shared
//                    memory), cut into 128-column groups, each written as three int8 terms
//                    x' ~ s (q0 + q1 / 128 + q2 / 128^2) with a power-of-two s per group and
//                    token: the tensor-core B operand, pre-swizzled, plus (s, sum of the terms)
//                    per group for the zero point.
//   qlin_mma_kernel  persistent CTAs stream the packed codes (bulk copies of several units at
//                    once into a ring of stages); eight warps turn each 128 x 128 blob into
//                    8-bit codes in tensor memory (one shift and one mask per four codes,
//                    tcgen05.st); tcgen05.mma kind::i8 multiplies them, exactly, with the int8
//                    terms of x'; four epilogue warps apply the grid, the group scale and the
//                    within-tile part of U^T, and write one partial per (CTA, row tile). Work is
//                    split over CTAs as contiguous ranges of (row tile, column group) units.
//   qlin_dp4a_kernel (one or two tokens, in place of qlin_mma_kernel) a producer warp streams
//                    each CTA's units of packed codes and grid into a shared-memory ring with
//                    bulk copies; four warps, one thread per row, take exact int32 dot products
//                    of the codes with the int8 terms (dp4a) and write the same partials.
//   qlin_out_kernel  sums each tile's partials in a fixed order (deterministic), applies the
//                    across-tile part of U^T, the signs and S_G^-1.
// The codes are the MMA's A operand (128 rows per instruction); a tcgen05 MMA costs about the
// same time for any N up to 256, so the tokens ride along in N, and 8-bit operands (32 columns
// per instruction, twice bf16's) halve the MMA time per code.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

constexpr int QL_TILE = 128;            // rows per tile, columns per group
constexpr int QL_NT_MAX = 32;           // tokens per pass
constexpr int QL_THREADS = 512;         // 16 warps
constexpr int QL_EPI_WARP0 = 4;         // warps 4..7: epilogue (TMEM lanes 32 (w % 4) ...)
constexpr int QL_DQ_WARP0 = 8;          // warps 8..15: dequantization
constexpr int QL_DQ_THREADS = 256;
constexpr int QL_MAX_STAGES = 16;
constexpr int QL_TERMS = 3;             // int8 terms of x'
constexpr int QL_DP_THREADS = 160;      // decode kernel: 4 consumer warps + 1 producer warp
constexpr int QL_DP_CTAS_PER_SM = 5;
constexpr int QL_DP_MAX_STAGES = 8;

__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// 1-D bulk copy global -> shared, completion on `bar` (no multicast).
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes),
      "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Named barrier that also returns the AND of a predicate over the participating threads.
__device__ __forceinline__ bool bar_and(int id, int count, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.b32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(out)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(count)
      : "memory");
  return out != 0;
}

// ---- thread-block clusters (distributed shared memory)
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_shared_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_dsmem(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// 32 lanes x 16 consecutive 32-bit TMEM columns.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// kind::i8: A unsigned 8-bit (codes), B signed 8-bit (terms of x'), both K-major, s32 accumulate.
__host__ __device__ constexpr uint32_t ql_idesc(int m, int n) {
  return (2u << 4) | (0u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

// ---------------------------------------------------------------------------------------------
// Packing
// ---------------------------------------------------------------------------------------------
// One thread per (padded row, chunk of 16 (b = 2), 8 (b = 4) or 32 (b = 3) columns) -> 1, 1 or 3
// words, written where the packed format puts them.
__global__ void pack_codes_kernel(const uint8_t* __restrict__ codes, int d_out, int d_in,
                                  int bits, int groups, int rows_pad, uint32_t* __restrict__ out) {
  const int cpg = bits == 2 ? 8 : (bits == 4 ? 16 : 4);     // chunks per 128-column group
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(rows_pad) * groups * cpg;
  if (idx >= total) return;
  const int chunk = static_cast<int>(idx % cpg);
  const int64_t rg = idx / cpg;
  const int g = static_cast<int>(rg % groups);
  const int row = static_cast<int>(rg / groups);
  const int t = row / QL_TILE, r = row % QL_TILE;
  const int width = QL_TILE / cpg;
  const int col0 = g * QL_TILE + chunk * width;
  auto code = [&](int k) -> uint32_t {
    const int col = col0 + k;
    return (row < d_out && col < d_in) ? codes[static_cast<int64_t>(row) * d_in + col] : 0u;
  };
  // word j of row r's string in blob (t, g): 8-byte piece j / 2 at 1024 (j / 2) + 8 r, word
  // j % 2 inside it
  uint32_t* blob = out + (static_cast<int64_t>(t) * groups + g) * (512 * bits);
  auto put = [&](int j, uint32_t w) { blob[(j >> 1) * 256 + 2 * r + (j & 1)] = w; };
  if (bits == 2) {
    uint32_t w = 0u;
    for (int k = 0; k < 4; ++k)
      for (int j = 0; j < 4; ++j) w |= (code(4 * k + j) & 3u) << (8 * j + 2 * k);
    put(chunk, w);
  } else if (bits == 4) {
    uint32_t w = 0u;
    for (int k = 0; k < 2; ++k)
      for (int j = 0; j < 4; ++j) w |= (code(4 * k + j) & 15u) << (8 * j + 4 * k);
    put(chunk, w);
  } else {
    uint32_t w[3] = {0u, 0u, 0u};
    for (int c = 0; c < 32; ++c) {
      const uint32_t v = code(c);
      const int cc = c & 15, k = cc >> 2, j = cc & 3;
      w[c >> 4] |= (v & 3u) << (8 * j + 2 * k);
      w[2] |= ((v >> 2) & 1u) << (8 * (c & 3) + (c >> 2));
    }
    for (int i = 0; i < 3; ++i) put(3 * chunk + i, w[i]);
  }
}

// ---------------------------------------------------------------------------------------------
// Input side: x' = V S_X^-1 x, split into the B operand
// ---------------------------------------------------------------------------------------------
struct QlInArgs {
  const void* x;
  int x_dtype;
  int64_t ld_x;
  int n_tok;           // tokens of this pass
  int d_in;
  int span;            // columns per CTA (a power of two, at least 128)
  int b_in;
  int cl;              // CTAs per Hadamard block (a thread-block cluster), b_in = cl span when > 1
  const float* s_x;
  const int8_t* sign_in;
  uint32_t flags;
  float inv_sqrt_b;
  int rows;            // B rows: 3 n_tok rounded up to 8
  int swz;             // 1: 128-byte swizzle (tensor-core operand), 0: plain rows
  uint8_t* bop;        // groups x [rows][128 bytes]: row 3 t + k = term k of token t
  float2* sums;        // groups x n_tok: (s, q0 + q1 / 128 + q2 / 128^2 summed over the group)
};

// One CTA per (span of columns, token). Hadamard blocks larger than a span are spread over a
// cluster of cl CTAs: each applies the stages of the low index bits to its own contiguous span
// (radix-16 passes: in the pass over bits [4p, 4p + 4) a thread gathers the 16 elements that
// differ only in those bits and applies four stages in registers), then, after a cluster
// barrier, combines element e of the cl spans through distributed shared memory:
// H_b = (H_cl (x) I_span)(I_cl (x) H_span), and this CTA keeps row `rank` of H_cl. At the end
// thread t (of span / 16) owns the 16 consecutive columns 16t .. 16t + 15.
__global__ void __launch_bounds__(1024) qlin_in_kernel(QlInArgs a) {
  // two buffers of span + span / 16 floats: element i at i + i / 16 (one pad per 16 elements,
  // so that the passes below are free of bank conflicts); the second takes the cluster result
  extern __shared__ float xs[];
  auto at = [](int i) { return i + (i >> 4); };
  griddep_launch_dependents();
  const int tid = threadIdx.x;
  const int nthr = blockDim.x;
  const int nwork = a.span >> 4;                // threads that own 16 columns
  const int t = blockIdx.y;
  const int j0 = blockIdx.x * a.span;
  const int len = min(a.span, a.d_in - j0);
  const bool rot = (a.flags & KRONQ_BIIP_ROTATE_IN) != 0;
  const bool scl = (a.flags & KRONQ_BIIP_SCALE_IN) != 0;
  // at most 16 elements per thread (nthr >= span / 16): all loads issued before any is used;
  // the layer's scales and signs while the preceding kernel still runs, x (which that kernel
  // may have written) after waiting for it
  {
    float xv[16], sv[16];
    int8_t sg[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const int j = tid + m * nthr;
      sv[m] = 1.f;
      sg[m] = 1;
      if (j < len) {
        if (scl) sv[m] = a.s_x[j0 + j];
        if (rot) sg[m] = a.sign_in[j0 + j];
      }
    }
    griddep_wait();
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const int j = tid + m * nthr;
      xv[m] = 0.f;
      if (j < len) {
        const int64_t o = static_cast<int64_t>(t) * a.ld_x + j0 + j;
        xv[m] = a.x_dtype == KRONQ_DTYPE_BF16
                    ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.x)[o])
                    : reinterpret_cast<const float*>(a.x)[o];
      }
    }
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const int j = tid + m * nthr;
      if (j < a.span) {
        float v = scl ? xv[m] / sv[m] : xv[m];
        xs[at(j)] = sg[m] < 0 ? -v : v;
      }
    }
  }
  __syncthreads();
  if (rot && a.b_in > 1) {
    const int L = 31 - __clz(min(a.b_in, a.span));   // stages inside this CTA's span
    int sh = 0;
    for (; sh + 4 <= L; sh += 4) {
      if (tid < nwork) {
        const int lo = tid & ((1 << sh) - 1);
        const int base = lo | ((tid >> sh) << (sh + 4));
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = xs[at(base + (j << sh))];
#pragma unroll
        for (int h = 1; h < 16; h <<= 1)
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (!(j & h)) {
              const float u = v[j], w = v[j + h];
              v[j] = u + w;
              v[j + h] = u - w;
            }
#pragma unroll
        for (int j = 0; j < 16; ++j) xs[at(base + (j << sh))] = v[j];
      }
      __syncthreads();
    }
    for (; sh < L; ++sh) {                      // remaining 1..3 stages, pairwise
      const int h = 1 << sh;
      for (int pi = tid; pi < a.span / 2; pi += nthr) {
        const int i = ((pi >> sh) << (sh + 1)) | (pi & (h - 1));
        const float u = xs[at(i)], w = xs[at(i + h)];
        xs[at(i)] = u + w;
        xs[at(i + h)] = u - w;
      }
      __syncthreads();
    }
  }
  float* xf = xs;                               // the transformed span
  if (rot && a.cl > 1) {
    float* xo = xs + a.span + a.span / 16;
    const uint32_t rank = cluster_ctarank();
    const uint32_t base = smem_u32(xs);
    cluster_sync_all();                         // every span of the block is transformed
    // all of a thread's remote loads (at most 4 elements x 8 spans) are issued before any sum
    constexpr int EPT = 4;                      // elements per thread: nthr = span / 4
    float z[EPT][8];
#pragma unroll
    for (int m = 0; m < EPT; ++m) {
      const uint32_t off = static_cast<uint32_t>(at(tid + m * nthr)) * 4u;
#pragma unroll
      for (int r2 = 0; r2 < 8; ++r2)
        z[m][r2] = r2 < a.cl ? ld_dsmem(map_shared_rank(base + off, static_cast<uint32_t>(r2)))
                             : 0.f;
    }
#pragma unroll
    for (int m = 0; m < EPT; ++m) {
      float v = 0.f;
#pragma unroll
      for (int r2 = 0; r2 < 8; ++r2)
        v += (__popc(rank & static_cast<uint32_t>(r2)) & 1) ? -z[m][r2] : z[m][r2];
      xo[at(tid + m * nthr)] = v;
    }
    cluster_sync_all();                         // no CTA leaves while another still reads it
    xf = xo;
  }
  // B operand: thread = 16 columns = one 16-byte unit of each of the token's three term rows;
  // a group's 128 columns belong to 8 consecutive threads (its maximum and sums by shuffles)
  float xv[16];
  float amax = 0.f;
  if (tid < nwork) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float v = 16 * tid + e < len ? (rot ? xf[17 * tid + e] * a.inv_sqrt_b
                                                : xf[17 * tid + e])
                                         : 0.f;
      xv[e] = v;
      amax = fmaxf(amax, fabsf(v));
    }
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  // s = the smallest power of two with 127 s >= max |x'| over the group (1 for a zero group)
  float sc = 1.f;
  if (amax > 0.f) {
    // exponent field of amax / 127, raised by one unless the mantissa is exactly 1; values
    // below the normal range are not reached by activations and round up to 2^-126
    const uint32_t bits = __float_as_uint(amax / 127.f);
    uint32_t e = bits & 0x7F800000u;
    if ((bits & 0x007FFFFFu) != 0u || e == 0u) e += 0x00800000u;
    sc = __uint_as_float(e);
  }
  const float inv_sc = 1.f / sc;                 // exact: a power of two
  int qsum[QL_TERMS] = {0, 0, 0};
  uint32_t wq[QL_TERMS][4];
  if (tid < nwork) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      float r = xv[e] * inv_sc;                   // exact; |r| <= 127
      int q[QL_TERMS];
#pragma unroll
      for (int k = 0; k < QL_TERMS; ++k) {
        q[k] = __float2int_rn(r);                 // |q0| <= 127, |q1|, |q2| <= 64
        r = (r - static_cast<float>(q[k])) * 128.f;   // exact
        qsum[k] += q[k];
      }
#pragma unroll
      for (int k = 0; k < QL_TERMS; ++k) {
        const uint32_t byte = static_cast<uint32_t>(q[k]) & 0xFFu;
        if ((e & 3) == 0) wq[k][e >> 2] = byte;
        else wq[k][e >> 2] |= byte << (8 * (e & 3));
      }
    }
    const int c0 = j0 + 16 * tid;                 // 16 columns never straddle a group
    const int g = c0 / QL_TILE, unit = (c0 % QL_TILE) >> 4;
    uint8_t* gb = a.bop + static_cast<int64_t>(g) * (128 * a.rows);
#pragma unroll
    for (int k = 0; k < QL_TERMS; ++k) {
      const int rho = QL_TERMS * t + k;
      *reinterpret_cast<uint4*>(gb + rho * 128 + ((a.swz ? unit ^ (rho & 7) : unit) << 4)) =
          make_uint4(wq[k][0], wq[k][1], wq[k][2], wq[k][3]);
    }
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1)
#pragma unroll
    for (int k = 0; k < QL_TERMS; ++k) qsum[k] += __shfl_xor_sync(0xffffffffu, qsum[k], o);
  if (tid < nwork && (tid & 7) == 0) {
    // exact integers, combined once in fp32
    const float qs = static_cast<float>(qsum[0]) + static_cast<float>(qsum[1]) * (1.f / 128.f) +
                     static_cast<float>(qsum[2]) * (1.f / 16384.f);
    a.sums[static_cast<int64_t>((j0 + 16 * tid) / QL_TILE) * a.n_tok + t] = make_float2(sc, qs);
  }
}

// ---------------------------------------------------------------------------------------------
// The tensor-core pass over the packed codes
// ---------------------------------------------------------------------------------------------
struct QlMmaArgs {
  const uint8_t* packed;
  const uint8_t* bop;
  const float2* sums;
  const float2* grid;  // packed (scale, zero): [tile][group][128] or [tile][128]
  float* partial;      // (C + T) segments x n_tok x 128
  int d_out, T, G;
  int n_tok, N;        // tokens; MMA N = 3 n_tok rounded up to 16
  int R;               // B rows in memory: 3 n_tok rounded up to 8
  int ku;              // units per pipeline stage (one bulk copy of codes, one of B)
  int grouped;         // 1: grid per row and 128-column group
  int rotate_out;
  int b_tile;          // Hadamard block inside a tile: min(b_out, 128) (1 without rotation)
  int64_t U;           // units = T G
  int stages;
  int* err;
};

__device__ __forceinline__ int64_t unit_begin(int64_t c, int64_t U, int64_t C) {
  return (c * U) / C;
}

// Dequantization of one row's half (64 columns) of a 128 x 128 blob into 16 registers of four
// 8-bit codes each (register j = columns 4j .. 4j + 3 of the half). The row's string is read as
// 8-byte pieces (piece p of row r at 1024 p + 8 r): the 32 lanes of a warp read 32 consecutive
// rows, so every read is free of bank conflicts.
template <int BITS>
__device__ __forceinline__ void dequant_half_row(const uint8_t* pk, int r, int kh,
                                                 uint32_t (&o)[16]);

template <>
__device__ __forceinline__ void dequant_half_row<2>(const uint8_t* pk, int r, int kh,
                                                    uint32_t (&o)[16]) {
  const uint2* pc = reinterpret_cast<const uint2*>(pk) + r;
  const uint2 a = pc[(2 * kh) * 128], b = pc[(2 * kh + 1) * 128];
  const uint32_t ws[4] = {a.x, a.y, b.x, b.y};            // 16 columns per word
#pragma unroll
  for (int w = 0; w < 4; ++w)
#pragma unroll
    for (int k = 0; k < 4; ++k) o[4 * w + k] = (ws[w] >> (2 * k)) & 0x03030303u;
}

template <>
__device__ __forceinline__ void dequant_half_row<4>(const uint8_t* pk, int r, int kh,
                                                    uint32_t (&o)[16]) {
  const uint2* pc = reinterpret_cast<const uint2*>(pk) + r;
#pragma unroll
  for (int p = 0; p < 4; ++p) {                            // 8 columns per word
    const uint2 a = pc[(4 * kh + p) * 128];
    o[4 * p + 0] = a.x & 0x0F0F0F0Fu;
    o[4 * p + 1] = (a.x >> 4) & 0x0F0F0F0Fu;
    o[4 * p + 2] = a.y & 0x0F0F0F0Fu;
    o[4 * p + 3] = (a.y >> 4) & 0x0F0F0F0Fu;
  }
}

template <>
__device__ __forceinline__ void dequant_half_row<3>(const uint8_t* pk, int r, int kh,
                                                    uint32_t (&o)[16]) {
  const uint2* pc = reinterpret_cast<const uint2*>(pk) + r;
  const uint2 a = pc[(3 * kh) * 128], b = pc[(3 * kh + 1) * 128], e = pc[(3 * kh + 2) * 128];
  const uint32_t ws[6] = {a.x, a.y, b.x, b.y, e.x, e.y};  // two runs of 32 columns
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    const uint32_t wh = ws[3 * m + 2];                      // top bits of the 32 columns
#pragma unroll
    for (int k8 = 0; k8 < 8; ++k8) {                         // columns 4 k8 .. 4 k8 + 3
      const uint32_t lo = (ws[3 * m + (k8 >> 2)] >> (2 * (k8 & 3))) & 0x03030303u;
      const uint32_t hi = (k8 >= 2 ? (wh >> (k8 - 2)) : (wh << (2 - k8))) & 0x04040404u;
      o[8 * m + k8] = lo | hi;
    }
  }
}

// 32 lanes x 16 consecutive 32-bit TMEM columns from registers: thread i -> lane (base + i).
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// D(tmem) (+)= A(tmem) * B(smem desc), kind::i8: A is read from tensor memory (K-major, row m
// in lane m, four 8-bit values per 32-bit column), D is int32.
__device__ __forceinline__ void umma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Tensor memory of qlin_mma_kernel (512 columns): four A tiles of 128 rows x 128 8-bit codes
// (32 columns each), then four int32 accumulators of N columns (N <= 96).
constexpr int QL_NA = 4;
constexpr int QL_NACC = 4;
constexpr uint32_t QL_A_COLS = 32;
constexpr uint32_t QL_ACC_COL0 = QL_NA * QL_A_COLS;
constexpr uint32_t QL_TMEM_COLS = 512;

// Shared memory of qlin_mma_kernel (offsets from a 1024-byte aligned base). A stage holds ku
// consecutive units: their B tiles ([R rows][128 B] each, then N rows of slack for the MMA's
// reads past the last tile's R rows) and their packed blobs, each block filled by one bulk
// copy (the blobs of consecutive units, and the B tiles of consecutive groups, are contiguous
// in global memory).
struct QlSmem {
  uint32_t stage0;
  uint32_t stage_bytes;
  uint32_t b_unit;     // B bytes per unit: 128 R
  uint32_t a_off;      // offset of the packed blobs inside a stage
  uint32_t bars;
  uint32_t xchg;       // 128 rows x 8 tokens of fp32 for the within-tile Hadamard
  uint32_t total;
};

__host__ __device__ inline QlSmem ql_smem(int bits, int N, int R, int ku, int stages) {
  QlSmem s;
  s.b_unit = 128u * static_cast<uint32_t>(R);
  s.a_off = static_cast<uint32_t>(ku) * s.b_unit + 128u * static_cast<uint32_t>(N);
  s.stage_bytes = s.a_off + static_cast<uint32_t>(ku) * 2048u * static_cast<uint32_t>(bits);
  s.stage0 = 0;
  s.bars = s.stage0 + static_cast<uint32_t>(stages) * s.stage_bytes;
  s.xchg = s.bars + 512;
  s.total = s.xchg + QL_TILE * 8 * 4 + 1024;   // + alignment slack
  return s;
}

template <int BITS, int NTC>
__global__ void __launch_bounds__(QL_THREADS, 1) qlin_mma_kernel(QlMmaArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const QlSmem L = ql_smem(BITS, p.N, p.R, p.ku, p.stages);
  const int S = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + QL_MAX_STAGES;
  // unit i uses A tile and accumulator i % 4: afull (dequantization done), mdone (its MMAs
  // done: the A tile is free and the accumulator full), accempty (the epilogue drained it)
  uint64_t* afull = empty + QL_MAX_STAGES;      // QL_NA
  uint64_t* mdone = afull + QL_NA;              // QL_NA
  uint64_t* accfull = mdone;                    // the same barrier, seen by the epilogue
  uint64_t* accempty = mdone + QL_NA;           // QL_NACC
  static_assert(QL_NA == 4 && QL_NACC == 4, "unit i uses slot i & 3 of both rings");
  volatile int* abort_flag = reinterpret_cast<volatile int*>(accempty + QL_NACC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accempty + QL_NACC) + 1;
  float* xchg = reinterpret_cast<float*>(smem + L.xchg);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t C = gridDim.x;
  const int64_t u0 = unit_begin(blockIdx.x, p.U, C);
  const int64_t u1 = unit_begin(blockIdx.x + 1, p.U, C);
  const int n_units = static_cast<int>(u1 - u0);
  const int ku = p.ku;
  const int n_stages = (n_units + ku - 1) / ku;
  const int g0 = static_cast<int>(u0 % p.G);     // group of the first unit
  const uint32_t pk_bytes = 2048u * BITS;
  auto stage_ptr = [&](int s) { return smem + L.stage0 + s * L.stage_bytes; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < QL_NA; ++i) {
      mbar_init(&afull[i], QL_DQ_THREADS / 32);
      mbar_init(&mdone[i], 1);
    }
    for (int i = 0; i < QL_NACC; ++i) {
      mbar_init(&accempty[i], 4);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, QL_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;


  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      const int pre = min(S, n_stages);
      bool ok = true;
      // the packed codes do not depend on the preceding kernel: start them before waiting
      for (int si = 0; si < pre; ++si) {
        const int i0 = si * ku, nu = min(ku, n_units - i0);
        mbar_arrive_expect_tx(&full[si], nu * (pk_bytes + L.b_unit));
        bulk_load(stage_ptr(si) + L.a_off, p.packed + (u0 + i0) * static_cast<int64_t>(pk_bytes),
                  nu * pk_bytes, &full[si]);
      }
      griddep_wait();
      int si = 0, g = g0, s = 0;
      uint32_t ph = 0;
      for (; si < n_stages && ok; ++si, s = (s + 1 == S) ? 0 : s + 1, ph ^= (s == 0)) {
        const int i0 = si * ku, nu = min(ku, n_units - i0);
        uint8_t* st = stage_ptr(s);
        if (si >= pre) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.err, DEV_ERR_TMA_WAIT)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], nu * (pk_bytes + L.b_unit));
          bulk_load(st + L.a_off, p.packed + (u0 + i0) * static_cast<int64_t>(pk_bytes),
                    nu * pk_bytes, &full[s]);
        }
        // B tiles of groups g .. g + nu - 1 (mod G): one copy per contiguous run
        for (int done = 0; done < nu;) {
          const int run = min(nu - done, p.G - g);
          bulk_load(st + done * L.b_unit, p.bop + static_cast<int64_t>(g) * L.b_unit,
                    run * L.b_unit, &full[s]);
          done += run;
          g += run;
          if (g == p.G) g = 0;
        }
      }
      if (!ok) {
        // copies already issued complete on their barriers before the CTA leaves
        for (int j = max(0, si - S); j < si; ++j)
          mbar_drain(&full[j % S], (j / S) & 1u, 1000000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = ql_idesc(128, p.N);
      // descriptor of a stage's first B tile; a tile k and a K step kk add (k b_unit + 32 kk)
      // bytes, i.e. (k b_unit + 32 kk) / 16 in the descriptor's address field
      const uint64_t bdesc0 = smem_desc_sw128(smem_u32(stage_ptr(0)), 16, 1024);
      const uint32_t stage_step = L.stage_bytes >> 4, unit_step = L.b_unit >> 4;
      int k = 0, s = 0;
      uint32_t ph = 0;
      uint64_t bstage = bdesc0;
      // one accumulator per unit (the scale of x' changes from group to group)
      for (int i = 0; i < n_units; ++i) {
        const int b = i & 3;
        const uint32_t bph = (i >> 2) & 1u;
        if (k == 0 && !mbar_wait(&full[s], ph, abort_flag, p.err, DEV_ERR_MMA_WAIT)) break;
        if (!mbar_wait(&afull[b], bph, abort_flag, p.err, DEV_ERR_MMA_WAIT)) break;
        if (!mbar_wait(&accempty[b], bph ^ 1u, abort_flag, p.err, DEV_ERR_MMA_WAIT)) break;
        tc_fence_after();
        const uint32_t a_tmem = tmem_base + b * QL_A_COLS;
        const uint32_t d_tmem = tmem_base + QL_ACC_COL0 + b * p.N;
        const uint64_t bd = bstage + k * unit_step;
        // K = 128 in four steps of 32 8-bit values (32 bytes of each A and B row)
        umma_i8_ts(d_tmem, a_tmem, bd, idesc, 0u);
        umma_i8_ts(d_tmem, a_tmem + 8, bd + 2, idesc, 1u);
        umma_i8_ts(d_tmem, a_tmem + 16, bd + 4, idesc, 1u);
        umma_i8_ts(d_tmem, a_tmem + 24, bd + 6, idesc, 1u);
        umma_commit(&mdone[b]);
        if (++k == ku || i == n_units - 1) {
          umma_commit(&empty[s]);          // the stage's codes and B tiles are consumed
          k = 0;
          if (++s == S) {
            s = 0;
            ph ^= 1u;
            bstage = bdesc0;
          } else {
            bstage += stage_step;
          }
        }
      }
    }
  } else if (warp >= QL_DQ_WARP0) {
    // ------------------------------------------------------------------ dequantization
    // warp w writes TMEM lanes 32 (w % 4) .. + 31 (its rows) for column half (w - 8) / 4
    const int q = warp & 3, kh = (warp - QL_DQ_WARP0) >> 2;
    const int r = q * 32 + lane;
    int k = 0, s = 0;
    uint32_t ph = 0;
    for (int i = 0; i < n_units; ++i) {
      const int ab = i & 3;
      const uint32_t aph = (i >> 2) & 1u;
      int ok = 1;
      if (lane == 0) {
        ok = (k != 0 || mbar_wait(&full[s], ph, abort_flag, p.err, DEV_ERR_MMA_WAIT)) &&
             mbar_wait(&mdone[ab], aph ^ 1u, abort_flag, p.err, DEV_ERR_MMA_WAIT);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      uint32_t o[16];
      dequant_half_row<BITS>(stage_ptr(s) + L.a_off + k * pk_bytes, r, kh, o);
      tmem_st_32x32b_x16(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ab * QL_A_COLS +
                             kh * 16,
                         o);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[ab]);
      if (++k == ku) {
        k = 0;
        if (++s == S) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
  } else if (warp >= QL_EPI_WARP0) {
    // ------------------------------------------------------------------ epilogue
    griddep_wait();                                   // the group sums come from qlin_in
    const int q = warp & 3;
    const int r = q * 32 + lane;                      // row inside the tile = TMEM lane
    float yacc[NTC];
#pragma unroll
    for (int k = 0; k < NTC; ++k) yacc[k] = 0.f;
    int g = g0;
    int tile = static_cast<int>(u0 / p.G);
    for (int i = 0; i < n_units; ++i) {
      const int gcur = g;
      const int tcur = tile;
      if (++g == p.G) {
        g = 0;
        ++tile;
      }
      // lane k holds token k's (s, sum of its terms) for this group; and this row's grid; both
      // loaded before waiting so that their latency overlaps the MMAs
      float sl = 0.f, ql = 0.f;
      if (lane < p.n_tok) {
        const float2 s2 = __ldg(&p.sums[static_cast<int64_t>(gcur) * p.n_tok + lane]);
        sl = s2.x;
        ql = s2.y;
      }
      const float2 gz = __ldg(&p.grid[p.grouped
                                          ? (static_cast<int64_t>(tcur) * p.G + gcur) * QL_TILE + r
                                          : static_cast<int64_t>(tcur) * QL_TILE + r]);
      const int acc = i & 3;
      const uint32_t cph = (i >> 2) & 1u;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&accfull[acc], cph, abort_flag, p.err, DEV_ERR_EPI_WAIT);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      // the four epilogue warps leave together (they meet at named barriers below)
      if (!bar_and(2, 128, ok != 0)) break;
      tc_fence_after();
      const float sc = gz.x, z = gz.y;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + QL_ACC_COL0 +
                             acc * p.N;
      // tokens in runs of 16 (48 int32 columns = three loads of 16)
#pragma unroll
      for (int t0 = 0; t0 < NTC; t0 += 16) {
        float f[48];
#pragma unroll
        for (int cb = 0; cb < 3; ++cb) {
          if (3 * t0 + 16 * cb < p.N) {
            uint32_t w[16];
            tmem_ld_32x32b_x16(taddr + 3 * t0 + 16 * cb, w);
            tmem_ld_wait();
            // |value| < 2^22: exact through the 1.5 * 2^23 bias
#pragma unroll
            for (int j = 0; j < 16; ++j)
              f[16 * cb + j] = __int_as_float(static_cast<int>(w[j]) + 0x4B400000) - 12582912.f;
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) f[16 * cb + j] = 0.f;
          }
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int tt = t0 + k;
          if (tt < NTC) {
            const float st = __shfl_sync(0xffffffffu, sl, tt);
            const float qt = __shfl_sync(0xffffffffu, ql, tt);
            if (tt < p.n_tok) {
              // sum_j c_j x'_j / s = t0 + t1 / 128 + t2 / 128^2 (exact int32 products)
              const float a = f[3 * k] + f[3 * k + 1] * (1.f / 128.f) +
                              f[3 * k + 2] * (1.f / 16384.f);
              yacc[tt] = fmaf(sc * st, fmaf(-z, qt, a), yacc[tt]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[acc]);
      // end of this CTA's part of the tile: within-tile Hadamard, then one partial
      if (i == n_units - 1 || gcur == p.G - 1) {
        if (p.rotate_out) {
#pragma unroll
          for (int h = 1; h < 32; h <<= 1) {
            if (h >= p.b_tile) break;
#pragma unroll
            for (int k = 0; k < NTC; ++k) {
              const float o = __shfl_xor_sync(0xffffffffu, yacc[k], h);
              yacc[k] = (lane & h) ? (o - yacc[k]) : (yacc[k] + o);
            }
          }
          for (int h = 32; h < p.b_tile; h <<= 1) {
#pragma unroll
            for (int k0 = 0; k0 < NTC; k0 += 8) {
              named_bar_sync(1, 128);
#pragma unroll
              for (int k = 0; k < 8; ++k)
                if (k0 + k < NTC) xchg[k * QL_TILE + r] = yacc[k0 + k];
              named_bar_sync(1, 128);
#pragma unroll
              for (int k = 0; k < 8; ++k)
                if (k0 + k < NTC) {
                  const float o = xchg[k * QL_TILE + (r ^ h)];
                  yacc[k0 + k] = (r & h) ? (o - yacc[k0 + k]) : (yacc[k0 + k] + o);
                }
            }
          }
        }
        const int64_t seg = blockIdx.x + tcur;
        float* out = p.partial + seg * p.n_tok * QL_TILE + r;
#pragma unroll
        for (int k = 0; k < NTC; ++k) {
          if (k < p.n_tok) out[k * QL_TILE] = yacc[k];
          yacc[k] = 0.f;
        }
      }
    }
  }

  griddep_launch_dependents();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, QL_TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------------
// Decode on the CUDA cores (1 or 2 tokens)
// ---------------------------------------------------------------------------------------------
// A tensor-core MMA costs the same for any N <= 256 and covers 128 rows x 32 bytes of the code
// matrix, which caps the tensor-core pass near 22 codes per cycle per SM. For a few tokens the
// CUDA cores do better: one thread per row and unit, codes masked in place (no shifts: a code in
// bit pair k of a byte is 4^k c, and each k keeps its own accumulator), and dp4a with the three
// int8 terms of x' (exact int32 sums, as on the tensor cores).
struct QlDpArgs {
  const uint8_t* packed;
  const uint8_t* bop;      // groups x [rows][128 bytes], plain rows, row 3 t + k = term k
  const float2* sums;      // groups x n_tok: (s, sum of the three terms)
  const float2* grid;
  float* partial;          // (C + T) segments x n_tok x 128
  int d_out, G, n_tok, rows;
  int grouped, rotate_out, b_tile;
  int stages;              // ring stages (<= QL_DP_MAX_STAGES)
  int64_t U;
  int* err;
};

__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// exact int -> float for |v| < 2^22
__device__ __forceinline__ float i2f_small(int v) {
  return __int_as_float(v + 0x4B400000) - 12582912.f;
}

template <int BITS>
struct DpCodes {
  static constexpr int PIECES = 2 * BITS;   // 8-byte pieces per row and unit
  uint2 p[PIECES];
};

__device__ __forceinline__ uint2 lds_u2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint4 lds_u4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// acc[term][part] += codes . x' terms over the unit's 128 columns; the parts carry the codes'
// bit-position factors (2 bits: 4^k, 4 bits: 16^k, 3 bits: 1)
template <int BITS, int NT>
__device__ __forceinline__ void dp_unit(const DpCodes<BITS>& c, uint32_t xg, int n_tok,
                                        int (&acc)[NT][QL_TERMS][4]) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(c.p);
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int k = 0; k < QL_TERMS; ++k)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[t][k][j] = 0;
  // 16 columns per step: the step's codes are masked once and used for every token and term
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint32_t cm[4];                               // four 4-column code words of the step
    if (BITS == 2) {
      // word q: columns 16q + 4k + j at bits 8j + 2k (code scaled by 4^k)
#pragma unroll
      for (int k = 0; k < 4; ++k) cm[k] = w[q] & (0x03030303u << (2 * k));
    } else if (BITS == 4) {
      // words 2q, 2q + 1: columns 8w + 4k + j at bits 8j + 4k (code scaled by 16^k)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        cm[2 * h] = w[2 * q + h] & 0x0F0F0F0Fu;
        cm[2 * h + 1] = w[2 * q + h] & 0xF0F0F0F0u;
      }
    } else {
      // 32 columns per three words: low bits in words 3m, 3m + 1, top bits in word 3m + 2
      const int m = q >> 1, half = q & 1;
      const uint32_t wl = w[3 * m + half], wh = w[3 * m + 2];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int k8 = 4 * half + k;
        const uint32_t lo = (wl >> (2 * k)) & 0x03030303u;
        const uint32_t hi = (k8 >= 2 ? (wh >> (k8 - 2)) : (wh << (2 - k8))) & 0x04040404u;
        cm[k] = lo | hi;
      }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      // a run-time bound for two tokens keeps their loads apart (no spills); none for one
      if (NT > 1 && t >= n_tok) break;
#pragma unroll
      for (int term = 0; term < QL_TERMS; ++term) {
        const uint4 xv = lds_u4(xg + (3 * t + term) * 128 + 16 * q);
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};   // columns 16q + 4k .. + 3
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          // part: 2 bits -> k (factor 4^k); 4 bits -> k & 1 (factor 16^(k & 1)); 3 bits -> 0
          const int part = BITS == 2 ? k : (BITS == 4 ? (k & 1) : 0);
          acc[t][term][part] = dp4a_us(cm[k], xw[k], acc[t][term][part]);
        }
      }
    }
  }
}

// Shared-memory layout of the decode kernel: the x' terms of the groups the CTA visits (3 n_tok
// rows of 128 bytes each), their (s, sum) pairs, then a ring of stages, each one unit's packed
// codes (2048 b bytes) and its 128 grid pairs, filled by bulk copies; the stages' full and
// empty barriers and the abort flag come last.
struct DpSmem {
  int x, sums, ring, stage, bars, total;
};
__host__ __device__ inline DpSmem dp_smem(int bits, int ng, int n_tok, int stages) {
  DpSmem L;
  L.x = 0;
  L.sums = ng * 384 * n_tok;
  L.ring = (L.sums + ng * n_tok * 8 + 127) / 128 * 128;
  L.stage = 2048 * bits + QL_TILE * 8;
  L.bars = L.ring + stages * L.stage;
  L.total = L.bars + 2 * QL_DP_MAX_STAGES * 8 + 16;
  return L;
}

// Four consumer warps (one thread per row of the 128-row unit) and one producer warp, whose
// first lane streams the CTA's units into the ring with bulk copies; the codes therefore need
// no registers while in flight, and the copies run as far ahead as the ring is deep.
template <int BITS, int NT>
__global__ void __launch_bounds__(QL_DP_THREADS, QL_DP_CTAS_PER_SM) qlin_dp4a_kernel(QlDpArgs p) {
  __shared__ float ys[NT][QL_TILE];
  extern __shared__ __align__(128) uint8_t dsm[];
  const int tid = threadIdx.x;
  const int r = tid;                                  // row of the tile (consumer threads)
  const int lane = tid & 31, warp = tid >> 5;
  const int64_t C = gridDim.x;
  const int64_t u0 = unit_begin(blockIdx.x, p.U, C);
  const int64_t u1 = unit_begin(blockIdx.x + 1, p.U, C);
  const int n_units = static_cast<int>(u1 - u0);
  const bool all_groups = n_units >= p.G;
  const int ng = all_groups ? p.G : n_units;
  const int S = p.stages;
  const DpSmem L = dp_smem(BITS, ng, p.n_tok, S);
  uint8_t* xstage = dsm + L.x;                        // group i: 3 n_tok rows of 128 bytes
  float2* sstage = reinterpret_cast<float2*>(dsm + L.sums);
  uint64_t* full = reinterpret_cast<uint64_t*>(dsm + L.bars);
  uint64_t* empty = full + QL_DP_MAX_STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + QL_DP_MAX_STAGES);
  const uint32_t pk = 2048u * BITS;
  auto stage_ptr = [&](int s) { return dsm + L.ring + s * L.stage; };
  auto grid_src = [&](int64_t u) {
    return p.grid + (p.grouped ? u * QL_TILE : (u / p.G) * QL_TILE);
  };
  auto issue = [&](int i, int s) {
    mbar_arrive_expect_tx(&full[s], pk + QL_TILE * 8);
    bulk_load(stage_ptr(s), p.packed + (u0 + i) * static_cast<int64_t>(pk), pk, &full[s]);
    bulk_load(stage_ptr(s) + pk, grid_src(u0 + i), QL_TILE * 8, &full[s]);
  };

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], QL_TILE / 32);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const bool producer = warp == QL_TILE / 32;
  // the packed codes and the grid do not depend on the preceding kernel: start them first
  const int pre = min(S, n_units);
  if (producer && lane == 0)
    for (int i = 0; i < pre; ++i) issue(i, i);
  griddep_wait();                                     // x' and its sums come from qlin_in
  {
    // x' terms of the groups this CTA visits: groups g0 .. g0 + ng - 1 (mod G) in visiting
    // order, or all G groups at their own index when the CTA visits every group; the scale
    // s carries 4^-(parts - 1) and the sum 4^(parts - 1), the factor of the combined parts
    const int gstart = all_groups ? 0 : static_cast<int>(u0 % p.G);
    const int tr = 3 * p.n_tok;                       // term rows per group
    const int words = ng * tr * 8;                    // 16-byte words
    for (int w = tid; w < words; w += blockDim.x) {
      const int gi = w / (tr * 8), off = w % (tr * 8);
      int gsrc = gstart + gi;
      if (gsrc >= p.G) gsrc -= p.G;
      reinterpret_cast<uint4*>(xstage)[w] = __ldg(
          reinterpret_cast<const uint4*>(p.bop + static_cast<int64_t>(gsrc) * 128 * p.rows) + off);
    }
    constexpr float kPart = BITS == 2 ? 64.f : (BITS == 4 ? 16.f : 1.f);
    for (int w = tid; w < ng * p.n_tok; w += blockDim.x) {
      int gsrc = gstart + w / p.n_tok;
      if (gsrc >= p.G) gsrc -= p.G;
      const float2 v = __ldg(&p.sums[static_cast<int64_t>(gsrc) * p.n_tok + w % p.n_tok]);
      sstage[w] = make_float2(v.x * (1.f / kPart), v.y * kPart);
    }
    __syncthreads();
  }

  if (producer) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      // unit i >= S refills stage i % S once the consumers released unit i - S: the empty
      // barrier's completion number i / S - 1, parity (i / S - 1) & 1
      int i = pre, s = 0;
      uint32_t eph = 0;
      for (; i < n_units; ++i) {
        if (!mbar_wait(&empty[s], eph, abort_flag, p.err, DEV_ERR_TMA_WAIT)) break;
        issue(i, s);
        if (++s == S) {
          s = 0;
          eph ^= 1u;
        }
      }
      if (i < n_units) {
        // copies already issued complete on their barriers before the CTA leaves
        for (int j = max(0, i - S); j < i; ++j)
          mbar_drain(&full[j % S], (j / S) & 1u, 1000000000ull);
      }
    }
  } else {
    // ------------------------------------------------------------------ consumers
    // Every consumer runs every unit, also after an abort (then on whatever the stage holds),
    // so that the named barriers of the within-tile Hadamard are always reached by all 128.
    float y[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) y[t] = 0.f;
    int g = static_cast<int>(u0 % p.G);
    int tile = static_cast<int>(u0 / p.G);
    // the kernel is instantiated for the call's token count: NT == p.n_tok
    constexpr int xb = 384 * NT;                     // staged bytes per group
    const uint32_t xs0 = smem_u32(xstage);
    const uint32_t ring_row = smem_u32(stage_ptr(0)) + 8 * r;   // this row's piece 0, stage 0
    int s = 0;                                       // stage of unit i, and its fill parity
    uint32_t ph = 0;
    for (int i = 0; i < n_units; ++i) {
      mbar_wait(&full[s], ph, abort_flag, p.err, DEV_ERR_LOAD_WAIT);
      DpCodes<BITS> cb;
      const uint32_t st = ring_row + s * L.stage;
#pragma unroll
      for (int k = 0; k < DpCodes<BITS>::PIECES; ++k) cb.p[k] = lds_u2(st + 1024 * k);
      const uint2 gzu = lds_u2(st + pk);             // (scale, zero) of this row
      const float2 gz = make_float2(__uint_as_float(gzu.x), __uint_as_float(gzu.y));
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++s == S) {
        s = 0;
        ph ^= 1u;
      }
      const int row = tile * QL_TILE + r;
      const int si = all_groups ? g : i;              // staged group index
      int acc[NT][QL_TERMS][4];
      dp_unit<BITS, NT>(cb, xs0 + si * xb, p.n_tok, acc);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        if (NT > 1 && t >= p.n_tok) break;
        const float2 sq = sstage[si * NT + t];
        float a[QL_TERMS];
#pragma unroll
        for (int term = 0; term < QL_TERMS; ++term) {
          // the parts combined at the factor of the highest one (exact: |v| < 2^22)
          int v = acc[t][term][0];
          if (BITS == 2)
            v = (v << 6) + (acc[t][term][1] << 4) + (acc[t][term][2] << 2) + acc[t][term][3];
          else if (BITS == 4)
            v = (v << 4) + acc[t][term][1];
          a[term] = i2f_small(v);
        }
        const float dot = a[0] + a[1] * (1.f / 128.f) + a[2] * (1.f / 16384.f);
        if (row < p.d_out) y[t] = fmaf(gz.x * sq.x, fmaf(-gz.y, sq.y, dot), y[t]);
      }
      // end of this CTA's part of the tile: within-tile Hadamard, then one partial
      const bool seg_end = (i == n_units - 1) || (g == p.G - 1);
      if (seg_end) {
        if (p.rotate_out) {
#pragma unroll
          for (int h = 1; h < 32; h <<= 1) {
            if (h >= p.b_tile) break;
#pragma unroll
            for (int t = 0; t < NT; ++t) {
              const float o = __shfl_xor_sync(0xffffffffu, y[t], h);
              y[t] = (lane & h) ? (o - y[t]) : (y[t] + o);
            }
          }
          for (int h = 32; h < p.b_tile; h <<= 1) {
            named_bar_sync(1, QL_TILE);
#pragma unroll
            for (int t = 0; t < NT; ++t) ys[t][r] = y[t];
            named_bar_sync(1, QL_TILE);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
              const float o = ys[t][r ^ h];
              y[t] = (r & h) ? (o - y[t]) : (y[t] + o);
            }
          }
        }
        float* out = p.partial + (static_cast<int64_t>(blockIdx.x) + tile) * NT * QL_TILE + r;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          out[t * QL_TILE] = y[t];
          y[t] = 0.f;
        }
      }
      if (++g == p.G) {
        g = 0;
        ++tile;
      }
    }
  }
  griddep_launch_dependents();
  __syncthreads();
}

// ---------------------------------------------------------------------------------------------
// Output side: sum of partials, across-tile Hadamard, signs, S_G^-1
// ---------------------------------------------------------------------------------------------
struct QlOutArgs {
  const float* partial;
  int n_tok, T, G;
  int64_t U, C;
  int qb;              // tiles per output Hadamard block (1 when b_out <= 128 or no rotation)
  int tpe;             // threads per output element in the partial-sum gather (power of two)
  int d_out;
  const float* s_g;
  const int8_t* sign_out;
  uint32_t flags;
  float inv_sqrt_b;
  float* y;
  int64_t ld_y;
};

// CTA that owns unit u under the split c -> [floor(c U / C), floor((c + 1) U / C)): the
// smallest c with floor((c + 1) U / C) > u, i.e. (c + 1) U >= (u + 1) C.
__device__ __forceinline__ int64_t cta_of_unit(int64_t u, int64_t U, int64_t C) {
  return ((u + 1) * C - 1) / U;
}

// One CTA per (token, output Hadamard block, 16-row slice of the tiles): thread e handles row
// (e mod 16) of the slice in tile e / 16 of the block.
__global__ void __launch_bounds__(1024) qlin_out_kernel(QlOutArgs a) {
  extern __shared__ float ys[];                   // qb x 16, then qb x 2 CTA bounds
  int* cbound = reinterpret_cast<int*>(ys + a.qb * 16);
  const int slice = blockIdx.x & 7;
  const int sb = blockIdx.x >> 3;
  const int tok = blockIdx.y;
  griddep_launch_dependents();
  for (int qi = threadIdx.x; qi < a.qb; qi += blockDim.x) {
    const int64_t tile = static_cast<int64_t>(sb) * a.qb + qi;
    cbound[2 * qi] = static_cast<int>(cta_of_unit(tile * a.G, a.U, a.C));
    cbound[2 * qi + 1] = static_cast<int>(cta_of_unit(tile * a.G + a.G - 1, a.U, a.C));
  }
  // output scale of this thread's first row (most CTAs give one row per thread), read while
  // the preceding kernel still runs
  const bool rot = (a.flags & KRONQ_BIIP_ROTATE_OUT) != 0;
  float oscale = 1.f;
  {
    const int e = threadIdx.x;
    const int64_t i = static_cast<int64_t>(sb * a.qb + (e >> 4)) * QL_TILE + slice * 16 + (e & 15);
    if (e < a.qb * 16 && i < a.d_out) {
      if (rot) oscale = a.sign_out[i] < 0 ? -a.inv_sqrt_b : a.inv_sqrt_b;
      if (a.flags & KRONQ_BIIP_SCALE_OUT) oscale = oscale / a.s_g[i];
    }
  }
  griddep_wait();
  __syncthreads();
  const int n = a.qb * 16;
  // a.tpe consecutive threads share an element: each sums every tpe-th of its segments, with
  // four loads in flight, then the tpe sums are combined by shuffles in a fixed order
  const int tpe = a.tpe;
  const int epw = 32 / tpe;                     // elements per warp and step
  const int wid = threadIdx.x >> 5, lid = threadIdx.x & 31;
  for (int base = wid * epw; base < n; base += (blockDim.x >> 5) * epw) {   // warp-uniform
    const int e0 = base + lid / tpe, sub = lid % tpe;
    float tot = 0.f;
    if (e0 < n) {
      const int qi = e0 >> 4, r = slice * 16 + (e0 & 15);
      const int64_t tile = static_cast<int64_t>(sb) * a.qb + qi;
      const int c0 = cbound[2 * qi], c1 = cbound[2 * qi + 1];
      const int64_t seg = static_cast<int64_t>(a.n_tok) * QL_TILE;      // next segment
      const float* ps = a.partial + ((c0 + tile) * a.n_tok + tok) * QL_TILE + r + sub * seg;
      const int64_t step = seg * tpe;                                     // next own segment
      const int cnt = c1 - c0 + 1;
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      int k = sub;
      for (; k + 3 * tpe < cnt; k += 4 * tpe, ps += 4 * step) {
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] += ps[j * step];
      }
      for (int j = 0; k < cnt; k += tpe, ++j, ps += step) v[j & 3] += *ps;
      tot = (v[0] + v[1]) + (v[2] + v[3]);
    }
    for (int o = 1; o < tpe; o <<= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    if (e0 < n && sub == 0) ys[e0] = tot;
  }
  __syncthreads();
  if (rot && a.qb > 1) {
    for (int sh = 0; (1 << sh) < a.qb; ++sh) {
      const int h = 1 << sh;
      for (int pidx = threadIdx.x; pidx < n / 2; pidx += blockDim.x) {
        // pairs of tiles (qi, qi + h) with bit sh of qi clear, same row
        const int r = pidx & 15, pq = pidx >> 4;
        const int qi = ((pq >> sh) << (sh + 1)) | (pq & (h - 1));
        const float u = ys[qi * 16 + r], w = ys[(qi + h) * 16 + r];
        ys[qi * 16 + r] = u + w;
        ys[(qi + h) * 16 + r] = u - w;
      }
      __syncthreads();
    }
  }
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const int qi = e >> 4, r = slice * 16 + (e & 15);
    const int64_t i = static_cast<int64_t>(sb * a.qb + qi) * QL_TILE + r;
    if (i >= a.d_out) continue;
    float os = oscale;
    if (e != threadIdx.x) {                     // rows past the first: scale read now
      os = 1.f;
      if (rot) os = a.sign_out[i] < 0 ? -a.inv_sqrt_b : a.inv_sqrt_b;
      if (a.flags & KRONQ_BIIP_SCALE_OUT) os = os / a.s_g[i];
    }
    a.y[tok * a.ld_y + i] = ys[e] * os;
  }
}

// (scale, zero) pairs in the order the epilogue reads them: per tile, per group (group-wise
// grid) or once (per-row grid), 128 rows; rows past d_out get (0, 0).
__global__ void pack_grid_kernel(const float* __restrict__ scale, const float* __restrict__ zero,
                                 int d_out, int groups, int rows_pad, float2* __restrict__ out) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(rows_pad) * groups;
  if (idx >= total) return;
  const int r = static_cast<int>(idx % QL_TILE);
  const int64_t tg = idx / QL_TILE;               // tile * groups + g
  const int g = static_cast<int>(tg % groups);
  const int t = static_cast<int>(tg / groups);
  const int row = t * QL_TILE + r;
  float2 v = make_float2(0.f, 0.f);
  if (row < d_out) {
    const int64_t src = static_cast<int64_t>(row) * groups + g;
    v = make_float2(scale[src], zero[src]);
  }
  out[idx] = v;
}

template <typename Kern, typename Arg>
kronq_status launch_pdl(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                        bool pdl, const char* what, Arg arg, int cluster = 1) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (cluster > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, arg);
  if (e != cudaSuccess) return fail(KRONQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return check_launch(what);
}

int pow2_factor(int d) { return d & (-d); }

constexpr int QL_DP_MAX_TOK = 2;   // up to this many tokens: the CUDA-core decode kernel
constexpr int QL_DP_MAX_UNITS = 48;   // units per CTA (its x' groups are staged in shared memory)

struct QlGeom {
  int T, G, C;
  int64_t U;
  int span;
  size_t bop_bytes, sums_bytes, partial_bytes;
};

QlGeom ql_geom(int d_out, int d_in, int n_tok_pass) {
  QlGeom g;
  g.T = (d_out + QL_TILE - 1) / QL_TILE;
  g.G = (d_in + QL_TILE - 1) / QL_TILE;
  g.U = static_cast<int64_t>(g.T) * g.G;
  // CTAs (one partial per CTA and tile): one per SM for the tensor-core pass, several per SM
  // for the CUDA-core decode kernel
  const bool decode = n_tok_pass <= QL_DP_MAX_TOK;
  const int per_sm = decode ? QL_DP_CTAS_PER_SM : 1;
  g.C = static_cast<int>(std::min<int64_t>(g.U, static_cast<int64_t>(per_sm) * sm_budget()));
  if (decode) {
    // at most QL_DP_MAX_UNITS units (and staged groups) per CTA
    g.C = static_cast<int>(std::max<int64_t>(g.C, (g.U + QL_DP_MAX_UNITS - 1) / QL_DP_MAX_UNITS));
  }
  g.span = std::max(pow2_factor(d_in), QL_TILE);
  g.bop_bytes = align256(static_cast<size_t>(g.G) * 128 * ((3 * n_tok_pass + 7) / 8 * 8));
  g.sums_bytes = align256(static_cast<size_t>(g.G) * n_tok_pass * sizeof(float2));
  g.partial_bytes =
      align256(static_cast<size_t>(g.C + g.T) * n_tok_pass * QL_TILE * sizeof(float));
  return g;
}

template <int BITS, int NTC>
kronq_status launch_mma_t(const QlMmaArgs& p, int C, size_t smem, cudaStream_t stream) {
  auto kern = qlin_mma_kernel<BITS, NTC>;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
  if (e != cudaSuccess) return fail(KRONQ_ERR_CUDA, "qlin_mma smem: %s", cudaGetErrorString(e));
  return launch_pdl(kern, dim3(C), dim3(QL_THREADS), smem, stream, true, "qlin_mma_kernel", p);
}

template <int BITS, int NT>
kronq_status launch_dp_t(const QlDpArgs& p, int C, size_t smem, cudaStream_t stream) {
  auto kern = qlin_dp4a_kernel<BITS, NT>;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
  if (e != cudaSuccess) return fail(KRONQ_ERR_CUDA, "qlin_dp4a smem: %s", cudaGetErrorString(e));
  return launch_pdl(kern, dim3(C), dim3(QL_DP_THREADS), smem, stream, true, "qlin_dp4a_kernel", p);
}

kronq_status launch_dp(int bits, int nt, const QlDpArgs& p, int C, size_t smem,
                       cudaStream_t stream) {
  if (nt != 1 && nt != 2) return fail(KRONQ_ERR_INVALID_ARG, "decode kernel: 1 or 2 tokens");
  if (bits == 2)
    return nt <= 1 ? launch_dp_t<2, 1>(p, C, smem, stream) : launch_dp_t<2, 2>(p, C, smem, stream);
  if (bits == 3)
    return nt <= 1 ? launch_dp_t<3, 1>(p, C, smem, stream) : launch_dp_t<3, 2>(p, C, smem, stream);
  return nt <= 1 ? launch_dp_t<4, 1>(p, C, smem, stream) : launch_dp_t<4, 2>(p, C, smem, stream);
}

kronq_status launch_mma(int bits, int ntc, const QlMmaArgs& p, int C, size_t smem,
                        cudaStream_t stream) {
  if (bits == 2) return ntc <= 8 ? launch_mma_t<2, 8>(p, C, smem, stream)
                                 : launch_mma_t<2, 32>(p, C, smem, stream);
  if (bits == 3) return ntc <= 8 ? launch_mma_t<3, 8>(p, C, smem, stream)
                                 : launch_mma_t<3, 32>(p, C, smem, stream);
  return ntc <= 8 ? launch_mma_t<4, 8>(p, C, smem, stream)
                  : launch_mma_t<4, 32>(p, C, smem, stream);
}

}  // namespace

size_t packed_code_bytes(int d_out, int d_in, int bits) {
  const size_t t = (d_out + QL_TILE - 1) / QL_TILE, g = (d_in + QL_TILE - 1) / QL_TILE;
  return t * g * 2048 * static_cast<size_t>(bits);
}

kronq_status run_pack_codes(const uint8_t* codes, int d_out, int d_in, int bits, void* packed,
                            cudaStream_t stream) {
  const int groups = (d_in + QL_TILE - 1) / QL_TILE;
  const int rows_pad = (d_out + QL_TILE - 1) / QL_TILE * QL_TILE;
  const int cpg = bits == 2 ? 8 : (bits == 4 ? 16 : 4);   // words-chunks per group row
  const int64_t total = static_cast<int64_t>(rows_pad) * groups * cpg;
  const int threads = 256;
  pack_codes_kernel<<<static_cast<unsigned>((total + threads - 1) / threads), threads, 0,
                      stream>>>(codes, d_out, d_in, bits, groups, rows_pad,
                                static_cast<uint32_t*>(packed));
  return check_launch("pack_codes_kernel");
}

size_t packed_grid_bytes(int d_out, int d_in, int group) {
  const size_t t = (d_out + QL_TILE - 1) / QL_TILE;
  const size_t g = group ? (d_in + QL_TILE - 1) / QL_TILE : 1;
  return t * g * QL_TILE * sizeof(float2);
}

kronq_status run_pack_grid(const float* scale, const float* zero, int d_out, int d_in, int group,
                           void* packed, cudaStream_t stream) {
  const int groups = group ? (d_in + QL_TILE - 1) / QL_TILE : 1;
  const int rows_pad = (d_out + QL_TILE - 1) / QL_TILE * QL_TILE;
  const int64_t total = static_cast<int64_t>(rows_pad) * groups;
  const int threads = 256;
  pack_grid_kernel<<<static_cast<unsigned>((total + threads - 1) / threads), threads, 0,
                     stream>>>(scale, zero, d_out, groups, rows_pad,
                               static_cast<float2*>(packed));
  return check_launch("pack_grid_kernel");
}

size_t qlinear_workspace_bytes(int d_out, int d_in, int n_tok) {
  const int ntp = std::min(std::max(n_tok, 1), QL_NT_MAX);
  const QlGeom g = ql_geom(d_out, d_in, ntp);
  return g.bop_bytes + g.sums_bytes + g.partial_bytes;
}

kronq_status run_qlinear(const QlinearArgs& q, void* ws, cudaStream_t stream) {
  const int ntp_max = std::min(q.n_tok, QL_NT_MAX);
  const QlGeom g = ql_geom(q.d_out, q.d_in, ntp_max);
  Carve cv{static_cast<uint8_t*>(ws)};
  uint8_t* bop = cv.p;
  cv.p += g.bop_bytes;
  float2* sums = reinterpret_cast<float2*>(cv.p);
  cv.p += g.sums_bytes;
  float* partial = reinterpret_cast<float*>(cv.p);

  const int b_in = pow2_factor(q.d_in), b_out = pow2_factor(q.d_out);
  const bool rot_in = (q.flags & KRONQ_BIIP_ROTATE_IN) != 0;
  const bool rot_out = (q.flags & KRONQ_BIIP_ROTATE_OUT) != 0;
  if (rot_in && b_in > 16384)
    return fail(KRONQ_ERR_UNSUPPORTED, "input Hadamard block %d > 16384", b_in);
  if (rot_out && b_out > 16384)
    return fail(KRONQ_ERR_UNSUPPORTED, "output Hadamard block %d > 16384", b_out);
  // columns per CTA and CTAs per Hadamard block (a cluster of at most 8)
  int span = QL_TILE, cl = 1;
  if (rot_in) {
    if (b_in <= 1024) {
      span = std::max(QL_TILE, b_in);
    } else {
      span = std::max(1024, b_in / 8);
      cl = b_in / span;
    }
  }
  const int in_threads = std::max(32, span / 4);
  const size_t in_smem = static_cast<size_t>(2 * (span + span / 16)) * sizeof(float);
  KQ_CUDA_TRY(cudaFuncSetAttribute(qlin_in_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   static_cast<int>(in_smem)));
  const int qb = (rot_out && b_out > QL_TILE) ? b_out / QL_TILE : 1;
  const size_t out_smem = static_cast<size_t>(qb) * (16 * sizeof(float) + 2 * sizeof(int));

  int dev = 0, max_smem = 0;
  KQ_CUDA_TRY(cudaGetDevice(&dev));
  KQ_CUDA_TRY(cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));

  const bool decode = q.n_tok <= QL_DP_MAX_TOK;
  for (int t0 = 0; t0 < q.n_tok; t0 += QL_NT_MAX) {
    const int nt = std::min(QL_NT_MAX, q.n_tok - t0);
    QlInArgs ia;
    ia.x = static_cast<const uint8_t*>(q.x) +
           static_cast<int64_t>(t0) * q.ld_x * (q.x_dtype == KRONQ_DTYPE_BF16 ? 2 : 4);
    ia.x_dtype = q.x_dtype;
    ia.ld_x = q.ld_x;
    ia.n_tok = nt;
    ia.d_in = q.d_in;
    ia.span = span;
    ia.b_in = rot_in ? b_in : 1;
    ia.cl = cl;
    ia.s_x = q.s_x;
    ia.sign_in = q.sign_in;
    ia.flags = q.flags;
    ia.inv_sqrt_b = static_cast<float>(1.0 / std::sqrt(static_cast<double>(b_in)));
    ia.rows = (3 * nt + 7) / 8 * 8;
    ia.swz = decode ? 0 : 1;
    ia.bop = bop;
    ia.sums = sums;
    const dim3 igrid((q.d_in + span - 1) / span, nt);
    // Chained to the previous kernel too: only the launch overlaps it, since qlin_in waits for
    // it to complete before reading x (which the previous kernel may have written); so this
    // call's workspace writes never race with a previous call's reads.
    KQ_TRY(launch_pdl(qlin_in_kernel, igrid, dim3(in_threads), in_smem, stream, true,
                      "qlin_in_kernel", ia, cl));

    if (decode) {
      QlDpArgs dpa;
      dpa.packed = static_cast<const uint8_t*>(q.packed);
      dpa.bop = bop;
      dpa.sums = sums;
      dpa.grid = static_cast<const float2*>(q.grid);
      dpa.partial = partial;
      dpa.d_out = q.d_out;
      dpa.G = g.G;
      dpa.n_tok = nt;
      dpa.rows = ia.rows;
      dpa.grouped = q.group ? 1 : 0;
      dpa.rotate_out = rot_out ? 1 : 0;
      dpa.b_tile = rot_out ? std::min(b_out, QL_TILE) : 1;
      dpa.U = g.U;
      dpa.err = device_error_word();
      if (!dpa.err) return fail(KRONQ_ERR_CUDA, "device error word unavailable");
      // the largest CTA's staged groups, and as many ring stages as leave room for
      // QL_DP_CTAS_PER_SM CTAs per SM (at least 2)
      const int64_t upc = (g.U + g.C - 1) / g.C;
      const int ng = static_cast<int>(std::min<int64_t>(upc, g.G));
      int per_sm_smem = 0;
      KQ_CUDA_TRY(cudaDeviceGetAttribute(&per_sm_smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor,
                                         dev));
      const int budget = per_sm_smem / QL_DP_CTAS_PER_SM - 1024 -
                         static_cast<int>(sizeof(float)) * nt * QL_TILE;
      const DpSmem L1 = dp_smem(q.bits, ng, nt, 1);
      dpa.stages = std::max(2, std::min(QL_DP_MAX_STAGES, (budget - (L1.total - L1.stage)) /
                                                              L1.stage));
      const size_t dsmem = static_cast<size_t>(dp_smem(q.bits, ng, nt, dpa.stages).total);
      if (static_cast<int>(dsmem) > max_smem)
        return fail(KRONQ_ERR_UNSUPPORTED, "qlinear decode: shared memory too small");
      KQ_TRY(launch_dp(q.bits, nt, dpa, g.C, dsmem, stream));
    } else {
    QlMmaArgs p;
    p.packed = static_cast<const uint8_t*>(q.packed);
    p.bop = bop;
    p.sums = sums;
    p.grid = static_cast<const float2*>(q.grid);
    p.partial = partial;
    p.d_out = q.d_out;
    p.T = g.T;
    p.G = g.G;
    p.n_tok = nt;
    p.N = std::max(16, (3 * nt + 15) / 16 * 16);
    p.grouped = q.group ? 1 : 0;
    p.rotate_out = rot_out ? 1 : 0;
    p.b_tile = rot_out ? std::min(b_out, QL_TILE) : 1;
    p.U = g.U;
    p.err = device_error_word();
    p.R = (3 * nt + 7) / 8 * 8;
    // about 48 KB of stage per bulk-copy pair: few, large copies keep the copy engine busy
    const int per_unit = 2048 * q.bits + 128 * p.R;
    p.ku = std::max(1, std::min(8, 49152 / per_unit));
    QlSmem L0 = ql_smem(q.bits, p.N, p.R, p.ku, 1);
    const int avail = max_smem - static_cast<int>(L0.total - L0.stage_bytes);
    p.stages = std::min(QL_MAX_STAGES, avail / static_cast<int>(L0.stage_bytes));
    if (p.stages < 2) return fail(KRONQ_ERR_UNSUPPORTED, "qlinear: shared memory too small");
    // at least 117 KB, so that one CTA (and its 512 TMEM columns) fills an SM
    const size_t smem = std::max<size_t>(ql_smem(q.bits, p.N, p.R, p.ku, p.stages).total,
                                         117 * 1024);
    KQ_TRY(launch_mma(q.bits, nt, p, g.C, smem, stream));
    }

    QlOutArgs oa;
    oa.partial = partial;
    oa.n_tok = nt;
    oa.T = g.T;
    oa.G = g.G;
    oa.U = g.U;
    oa.C = g.C;
    oa.qb = qb;
    oa.d_out = q.d_out;
    oa.s_g = q.s_g;
    oa.sign_out = q.sign_out;
    oa.flags = q.flags;
    oa.inv_sqrt_b = static_cast<float>(1.0 / std::sqrt(static_cast<double>(b_out)));
    oa.y = q.y + static_cast<int64_t>(t0) * q.ld_y;
    oa.ld_y = q.ld_y;
    // threads per element: enough to give each at most about four segments, within 1024
    // threads per CTA (qb * 16 elements)
    const int64_t segs = (g.C + g.T - 1) / g.T + 1;     // partials per tile, at most
    int tpe = 1;
    while (tpe < 32 && tpe * 4 < segs && qb * 16 * tpe * 2 <= 1024) tpe *= 2;
    oa.tpe = tpe;
    const dim3 ogrid(8 * (g.T / qb), nt);
    KQ_TRY(launch_pdl(qlin_out_kernel, ogrid,
                      dim3(std::min(1024, std::max(32, qb * 16 * tpe))), out_smem, stream, true,
                      "qlin_out_kernel", oa));
  }
  return KRONQ_OK;
}

}  // namespace kq
