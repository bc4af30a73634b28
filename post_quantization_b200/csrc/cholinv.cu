// Damped inverse Cholesky factor K (upper, K^T K = (H + lambda I)^-1).
//
// KronQ (hyper.ai summary), Method, OBS update: the rows "[H_X^-1]_p,p+1:" that the column
// update subtracts are the rows of K. Route: reverse-order (UL) Cholesky H + lambda I = R R^T
// with R upper, and K = R^-1 (by uniqueness of the Cholesky factorization, K is the upper
// Cholesky factor of the damped inverse). lambda = damp_rel * mean(diag H).
//
// Recursive blocked algorithm on a diagonal block A = [[A11, A12], [A12^T, A22]] (upper triangle
// stored, lower triangle zero), which it overwrites with K:
//   K22 = chol_inv(A22)
//   R12 = A12 K22^T                 (A12 = R12 R22^T)
//   A11 <- A11 - R12 R12^T          (upper triangle)
//   K11 = chol_inv(A11)
//   K12 = -K11 R12 K22              ([[R11, R12], [0, R22]]^-1)
// Leaves of at most 128 columns are factored and inverted in shared memory by one CTA. The four
// products of a level are square GEMMs: on the tensor cores (operands split into three bf16
// pieces, fp32-accurate, skipping the zero triangles of K) where a half exceeds 256, and on the
// CUDA cores in fp32 below that, where a product is a handful of tiles and latency, not arithmetic, decides.
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace kq {

namespace {

constexpr int NB = 128;   // leaf size

// lambda = damp_rel * mean(diag A); info = -1.
__global__ void damping_kernel(const float* __restrict__ a, int d, float damp_rel,
                               float* __restrict__ lam, int32_t* __restrict__ info) {
  __shared__ double red[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) s += a[static_cast<int64_t>(i) * d + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) {
      *lam = static_cast<float>(static_cast<double>(damp_rel) * v / d);
      *info = -1;
    }
  }
}

// A_ii += lambda, strict lower triangle := 0 (only the upper triangle is used from here on).
__global__ void prep_kernel(float* __restrict__ a, int d, const float* __restrict__ lam) {
  const int i = blockIdx.y;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j <= i && j < d; j += gridDim.x * blockDim.x) {
    float* p = a + static_cast<int64_t>(i) * d + j;
    if (j < i)
      *p = 0.f;
    else
      *p += *lam;
  }
}

// Leaf: factor the nb x nb diagonal block at a (ld) as A = R R^T (R upper) and overwrite its
// upper triangle with K = R^-1 (strict lower triangle := 0). One CTA of 512 threads; the block is
// padded to 128 with an identity bottom-right part, which factors to itself and leaves the rest
// unchanged.
//
// Blocked by 32-column panels P = [p0, p0 + 32), right to left, on the Schur-updated matrix S:
//   S_PP = R_PP R_PP^T and K_PP = R_PP^-1      one warp, in registers (shuffles, no barriers)
//   R_{<p0,P} = S_{<p0,P} K_PP^T               (S_{<p0,P} = R_{<p0,P} R_PP^T)
//   S_{<p0,<p0} -= R_{<p0,P} R_{<p0,P}^T        (upper triangle)
// then the off-diagonal blocks of K = R^-1 by block rows, bottom up:
//   K_ij = -K_ii sum_{l=i+1..j} R_il K_lj       (j > i; from R K = I)
// The products run from shared memory, a 16 x 32 tile per warp with a 4 x 4 register block per
// lane. K's blocks are kept transposed in the (otherwise free) lower part of the R buffer, so
// every product reads both operands along rows.
constexpr int LEAF_THREADS = 512;
constexpr int PW = 32;                  // panel width
constexpr int LDS = NB + 4;             // row stride: 16-byte rows, consecutive rows 4 banks apart
constexpr int LDT = PW + 4;
constexpr size_t LEAF_SMEM = sizeof(float) * (2 * NB * LDS + (NB - PW) * LDT) + 16;

// acc[i][j] += sum_{m in [m0, m1)} X[r_i][m] * Y[c_j][m] for this lane's rows r_i = tr + ly + 4i
// and columns c_j = tc + lx + 8j of a 16 x 32 warp tile (m0, m1 multiples of 4). Both reads are
// conflict-free: the 4 (8) distinct rows of one read sit 4 banks apart.
__device__ __forceinline__ void tile_acc(float (&acc)[4][4], const float* __restrict__ x, int ldx,
                                         const float* __restrict__ y, int ldy, int tr, int tc,
                                         int m0, int m1, int lane) {
  const int ly = lane >> 3, lx = lane & 7;
  const float* xr = x + (tr + ly) * ldx;
  const float* yr = y + (tc + lx) * ldy;
#pragma unroll 2
  for (int m = m0; m < m1; m += 4) {
    float4 xv[4], yv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) xv[i] = *reinterpret_cast<const float4*>(xr + 4 * i * ldx + m);
#pragma unroll
    for (int j = 0; j < 4; ++j) yv[j] = *reinterpret_cast<const float4*>(yr + 8 * j * ldy + m);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc[i][j] = fmaf(xv[i].x, yv[j].x, acc[i][j]);
        acc[i][j] = fmaf(xv[i].y, yv[j].y, acc[i][j]);
        acc[i][j] = fmaf(xv[i].z, yv[j].z, acc[i][j]);
        acc[i][j] = fmaf(xv[i].w, yv[j].w, acc[i][j]);
      }
  }
}

__device__ __forceinline__ void zero4x4(float (&acc)[4][4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
}

__global__ void __launch_bounds__(LEAF_THREADS, 1) leaf_kernel(float* __restrict__ a, int64_t ld,
                                                            int nb, int j0,
                                                            int32_t* __restrict__ info) {
  extern __shared__ __align__(16) float leaf_smem[];
  float* S = leaf_smem;                 // NB x LDS: S (upper), then K_ii in the diagonal blocks
  float* R = S + NB * LDS;              // NB x LDS: R off-diagonal blocks (upper), K^T (lower)
  float* T = R + NB * LDS;              // (NB - PW) x LDT: one block row of sum R_il K_lj,
                                        // transposed (the panel warp's scratch before that)
  int* bad = reinterpret_cast<int*>(T + (NB - PW) * LDT);
  if (*info >= 0) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ly = lane >> 3, lx = lane & 7;
  constexpr int NWARPS = LEAF_THREADS / 32;

  // the loads of a batch in flight together, then their stores (the zero fill goes through the
  // same pointer, so it must not sit between loads)
  constexpr int PER = NB * NB / LEAF_THREADS, BATCH = 16;
#pragma unroll 1
  for (int u0 = 0; u0 < PER; u0 += BATCH) {
    float v[BATCH];
#pragma unroll
    for (int u = 0; u < BATCH; ++u) {
      const int r = (tid >> 7) + (u0 + u) * (LEAF_THREADS / NB), c = tid & (NB - 1);
      if (r < nb && c < nb)
        v[u] = c >= r ? a[r * ld + c] : 0.f;
      else
        v[u] = r == c ? 1.f : 0.f;
    }
#pragma unroll
    for (int u = 0; u < BATCH; ++u) {
      const int r = (tid >> 7) + (u0 + u) * (LEAF_THREADS / NB), c = tid & (NB - 1);
      S[r * LDS + c] = v[u];
      if (r > c && (r >> 5) != (c >> 5) && r < nb && c < nb) a[r * ld + c] = 0.f;
    }
  }
  if (tid == 0) *bad = -1;
  __syncthreads();

  for (int p0 = NB - PW; p0 >= 0; p0 -= PW) {
    if (warp == 0) {
      // lane k holds column k of the symmetric panel block (both triangles, so that the
      // multiplier S_ck of lane k is a register with a compile-time index). The column that
      // drives a step is published in shared memory by its lane and read back as broadcasts;
      // T is free until the off-diagonal blocks of K are formed.
      float* pub = T;                  // PW x LDT: published columns of the factor step
      float* rt = T + PW * LDT;        // PW x LDT: R_PP^T, 1/R_ii in the padding column PW
      float s[PW];
#pragma unroll
      for (int i = 0; i < PW; ++i) {
        const int r = i < lane ? i : lane, c = i < lane ? lane : i;
        s[i] = S[(p0 + r) * LDS + p0 + c];
      }
      float mypiv = 1.f;
      int fail = -1;
#pragma unroll
      for (int c = PW - 1; c >= 0; --c) {
        if (lane == c) {
#pragma unroll
          for (int i4 = 0; i4 <= c / 4; ++i4)
            *reinterpret_cast<float4*>(pub + c * LDT + 4 * i4) =
                make_float4(s[4 * i4], s[4 * i4 + 1], s[4 * i4 + 2], s[4 * i4 + 3]);
        }
        __syncwarp();
        const float piv = pub[c * LDT + c];
        if (fail < 0 && !(piv > 0.f && isfinite(piv))) fail = c;   // the same on every lane
        mypiv = lane == c ? piv : mypiv;
        const float rp = rsqrtf(piv);
        // finished columns (lanes >= c) take a zero multiplier and stay as they are
        const float f = lane < c ? s[c] * (rp * rp) : 0.f;
#pragma unroll
        for (int i4 = 0; i4 < (c + 3) / 4; ++i4) {
          const float4 v = *reinterpret_cast<const float4*>(pub + c * LDT + 4 * i4);
          if (4 * i4 < c) s[4 * i4] = fmaf(-v.x, f, s[4 * i4]);
          if (4 * i4 + 1 < c) s[4 * i4 + 1] = fmaf(-v.y, f, s[4 * i4 + 1]);
          if (4 * i4 + 2 < c) s[4 * i4 + 2] = fmaf(-v.z, f, s[4 * i4 + 2]);
          if (4 * i4 + 3 < c) s[4 * i4 + 3] = fmaf(-v.w, f, s[4 * i4 + 3]);
        }
      }
      if (fail >= 0) {
        if (lane == 0) *bad = p0 + fail;
      } else {
        // lane k: column k of R_PP (row k of R_PP^T), then column k of K_PP = R_PP^-1 by
        // right-looking substitution, reading column i of R_PP as broadcasts
        const float rs = rsqrtf(mypiv), sq = sqrtf(mypiv);
#pragma unroll
        for (int i = 0; i < PW; ++i) s[i] = i < lane ? s[i] * rs : (i == lane ? sq : 0.f);
#pragma unroll
        for (int i4 = 0; i4 < PW / 4; ++i4)
          *reinterpret_cast<float4*>(rt + lane * LDT + 4 * i4) =
              make_float4(s[4 * i4], s[4 * i4 + 1], s[4 * i4 + 2], s[4 * i4 + 3]);
        rt[lane * LDT + PW] = rs;      // 1 / R_kk
        __syncwarp();
        float k[PW];
#pragma unroll
        for (int i = 0; i < PW; ++i) k[i] = 0.f;
#pragma unroll
        for (int i = PW - 1; i >= 0; --i) {
          k[i] = ((lane == i ? 1.f : 0.f) - k[i]) * rt[i * LDT + PW];
#pragma unroll
          for (int r4 = 0; r4 < (i + 3) / 4; ++r4) {
            const float4 v = *reinterpret_cast<const float4*>(rt + i * LDT + 4 * r4);
            if (4 * r4 < i) k[4 * r4] = fmaf(v.x, k[i], k[4 * r4]);
            if (4 * r4 + 1 < i) k[4 * r4 + 1] = fmaf(v.y, k[i], k[4 * r4 + 1]);
            if (4 * r4 + 2 < i) k[4 * r4 + 2] = fmaf(v.z, k[i], k[4 * r4 + 2]);
            if (4 * r4 + 3 < i) k[4 * r4 + 3] = fmaf(v.w, k[i], k[4 * r4 + 3]);
          }
        }
#pragma unroll
        for (int i = 0; i < PW; ++i) {
          S[(p0 + i) * LDS + p0 + lane] = k[i];        // K_PP
          if (p0 + i < nb && p0 + lane < nb) a[(p0 + i) * ld + p0 + lane] = k[i];
        }
#pragma unroll
        for (int i4 = 0; i4 < PW / 4; ++i4)            // K_PP^T
          *reinterpret_cast<float4*>(R + (p0 + lane) * LDS + p0 + 4 * i4) =
              make_float4(k[4 * i4], k[4 * i4 + 1], k[4 * i4 + 2], k[4 * i4 + 3]);
      }
    }
    __syncthreads();
    if (*bad >= 0) {
      if (tid == 0 && *bad < nb) *info = j0 + *bad;
      return;                                  // uniform
    }
    if (p0 == 0) break;
    // R_{<p0,P} = S_{<p0,P} K_PP^T: p0 / 16 tiles of 16 x 32
    for (int t = warp; t < p0 / 16; t += NWARPS) {
      float acc[4][4];
      zero4x4(acc);
      tile_acc(acc, S + p0, LDS, S + p0 * LDS + p0, LDS, 16 * t, 0, 0, PW, lane);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) R[(16 * t + ly + 4 * i) * LDS + p0 + lx + 8 * j] = acc[i][j];
    }
    __syncthreads();
    // S_{<p0,<p0} -= R_{<p0,P} R_{<p0,P}^T on the tiles that meet the upper triangle
    {
      const int tcols = p0 / 32, ntiles = (p0 / 16) * tcols;
      for (int t = warp; t < ntiles; t += NWARPS) {
        const int tr = 16 * (t / tcols), tc = 32 * (t % tcols);
        if (tr >= tc + 32) continue;
        float acc[4][4];
        zero4x4(acc);
        tile_acc(acc, R + p0, LDS, R + p0, LDS, tr, tc, 0, PW, lane);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) S[(tr + ly + 4 * i) * LDS + tc + lx + 8 * j] -= acc[i][j];
      }
    }
    __syncthreads();
  }

  // K_ij (j > i), block rows bottom up
  for (int bi = NB / PW - 2; bi >= 0; --bi) {
    const int i0 = PW * bi, nj = NB / PW - 1 - bi;
    // T_ij = sum_{l=i+1..j} R_il K_lj, stored transposed: T[32 (j - i - 1) + c][r]
    for (int t = warp; t < 2 * nj; t += NWARPS) {
      const int jj = t >> 1, tr = i0 + 16 * (t & 1), tc = i0 + PW * (jj + 1);
      float acc[4][4];
      zero4x4(acc);
      tile_acc(acc, R, LDS, R, LDS, tr, tc, i0 + PW, tc + PW, lane);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          T[(PW * jj + lx + 8 * j) * LDT + tr - i0 + ly + 4 * i] = acc[i][j];
    }
    __syncthreads();
    // K_ij = -K_ii T_ij: into K^T (lower part of R) and to global memory
    for (int t = warp; t < 2 * nj; t += NWARPS) {
      const int jj = t >> 1, tr = i0 + 16 * (t & 1), tc = i0 + PW * (jj + 1);
      float acc[4][4];
      zero4x4(acc);
      tile_acc(acc, S + i0, LDS, T + PW * jj * LDT, LDT, tr, 0, 0, PW, lane);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = tr + ly + 4 * i, c = tc + lx + 8 * j;
          R[c * LDS + r] = -acc[i][j];
          if (r < nb && c < nb) a[r * ld + c] = -acc[i][j];
        }
    }
    __syncthreads();
  }
}

// fp32 GEMM on the CUDA cores for the bottom levels of the recursion (m, n, k <= 256), where
// a product is a handful of tiles and latency, not arithmetic, decides:
//   C = alpha * A op(B) + beta * C,  op(B) = B^T (B given n x k) or B (B given k x n).
// C must not alias A or B. CTA tile 32 x 64, 128 threads, each a 4 x 4 block (rows ty + 8i,
// columns tx + 16j); K in chunks of 32, both operands staged along K in shared memory and read
// as 16-byte vectors, the next chunk's loads in flight (registers) while this one is used.
// k0 (A upper triangular) starts the K loop at the tile's first row.
constexpr int SG_TM = 32, SG_TN = 64, SG_KC = 32, SG_LD = SG_KC + 4, SG_THREADS = 128;

struct SgChunk {
  float4 a[2];   // 32 x 32 of A: 256 float4, two per thread
  float4 b[4];   // 64 x 32 of B: 512 float4, four per thread
};

__device__ __forceinline__ float4 ld4_guard(const float* p, int valid) {
  // valid: how many of the 4 floats at p exist (0..4); the pointer is 16-byte aligned if 4
  if (valid >= 4) return *reinterpret_cast<const float4*>(p);
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (valid > 0) v.x = p[0];
  if (valid > 1) v.y = p[1];
  if (valid > 2) v.z = p[2];
  return v;
}

__global__ void __launch_bounds__(SG_THREADS) sgemm_small_kernel(
    int m, int n, int k, float alpha, const float* __restrict__ a, int64_t lda,
    const float* __restrict__ b, int64_t ldb, int b_mn, float beta, float* __restrict__ c,
    int64_t ldc, int upper_only, int a_upper, int vec, const int32_t* __restrict__ skip) {
  if (skip && *skip >= 0) return;
  __shared__ __align__(16) float as[2][SG_TM * SG_LD];
  __shared__ __align__(16) float bs[2][SG_TN * SG_LD];
  const int t = threadIdx.x, ty = t >> 4, tx = t & 15;
  const int row0 = blockIdx.y * SG_TM, col0 = blockIdx.x * SG_TN;
  if (upper_only && row0 > col0 + SG_TN - 1) return;
  const int kbeg = a_upper ? (row0 / SG_KC) * SG_KC : 0;

  // load mapping: A: float4 index e = t + 128 u (u < 2): row e / 8, k4 (e % 8) * 4
  //   B K-major: e = t + 128 u (u < 4): col e / 8, k4 (e % 8) * 4
  //   B MN-major: e = t + 128 u: k-row e / 16, col4 (e % 16) * 4
  auto load = [&](int k0, SgChunk& ch) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int e = t + SG_THREADS * u, r = row0 + e / 8, kk = k0 + (e % 8) * 4;
      ch.a[u] = (r < m) ? (vec ? ld4_guard(a + r * lda + kk, k - kk)
                               : make_float4(kk < k ? a[r * lda + kk] : 0.f,
                                             kk + 1 < k ? a[r * lda + kk + 1] : 0.f,
                                             kk + 2 < k ? a[r * lda + kk + 2] : 0.f,
                                             kk + 3 < k ? a[r * lda + kk + 3] : 0.f))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = t + SG_THREADS * u;
      if (!b_mn) {
        const int cc = col0 + e / 8, kk = k0 + (e % 8) * 4;
        ch.b[u] = (cc < n) ? (vec ? ld4_guard(b + cc * ldb + kk, k - kk)
                                  : make_float4(kk < k ? b[cc * ldb + kk] : 0.f,
                                                kk + 1 < k ? b[cc * ldb + kk + 1] : 0.f,
                                                kk + 2 < k ? b[cc * ldb + kk + 2] : 0.f,
                                                kk + 3 < k ? b[cc * ldb + kk + 3] : 0.f))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        const int kk = k0 + e / 16, cc = col0 + (e % 16) * 4;
        ch.b[u] = (kk < k) ? (vec ? ld4_guard(b + kk * ldb + cc, n - cc)
                                  : make_float4(cc < n ? b[kk * ldb + cc] : 0.f,
                                                cc + 1 < n ? b[kk * ldb + cc + 1] : 0.f,
                                                cc + 2 < n ? b[kk * ldb + cc + 2] : 0.f,
                                                cc + 3 < n ? b[kk * ldb + cc + 3] : 0.f))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  };
  auto store = [&](const SgChunk& ch, int buf) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int e = t + SG_THREADS * u;
      *reinterpret_cast<float4*>(&as[buf][(e / 8) * SG_LD + (e % 8) * 4]) = ch.a[u];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = t + SG_THREADS * u;
      if (!b_mn) {
        *reinterpret_cast<float4*>(&bs[buf][(e / 8) * SG_LD + (e % 8) * 4]) = ch.b[u];
      } else {
        const int kk = e / 16, cc = (e % 16) * 4;
        bs[buf][(cc + 0) * SG_LD + kk] = ch.b[u].x;
        bs[buf][(cc + 1) * SG_LD + kk] = ch.b[u].y;
        bs[buf][(cc + 2) * SG_LD + kk] = ch.b[u].z;
        bs[buf][(cc + 3) * SG_LD + kk] = ch.b[u].w;
      }
    }
  };

  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  SgChunk ch;
  int buf = 0;
  if (kbeg < k) {
    load(kbeg, ch);
    store(ch, 0);
  }
  __syncthreads();
  for (int k0 = kbeg; k0 < k; k0 += SG_KC) {
    const bool more = k0 + SG_KC < k;
    if (more) load(k0 + SG_KC, ch);          // in flight during the products below
    const float* ap = &as[buf][ty * SG_LD];
    const float* bp = &bs[buf][tx * SG_LD];
#pragma unroll
    for (int k4 = 0; k4 < SG_KC; k4 += 4) {
      float4 av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = *reinterpret_cast<const float4*>(ap + 8 * i * SG_LD + k4);
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = *reinterpret_cast<const float4*>(bp + 16 * j * SG_LD + k4);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(av[i].x, bv[j].x, acc[i][j]);
          acc[i][j] = fmaf(av[i].y, bv[j].y, acc[i][j]);
          acc[i][j] = fmaf(av[i].z, bv[j].z, acc[i][j]);
          acc[i][j] = fmaf(av[i].w, bv[j].w, acc[i][j]);
        }
    }
    if (more) store(ch, buf ^ 1);
    __syncthreads();
    buf ^= 1;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = row0 + ty + 8 * i;
    if (r >= m) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int cc = col0 + tx + 16 * j;
      if (cc >= n || (upper_only && cc < r)) continue;
      float* p = c + r * ldc + cc;
      *p = beta != 0.f ? fmaf(beta, *p, alpha * acc[i][j]) : alpha * acc[i][j];
    }
  }
}
kronq_status sgemm_small(int m, int n, int k, float alpha, const float* a, int64_t lda,
                         const float* b, int64_t ldb, bool b_mn_major, float beta, float* c,
                         int64_t ldc, bool upper_only, bool a_upper, const int32_t* skip,
                         cudaStream_t stream) {
  if (m <= 0 || n <= 0) return KRONQ_OK;
  if (k <= 0) return fail(KRONQ_ERR_SHAPE, "sgemm_small: k must be >= 1");
  const int vec = (reinterpret_cast<uintptr_t>(a) & 15u) == 0 &&
                  (reinterpret_cast<uintptr_t>(b) & 15u) == 0 && lda % 4 == 0 && ldb % 4 == 0;
  dim3 grid(static_cast<unsigned>((n + SG_TN - 1) / SG_TN),
            static_cast<unsigned>((m + SG_TM - 1) / SG_TM));
  sgemm_small_kernel<<<grid, SG_THREADS, 0, stream>>>(m, n, k, alpha, a, lda, b, ldb, b_mn_major,
                                                      beta, c, ldc, upper_only, a_upper, vec,
                                                      skip);
  return check_launch("sgemm_small_kernel");
}

struct Ctx {
  int64_t ld;
  float* t;          // n1 x n2 product T of the top level (largest)
  int32_t* info;
  cudaStream_t stream;
};

void halves(int n, int& n1, int& n2) {
  // bottom-right part: a multiple of NB columns, about half
  n2 = ((n / 2 + NB - 1) / NB) * NB;
  if (n2 >= n) n2 = n - NB;
  n1 = n - n2;
}

// Split-operand scratch of one recursion node and everything below it. A node keeps the splits
// of K22 and of A12 / R12 from the first GEMM to the last (across the K11 recursion), so each is
// split once; the K11 recursion and the (K11, T) pair use the space after them.
size_t area_bytes(int n) {
  if (n <= NB) return 0;
  int n1, n2;
  halves(n, n1, n2);
  if (n1 <= 256 && n2 <= 256)
    return std::max(area_bytes(n2),
                    align256(2 * sizeof(float) * static_cast<size_t>(n1) * n2) + area_bytes(n1));
  const size_t own = split_bytes(n2, n2) + split_bytes(n1, n2);
  const size_t tail = std::max(area_bytes(n1), split_bytes(n1, n1) + split_bytes(n1, n2));
  return std::max(area_bytes(n2), own + tail);
}

// Overwrite the n x n diagonal block at a (global index j0) with K.
kronq_status chol_inv_rec(const Ctx& c, float* a, int n, int j0, uint8_t* area) {
  if (n <= NB) {
    leaf_kernel<<<1, LEAF_THREADS, LEAF_SMEM, c.stream>>>(a, c.ld, n, j0, c.info);
    return check_launch("leaf_kernel");
  }
  int n1, n2;
  halves(n, n1, n2);
  float* a11 = a;
  float* a12 = a + n1;
  float* a22 = a + static_cast<int64_t>(n1) * c.ld + n1;
  const int64_t ld = c.ld;
  cudaStream_t st = c.stream;

  KQ_TRY(chol_inv_rec(c, a22, n2, j0 + n1, area));                         // K22
  if (n1 <= 256 && n2 <= 256) {
    // small node: the four products on the CUDA cores, straight from the fp32 blocks; R12 and
    // T live in this node's scratch, the K11 recursion uses the space after them
    float* r12 = reinterpret_cast<float*>(area);
    float* tt = r12 + static_cast<int64_t>(n1) * n2;
    uint8_t* rest = reinterpret_cast<uint8_t*>(tt + static_cast<int64_t>(n1) * n2);
    KQ_TRY(sgemm_small(n1, n2, n2, 1.f, a12, ld, a22, ld, false, 0.f, r12, n2, false, false,
                       c.info, st));                                        // R12 = A12 K22^T
    KQ_TRY(sgemm_small(n1, n1, n2, -1.f, r12, n2, r12, n2, false, 1.f, a11, ld, true, false,
                       c.info, st));                                        // A11 -= R12 R12^T
    KQ_TRY(chol_inv_rec(c, a11, n1, j0, rest));                            // K11
    KQ_TRY(sgemm_small(n1, n2, n2, 1.f, r12, n2, a22, ld, true, 0.f, tt, n2, false, false,
                       c.info, st));                                        // T = R12 K22
    return sgemm_small(n1, n2, n1, -1.f, a11, ld, tt, n2, true, 0.f, a12, ld, false, true,
                       c.info, st);                                         // K12 = -K11 T
  }
  Carve cv{area};
  const Split3 s22 = cv.split(n2, n2);    // K22, kept to the end of the node
  const Split3 s12 = cv.split(n1, n2);    // A12, then R12
  uint8_t* rest = cv.p;
  // R12 = A12 K22^T, written over A12
  KQ_TRY(split_bf16x3_2(a22, ld, n2, n2, s22, a12, ld, n1, n2, s12, st));
  KQ_TRY(tgemm(n1, n2, n2, 1.f, s12, s22, false, 0.f, a12, ld, false, GEMM_B_LOWER, c.info, st));
  // A11 -= R12 R12^T (upper triangle)
  KQ_TRY(split_bf16x3(a12, ld, n1, n2, s12, st));
  KQ_TRY(tgemm(n1, n1, n2, -1.f, s12, s12, false, 1.f, a11, ld, true, 0, c.info, st));
  KQ_TRY(chol_inv_rec(c, a11, n1, j0, rest));                              // K11
  // T = R12 K22
  KQ_TRY(tgemm(n1, n2, n2, 1.f, s12, s22, true, 0.f, c.t, n2, false, GEMM_B_UPPER, c.info, st));
  // K12 = -K11 T
  Carve cr{rest};
  const Split3 s11 = cr.split(n1, n1), tt = cr.split(n1, n2);
  KQ_TRY(split_bf16x3_2(a11, ld, n1, n1, s11, c.t, n2, n1, n2, tt, st));
  KQ_TRY(tgemm(n1, n2, n1, -1.f, s11, tt, true, 0.f, a12, ld, false, GEMM_A_UPPER, c.info, st));
  return KRONQ_OK;
}

size_t t_bytes(int d) {
  if (d <= NB) return align256(sizeof(float));
  int n1, n2;
  halves(d, n1, n2);
  return align256(sizeof(float) * static_cast<size_t>(n1) * n2);
}

}  // namespace

size_t cholinv_workspace_bytes(int d) { return 256 + t_bytes(d) + area_bytes(d); }

kronq_status run_cholinv(float* a, int d, float damp_rel, int32_t* info, void* ws,
                         cudaStream_t stream) {
  uint8_t* p = static_cast<uint8_t*>(ws);
  float* lam = reinterpret_cast<float*>(p);
  p += 256;
  float* t = reinterpret_cast<float*>(p);
  p += t_bytes(d);
  damping_kernel<<<1, 1024, 0, stream>>>(a, d, damp_rel, lam, info);
  KQ_TRY(check_launch("damping_kernel"));
  {
    dim3 grid((d + 255) / 256, d);
    prep_kernel<<<grid, 256, 0, stream>>>(a, d, lam);
    KQ_TRY(check_launch("prep_kernel"));
  }
  // per device and cheap on the host, so set on every call
  KQ_CUDA_TRY(cudaFuncSetAttribute(leaf_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   static_cast<int>(LEAF_SMEM)));
  Ctx c{d, t, info, stream};
  return chol_inv_rec(c, a, d, 0, p);
}

}  // namespace kq
