// C ABI of the KronQ library: argument validation, workspace carving and dispatch to the
// kernels. Declarations and the contract of every call are in include/kronq.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace kq {

namespace {
thread_local char g_detail[512] = "";
__device__ int g_device_error_word = 0;
constexpr int kMaxDevices = 64;
int* g_err_ptr[kMaxDevices] = {nullptr};
std::mutex g_err_mu;
}  // namespace

void set_detail(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
  va_end(ap);
}

kronq_status fail(kronq_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
  va_end(ap);
  return s;
}

std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_sm_budget{0};

int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    sms = 148;
  return sms;
}

int sm_budget() {
  static thread_local int cached_dev = -1, cached_sms = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev != cached_dev) {
    cached_sms = device_sms();
    cached_dev = dev;
  }
  const int b = g_sm_budget.load(std::memory_order_relaxed);
  return (b > 0 && b < cached_sms) ? b : cached_sms;
}

kronq_status check_launch(const char* what) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(KRONQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return KRONQ_OK;
}

kronq_status encode_tiled_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank,
                              const void* base, const uint64_t* dims, const uint64_t* strides,
                              const uint32_t* box, CUtensorMapSwizzle swizzle) {
  using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                     const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                     const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                     CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static EncodeTiledFn enc = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(ptr);
    return static_cast<EncodeTiledFn>(nullptr);
  }();
  if (!enc) return fail(KRONQ_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  if (rank < 1 || rank > 5) return fail(KRONQ_ERR_INVALID_ARG, "tensor map rank %d", rank);
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides[i];
  }
  const CUresult r = enc(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d,
                         st, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KRONQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return KRONQ_OK;
}

int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  // the address is per device; host threads making their first call on one device together
  // look it up under the lock
  std::lock_guard<std::mutex> lock(g_err_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error_word) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<int*>(p);
  }
  return g_err_ptr[dev];
}

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

kronq_status check_ws(void* ws, size_t have, size_t need) {
  if (need == 0) return KRONQ_OK;
  if (!ws) return fail(KRONQ_ERR_WORKSPACE, "workspace is NULL, %zu bytes needed", need);
  if (!aligned(ws, 256)) return fail(KRONQ_ERR_WORKSPACE, "workspace not 256-byte aligned");
  if (have < need)
    return fail(KRONQ_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", have, need);
  return KRONQ_OK;
}

kronq_status check_bf16_matrix(const void* p, int64_t ld, int cols, const char* name) {
  if (!p) return fail(KRONQ_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned(p, 16)) return fail(KRONQ_ERR_INVALID_ARG, "%s not 16-byte aligned", name);
  if (ld < cols) return fail(KRONQ_ERR_SHAPE, "%s: stride %lld < width %d", name, (long long)ld, cols);
  if ((ld * 2) % 16 != 0)
    return fail(KRONQ_ERR_INVALID_ARG, "%s: stride %lld elements is not a multiple of 16 bytes",
                name, (long long)ld);
  return KRONQ_OK;
}

constexpr int64_t kDriftChunk = 32768;   // tokens per fp16 conversion (workspace bound)

size_t drift_ld(int d_in) { return static_cast<size_t>((d_in + 7) / 8 * 8); }

// [amax pair: 256 B][fp16 X - X~ chunk][fp16 X~ chunk]
size_t drift_ws(int64_t n, int d_in) {
  const int64_t rows = std::min<int64_t>(n, kDriftChunk);
  if (rows <= 0) return 0;
  return 256 + 2 * align256(static_cast<size_t>(rows) * drift_ld(d_in) * 2);
}

}  // namespace
}  // namespace kq

using namespace kq;

extern "C" {

const char* kronq_status_string(kronq_status s) {
  switch (s) {
    case KRONQ_OK: return "ok";
    case KRONQ_ERR_INVALID_ARG: return "invalid argument";
    case KRONQ_ERR_SHAPE: return "invalid shape";
    case KRONQ_ERR_NOT_PD: return "matrix not positive definite";
    case KRONQ_ERR_CUDA: return "CUDA error";
    case KRONQ_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case KRONQ_ERR_UNSUPPORTED: return "unsupported device or parameter";
    case KRONQ_ERR_TIMEOUT: return "a kernel gave up a bounded wait";
  }
  return "unknown status";
}

const char* kronq_last_error_detail(void) { return g_detail; }

int kronq_version(void) { return 100; }

uint64_t kronq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

void kronq_set_sm_budget(int32_t sms) { kq::g_sm_budget.store(sms > 0 ? sms : 0); }

int32_t kronq_sm_budget(void) { return kq::g_sm_budget.load(); }

kronq_status kronq_device_check(void) {
  int dev = 0;
  KQ_CUDA_TRY(cudaGetDevice(&dev));
  int major = 0, minor = 0;
  KQ_CUDA_TRY(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  KQ_CUDA_TRY(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
  if (major != 10 || minor != 0)
    return fail(KRONQ_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a",
                dev, major, minor);
  return KRONQ_OK;
}

kronq_status kronq_device_error(int32_t* code_out, kronq_stream_t stream) {
  if (!code_out) return fail(KRONQ_ERR_INVALID_ARG, "code_out is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* w = device_error_word();
  if (!w) return fail(KRONQ_ERR_CUDA, "device error word unavailable");
  int host = 0;
  KQ_CUDA_TRY(cudaMemcpyAsync(&host, w, sizeof(int), cudaMemcpyDeviceToHost, s));
  KQ_CUDA_TRY(cudaStreamSynchronize(s));
  *code_out = host;
  if (host != 0) {
    KQ_CUDA_TRY(cudaMemsetAsync(w, 0, sizeof(int), s));
    KQ_CUDA_TRY(cudaStreamSynchronize(s));
  }
  return KRONQ_OK;
}

// ----------------------------------------------------------------------------- accumulate
size_t kronq_accumulate_workspace_size(int64_t n, int32_t d_in, int32_t d_out, int with_dxx) {
  (void)d_out;
  if (!with_dxx || n <= 0 || d_in <= 0) return 0;
  return drift_ws(n, d_in);
}

kronq_status kronq_accumulate(const void* xq, int64_t ld_xq, const void* xfp, int64_t ld_xfp,
                              const void* g, int64_t ld_g, int64_t n, int32_t d_in,
                              int32_t d_out, float* hx_sum, float* hg_sum, float* dxx_sum,
                              void* workspace, size_t workspace_bytes, kronq_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (n < 0) return fail(KRONQ_ERR_SHAPE, "n < 0");
  if (!hx_sum && !hg_sum && !dxx_sum) return fail(KRONQ_ERR_INVALID_ARG, "no output requested");
  if (n == 0) return KRONQ_OK;   // nothing to add (inputs may be empty/NULL)
  if ((hx_sum || dxx_sum) && d_in <= 0) return fail(KRONQ_ERR_SHAPE, "d_in <= 0");
  if (hg_sum && d_out <= 0) return fail(KRONQ_ERR_SHAPE, "d_out <= 0");
  if (hx_sum || dxx_sum) KQ_TRY(check_bf16_matrix(xq, ld_xq, d_in, "xq"));
  if (dxx_sum) KQ_TRY(check_bf16_matrix(xfp, ld_xfp, d_in, "xfp"));
  if (hg_sum) KQ_TRY(check_bf16_matrix(g, ld_g, d_out, "g"));
  for (const float* o : {hx_sum, hg_sum, dxx_sum})
    if (o && !aligned(o, 16)) return fail(KRONQ_ERR_INVALID_ARG, "output not 16-byte aligned");
  if (dxx_sum) KQ_TRY(check_ws(workspace, workspace_bytes, drift_ws(n, d_in)));
  KQ_TRY(kronq_device_check());

  if (hx_sum) {
    KQ_TRY(launch_accumulate_tc(xq, ld_xq, xq, ld_xq, n, d_in, d_in, hx_sum, d_in, true, s));
    KQ_TRY(launch_mirror_upper(hx_sum, d_in, d_in, s));
  }
  if (hg_sum) {
    KQ_TRY(launch_accumulate_tc(g, ld_g, g, ld_g, n, d_out, d_out, hg_sum, d_out, true, s));
    KQ_TRY(launch_mirror_upper(hg_sum, d_out, d_out, s));
  }
  if (dxx_sum) {
    // D += (X - X~)^T X~ as one fp16 product per token chunk: both operands rescaled by powers
    // of two from their largest magnitude over all n tokens (X~ exact, X - X~ rounded once)
    const int64_t ld = static_cast<int64_t>(drift_ld(d_in));
    const int64_t rows = std::min<int64_t>(n, kDriftChunk);
    float* amax = static_cast<float*>(workspace);
    uint8_t* da = static_cast<uint8_t*>(workspace) + 256;
    uint8_t* xb = da + align256(static_cast<size_t>(rows) * ld * 2);
    const uint16_t* xq16 = static_cast<const uint16_t*>(xq);
    const uint16_t* xf16 = static_cast<const uint16_t*>(xfp);
    KQ_TRY(launch_drift_amax(xfp, ld_xfp, xq, ld_xq, n, d_in, amax, s));
    for (int64_t t0 = 0; t0 < n; t0 += kDriftChunk) {
      const int64_t cnt = std::min<int64_t>(kDriftChunk, n - t0);
      KQ_TRY(launch_drift_fp16(xf16 + t0 * ld_xfp, ld_xfp, xq16 + t0 * ld_xq, ld_xq, cnt, d_in,
                               amax, da, xb, ld, s));
      KQ_TRY(launch_accumulate_tc(da, ld, xb, ld, cnt, d_in, d_in, dxx_sum, d_in, false, s,
                                  true, amax));
    }
  }
  return KRONQ_OK;
}

size_t kronq_accumulate_diag_workspace_size(int64_t n, int32_t d) {
  return accumulate_diag_workspace_bytes(n, d);
}

kronq_status kronq_accumulate_diag(const void* g, int64_t ld_g, int64_t n, int32_t d,
                                   float* diag_sum, void* workspace, size_t workspace_bytes,
                                   kronq_stream_t stream) {
  if (n < 0) return fail(KRONQ_ERR_SHAPE, "n < 0");
  if (d <= 0) return fail(KRONQ_ERR_SHAPE, "d <= 0");
  if (!diag_sum) return fail(KRONQ_ERR_INVALID_ARG, "diag_sum is required");
  if (n == 0) return KRONQ_OK;
  if (n > kMaxDiagTokens)
    return fail(KRONQ_ERR_SHAPE, "n = %lld tokens exceeds the %lld tokens one call takes; "
                "split the tokens over several calls (the sums add)", (long long)n,
                (long long)kMaxDiagTokens);
  KQ_TRY(check_bf16_matrix(g, ld_g, d, "g"));
  KQ_TRY(check_ws(workspace, workspace_bytes, accumulate_diag_workspace_bytes(n, d)));
  KQ_TRY(kronq_device_check());
  return launch_accumulate_diag(g, ld_g, n, d, diag_sum, workspace,
                                reinterpret_cast<cudaStream_t>(stream));
}

// ----------------------------------------------------------------------------- biip
size_t kronq_biip_workspace_size(int32_t d_out, int32_t d_in) {
  if (d_out <= 0 || d_in <= 0) return 0;
  return biip_workspace_bytes(d_out, d_in);
}

kronq_status kronq_biip(const void* w, int32_t w_dtype, float* w_out, float* hx, float* hg,
                        float* dxx, double inv_n, const int8_t* sign_in, const int8_t* sign_out,
                        int32_t d_out, int32_t d_in, uint32_t flags, float* s_x, float* s_g,
                        double* tr_hx, double* tr_hg, void* workspace, size_t workspace_bytes,
                        kronq_stream_t stream) {
  if (d_out <= 0 || d_in <= 0) return fail(KRONQ_ERR_SHAPE, "d_out and d_in must be positive");
  if (!w || !w_out || !hx || !s_x || !s_g || !tr_hx)
    return fail(KRONQ_ERR_INVALID_ARG, "w, w_out, hx, s_x, s_g and tr_hx are required");
  if (w_dtype != KRONQ_DTYPE_BF16 && w_dtype != KRONQ_DTYPE_F32)
    return fail(KRONQ_ERR_INVALID_ARG, "w_dtype must be KRONQ_DTYPE_BF16 or KRONQ_DTYPE_F32");
  if (flags & ~static_cast<uint32_t>(63))
    return fail(KRONQ_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
  if ((flags & KRONQ_BIIP_SCALE_OUT) && !hg)
    return fail(KRONQ_ERR_INVALID_ARG, "KRONQ_BIIP_SCALE_OUT needs hg");
  if ((flags & KRONQ_BIIP_HG_DIAG) && !hg)
    return fail(KRONQ_ERR_INVALID_ARG, "KRONQ_BIIP_HG_DIAG needs hg (the diagonal sums)");
  if ((flags & KRONQ_BIIP_HG_DIAG) && (flags & KRONQ_BIIP_WRITE_HG))
    return fail(KRONQ_ERR_INVALID_ARG, "KRONQ_BIIP_WRITE_HG needs the full H_G, not its diagonal");
  if ((flags & KRONQ_BIIP_ROTATE_IN) && !sign_in)
    return fail(KRONQ_ERR_INVALID_ARG, "KRONQ_BIIP_ROTATE_IN needs sign_in");
  if ((flags & KRONQ_BIIP_ROTATE_OUT) && !sign_out)
    return fail(KRONQ_ERR_INVALID_ARG, "KRONQ_BIIP_ROTATE_OUT needs sign_out");
  if (!(inv_n > 0.0) || !std::isfinite(inv_n)) return fail(KRONQ_ERR_INVALID_ARG, "inv_n must be > 0");
  if (w == w_out) return fail(KRONQ_ERR_INVALID_ARG, "w and w_out must not alias");
  KQ_TRY(check_ws(workspace, workspace_bytes, biip_workspace_bytes(d_out, d_in)));
  KQ_TRY(kronq_device_check());
  BiipArgs a{w, w_dtype, w_out, hx, hg, dxx, inv_n, sign_in, sign_out, d_out, d_in, flags,
             s_x, s_g, tr_hx, tr_hg};
  return run_biip(a, workspace, reinterpret_cast<cudaStream_t>(stream));
}

// ----------------------------------------------------------------------------- cholinv
size_t kronq_cholinv_workspace_size(int32_t d) {
  if (d <= 0) return 0;
  return cholinv_workspace_bytes(d);
}

kronq_status kronq_cholinv(float* h_to_k, int32_t d, float damp_rel, int32_t* info,
                           uint32_t flags, void* workspace, size_t workspace_bytes,
                           kronq_stream_t stream) {
  if (d <= 0) return fail(KRONQ_ERR_SHAPE, "d must be positive");
  if (!h_to_k || !info) return fail(KRONQ_ERR_INVALID_ARG, "h_to_k and info are required");
  if (!(damp_rel >= 0.f) || !std::isfinite(damp_rel))
    return fail(KRONQ_ERR_INVALID_ARG, "damp_rel must be finite and >= 0");
  if (flags & ~static_cast<uint32_t>(KRONQ_CHOLINV_SYNC))
    return fail(KRONQ_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
  KQ_TRY(check_ws(workspace, workspace_bytes, cholinv_workspace_bytes(d)));
  KQ_TRY(kronq_device_check());
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  KQ_TRY(run_cholinv(h_to_k, d, damp_rel, info, workspace, s));
  if (flags & KRONQ_CHOLINV_SYNC) {
    int32_t host = -1;
    KQ_CUDA_TRY(cudaMemcpyAsync(&host, info, sizeof(int32_t), cudaMemcpyDeviceToHost, s));
    KQ_CUDA_TRY(cudaStreamSynchronize(s));
    if (host >= 0)
      return fail(KRONQ_ERR_NOT_PD, "pivot %d of the damped H_X is not positive", host);
  }
  return KRONQ_OK;
}

// ----------------------------------------------------------------------------- quantize
size_t kronq_quantize_layer_workspace_size(int32_t d_out, int32_t d_in, int32_t block,
                                           int with_dxx) {
  if (d_out <= 0 || d_in <= 0) return 0;
  return quantize_workspace_bytes(d_out, d_in, block, with_dxx != 0);
}

kronq_status kronq_quantize_layer(const float* w, const float* k, const float* dxx,
                                  int32_t d_out, int32_t d_in, int32_t bits, int32_t block,
                                  int32_t group, uint8_t* codes, float* scale, float* zero,
                                  float* w_hat, void* workspace, size_t workspace_bytes,
                                  kronq_stream_t stream) {
  if (d_out <= 0 || d_in <= 0) return fail(KRONQ_ERR_SHAPE, "d_out and d_in must be positive");
  if (!w || !k || !codes || !scale || !zero || !w_hat)
    return fail(KRONQ_ERR_INVALID_ARG, "w, k, codes, scale, zero and w_hat are required");
  if (bits < 2 || bits > 8) return fail(KRONQ_ERR_UNSUPPORTED, "bits must be in 2..8");
  if (block != 128) return fail(KRONQ_ERR_UNSUPPORTED, "block must be 128");
  if (group != 0 && group != block)
    return fail(KRONQ_ERR_UNSUPPORTED, "group must be 0 (per row) or the block width (128)");
  if (w == w_hat) return fail(KRONQ_ERR_INVALID_ARG, "w and w_hat must not alias");
  KQ_TRY(check_ws(workspace, workspace_bytes,
                  quantize_workspace_bytes(d_out, d_in, block, dxx != nullptr)));
  KQ_TRY(kronq_device_check());
  return run_quantize(w, k, dxx, d_out, d_in, bits, block, group, codes, scale, zero, w_hat,
                      workspace, reinterpret_cast<cudaStream_t>(stream));
}

// ----------------------------------------------------------------------------- two-sided
size_t kronq_quantize_layer_twosided_workspace_size(int32_t d_out, int32_t d_in) {
  if (d_out <= 0 || d_in <= 0) return 0;
  return twosided_workspace_bytes(d_out, d_in);
}

kronq_status kronq_quantize_layer_twosided(const float* w, const float* k_in, const float* k_out,
                                           int32_t d_out, int32_t d_in, int32_t bits,
                                           uint8_t* codes, float* scale, float* zero,
                                           float* w_hat, int32_t* iterations, void* workspace,
                                           size_t workspace_bytes, kronq_stream_t stream) {
  if (d_out <= 0 || d_in <= 0) return fail(KRONQ_ERR_SHAPE, "d_out and d_in must be positive");
  if (!w || !k_in || !k_out || !codes || !scale || !zero || !w_hat)
    return fail(KRONQ_ERR_INVALID_ARG, "w, k_in, k_out, codes, scale, zero and w_hat are required");
  if (bits < 2 || bits > 8) return fail(KRONQ_ERR_UNSUPPORTED, "bits must be in 2..8");
  if (w == w_hat) return fail(KRONQ_ERR_INVALID_ARG, "w and w_hat must not alias");
  if (d_out > 65535 || d_in > 65535)
    return fail(KRONQ_ERR_SHAPE, "two-sided rounding takes at most 65535 rows and columns");
  KQ_TRY(check_ws(workspace, workspace_bytes, twosided_workspace_bytes(d_out, d_in)));
  KQ_TRY(kronq_device_check());
  return run_twosided(w, k_in, k_out, d_out, d_in, bits, codes, scale, zero, w_hat, iterations,
                      workspace, reinterpret_cast<cudaStream_t>(stream));
}

// ----------------------------------------------------------------------------- inference
size_t kronq_packed_codes_bytes(int32_t d_out, int32_t d_in, int32_t bits) {
  if (d_out <= 0 || d_in <= 0 || bits < 2 || bits > 4) return 0;
  return packed_code_bytes(d_out, d_in, bits);
}

kronq_status kronq_pack_codes(const uint8_t* codes, int32_t d_out, int32_t d_in, int32_t bits,
                              void* packed, size_t packed_bytes, kronq_stream_t stream) {
  if (d_out <= 0 || d_in <= 0) return fail(KRONQ_ERR_SHAPE, "d_out and d_in must be positive");
  if (bits < 2 || bits > 4) return fail(KRONQ_ERR_UNSUPPORTED, "packed codes have 2, 3 or 4 bits");
  if (!codes || !packed) return fail(KRONQ_ERR_INVALID_ARG, "codes and packed are required");
  if (!aligned(packed, 16)) return fail(KRONQ_ERR_INVALID_ARG, "packed not 16-byte aligned");
  if (packed_bytes < packed_code_bytes(d_out, d_in, bits))
    return fail(KRONQ_ERR_SHAPE, "packed buffer too small: %zu < %zu bytes", packed_bytes,
                packed_code_bytes(d_out, d_in, bits));
  KQ_TRY(kronq_device_check());
  return run_pack_codes(codes, d_out, d_in, bits, packed, reinterpret_cast<cudaStream_t>(stream));
}

size_t kronq_packed_grid_bytes(int32_t d_out, int32_t d_in, int32_t group) {
  if (d_out <= 0 || d_in <= 0 || (group != 0 && group != 128)) return 0;
  return packed_grid_bytes(d_out, d_in, group);
}

kronq_status kronq_pack_grid(const float* scale, const float* zero, int32_t d_out, int32_t d_in,
                             int32_t group, void* packed_grid, size_t packed_grid_bytes_,
                             kronq_stream_t stream) {
  if (d_out <= 0 || d_in <= 0) return fail(KRONQ_ERR_SHAPE, "d_out and d_in must be positive");
  if (group != 0 && group != 128)
    return fail(KRONQ_ERR_UNSUPPORTED, "group must be 0 (per row) or 128");
  if (!scale || !zero || !packed_grid)
    return fail(KRONQ_ERR_INVALID_ARG, "scale, zero and packed_grid are required");
  if (!aligned(packed_grid, 8)) return fail(KRONQ_ERR_INVALID_ARG, "packed_grid not 8-byte aligned");
  if (packed_grid_bytes_ < packed_grid_bytes(d_out, d_in, group))
    return fail(KRONQ_ERR_SHAPE, "packed_grid too small: %zu < %zu bytes", packed_grid_bytes_,
                packed_grid_bytes(d_out, d_in, group));
  KQ_TRY(kronq_device_check());
  return run_pack_grid(scale, zero, d_out, d_in, group, packed_grid,
                       reinterpret_cast<cudaStream_t>(stream));
}

size_t kronq_qlinear_workspace_size(int32_t d_out, int32_t d_in, int32_t n_tok) {
  if (d_out <= 0 || d_in <= 0 || n_tok <= 0) return 0;
  return qlinear_workspace_bytes(d_out, d_in, n_tok);
}

kronq_status kronq_qlinear(const void* x, int32_t x_dtype, int64_t ld_x, int32_t n_tok,
                           const void* packed, const void* packed_grid, int32_t group, const float* s_x, const float* s_g,
                           const int8_t* sign_in, const int8_t* sign_out, uint32_t flags,
                           int32_t d_out, int32_t d_in, int32_t bits, float* y, int64_t ld_y,
                           void* workspace, size_t workspace_bytes, kronq_stream_t stream) {
  if (d_out <= 0 || d_in <= 0 || n_tok < 0)
    return fail(KRONQ_ERR_SHAPE, "d_out, d_in must be positive and n_tok >= 0");
  if (bits < 2 || bits > 4) return fail(KRONQ_ERR_UNSUPPORTED, "packed codes have 2, 3 or 4 bits");
  if (group != 0 && group != 128)
    return fail(KRONQ_ERR_UNSUPPORTED, "group must be 0 (per row) or 128");
  if (flags & ~static_cast<uint32_t>(KRONQ_BIIP_FULL))
    return fail(KRONQ_ERR_INVALID_ARG, "flags may only hold the four transform bits");
  if (x_dtype != KRONQ_DTYPE_BF16 && x_dtype != KRONQ_DTYPE_F32)
    return fail(KRONQ_ERR_INVALID_ARG, "x_dtype must be KRONQ_DTYPE_BF16 or KRONQ_DTYPE_F32");
  if (n_tok == 0) return KRONQ_OK;
  if (!x || !packed || !packed_grid || !y)
    return fail(KRONQ_ERR_INVALID_ARG, "x, packed, packed_grid and y are required");
  if ((flags & KRONQ_BIIP_SCALE_IN) && !s_x) return fail(KRONQ_ERR_INVALID_ARG, "s_x is NULL");
  if ((flags & KRONQ_BIIP_SCALE_OUT) && !s_g) return fail(KRONQ_ERR_INVALID_ARG, "s_g is NULL");
  if ((flags & KRONQ_BIIP_ROTATE_IN) && !sign_in)
    return fail(KRONQ_ERR_INVALID_ARG, "sign_in is NULL");
  if ((flags & KRONQ_BIIP_ROTATE_OUT) && !sign_out)
    return fail(KRONQ_ERR_INVALID_ARG, "sign_out is NULL");
  if (ld_x < d_in || ld_y < d_out) return fail(KRONQ_ERR_SHAPE, "row stride below the width");
  if (!aligned(x, x_dtype == KRONQ_DTYPE_BF16 ? 2 : 4) || !aligned(y, 4))
    return fail(KRONQ_ERR_INVALID_ARG, "x or y not aligned to its element size");
  if (!aligned(packed, 16)) return fail(KRONQ_ERR_INVALID_ARG, "packed not 16-byte aligned");
  if (!aligned(packed_grid, 16))
    return fail(KRONQ_ERR_INVALID_ARG, "packed_grid not 16-byte aligned");
  const int b_in = d_in & (-d_in), b_out = d_out & (-d_out);
  if (((flags & KRONQ_BIIP_ROTATE_IN) && b_in > 16384) ||
      ((flags & KRONQ_BIIP_ROTATE_OUT) && b_out > 16384))
    return fail(KRONQ_ERR_UNSUPPORTED, "Hadamard blocks above 16384 are not supported");
  KQ_TRY(check_ws(workspace, workspace_bytes, qlinear_workspace_bytes(d_out, d_in, n_tok)));
  KQ_TRY(kronq_device_check());
  QlinearArgs q;
  q.x = x;
  q.x_dtype = x_dtype;
  q.ld_x = ld_x;
  q.n_tok = n_tok;
  q.packed = packed;
  q.grid = packed_grid;
  q.group = group;
  q.s_x = s_x;
  q.s_g = s_g;
  q.sign_in = sign_in;
  q.sign_out = sign_out;
  q.flags = flags;
  q.d_out = d_out;
  q.d_in = d_in;
  q.bits = bits;
  q.y = y;
  q.ld_y = ld_y;
  return run_qlinear(q, workspace, reinterpret_cast<cudaStream_t>(stream));
}

// ----------------------------------------------------------------------------- allocation
kronq_status kronq_score_allocate(const double* tr_hx, const double* tr_hg,
                                  const int64_t* n_params, int32_t L, const int32_t* choices,
                                  int32_t n_choices, double avg_bits, double* score_out,
                                  int32_t* bits_out) {
  if (L <= 0 || n_choices <= 0) return fail(KRONQ_ERR_SHAPE, "L and n_choices must be positive");
  if (!tr_hx || !tr_hg || !n_params || !choices || !bits_out)
    return fail(KRONQ_ERR_INVALID_ARG, "null pointer");
  std::vector<double> s(L);
  int64_t total = 0;
  for (int l = 0; l < L; ++l) {
    s[l] = tr_hg[l] * tr_hx[l];
    if (std::isnan(s[l])) return fail(KRONQ_ERR_INVALID_ARG, "score of sublayer %d is NaN", l);
    if (n_params[l] < 0) return fail(KRONQ_ERR_SHAPE, "n_params[%d] < 0", l);
    total += n_params[l];
  }
  std::vector<int32_t> ch(choices, choices + n_choices);
  std::sort(ch.begin(), ch.end());
  ch.erase(std::unique(ch.begin(), ch.end()), ch.end());
  if (ch.front() <= 0) return fail(KRONQ_ERR_INVALID_ARG, "bit widths must be positive");
  const int64_t budget = static_cast<int64_t>(std::floor(avg_bits * static_cast<double>(total)));
  int64_t used = static_cast<int64_t>(ch.front()) * total;
  if (used > budget)
    return fail(KRONQ_ERR_INVALID_ARG, "budget %lld bits is below the smallest width",
                (long long)budget);
  std::vector<int> order(L);
  for (int l = 0; l < L; ++l) order[l] = l;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
    if (s[a] != s[b]) return s[a] > s[b];
    return a < b;
  });
  for (int l = 0; l < L; ++l) bits_out[l] = ch.front();
  for (int l : order) {
    for (auto it = ch.rbegin(); it != ch.rend(); ++it) {
      const int b = *it;
      if (b <= bits_out[l]) break;
      const int64_t extra = static_cast<int64_t>(b - bits_out[l]) * n_params[l];
      if (used + extra <= budget) {
        used += extra;
        bits_out[l] = b;
        break;
      }
    }
  }
  if (score_out)
    for (int l = 0; l < L; ++l) score_out[l] = s[l];
  return KRONQ_OK;
}

}  // extern "C"
