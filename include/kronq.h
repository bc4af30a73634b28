/*
 * kronq.h - C ABI of the KronQ per-layer quantization hot path on NVIDIA B200 (sm_100a).
 *
 * KronQ quantizes one linear layer y = W x (W: d_out x d_in) with a Kronecker-factored
 * Hessian H ~ H_X (x) H_G, bidirectional incoherence processing (BiIP), a damped inverse
 * Cholesky factor and a column-wise OBS/GPTAQ solve, and ranks sublayers by
 * s = tr(H_G) * tr(H_X) for mixed precision. Sources of each operation are cited per call:
 *   [KronQ-hyper] "KronQ: LLM Quantization via Kronecker-Factored Hessian", hyper.ai summary,
 *                 Method section (the page that prints the equations);
 *   [KronQ-gist]  the same paper, gist.science technical summary (Methodology, Results).
 *
 * Conventions shared by every call
 *   - Matrices are row-major. Pointers marked (device) are CUDA device pointers owned by the
 *     caller; (host) pointers are ordinary host memory owned by the caller. The library never
 *     frees or retains a pointer after the call returns.
 *   - The library allocates no device memory. Calls that need scratch space take a caller
 *     workspace (device, 256-byte aligned) whose minimum size is returned by the matching
 *     kronq_*_workspace_size() query. A smaller workspace gives KRONQ_ERR_WORKSPACE.
 *   - Device work is enqueued on `stream` and is asynchronous unless stated otherwise. A status
 *     other than KRONQ_OK means nothing was enqueued (argument errors) or a CUDA launch failed;
 *     faults of earlier asynchronous work surface as KRONQ_ERR_CUDA at a later call.
 *   - bf16 arrays are IEEE bfloat16 (1 sign, 8 exponent, 7 mantissa bits) stored as uint16.
 *   - kronq_last_error_detail() returns a thread-local text of the last failure of this thread.
 *   - All entry points are safe to call from several host threads on distinct streams; calls
 *     that share output buffers must be ordered by the caller.
 */
#ifndef KRONQ_H_
#define KRONQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KRONQ_API __attribute__((visibility("default")))
#else
#define KRONQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream; binary-compatible with cudaStream_t / CUstream (NULL = legacy stream). */
typedef struct CUstream_st* kronq_stream_t;

typedef enum kronq_status {
  KRONQ_OK = 0,
  KRONQ_ERR_INVALID_ARG = 1,  /* null pointer, bad enum, misaligned pointer or stride */
  KRONQ_ERR_SHAPE = 2,        /* non-positive or inconsistent sizes */
  KRONQ_ERR_NOT_PD = 3,       /* damped H_X not positive definite (kronq_cholinv) */
  KRONQ_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  KRONQ_ERR_WORKSPACE = 5,    /* workspace pointer null/misaligned or smaller than required */
  KRONQ_ERR_UNSUPPORTED = 6,  /* device is not sm_100 or a parameter is outside the supported range */
  KRONQ_ERR_TIMEOUT = 7       /* a kernel gave up a bounded wait (see kronq_device_error) */
} kronq_status;

/* Element types of the weight input of kronq_biip. */
enum { KRONQ_DTYPE_BF16 = 0, KRONQ_DTYPE_F32 = 1 };

/* Flags of kronq_biip ([KronQ-hyper] Method, BiIP equations). */
enum {
  KRONQ_BIIP_SCALE_IN = 1,    /* W <- W S_X,  S_X = diag(H_X,jj / |W_:,j|^2)^(1/4)          */
  KRONQ_BIIP_SCALE_OUT = 2,   /* W <- S_G W,  S_G = diag(H_G,ii / |W_i,:|^2)^(1/4)          */
  KRONQ_BIIP_ROTATE_IN = 4,   /* W <- W V^T,  H_X <- V H_X V^T, dXX^T <- V dXX^T V^T         */
  KRONQ_BIIP_ROTATE_OUT = 8,  /* W <- U W,    H_G <- U H_G U^T                               */
  KRONQ_BIIP_WRITE_HG = 16,   /* also write the normalised, transformed H_G into `hg`        */
  KRONQ_BIIP_HG_DIAG = 32,    /* `hg` is only the d_out diagonal sums (kronq_accumulate_diag) */
  KRONQ_BIIP_FULL = 15        /* the four transforms of BiIP                                  */
};

/* Flags of kronq_cholinv. */
enum { KRONQ_CHOLINV_SYNC = 1 };

KRONQ_API const char* kronq_status_string(kronq_status status);
KRONQ_API const char* kronq_last_error_detail(void);
KRONQ_API int kronq_version(void);

/* Checks that the current CUDA device is a compute-capability 10.0 (B200-class) GPU. */
KRONQ_API kronq_status kronq_device_check(void);

/* Number of kernels this library has launched in this process (all devices, all threads). */
KRONQ_API uint64_t kronq_launch_count(void);

/* SM budget for the persistent kernels (the statistics kernel of kronq_accumulate and the
 * tensor-core GEMMs inside kronq_cholinv and kronq_quantize_layer): launches made while a budget
 * of n > 0 is set use at most n CTAs, one per SM, so that work on other streams keeps the rest
 * of the GPU. 0 (the default) lifts it. Process-wide, read at launch time (a captured CUDA graph
 * keeps the grid it was captured with); it changes no result. Not a reservation: nothing stops
 * other kernels from using the budgeted SMs. */
KRONQ_API void kronq_set_sm_budget(int32_t sms);
KRONQ_API int32_t kronq_sm_budget(void);

/* Reads and clears the device-side error word (bounded waits that gave up). Synchronizes
 * `stream`. *code_out = 0 when no kernel reported an error since the last call, else the first
 * code recorded: 1 a TMA producer found no free pipeline stage, 2 a tensor-core issuer waited for
 * operands or an accumulator, 3 an epilogue waited for an accumulator, 4 a streaming pass (the
 * Hadamard passes of kronq_biip) waited for a tile load. Each wait gives up after 4 s; the kernel
 * then lets its copies in flight land and returns, leaving its outputs incomplete. */
KRONQ_API kronq_status kronq_device_error(int32_t* code_out, kronq_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * 1. kronq_accumulate - Kronecker-factor sums over calibration tokens.
 *
 * [KronQ-hyper] Method: for y = W x with g = dL/dy, the empirical Fisher is
 * E[x x^T (x) g g^T] ~ H_X (x) H_G with H_X = E[x x^T], H_G = E[g g^T]; the asymmetric
 * (GPTAQ) objective adds the input-drift term dX X^T. This call adds, over n tokens,
 *     hx_sum  += X~^T X~            (d_in x d_in)   if hx_sum  != NULL
 *     hg_sum  += G^T G              (d_out x d_out) if hg_sum  != NULL
 *     dxx_sum += (X - X~)^T X~      (d_in x d_in)   if dxx_sum != NULL
 * where X~ (xq) is the input the quantized layer sees and X (xfp) the full-precision input.
 * The sums are un-normalised (divide by the total token count later, see kronq_biip).
 *
 *   xq, xfp  (device, bf16) n x d_in, row stride ld_xq / ld_xfp elements (one token per row)
 *   g        (device, bf16) n x d_out, row stride ld_g
 *   hx_sum, dxx_sum (device, fp32) d_in x d_in contiguous; hg_sum d_out x d_out contiguous.
 *            Both triangles of hx_sum / hg_sum are valid on return (symmetric).
 *   Requirements: strides >= width, stride*2 bytes a multiple of 16, base pointers 16-byte
 *   aligned; hx_sum needs xq; dxx_sum needs xq and xfp; hg_sum needs g. n = 0 is a no-op.
 *   Accumulation: bf16 products (exact), fp32 sums on tcgen05 tensor cores. For the drift
 *   term, X~ and X - X~ are first rescaled by powers of two chosen from their largest magnitude
 *   over the n tokens and converted to fp16: X~ stays exact, X - X~ is rounded once to 2^-11
 *   relative; the fp16 products are summed in fp32 and the rescale is undone exactly. Inputs
 *   must be finite. Scratch for the drift term (kronq_accumulate_workspace_size): 256 bytes
 *   plus two fp16 copies of up to 32768 tokens of width d_in.
 * ------------------------------------------------------------------------------------- */
KRONQ_API size_t kronq_accumulate_workspace_size(int64_t n, int32_t d_in, int32_t d_out, int with_dxx);
KRONQ_API kronq_status kronq_accumulate(const void* xq, int64_t ld_xq, const void* xfp, int64_t ld_xfp,
                              const void* g, int64_t ld_g, int64_t n, int32_t d_in,
                              int32_t d_out, float* hx_sum, float* hg_sum, float* dxx_sum,
                              void* workspace, size_t workspace_bytes, kronq_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * 1b. kronq_accumulate_diag - the diagonal of H_G alone.
 *
 * [KronQ-hyper] Method: S_G (BiIP equations) and the sensitivity tr(H_G) read only the diagonal
 * of H_G, and Proposition 1 takes H_G out of the column update. A caller that quantizes without
 * evaluating the objective or the incoherence of H_G therefore needs diag(G^T G) only. This call
 * adds, over n tokens,
 *     diag_sum[j] += sum_t G[t][j]^2        (j < d)
 * in one streaming read of G instead of the G^T G product. Pass the result to kronq_biip as `hg`
 * with KRONQ_BIIP_HG_DIAG.
 *
 *   g         (device, bf16) n x d, row stride ld_g elements (ld_g >= d, ld_g*2 bytes a multiple
 *             of 16, base 16-byte aligned); one token per row
 *   diag_sum  (device, fp32) d entries, += the column sums of squares (un-normalised)
 *   workspace kronq_accumulate_diag_workspace_size(n, d) bytes (partial sums of blocks of 2048
 *             tokens); NULL when that size is 0. n = 0 is a no-op.
 *   Accumulation: squares of bf16 values are exact in fp32; each block of 2048 tokens is summed
 *   in fp32, the blocks are added in a fixed order in fp64, so the result does not depend on
 *   scheduling.
 * ------------------------------------------------------------------------------------- */
KRONQ_API size_t kronq_accumulate_diag_workspace_size(int64_t n, int32_t d);
KRONQ_API kronq_status kronq_accumulate_diag(const void* g, int64_t ld_g, int64_t n, int32_t d,
                                             float* diag_sum, void* workspace,
                                             size_t workspace_bytes, kronq_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * 2. kronq_biip - normalisation and bidirectional incoherence processing of one sublayer.
 *
 * [KronQ-hyper] Method, BiIP equations:
 *     W <- S_G W S_X,  S_X = diag([H_X]_jj / |W_:,j|^2)^(1/4),  S_G = diag([H_G]_ii / |W_i,:|^2)^(1/4)
 *     W <- U W V^T,  H_X <- V H_X V^T,  H_G <- U H_G U^T,  dXX^T <- V dXX^T V^T
 * with U, V random-sign Hadamard transforms, here U = (1/sqrt(b)) (I (x) H_b) diag(sign_out)
 * (Sylvester H_b, b = largest power of two dividing d_out) and V likewise on the input side.
 * The Hessians follow the diagonal scaling as H_X <- S_X^-1 H_X S_X^-1 (same for dXX^T) and
 * H_G <- S_G^-1 H_G S_G^-1, which leaves tr[H_G dW H_X dW^T] unchanged. Both scales use the
 * original W; a zero norm or zero diagonal gives scale 1. Also returns the traces used by the
 * sensitivity score s = tr(H_G) tr(H_X) ([KronQ-hyper] Method: sensitivity), taken after BiIP.
 *
 *   w        (device) d_out x d_in, w_dtype KRONQ_DTYPE_BF16 or KRONQ_DTYPE_F32; not modified
 *   w_out    (device, fp32) d_out x d_in: W' = U S_G W S_X V^T
 *   hx       (device, fp32) d_in x d_in: in: raw sum X~^T X~; out: V S_X^-1 (inv_n hx) S_X^-1 V^T
 *   hg       (device, fp32) d_out x d_out raw sum G^T G, or NULL (then SCALE_OUT is invalid).
 *            Read-only unless KRONQ_BIIP_WRITE_HG, in which case it is replaced by
 *            U S_G^-1 (inv_n hg) S_G^-1 U^T. With KRONQ_BIIP_HG_DIAG it is instead the d_out
 *            raw diagonal sums from kronq_accumulate_diag: S_G and tr_hg need only those, and
 *            WRITE_HG is then invalid.
 *   dxx      (device, fp32) d_in x d_in raw drift sum or NULL; out: V S_X^-1 (inv_n dxx) S_X^-1 V^T
 *   inv_n    1 / total token count
 *   sign_in  (device, int8 +-1) d_in; needed with ROTATE_IN. sign_out likewise d_out.
 *   s_x, s_g (device, fp32) d_in / d_out diagonal scales (1 where the flag is off)
 *   tr_hx, tr_hg (device, fp64, one element each): traces after BiIP; tr_hg may be NULL and is
 *            left untouched when hg is NULL.
 * ------------------------------------------------------------------------------------- */
KRONQ_API size_t kronq_biip_workspace_size(int32_t d_out, int32_t d_in);
KRONQ_API kronq_status kronq_biip(const void* w, int32_t w_dtype, float* w_out, float* hx, float* hg,
                        float* dxx, double inv_n, const int8_t* sign_in, const int8_t* sign_out,
                        int32_t d_out, int32_t d_in, uint32_t flags, float* s_x, float* s_g,
                        double* tr_hx, double* tr_hg, void* workspace, size_t workspace_bytes,
                        kronq_stream_t stream);

/* kronq_biip_noalloc - kronq_biip for callers that cannot allocate device memory.
 *
 * The paper has no counterpart to this call; it exists for deployment. Some callers cannot call
 * cudaMalloc or hand the library a workspace: code running while a CUDA graph is being captured,
 * plug-ins and host runtimes that only see buffers handed to them by their host framework, and
 * services that reserve all device memory up front. This variant takes the same arguments as
 * kronq_biip minus the workspace and uses a fixed scratch array of 1 MiB that lives in device
 * memory (every GPU that loads this library holds it until the process exits). That limits it
 * to about 16.03 * (d_out + d_in) + 2 KB <= 1 MiB (d_out + d_in up to about 65000, every LLaMA
 * shape); larger layers get KRONQ_ERR_UNSUPPORTED with the needed size in the error detail.
 * The first call on a device looks up the array's device address; make that first call before
 * any stream capture. All calls in the process share the one array, so calls whose execution
 * overlaps on the GPU (several streams or threads) race on it and must be ordered by the caller.
 * The array keeps the last call's contents; the call clears what it needs cleared itself. */
KRONQ_API kronq_status kronq_biip_noalloc(const void* w, int32_t w_dtype, float* w_out, float* hx,
                                          float* hg, float* dxx, double inv_n,
                                          const int8_t* sign_in, const int8_t* sign_out,
                                          int32_t d_out, int32_t d_in, uint32_t flags,
                                          float* s_x, float* s_g, double* tr_hx, double* tr_hg,
                                          kronq_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * 3. kronq_cholinv - damped inverse Cholesky factor.
 *
 * [KronQ-hyper] Method, OBS update: the rows "[H_X^-1]_p,p+1:" of the column update are the
 * rows of K, the upper-triangular factor with K^T K = (H_X + lambda I)^-1 (positive diagonal),
 * lambda = damp_rel * mean(diag H_X). Computed as a blocked reverse-order Cholesky
 * H_X + lambda I = R R^T (R upper) followed by a blocked triangular inverse K = R^-1.
 *
 *   h_to_k   (device, fp32) d x d, in: symmetric H_X (upper triangle read); out: K in the upper
 *            triangle, zeros below the diagonal.
 *   info     (device, int32): -1 when positive definite, else the index of the first pivot that
 *            was not positive (pivots are taken from the last index down).
 *   flags    KRONQ_CHOLINV_SYNC: synchronize `stream` and return KRONQ_ERR_NOT_PD when
 *            info >= 0. Without it the call is asynchronous and the caller reads info.
 *   On failure K is unspecified.
 * ------------------------------------------------------------------------------------- */
KRONQ_API size_t kronq_cholinv_workspace_size(int32_t d);
KRONQ_API kronq_status kronq_cholinv(float* h_to_k, int32_t d, float damp_rel, int32_t* info,
                           uint32_t flags, void* workspace, size_t workspace_bytes,
                           kronq_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * 4. kronq_quantize_layer - column-wise OBS / GPTAQ solve onto a b-bit per-row grid.
 *
 * [KronQ-hyper] Method, OBS update (H_G cancels, Proposition 1 - the solve takes no H_G):
 *     dW_:,p+1: = -delta_p [H_X^-1]_p,p+1: + W_:,p P_p,p+1:
 * with delta_p = (w_p - deq(q(w_p))) / K_pp, K from kronq_cholinv and P the GPTAQ correction
 * matrix, read as P = striu(D K^T) K with D the processed drift term (P = 0 when dxx is NULL).
 * Because the P term uses the weights before any update, it is applied up front: the solve runs
 * on W (I + P) and then proceeds in 128-column blocks with lazy trailing updates.
 * Grid: per output row, lo/hi = min/max of W (before the solve), scale = (hi - lo)/(2^bits - 1)
 * (1 if hi == lo), zero = rint(-lo/scale), code = clamp(rint(w/scale) + zero, 0, 2^bits - 1),
 * deq = scale * (code - zero), all in fp32 with round-half-to-even.
 *
 *   w        (device, fp32) d_out x d_in processed weights W' (from kronq_biip); not modified
 *   k        (device, fp32) d_in x d_in, upper triangle = K (from kronq_cholinv)
 *   dxx      (device, fp32) d_in x d_in processed drift term, or NULL
 *   bits     2..8;  block: column block width, 128 (others give KRONQ_ERR_UNSUPPORTED)
 *   group    0: one grid per output row, from W before the solve (as above);
 *            128 (= block): one grid per row and per 128 consecutive columns ([KronQ-hyper]
 *            Experiments, g = 128), taken when the solve reaches the group's first column from
 *            the weights it is about to quantize, i.e. the rows of W (I + P) after the updates
 *            of every earlier column (lo/hi over the group's columns, same formulas);
 *            other values give KRONQ_ERR_UNSUPPORTED
 *   codes    (device, uint8) d_out x d_in
 *   scale, zero (device, fp32) d_out each (group 0), or d_out x ceil(d_in / group) row-major
 *   w_hat    (device, fp32) d_out x d_in: dequantized weights W^ (also the solve's working copy)
 * ------------------------------------------------------------------------------------- */
KRONQ_API size_t kronq_quantize_layer_workspace_size(int32_t d_out, int32_t d_in, int32_t block,
                                           int with_dxx);
KRONQ_API kronq_status kronq_quantize_layer(const float* w, const float* k, const float* dxx,
                                  int32_t d_out, int32_t d_in, int32_t bits, int32_t block,
                                  int32_t group, uint8_t* codes, float* scale, float* zero,
                                  float* w_hat,
                                  void* workspace, size_t workspace_bytes,
                                  kronq_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * 5. kronq_score_allocate - sensitivity scores and mixed-precision bit allocation (host).
 *
 * [KronQ-hyper] Method: s_l = tr(H_G^(l)) * tr(H_X^(l)), computed after BiIP; sublayers with a
 * larger s get more bits. [KronQ-gist] Results: the higher-scored sublayer is upgraded first.
 * Rule: budget T = floor(avg_bits * sum n_l) bits; every sublayer starts at min(choices);
 * sublayers are visited by s descending (ties: lower index first) and each takes the largest
 * choice that keeps the total <= T. Deterministic, integer budget arithmetic.
 *
 *   tr_hx, tr_hg (host, fp64) L each; n_params (host, int64) L; choices (host) n_choices widths
 *   score_out (host, fp64) L, may be NULL; bits_out (host, int32) L
 *   Errors: KRONQ_ERR_INVALID_ARG for a NaN score or a budget below L * min(choices).
 * ------------------------------------------------------------------------------------- */
KRONQ_API kronq_status kronq_score_allocate(const double* tr_hx, const double* tr_hg,
                                  const int64_t* n_params, int32_t L, const int32_t* choices,
                                  int32_t n_choices, double avg_bits, double* score_out,
                                  int32_t* bits_out);

/* ---------------------------------------------------------------------------------------
 * 5b. Comparison variant (prior art, not KronQ): rounding with output-side feedback too.
 *
 * [YAQA notes], generalized LDLQ: for a Kronecker proxy H_O (x) H_I of the layer Hessian with
 * unit upper triangular factors L_O, L_I (H = L diag L^T) and L' = L - I, the quantized W^ is
 * the fixed point of
 *     W^ = Q(W + L_O'^T D L_I' + L_O'^T D + D L_I'),   D = W - W^,
 * reached within d_out + d_in - 1 updates of all elements at once. KronQ's own solve
 * (kronq_quantize_layer) keeps only the input side, the D L_I' term: with H_G it cancels
 * ([KronQ-hyper] Method, Proposition 1). This call takes H_I = H_X' and H_O = H_G' through their
 * damped inverse factors and exists to measure what the output side adds.
 *
 *   w        (device, fp32) d_out x d_in, W' from kronq_biip (contiguous)
 *   k_in     (device, fp32) d_in x d_in, kronq_cholinv of H_X' (upper, K^T K = (H_X'+lI)^-1)
 *   k_out    (device, fp32) d_out x d_out, kronq_cholinv of the full H_G' (kronq_biip with
 *            KRONQ_BIIP_WRITE_HG gives H_G')
 *   bits 2..8; grid: one per row from w (as kronq_quantize_layer with group 0)
 *   codes (uint8), scale, zero (d_out), w_hat (fp32): outputs as for kronq_quantize_layer
 *   iterations (host, may be NULL): the update passes run, the last one changing no code
 *   Arithmetic: L from the inverse factors (the inverse factor of K K^T is K^-1, U U^T = H +
 *   lambda I); each update is two fp32-accurate tensor-core products with the strictly
 *   triangular parts of L_I and L_O; decisions in fp32. Synchronizes `stream` once per update
 *   (it reads how many codes changed). d_out, d_in <= 65535.
 *   Errors: KRONQ_ERR_NOT_PD if k_in or k_out is not an invertible upper factor (its K K^T
 *   has a non-positive pivot); KRONQ_ERR_CUDA if no fixed point is reached within d_out + d_in
 *   updates.
 * ------------------------------------------------------------------------------------- */
KRONQ_API size_t kronq_quantize_layer_twosided_workspace_size(int32_t d_out, int32_t d_in);
KRONQ_API kronq_status kronq_quantize_layer_twosided(const float* w, const float* k_in,
                                                     const float* k_out, int32_t d_out,
                                                     int32_t d_in, int32_t bits, uint8_t* codes,
                                                     float* scale, float* zero, float* w_hat,
                                                     int32_t* iterations, void* workspace,
                                                     size_t workspace_bytes,
                                                     kronq_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * 6. The quantized layer at inference: packed codes and y = W^ x.
 *
 * [KronQ-gist] Limitations: once quantized, the layer's inference overhead is only the
 * orthogonal transforms (the same as QuIP#'s). The solve works on W' = U S_G W S_X V^T and
 * returns codes, scale, zero with W^' = scale (codes - zero); in the original basis the layer is
 *     y = S_G^-1 U^T W^' V S_X^-1 x,
 * computed here without forming W^ or W^' in memory: x is transformed, multiplied by the
 * packed codes as 8-bit integers, and the result transformed back.
 *
 * Packed code format (this library's storage, the pages fix none). Bits b = 2, 3 or 4. Rows
 * are cut into tiles of 128 and columns into groups of 128 (past the matrix: code 0). Tile t,
 * group g is one blob of 2048 b bytes at byte offset (t G + g) 2048 b, G = ceil(d_in / 128).
 *   Row strings: row r (0..127) of the blob owns a string of 16 b bytes, read as little-endian
 *   32-bit words w[0 .. 4b-1]. The string is stored in 8-byte pieces: byte 8 p + k of row r's
 *   string (p = 0 .. 2b-1, k = 0..7) is blob byte 1024 p + 8 r + k, so the 32 rows a warp
 *   reads at once are contiguous.
 *   Codes in the words: the code of column c (0..127 within the group) sits in byte lane
 *   j = c mod 4 of its word, so one mask gives the codes of four consecutive columns:
 *     b = 2: word floor(c / 16), bits 8 j + 2 q and 8 j + 2 q + 1, q = floor((c mod 16) / 4);
 *     b = 4: word floor(c / 8), bits 8 j + 4 q .. 8 j + 4 q + 3, q = floor((c mod 8) / 4);
 *     b = 3: with m = floor(c / 32), e = c mod 32: code bits 0 and 1 as for b = 2 in word
 *            3 m + floor(e / 16) (q = floor((e mod 16) / 4)); code bit 2 in word 3 m + 2 at
 *            bit 8 j + floor(e / 4).
 * ------------------------------------------------------------------------------------- */
/* Size in bytes of the packed form of a d_out x d_in code matrix (0 for an unsupported b). */
KRONQ_API size_t kronq_packed_codes_bytes(int32_t d_out, int32_t d_in, int32_t bits);

/* kronq_pack_codes - codes (device, uint8, d_out x d_in contiguous, each < 2^bits) -> packed
 * (device, 16-byte aligned, packed_bytes >= kronq_packed_codes_bytes). Bits 2, 3, 4; others
 * give KRONQ_ERR_UNSUPPORTED. Codes >= 2^bits are not checked (their extra bits spill into
 * neighbouring codes). */
KRONQ_API kronq_status kronq_pack_codes(const uint8_t* codes, int32_t d_out, int32_t d_in,
                                        int32_t bits, void* packed, size_t packed_bytes,
                                        kronq_stream_t stream);

/* kronq_pack_grid - the grid (scale, zero from kronq_quantize_layer: d_out values each for
 * group 0, d_out x ceil(d_in / 128) row-major for group 128) re-laid out for kronq_qlinear:
 * (scale, zero) fp32 pairs, tile by tile of 128 rows, and within a tile group by group (group
 * 128) or once (group 0): pair (t, g, r) at index (t G' + g) 128 + r, G' = ceil(d_in / 128) or 1;
 * rows past d_out hold (0, 0). packed_grid: device, 8-byte aligned, at least
 * kronq_packed_grid_bytes bytes (kronq_qlinear reads it with bulk copies and needs it 16-byte
 * aligned). The values are copied, not changed. */
KRONQ_API size_t kronq_packed_grid_bytes(int32_t d_out, int32_t d_in, int32_t group);
KRONQ_API kronq_status kronq_pack_grid(const float* scale, const float* zero, int32_t d_out,
                                       int32_t d_in, int32_t group, void* packed_grid,
                                       size_t packed_grid_bytes, kronq_stream_t stream);

/* kronq_qlinear - y = S_G^-1 U^T W^' V S_X^-1 x for n_tok tokens.
 *
 *   x        (device) n_tok x d_in, x_dtype KRONQ_DTYPE_BF16 or KRONQ_DTYPE_F32, row stride ld_x
 *            elements (>= d_in), aligned to its element size
 *   packed   (device, 16-byte aligned) codes in the packed format above
 *   packed_grid (device, 16-byte aligned) the grid from kronq_pack_grid with the same group
 *   s_x, s_g, sign_in, sign_out, flags: the transforms of kronq_biip (KRONQ_BIIP_SCALE_IN,
 *            _SCALE_OUT, _ROTATE_IN, _ROTATE_OUT; a flag that is off drops its factor and its
 *            pointer may be NULL). Hadamard blocks up to 16384.
 *   y        (device, fp32) n_tok x d_out, row stride ld_y (>= d_out)
 *   Tokens are processed 32 at a time; each pass of up to 32 tokens reads the packed codes
 *   once. Deterministic: the same inputs give the same bits.
 *   Arithmetic: x' = V S_X^-1 x in fp32; each 128-column group of x' and each token is written
 *   as three int8 terms, x' ~ s (q0 + q1 / 128 + q2 / 128^2) with a power-of-two s per group and
 *   token (relative error about 1e-6 of the group's largest entry). The codes multiply the terms
 *   exactly in int32: with 1 or 2 tokens on the CUDA cores (dp4a, u8 codes x s8 terms), with 3
 *   to 32 tokens on the tensor cores (tcgen05.mma kind::i8, codes as the A operand in tensor
 *   memory). The grid, zero point, group scale and output transforms are applied in fp32.
 * ------------------------------------------------------------------------------------- */
KRONQ_API size_t kronq_qlinear_workspace_size(int32_t d_out, int32_t d_in, int32_t n_tok);
KRONQ_API kronq_status kronq_qlinear(const void* x, int32_t x_dtype, int64_t ld_x, int32_t n_tok,
                                     const void* packed, const void* packed_grid,
                                     int32_t group, const float* s_x, const float* s_g,
                                     const int8_t* sign_in, const int8_t* sign_out,
                                     uint32_t flags, int32_t d_out, int32_t d_in, int32_t bits,
                                     float* y, int64_t ld_y, void* workspace,
                                     size_t workspace_bytes, kronq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KRONQ_H_ */
