/*
 * aqnf4.h -- C ABI of libaqnf4: the per-layer NF4 pass on NVIDIA B200 (sm_100a).
 *
 * The pass quantizes each linear layer of a model to 4-bit NormalFloat (NF4) in blocks of
 * 64 elements, double-quantizes the per-block absmax constants to 8 bits in blocks of 256,
 * measures each layer's relative reconstruction error, and picks the K largest-error layers
 * to stay in 16 bits within a byte budget.  A standalone NF4 -> 16-bit dequantization comes with it.
 *
 * Sources (page title, section):
 *   "QLoRA" (ai360xpert.com), "How It Works": NF4 spreads the weights evenly over its 16
 *       values; the per-block scales get an 8-bit encoding of their own, worth about 0.37
 *       bits per weight; training turns the 4-bit weights back into 16-bit values whenever
 *       a pass needs them.
 *   "QLoRA Explained" (devtoolshub.net), "NF4", "Double Quantization".
 *   arxivdaily 2608.23816, "English abstract": a single sweep over the weights orders the
 *       layers by their NF4 error and holds the highest-error ones in 16 bits, as many as a
 *       byte budget allows.
 *   "AQLoRA: A Zero-Search Recipe for Fast Quantized LoRA Fine-Tuning", "Technical Details":
 *       every layer is ranked; the memory budget is configurable.
 *
 * Conventions for every call:
 *   - The caller owns every buffer.  The library allocates nothing and frees nothing; the one
     exception is the fixed scratch array that aqnf4_layer_error_noalloc uses (8 MiB of
     static device memory per device, with its address cached per device after the first
     call; the cache is not refreshed after cudaDeviceReset).
 *   - Pointers named "device" must be CUDA device (or managed) memory of the current device.
 *   - Calls with a stream argument are asynchronous on that stream (0 = legacy default
 *     stream).  The returned status covers the synchronous argument checks and the launch;
 *     data-dependent conditions are reported through a device flag word (below).
 *   - dev_flag (optional, device int32): when any input element is NaN or infinite the
 *     kernels store AQNF4_ERR_NONFINITE there; nothing is stored otherwise, so the caller
 *     zeroes it before the call and reads it after synchronizing.  The outputs of such a
 *     block are still written (see aqnf4_quantize) but are not meaningful.
 *   - 16-bit weights are either IEEE binary16 (AQNF4_F16) or bfloat16 (AQNF4_BF16).
 *   - Layout of the NF4 data of an n-element tensor (flattened row-major):
 *       packed  uint8[ceil(n/2)]   byte i = code[2i] << 4 | code[2i+1]; an odd n leaves the
 *                                  low nibble of the last byte 0.
 *       absmax  float[ceil(n/64)]  max |x| of each 64-element block (the last may be short).
 *       codes8  uint8[ceil(n/64)]  double-quantized absmax, see aqnf4_double_quant.
 *       scales  float[ceil(ceil(n/64)/256)]
 *   - Codes index the ascending 16-level codebook returned by aqnf4_codebook; code 7 is the
 *     exact zero.
 */
#ifndef AQNF4_H
#define AQNF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* cudaStream_t;

#if defined(__GNUC__)
#define AQNF4_API __attribute__((visibility("default")))
#else
#define AQNF4_API
#endif

typedef enum {
  AQNF4_OK = 0,
  AQNF4_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad count or budget */
  AQNF4_ERR_ALIGNMENT = 2,   /* a pointer lacks the alignment stated for it */
  AQNF4_ERR_DTYPE = 3,       /* dtype is neither AQNF4_F16 nor AQNF4_BF16 */
  AQNF4_ERR_NONFINITE = 4,   /* (device flag only) an input element is NaN or infinite */
  AQNF4_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed */
  AQNF4_ERR_TIMEOUT = 6,     /* (device flag only) a bounded wait inside a kernel ran out */
  AQNF4_ERR_WORKSPACE = 7    /* workspace missing, misaligned or smaller than required */
} aqnf4_status;

typedef enum { AQNF4_F16 = 0, AQNF4_BF16 = 1 } aqnf4_dtype;

/* aqnf4_layer.flags bits. */
enum {
  /* Score the layer as NF4 + double quantization stores it ("QLoRA", "How It Works": the
     block scales are themselves stored at 8 bits): w_hat is rebuilt from the DQ constant
     a'_b = fl(fl(code8_b / 255) * s) of its block, exactly what aqnf4_dequantize returns
     from packed + codes8 + scales, instead of the binary32 absmax a_b.  The codes, packed
     bytes, absmax, codes8 and scales written are the same either way. */
  AQNF4_SCORE_DQ_ABSMAX = 1,
  /* Score the layer as NF4 with mean-centred double quantization would store it
     (aqnf4_double_quant_centered, a format from outside the pages): w_hat is rebuilt from
     a'_b = fl(fl(fl((code8_b - 128) / 127) * h) + mu) of its DQ block, exactly what
     aqnf4_dequantize_centered returns.  The stored outputs are still the plain format's.
     At most one of the two score flags may be set. */
  AQNF4_SCORE_DQ_CENTERED = 2
};

/* One linear layer for aqnf4_layer_error.  All pointers are device pointers.
   w      : numel 16-bit weights, 16-byte aligned (required).
   packed : optional output, ceil(numel/2) bytes, 16-byte aligned.
   absmax : optional output, ceil(numel/64) floats, 4-byte aligned.
   codes8 : optional output, ceil(numel/64) bytes (double-quantized absmax).
   scales : optional output, ceil(ceil(numel/64)/256) floats, 4-byte aligned; required
            when codes8 is given, ignored otherwise. */
typedef struct {
  const void* w;
  int64_t numel;
  int32_t dtype; /* aqnf4_dtype */
  int32_t flags; /* AQNF4_SCORE_* bits; other bits must be 0 */
  uint8_t* packed;
  float* absmax;
  uint8_t* codes8;
  float* scales;
} aqnf4_layer;

/* Human-readable name of a status code (static string). */
AQNF4_API const char* aqnf4_status_string(aqnf4_status st);

/* The NF4 codebook ("QLoRA", "How It Works"; "QLoRA Explained", "NF4").  Host only.
   levels[16]: ascending, levels[0] = -1, levels[7] = 0 exactly, levels[15] = +1.  The 8
   positive levels are standard-normal quantiles at probabilities spaced evenly from 1/2
   (excluded) to p_max, the 7 negative ones likewise, all divided by the quantile of p_max;
   computed in binary64 and rounded to binary32.
   mids[15]: mids[j] = binary32 rounding of (levels[j] + levels[j+1]) / 2 taken in binary64.
   p_max <= 0 selects the default 1 - (1/32 + 1/30)/2, which the kernels use.
   Returns AQNF4_ERR_INVALID_ARG for null pointers or p_max outside (1/2, 1). */
AQNF4_API aqnf4_status aqnf4_codebook(double p_max, float levels[16], float mids[15]);

/* Blockwise absmax NF4 quantization of one tensor ("QLoRA", "How It Works").
   w (device, 16-byte aligned): n elements of dtype.  For each 64-element block b:
     a_b = max |x| (NaN if any element is NaN);
     v = fl(x * fl(1/a_b)) (a block with a_b below 2^-126 is scaled by 2^64 first; a block
         with a_b = 0 gets code 7 throughout);
     code = number of midpoints m_j with v > m_j.
   packed (device, 16-byte aligned, ceil(n/2) bytes) and absmax (device, 4-byte aligned,
   ceil(n/64) floats) are outputs; either may be NULL.  dev_flag may be NULL.
   Errors: INVALID_ARG (w NULL, n < 1), ALIGNMENT, DTYPE, CUDA. */
AQNF4_API aqnf4_status aqnf4_quantize(const void* w, int32_t dtype, int64_t n, uint8_t* packed,
                            float* absmax, int32_t* dev_flag, cudaStream_t stream);

/* Double quantization of an absmax array ("QLoRA", "How It Works": the block scales get
   an 8-bit encoding of their own; "QLoRA Explained", "Double Quantization").
   absmax (device, 4-byte aligned): nb constants.  For each block of 256 constants
   s = max a (NaN if any is NaN) is stored in scales[d] and each constant becomes
   code8 = round_half_even(fl(fl(a / s) * 255)); s = 0 gives codes 0; a NaN or infinite s
   gives codes 0 and sets dev_flag.  Storage per parameter: 8/64 + 32/(64*256) bits instead
   of 32/64, i.e. 0.373 bits saved.
   codes8 (device, nb bytes), scales (device, 4-byte aligned, ceil(nb/256) floats).
   Errors: INVALID_ARG (NULL pointer, nb < 1), ALIGNMENT, CUDA. */
AQNF4_API aqnf4_status aqnf4_double_quant(const float* absmax, int64_t nb, uint8_t* codes8,
                                float* scales, int32_t* dev_flag, cudaStream_t stream);

/* NF4 -> 16-bit dequantization ("QLoRA", "How It Works": the 16-bit values training computes
   with are rebuilt from the 4-bit storage when needed).
   packed (device, 16-byte aligned): ceil(n/2) bytes.  The block constant is
   a' = fl(fl(code8/255) * scales[b/256]) when codes8 is non-NULL (then scales is required),
   else a' = absmax[b].  out[i] = dtype_rn(fl(levels[code_i] * a')).
   out (device, 16-byte aligned): n elements of out_dtype.
   Errors: INVALID_ARG (NULL pointers, n < 1), ALIGNMENT, DTYPE, CUDA. */
AQNF4_API aqnf4_status aqnf4_dequantize(const uint8_t* packed, const uint8_t* codes8,
                              const float* scales, const float* absmax, int64_t n,
                              int32_t out_dtype, void* out, cudaStream_t stream);

/* Mean-centred double quantization, a second storage format for the block constants.  The
   pages give only the 0.37-bit saving ("QLoRA", "How It Works"); centring the constants on
   their mean before a symmetric 8-bit code is a reading from outside them, offered as an
   option beside aqnf4_double_quant.  Per block of 256 constants (the last may be short,
   len of them): S = their binary64 sum over a balanced binary tree of the 256 slots in index
   order (missing slots hold +0); mean mu = fl32(fl64(S / len)); h = max |fl(a - mu)|;
   code8 = rint_even(fl(fl(fl(a - mu) / h) * 127)) + 128 in [1, 255] (h = 0: 128).  The
   constant rebuilt is a' = fl(fl(fl((code8 - 128) / 127) * h) + mu).  Storage: 8/64 +
   64/(64*256) bits per weight (0.371 below binary32 constants).
   absmax (device, 4-byte aligned, nb floats) in; codes8 (device, nb bytes), scales = h and
   means = mu (device, 4-byte aligned, ceil(nb/256) floats each) out.  A NaN or infinite
   constant makes its block's mu or h non-finite: the block's codes are 0 and dev_flag
   (optional) receives AQNF4_ERR_NONFINITE.
   Errors: INVALID_ARG (NULL pointer, nb < 1), ALIGNMENT, CUDA. */
AQNF4_API aqnf4_status aqnf4_double_quant_centered(const float* absmax, int64_t nb,
                                                   uint8_t* codes8, float* scales, float* means,
                                                   int32_t* dev_flag, cudaStream_t stream);

/* NF4 -> 16-bit dequantization from mean-centred DQ storage (aqnf4_double_quant_centered):
   as aqnf4_dequantize with the block constant a' = fl(fl(fl((code8 - 128) / 127) *
   scales[b/256]) + means[b/256]).  All pointers required; packed and out 16-byte aligned,
   scales and means 4-byte aligned.  Errors: INVALID_ARG, ALIGNMENT, DTYPE, CUDA. */
AQNF4_API aqnf4_status aqnf4_dequantize_centered(const uint8_t* packed, const uint8_t* codes8,
                                                 const float* scales, const float* means,
                                                 int64_t n, int32_t out_dtype, void* out,
                                                 cudaStream_t stream);

/* Bytes of device workspace aqnf4_layer_error needs for these layers (host only; 0 when
   the arguments are invalid). */
AQNF4_API size_t aqnf4_workspace_size(const aqnf4_layer* layers, int32_t num_layers);

/* The AQLoRA scoring pass (arxivdaily 2608.23816, "English abstract": layers ranked by NF4
   reconstruction error), fused with NF4 quantization, packing and double quantization.
   layers: HOST array of num_layers descriptors (device pointers inside).  Each layer is
   quantized as in aqnf4_quantize; its optional outputs (packed, absmax, codes8 + scales)
   are written; and, with w_hat = dtype_rn(fl(levels[code] * a_b)) (a_b replaced by the
   double-quantized a'_b for a layer flagged AQNF4_SCORE_DQ_ABSMAX or
   AQNF4_SCORE_DQ_CENTERED),
     sq_err[l] = sum (x - w_hat)^2,  sq_w[l] = sum x^2,
     rel_err[l] = sqrt(sq_err[l] / sq_w[l])  (0 when sq_w[l] = 0; NaN after a NaN/inf input).
   The sums are taken in a fixed order, so repeated calls give identical bits.
   workspace (device, 256-byte aligned) of at least aqnf4_workspace_size bytes, contents
   ignored on entry.  sq_err, sq_w (device double[num_layers]) and rel_err (device
   float[num_layers]) are outputs; any may be NULL.
   Errors: INVALID_ARG, ALIGNMENT, DTYPE, WORKSPACE, CUDA. */
AQNF4_API aqnf4_status aqnf4_layer_error(const aqnf4_layer* layers, int32_t num_layers, void* workspace,
                               size_t ws_bytes, double* sq_err, double* sq_w, float* rel_err,
                               int32_t* dev_flag, cudaStream_t stream);

/* Same as aqnf4_layer_error but without a workspace argument (no counterpart on the
   pages: this is a calling convenience).  For callers that have no way to provide device
   memory at the call site -- for example a plugin or C FFI layer that only receives device
   pointers from its host framework, or code running where the framework forbids new device
   allocations -- the per-tile partial sums go to a scratch array built into the library
   (8 MiB per device, held until the process exits).  Limit: the layers may span at most
   2^19 tiles of 16384 elements (8.6e9 weights); larger requests return AQNF4_ERR_WORKSPACE
   and should be split.  The first call on a device looks up the scratch address with that
   device current; make it before any stream capture.  All calls on a device share the
   scratch, so calls that overlap on the GPU race: serialise them.  The library allocates
   nothing here either.  Other arguments and errors as for aqnf4_layer_error. */
AQNF4_API aqnf4_status aqnf4_layer_error_noalloc(const aqnf4_layer* layers, int32_t num_layers,
                                                 double* sq_err, double* sq_w, float* rel_err,
                                                 int32_t* dev_flag, cudaStream_t stream);

/* Forward product of a layer stored in NF4 + DQ ("QLoRA", "How It Works": a training pass
   works on 16-bit values rebuilt from the 4-bit storage), on the tensor cores with the
   dequantization fused in: y = x w_hat^T, where w_hat (N x K) is exactly what
   aqnf4_dequantize(packed, codes8, scales, NULL, N*K, dtype, ...) returns for the layer's
   storage, and the products are summed in binary32.
   x (device, M x K, row-major, dtype, 16-byte aligned); packed (device, N*K/2 bytes,
   16-byte aligned), codes8 (device, N*K/64 bytes), scales (device, ceil(N*K/16384) floats):
   the layer's storage as aqnf4_layer_error writes it; y (device, M x N, row-major,
   16-byte aligned): float when out_f32 != 0, else dtype.  K must be a positive multiple of 64, so that each row of
   the layer is whole NF4 blocks.  When the output has too few 256 x 256 tiles to fill the
   GPU, K is split over aqnf4_nf4_linear_splits(M, N, K) thread blocks that form one cluster
   per tile and add their binary32 partial sums on chip, in split order (the result does not
   depend on scheduling, and no workspace is needed).  Otherwise, with more than 256 rows,
   two row tiles share each dequantized weight tile on a pair of thread blocks.  dev_flag (optional, device int32)
   receives AQNF4_ERR_TIMEOUT if a bounded wait inside the kernel gave up; the tiles that
   wait belonged to are then not written (without a dev_flag a timeout goes unreported and y
   is undefined).
   Errors: INVALID_ARG (NULL pointer, M < 1, N < 1, K not a positive multiple of 64, sizes
   above 2^31, M above 65535 * 256 = 16776960 rows), DTYPE, ALIGNMENT, CUDA. */
AQNF4_API aqnf4_status aqnf4_nf4_linear(const void* x, int32_t dtype, int64_t M, int64_t K,
                                        const uint8_t* packed, const uint8_t* codes8,
                                        const float* scales, int64_t N, void* y,
                                        int32_t out_f32, int32_t* dev_flag,
                                        cudaStream_t stream);

/* How many thread blocks aqnf4_nf4_linear splits K over for this shape on the current device
   (1: no split; at most 8; 0: invalid shape).  Host only. */
AQNF4_API int32_t aqnf4_nf4_linear_splits(int64_t M, int64_t N, int64_t K);

/* Top-K under a byte budget (arxivdaily 2608.23816, "English abstract": the highest-error
   layers stay in 16 bits while a byte budget allows; "AQLoRA: ...", "Technical Details":
   the budget is a setting).
   Layers are ranked by rel_err descending, equal scores by lower index first, NaN scores
   last.  Walking the ranking, layers are kept until the next one would exceed k_cap layers
   (k_cap < 0: no cap) or push the summed cost_bytes above budget_bytes.
   rel_err (device float[L]), cost_bytes (device int64[L]) are inputs; sel_idx (device
   int32[L]) receives the whole ranking, of which the first *k_out entries are the kept
   layers; k_out (device int32[1]).  Runs in one thread block, O(L^2 / 1024) time.
   Errors: INVALID_ARG (NULL pointer, L < 1, budget_bytes < 0), ALIGNMENT, CUDA. */
AQNF4_API aqnf4_status aqnf4_select_topk(const float* rel_err, const int64_t* cost_bytes, int32_t L,
                               int64_t budget_bytes, int32_t k_cap, int32_t* sel_idx,
                               int32_t* k_out, cudaStream_t stream);

/* Diagnostic for failure detection (no counterpart on the pages).  Runs the bounded wait
   that every bulk-copy consumer in this library uses, on an mbarrier that nothing ever
   completes, with a limit of timeout_ns (1 ns .. 2 s; the kernels themselves use 2 s).  The
   wait gives up, the kernel stores AQNF4_ERR_TIMEOUT in *dev_flag (device int32, required)
   and, if waited_ns (device int64) is non-NULL, the nanoseconds it waited; then it returns
   normally, leaving the context usable.  Errors: INVALID_ARG, ALIGNMENT, CUDA. */
AQNF4_API aqnf4_status aqnf4_selftest_wait_timeout(int64_t timeout_ns, int32_t* dev_flag,
                                                   int64_t* waited_ns, cudaStream_t stream);

/* Diagnostic (no counterpart on the pages).  The fused pass takes fl(1/a) and fl(a/s) with a
   short Newton-Raphson form (the hardware reciprocal approximation and one fused
   multiply-add correction) that is exact for the 16-bit values it meets.  This call
   evaluates, for each i < n, out[4i] = that reciprocal of a[i], out[4i+1] = CUDA's
   correctly rounded __frcp_rn(a[i]), out[4i+2] = the short quotient a[i] / s[i] and
   out[4i+3] = CUDA's __fdiv_rn(a[i], s[i]), so a test can compare them.  a, s (device
   float[n]) are inputs, out (device float[4n], 16-byte aligned) the output.
   Errors: INVALID_ARG, ALIGNMENT, CUDA. */
AQNF4_API aqnf4_status aqnf4_selftest_division(const float* a, const float* s, int64_t n,
                                               float* out, cudaStream_t stream);

/* Incremental bytes of keeping an n-element layer in 16 bits instead of its NF4 storage
   (packed + codes8 + scales): 2n - (ceil(n/2) + ceil(n/64) + 4*ceil(ceil(n/64)/256)).
   Host only; -1 for n < 1.  (The 0.2 GiB extra memory of the abstract's quality setting is
   read as a budget on this quantity.) */
AQNF4_API int64_t aqnf4_cost_bytes(int64_t n);

/* Block-level selection for the speed setting (arxivdaily 2608.23816, "English abstract":
   a speed setting adapts only the top blocks, so the backward pass stops early; "AQLoRA:
   ...", "Technical Details": it promotes only the top blocks).  Layer l belongs to
   transformer block block_of[l] in [0, num_blocks).  A block costs the sum of its layers'
   cost_bytes.  Its score block_err is the relative error of its layers together,
   sqrt(sum sq_err / sum sq_w), summed in binary64 in layer order (0 when sum sq_w = 0; NaN
   after a NaN input).  order AQNF4_BLOCKS_BY_DEPTH ranks the blocks from the last one down
   (the pages' "top blocks"; the lowest kept block is where the backward pass can stop);
   AQNF4_BLOCKS_BY_ERROR ranks them by block_err descending (equal scores: lower index
   first; NaN last).  The kept blocks are the longest prefix of the ranking whose summed
   cost is within budget_bytes.
   sq_err, sq_w (device double[num_layers], e.g. aqnf4_layer_error's outputs), block_of
   (device int32[num_layers]) and cost_bytes (device int64[num_layers]) are inputs;
   block_rank (device int32[num_blocks]) receives the whole ranking, block_err (optional,
   device float[num_blocks]) the scores and k_out (device int32[1]) the number of blocks kept.
   A block_of entry outside [0, num_blocks) is a data error: the kernel stores
   AQNF4_ERR_INVALID_ARG in *dev_flag (optional device int32, zeroed by the caller) and -1 in
   *k_out, and the other outputs are then meaningless.  1 <= num_blocks <= 2048.  One thread
   block.
   Errors: INVALID_ARG (NULL pointer, a size out of range, budget_bytes < 0, unknown order),
   ALIGNMENT, CUDA. */
enum { AQNF4_BLOCKS_BY_DEPTH = 0, AQNF4_BLOCKS_BY_ERROR = 1 };
AQNF4_API aqnf4_status aqnf4_select_blocks(const double* sq_err, const double* sq_w,
                                           const int32_t* block_of, const int64_t* cost_bytes,
                                           int32_t num_layers, int32_t num_blocks,
                                           int64_t budget_bytes, int32_t order,
                                           int32_t* block_rank, float* block_err,
                                           int32_t* k_out, int32_t* dev_flag,
                                           cudaStream_t stream);

/* The fused pass's code lookup, for inspection (host only; no counterpart on the pages,
   which define the code as the nearest level, i.e. the number of midpoints below v).
   curve[2] = (a, b); slot_mid[32], slot_level[32].  For a normalised value v with
   |v| <= 1 + 2^-20 the kernels compute, in binary32, s = fma(v*v, b, a) and
   k = round_to_nearest(fma(v, s, 2^23 + 8)) - 2^23, and take
   code = k - 1 + (v > slot_mid[k]) and level = slot_level[code + 1].  The library checks
   when it builds the tables that this equals the midpoint count for every such v.
   Host arrays, caller-owned.  Errors: INVALID_ARG (null pointer), CUDA (tables failed). */
AQNF4_API aqnf4_status aqnf4_slot_tables(float* curve, float* slot_mid, float* slot_level);

/* Number of kernels this library has launched in this process (host counter). */
AQNF4_API uint64_t aqnf4_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* AQNF4_H */
