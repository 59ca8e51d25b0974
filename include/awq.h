/*
 * awq.h -- C ABI of libawq_b200, a W4A16 linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer is y = x . W'^T where W' is decoded on the fly from group-wise
 * 4-bit codes: w' = (q - z) * s (asymmetric, zero point z) or w' = s * (q - 8)
 * (symmetric). Groups are 128 consecutive input channels of one output
 * channel. Activations and outputs are fp16, accumulation is fp32.
 *
 * Sources, by page and section:
 *   "AutoAWQ" code tour (pyshine.com): "The Quantization Flow Up Close"
 *     (pseudo-quantization rounds each group to integer levels against its
 *     scale and zero point), "The big picture" (WQLinear_GEMM for batched
 *     requests, WQLinear_GEMV for single-token decode), "From Install to Your
 *     First Model" (zero_point, q_group_size = 128, w_bit = 4).
 *   "AutoAWQ" capability page (unfragile.ai): the WQLinear kernels dequantize
 *     inside the fused matmul and never materialize fp16 weights.
 *   "AWQ > Implementation" (Language AI Handbook), "Understanding the
 *     Quantization Structure": eight 4-bit codes per int32, fp16 scales, one
 *     scale and zero per 128 weights.
 *   "AWQ Quantization Support" (fak explainer), "Dequantization Formula":
 *     weight = scale x (code - 8); "Integration with Forward Pass": a
 *     matrix-vector entry for decode and a batched matmul entry for P tokens.
 *
 * ---------------------------------------------------------------------------
 * Data layout (all row-major, K contiguous; N output channels, K input
 * channels, G = K / group_size groups per row):
 *
 *   W        fp16   [N][K]      (quantizer input; awq_dequant output)
 *   x        fp16   [M][K]
 *   y        fp16   [M][N]
 *   qweight  int32  [N][K/8]    word w of row n covers k = 8w .. 8w+7; nibble
 *                               slot i (bits 4i .. 4i+3) holds the code of
 *                               k = 8w + {0,2,4,6,1,3,5,7}[i]. With this
 *                               order, (word >> 4j) & 0x000F000F holds the
 *                               codes of the consecutive pair k = 8w+2j,
 *                               8w+2j+1 in its low and high 16-bit halves.
 *   scales   fp16   [G][N]      s[j][n] for k in [128j, 128j + 128) of row n
 *                               (group-major, as AutoAWQ stores scales)
 *   zeros    fp16   [G][N]      integer zero points 0..15 stored as fp16,
 *                               group-major (asymmetric only; NULL for
 *                               symmetric)
 *
 * fp16 buffers are passed as uint16_t pointers holding IEEE binary16 bits.
 *
 * Ownership and execution: every pointer is device memory owned by the
 * caller (the library allocates nothing and keeps no per-call state). Every
 * entry point validates its arguments on the host, then enqueues its work on
 * `stream` (a cudaStream_t; NULL = the legacy default stream) and returns
 * without synchronizing. A non-OK status means nothing was enqueued, except
 * AWQ_ERR_CUDA, which reports a launch error from the CUDA runtime.
 * Device pointers must be 16-byte aligned. Sizes are element counts.
 * Inputs must be finite (no NaN or infinity); the results for non-finite
 * inputs are unspecified.
 * ---------------------------------------------------------------------------
 */
#ifndef AWQ_B200_H
#define AWQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define AWQ_ABI_VERSION 8

#if defined(__GNUC__)
#define AWQ_API __attribute__((visibility("default")))
#else
#define AWQ_API
#endif

typedef enum awq_status {
  AWQ_OK = 0,
  AWQ_ERR_NULL = 1,        /* a required pointer is NULL                     */
  AWQ_ERR_SHAPE = 2,       /* a size is negative, out of range or mismatched */
  AWQ_ERR_ALIGN = 3,       /* a device pointer is not 16-byte aligned        */
  AWQ_ERR_UNSUPPORTED = 4, /* group size / variant not implemented           */
  AWQ_ERR_CUDA = 5,        /* the CUDA runtime reported an error             */
  AWQ_ERR_WORKSPACE = 6    /* workspace missing or smaller than required     */
} awq_status_t;

/* Quantization configuration ("AutoAWQ" code tour, "From Install to Your
 * First Model": q_group_size, zero_point; w_bit is fixed at 4).
 * group_size must be 128. zero_point: 1 = asymmetric, 0 = symmetric.
 * flags: a bitwise OR of AWQ_FLAG_* values (0 for none); bits this library
 * does not define are rejected with AWQ_ERR_UNSUPPORTED. */
typedef struct awq_qconfig {
  int32_t group_size;
  int32_t zero_point;
  uint32_t flags;
} awq_qconfig_t;

/* awq_gemv / awq_gemv_noalloc may start reading qweight, scales and zeros
 * before the kernel launched just before them on the same stream has
 * finished (it still waits for that kernel before it reads x or writes y).
 * Set it only when no work still running on the stream writes those three
 * arrays, for instance in a decode loop over weights loaded once. The other
 * entry points ignore it. */
#define AWQ_FLAG_WEIGHTS_STATIC 1u

/* Fused MLP input projection ("AutoAWQ" code tour, "The Quantization Flow Up
 * Close": the fuser merges the gate and up projections into one quantized
 * MLP block; "AutoAWQ" capability page: fused blocks save launches and
 * intermediate tensors). With this flag awq_gemv, awq_gemv_noalloc and
 * awq_gemm read qweight / scales / zeros as N rows in which 16-row tiles
 * alternate between a gate and an up projection of N/2 rows each -- tile 2j
 * holds gate rows 16j .. 16j+15, tile 2j+1 up rows 16j .. 16j+15 (scales and
 * zeros: the same order along their N columns); awq_interleave_gate_up
 * builds it -- and write y[M][N/2] with
 *   y[m][n] = fp16( silu(g) * u ),  silu(v) = v / (1 + exp(-v)),
 * g and u the fp32 sums of gate row n and up row n (the values awq_gemv /
 * awq_gemm would round to fp16 for those rows), silu and the product in
 * fp32 with the fast exponential and division intrinsics (within a few fp32
 * ulp of the exact silu). Requires N % 32 == 0. awq_workspace_bytes takes
 * the flag. */
#define AWQ_FLAG_SILU_MUL 2u

/* Packed zero points ("AWQ > Implementation", "Understanding the Quantization
 * Structure": a quantized layer holds qweight, scales and qzeros, its 4-bit
 * values stored eight per int32). With this flag the `zeros` argument of
 * awq_gemv, awq_gemv_noalloc and awq_dequant points to int32
 * qzeros[K/128][N/8] instead of fp16 zeros[K/128][N]: word w of group row j
 * holds the zero points of output channels 8w .. 8w+7 of that group, channel
 * 8w+i in bits 4i .. 4i+3 (awq_pack_zeros writes it from the fp16 array).
 * Results are identical to the fp16 form of the same zero points. The GEMV
 * reads the packed words directly; awq_gemm unpacks them into its workspace
 * first (G x N x 2 bytes, which awq_workspace_bytes counts for M > 16). Needs
 * zero_point = 1 (else AWQ_ERR_UNSUPPORTED); N % 32 == 0 for awq_gemv,
 * awq_gemv_noalloc and awq_gemm (a group row of qzeros is then whole 16-byte
 * runs), N % 8 == 0 for awq_dequant (else AWQ_ERR_SHAPE). Every other entry
 * point returns AWQ_ERR_UNSUPPORTED for it (awq_unpack_zeros restores the
 * fp16 form). */
#define AWQ_FLAG_PACKED_ZEROS 4u

/* ABI version of the loaded library (AWQ_ABI_VERSION at build time). */
AWQ_API int awq_abi_version(void);

/* Static description of a status code. Never NULL. */
AWQ_API const char* awq_status_string(awq_status_t status);

/*
 * awq_pseudo_quantize_pack -- quantize fp16 W[N][K] group-wise and pack it.
 * ("AutoAWQ" code tour, "The Quantization Flow Up Close": each group of
 * weights is rounded to integer levels against its scale and zero point.)
 *
 * Per row n and group j, with w the 128 values in fp32 and IEEE fp32
 * arithmetic rounded to nearest even:
 *   asymmetric: s = fp16(max((max w - min w) / 15, 1e-5)),
 *               z = clamp(-rint(min w / s), 0, 15),
 *               q = clamp(rint(w / s) + z, 0, 15)
 *   symmetric:  s = fp16(max(max|w| / 7, 1e-5)),
 *               q = clamp(rint(w / s), -8, 7) + 8
 * rint rounds half to even; s is used at its fp16 value.
 *
 * In:  W [N][K] fp16.  Out: qweight [N][K/8], scales [G][N], zeros [G][N]
 * (asymmetric; must be NULL for symmetric).
 * N >= 0 (N == 0: no work), K > 0 and K % group_size == 0.
 * Results are bit-exact: a given W always yields the same bits.
 */
AWQ_API awq_status_t awq_pseudo_quantize_pack(const uint16_t* W, int64_t N, int64_t K,
                                      awq_qconfig_t cfg, int32_t* qweight,
                                      uint16_t* scales, uint16_t* zeros,
                                      void* stream);

/*
 * awq_dequant -- decode packed weights to fp16 W'[N][K] (for checks).
 * ("AWQ Quantization Support", "Dequantization Formula": weight =
 * scale x (code - 8); asymmetric: (q - z) x s.)
 * w'[n][k] = fp16((q - z) * s), one rounding to nearest even ((q - z) * s is
 * exact in fp32), z = 8 for symmetric. Bit-exact.
 * N >= 0, K > 0, K % group_size == 0; zeros NULL iff symmetric.
 * cfg.flags may hold AWQ_FLAG_PACKED_ZEROS (zeros is then int32 qzeros).
 */
AWQ_API awq_status_t awq_dequant(const int32_t* qweight, const uint16_t* scales,
                         const uint16_t* zeros, int64_t N, int64_t K,
                         awq_qconfig_t cfg, uint16_t* W_out, void* stream);

/*
 * awq_pack_zeros -- fp16 zero points [G][N] (as awq_pseudo_quantize_pack
 * writes them) -> int32 qzeros [G][N/8] in the AWQ_FLAG_PACKED_ZEROS layout.
 * Each value is rounded to the nearest integer (ties to even) and clamped to
 * 0..15 (NaN -> 0); the quantizer's zero points are integers 0..15 already.
 * G >= 0, N >= 0, N % 8 == 0 (either 0: no work); zeros and qzeros
 * device pointers, 16-byte aligned, caller-owned. One kernel on `stream`.
 *
 * awq_unpack_zeros -- the inverse: qzeros [G][N/8] -> fp16 zeros [G][N]
 * holding the integers 0..15. Same limits.
 */
AWQ_API awq_status_t awq_pack_zeros(const uint16_t* zeros, int64_t G, int64_t N,
                                    int32_t* qzeros, void* stream);
AWQ_API awq_status_t awq_unpack_zeros(const int32_t* qzeros, int64_t G, int64_t N,
                                      uint16_t* zeros, void* stream);

/*
 * awq_workspace_bytes -- bytes of workspace awq_gemv / awq_gemm need for
 * (M, N, K) on the current device. *bytes is 0 when none is needed.
 * The workspace holds split-K partial sums and arrival counters. It must be
 * zero-filled before its first use; every call that completes brings the
 * counters back to zero (the partial sums need no clearing), so one memset
 * at allocation suffices. Calls that may run concurrently need separate
 * workspaces.
 */
AWQ_API awq_status_t awq_workspace_bytes(int64_t M, int64_t N, int64_t K,
                                 awq_qconfig_t cfg, size_t* bytes);

/*
 * awq_gemv -- y[M][N] = x[M][K] . W'^T for small batches (decode), 1 <= M <= 16.
 * ("AutoAWQ" code tour, "The big picture": the GEMV variant for single-token
 * decoding; "AutoAWQ" capability page: dequantization fused into the matmul.)
 * y[m][n] = fp16( sum_k x[m][k] * (q[n][k] - z[k/128][n]) * s[k/128][n] ),
 * products and sums in fp32 (the per-group factor s is applied to the fp32
 * partial sum of each group). The summation order is fixed for a given
 * device and shape, so results are reproducible run to run.
 * M in [1, 16]; N >= 0 and N % 8 == 0 (0: no work); K > 0, K % group_size == 0.
 * (N % 8 keeps every 8-row run of scales and zero points 16-byte aligned.)
 * cfg.flags may hold AWQ_FLAG_WEIGHTS_STATIC, AWQ_FLAG_SILU_MUL and
 * AWQ_FLAG_PACKED_ZEROS (see there; with AWQ_FLAG_SILU_MUL y is [M][N/2]).
 * workspace: at least awq_workspace_bytes(M, N, K) bytes, zero-filled before
 * first use (see above); may be NULL when that size is 0, which is the case
 * whenever N / 16 is at least the device's SM count.
 */
AWQ_API awq_status_t awq_gemv(const uint16_t* x, const int32_t* qweight,
                      const uint16_t* scales, const uint16_t* zeros,
                      int64_t M, int64_t N, int64_t K, awq_qconfig_t cfg,
                      uint16_t* y, void* workspace, size_t workspace_bytes,
                      void* stream);

/*
 * awq_gemv_noalloc -- awq_gemv without a caller-provided workspace, for
 * callers that cannot allocate device memory when they run the layer: for
 * example a plugin inside a host engine that owns all device memory and
 * passes in only the input and output buffers, or a decode loop that must
 * not allocate after start-up. The AWQ pages have no counterpart to this
 * entry point.
 *
 * Same arguments, limits, arithmetic and results as awq_gemv; the split-K
 * scratch lives in one fixed array of AWQ_GEMV_STATIC_WORKSPACE_BYTES inside
 * the library, which every GPU that loads the library keeps until the
 * process exits. Shapes whose scratch would not fit return
 * AWQ_ERR_WORKSPACE. The call allocates nothing: it does not call cudaMalloc,
 * cudaFree or any allocating routine. It enqueues a cudaMemsetAsync of the
 * array's counter region and then the GEMV kernel, both on `stream`.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current and caches it with the
 * device's current context (a new context after cudaDeviceReset is looked
 * up again, by its first call); make that first call before any stream
 * capture. All calls on a device share the
 * array: calls that may overlap on the GPU (different streams, or
 * concurrent host threads) race and must be serialized by the caller.
 */
#define AWQ_GEMV_STATIC_WORKSPACE_BYTES (1u << 20)
AWQ_API awq_status_t awq_gemv_noalloc(const uint16_t* x, const int32_t* qweight,
                                      const uint16_t* scales, const uint16_t* zeros,
                                      int64_t M, int64_t N, int64_t K, awq_qconfig_t cfg,
                                      uint16_t* y, void* stream);

/*
 * awq_gemv_chain -- several decode products in one launch, where a layer's
 * input may be the output of an earlier layer of the same call.
 * ("AutoAWQ" code tour, "The big picture": the GEMV kernel for single-token
 * decoding; "AutoAWQ" capability page, WQLinear paragraph: the INT4 layer is
 * bound by memory at small batch, and fused-blocks paragraph: fused blocks
 * save launches.)
 *
 * For l = 0 .. n_layers - 1, in order:
 *   layers[l].y[M][N_l] = layers[l].x[M][K_l] . W_l'^T
 * with the arithmetic, results and flags of awq_gemv (AWQ_FLAG_SILU_MUL:
 * y is [M][N_l/2]). The results are bit-identical to n_layers awq_gemv
 * calls made in order on the same stream whenever each layer's split of K
 * is the same (it is whenever N_l / 16 is at least twice the SM count).
 * The launch streams the weights of all layers back to back; a layer that
 * reads an earlier layer's output takes its x from a copy of that output in
 * the workspace and uses each value only once it has been written.
 *
 * x_from = -1: x is ready when the call starts (written by earlier work on
 * the stream). x_from = d (0 <= d < l): x is layer d's y of this call; x
 * must then equal layers[d].y and K_l the column count of that y.
 * A layer's y must not overlap any other layer's x or y, except as the x
 * of the layers that name it in x_from.
 * 1 <= n_layers <= AWQ_CHAIN_MAX_LAYERS; 1 <= M <= 16; per layer: N >= 8,
 * N % 8 == 0 (N % 32 with AWQ_FLAG_SILU_MUL or AWQ_FLAG_PACKED_ZEROS);
 * K % 128 == 0; every layer has the same zero-point form (symmetric, fp16
 * zeros or packed zeros); pointers 16-byte aligned. The weights may be read
 * before the kernel launched just before this one on the stream has
 * finished only if every layer carries AWQ_FLAG_WEIGHTS_STATIC.
 * layers: host memory, read before the call returns.
 * workspace: at least awq_gemv_chain_workspace_bytes() bytes of device
 * memory, zero-filled before its first use and then kept for calls with the
 * same M and layers (shapes, flags, x_from; the pointers may change) and not
 * written by anything else: between calls it holds a launch count and the
 * half of the output-copy region that the next call reads, zeroed (every
 * call that completes, also one whose waits gave up, leaves it so). A call
 * with other layers needs its own workspace, or this one zero-filled again.
 * Calls that may run concurrently need separate workspaces.
 * Every CTA of the launch must be resident at once (the grid is sized from
 * the occupancy of the kernel on this device): do not run other kernels
 * concurrently on the same device that could hold SMs for a long time, or
 * the dependency waits reach their time limit and the call gives up
 * (reported by awq_device_error, bit 2).
 */
#define AWQ_CHAIN_MAX_LAYERS 32
typedef struct awq_gemv_layer {
  const uint16_t* x;        /* [M][K] fp16 */
  const int32_t* qweight;   /* [N][K/8] */
  const uint16_t* scales;   /* [K/128][N] fp16 */
  const uint16_t* zeros;    /* [K/128][N] fp16, int32 [K/128][N/8] with
                               AWQ_FLAG_PACKED_ZEROS, or NULL (symmetric) */
  uint16_t* y;              /* [M][N] fp16 ([M][N/2] with AWQ_FLAG_SILU_MUL) */
  int64_t N, K;
  awq_qconfig_t cfg;
  int32_t x_from;           /* -1, or the index of the layer whose y x is */
} awq_gemv_layer_t;

AWQ_API awq_status_t awq_gemv_chain_workspace_bytes(const awq_gemv_layer_t* layers, int n_layers,
                                                    int64_t M, size_t* bytes);
AWQ_API awq_status_t awq_gemv_chain(const awq_gemv_layer_t* layers, int n_layers, int64_t M,
                                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * awq_debug_set_wait_limit_ns -- test hook: the time limit after which a
 * pipeline wait inside awq_gemv_chain gives up (0 restores the default of
 * 2 s; at most 2 s). Copies already in flight are always waited for with
 * the full limit. Synchronizes `stream`. The pages have no counterpart; it
 * exists so that tests can make a wait run out without a fault.
 */
AWQ_API awq_status_t awq_debug_set_wait_limit_ns(uint64_t ns, void* stream);

/*
 * awq_gemm -- y[M][N] = x[M][K] . W'^T for any M >= 1 (prefill).
 * ("AutoAWQ" code tour, "The big picture": the GEMM variant for batched
 * requests; "AWQ Quantization Support", "Integration with Forward Pass":
 * the batched product over P tokens.)
 * Tiles of W' are decoded bit-exactly (as awq_dequant) into shared memory and
 * multiplied on the tensor cores (tcgen05, fp16 inputs, fp32 accumulation in
 * tensor memory); y = fp16 of the fp32 sum.
 * M >= 0, N >= 0 (either 0: no work); K > 0, K % group_size == 0.
 * cfg.flags may hold AWQ_FLAG_SILU_MUL (y is then [M][N/2]) and
 * AWQ_FLAG_PACKED_ZEROS (see there).
 * Workspace as for awq_gemv: awq_workspace_bytes(M, N, K, cfg) bytes, 0
 * (NULL allowed) unless the zero points are packed.
 */
AWQ_API awq_status_t awq_gemm(const uint16_t* x, const int32_t* qweight,
                      const uint16_t* scales, const uint16_t* zeros,
                      int64_t M, int64_t N, int64_t K, awq_qconfig_t cfg,
                      uint16_t* y, void* workspace, size_t workspace_bytes,
                      void* stream);

/*
 * awq_interleave_gate_up -- build the AWQ_FLAG_SILU_MUL weight layout from
 * a gate and an up projection packed by awq_pseudo_quantize_pack (same K,
 * config and N rows each): qweight_out [2N][K/8], scales_out [G][2N],
 * zeros_out [G][2N] (NULL iff symmetric) in 16-row tiles alternating gate,
 * up. Copies only (cudaMemcpy2DAsync on `stream`); the outputs must not
 * overlap the inputs. N >= 0 and N % 16 == 0; K > 0, K % group_size == 0.
 */
AWQ_API awq_status_t awq_interleave_gate_up(const int32_t* qweight_gate, const uint16_t* scales_gate,
                                            const uint16_t* zeros_gate, const int32_t* qweight_up,
                                            const uint16_t* scales_up, const uint16_t* zeros_up,
                                            int64_t N, int64_t K, awq_qconfig_t cfg,
                                            int32_t* qweight_out, uint16_t* scales_out,
                                            uint16_t* zeros_out, void* stream);

/*
 * awq_concat_rows -- concatenate `parts` packed projections that share K and
 * config along N ("AutoAWQ" code tour, "The Quantization Flow Up Close": the
 * fuser concatenates the q, k and v projections through fuse_qkv), so one
 * awq_gemv / awq_gemm computes all of them: part p's rows follow those of
 * parts 0 .. p-1 in qweight_out [sum N][K/8], and its columns those of parts
 * 0 .. p-1 in scales_out / zeros_out [G][sum N] (zeros NULL iff symmetric,
 * for every part). qweights / scales / zeros are arrays of `parts` device
 * pointers (zeros may be NULL when symmetric), Ns their row counts (host
 * memory, read before the call returns). Copies only (cudaMemcpy2DAsync on
 * `stream`); outputs must not overlap inputs. 1 <= parts <= 16, every
 * N_p >= 0, K > 0, K % group_size == 0.
 */
AWQ_API awq_status_t awq_concat_rows(int parts, const int32_t* const* qweights, const uint16_t* const* scales,
                                     const uint16_t* const* zeros, const int64_t* Ns, int64_t K,
                                     awq_qconfig_t cfg, int32_t* qweight_out, uint16_t* scales_out,
                                     uint16_t* zeros_out, void* stream);

/*
 * awq_search_scale -- activation-aware per-input-channel scale search.
 * ("AutoAWQ" code tour, "The Quantization Flow Up Close": a per-channel mean
 * of normalized weights and a float32 mean of activations, the fp16 module
 * run once as the reference, the candidate scaling with the lowest output
 * error kept; "From Install to Your First Model": duo_scaling.)
 * With x_mean[k] = mean_m |X[m][k]| and w_mean[k] = mean_n |W[n][k]| /
 * max|W[n][group of k]| (fp32), grid point i (alpha = i / n_grid) tries
 *   s = max(x_mean^alpha / (w_mean^(1 - alpha) + 1e-4), 1e-4)  (duo != 0)
 *   s = max(x_mean^alpha, 1e-4)                                 (duo == 0)
 * divided by sqrt(max s * min s); its loss is the mean over outputs of
 * (fp16(X . W^T) - fp16((X / s) . Q(W diag(s))'^T))^2, Q the quantizer of
 * awq_pseudo_quantize_pack and the product that of awq_gemv / awq_gemm,
 * X / s and W diag(s) rounded to fp16. losses_out [n_grid] (device fp32)
 * receives the losses, scales_out [K] (device fp32) the scales of the first
 * minimum. To use them: quantize W diag(s) (awq_apply_scale, then
 * awq_pseudo_quantize_pack) and divide the layer's input by s upstream.
 * W [N][K], X [Ms][K] fp16 device; N >= 1, N % 8 == 0, K % group_size == 0,
 * 1 <= Ms <= 2^24, 1 <= n_grid <= 64, cfg.flags == 0.
 * workspace: awq_search_scale_workspace_bytes(N, K, Ms, cfg) bytes of device
 * memory, 16-byte aligned, contents irrelevant. Stream-ordered, no host
 * synchronization; same inputs give the same bits.
 */
AWQ_API awq_status_t awq_search_scale_workspace_bytes(int64_t N, int64_t K, int64_t Ms, awq_qconfig_t cfg,
                                                      size_t* bytes);
AWQ_API awq_status_t awq_search_scale(const uint16_t* W, int64_t N, int64_t K, const uint16_t* X, int64_t Ms,
                                      awq_qconfig_t cfg, int n_grid, int duo, float* scales_out,
                                      float* losses_out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * awq_apply_scale -- W_out[n][k] = fp16(W[n][k] * s[k]) (fp32 product, one
 * rounding): the weights of a layer whose input will be divided by s.
 * W, W_out [N][K] fp16 device (16-byte aligned), s [K] fp32 device.
 * N >= 0, K > 0, K % 8 == 0.
 */
AWQ_API awq_status_t awq_apply_scale(const uint16_t* W, const float* s, int64_t N, int64_t K, uint16_t* W_out,
                                     void* stream);

/*
 * awq_search_clip -- per (row, group) clipping-ratio search.
 * ("AutoAWQ" code tour, "The Quantization Flow Up Close": the clipping pass
 * shrinks extreme weights group by group where that lowers the output error;
 * apply_clip switches it.) For row n and group j, grid point i tries
 * r = 1 - max_shrink * i / n_grid (fp32): the group is clipped to [-t, t],
 * t = r * max|w| of the group (fp32), the values rounded to fp16 and
 * quantized as by awq_pseudo_quantize_pack; the error is d^T G_j d with
 * d = w - w' (fp32) and G_j = X_j^T X_j (fp32) the Gram matrix of the
 * calibration inputs over the group's input channels. ratios_out [G][N]
 * (device fp32, group-major like the scales) receives the first ratio with
 * the lowest error. To use them: awq_apply_clip, then
 * awq_pseudo_quantize_pack. W [N][K], X [Ms][K] fp16 device; N >= 1,
 * N % 8 == 0, K % group_size == 0, 1 <= Ms <= 2^24, 1 <= n_grid <= 64,
 * 0 <= max_shrink < 1, cfg.flags == 0. workspace:
 * awq_search_clip_workspace_bytes(K) bytes (the Gram matrices), 16-byte
 * aligned, contents irrelevant. Stream-ordered; same inputs, same bits.
 */
AWQ_API awq_status_t awq_search_clip_workspace_bytes(int64_t K, size_t* bytes);
AWQ_API awq_status_t awq_search_clip(const uint16_t* W, int64_t N, int64_t K, const uint16_t* X, int64_t Ms,
                                     awq_qconfig_t cfg, int n_grid, float max_shrink, float* ratios_out,
                                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * awq_apply_clip -- W_out = W with each (row n, group j) clipped to [-t, t],
 * t = ratios[j][n] * max|w| of the group (fp32), rounded to fp16.
 * W, W_out [N][K] fp16 device (16-byte aligned), ratios [G][N] fp32 device.
 */
AWQ_API awq_status_t awq_apply_clip(const uint16_t* W, const float* ratios, int64_t N, int64_t K,
                                    uint16_t* W_out, void* stream);

/*
 * awq_device_error -- read and clear the device-side error word of the
 * current device (synchronizes `stream`). Bit 0: a pipeline wait inside
 * awq_gemm passed its time limit (2 s) and the kernel abandoned its tiles;
 * bit 1: the same inside awq_gemv; bit 2: a pipeline or dependency wait
 * inside awq_gemv_chain. The output is then incomplete. 0 means
 * no error was recorded. No kernel traps: a wait that gives up records the
 * bit, lets its copies in flight land, frees what it holds and returns.
 */
AWQ_API awq_status_t awq_device_error(uint32_t* error_word, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* AWQ_B200_H */
