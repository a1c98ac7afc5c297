/*
 * qe.h -- C ABI of the B200 (sm_100a) Quant Experts (QE) linear-layer library.
 *
 * The layer (Quant Experts: Token-aware Adaptive Error Reconstruction with
 * Mixture of Experts for Large Vision-Language Models Quantization; method
 * text on the MCISLAB DeepRead summary page, section "Method"; cost model in
 * Table 7 of the thelatestinai listing):
 *
 *   Y = dequant(Q_A(X/s)) . dequant(Q_W(W.s))^T  +  X.A_s.B_s  +  X.A_r[e(t)].B_r[e(t)]
 *
 * - W.s / X/s: channel-wise scaling (Method, "Shared Expert"), with s_inv = 1/s
 *   stored per input channel.
 * - Q_W: symmetric group RTN, W4 or W3, one fp32 scale per (output row, group).
 * - Q_A: symmetric per-token RTN, A8 or A6 (a_bits 8/6). a_bits 16 means
 *   weight-only (W3A16 / W4A16): bf16(x/s) against the dequantized weight.
 * - A_s.B_s: the shared low-rank expert, applied to every token (Method,
 *   "Shared Expert").
 * - A_r[e].B_r[e]: one routed low-rank expert per token (Method, "Routed
 *   Experts"). e(t) = argmin_e (X.G)[t,e], a router that predicts each
 *   expert's residual error and takes the smallest. Table 7 prices it at
 *   s*d*N_r, so it is a single d_in x N_r linear map.
 *
 * Conventions for every entry point
 * - Pointers marked (device) are CUDA device pointers. The caller allocates
 *   and owns all of them. The library allocates no device memory at run
 *   time and never frees anything it did not allocate. Its own device state
 *   is static, on every device that loads the library: one error word
 *   (qe_device_error) and the fixed scratch array of
 *   qe_linear_forward_noalloc (QE_NOALLOC_WORKSPACE_BYTES).
 * - Matrices are row-major. W is [d_out, d_in] (the nn.Linear convention),
 *   X is [T, d_in] and Y is [T, d_out].
 * - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *   default stream). Arguments are validated synchronously before anything
 *   is launched. On a non-OK return nothing was launched.
 * - Every device pointer must be 16-byte aligned. d_in must be a multiple of
 *   the group (64 or 128). Row pitches equal the row width (dense).
 * - Kernels never trap. A device-side wait that runs out (2 s) records a code
 *   that qe_device_error() returns. The caller should then treat that call's
 *   outputs as invalid.
 * - No exception crosses this ABI.
 */
#ifndef QE_H_
#define QE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QE_API __attribute__((visibility("default")))
#else
#define QE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QE_OK = 0,
  QE_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, inconsistent shape */
  QE_ERR_UNSUPPORTED = 2,  /* a combination this build does not implement (bits, group, ranks) */
  QE_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned */
  QE_ERR_WORKSPACE = 4,    /* workspace pointer null or smaller than qe_linear_workspace_bytes */
  QE_ERR_CUDA = 5,         /* a CUDA launch or driver call failed (see qe_last_cuda_error) */
  QE_ERR_TIMEOUT = 6       /* a device wait ran out (returned by qe_device_error) */
} qe_status;

typedef enum { QE_F32 = 0, QE_BF16 = 1 } qe_dtype;

/* Shape and precision of one QE linear layer. */
typedef struct {
  int32_t d_in;         /* K, multiple of group, >= 128                           */
  int32_t d_out;        /* N, any positive value                                  */
  int32_t group;        /* weight quantization group along K: 64 or 128           */
  int32_t w_bits;       /* 4 (W4) or 3 (W3)                                        */
  int32_t a_bits;       /* 8 (A8), 6 (A6) or 16 (weight-only, bf16 activations)   */
  int32_t rank_shared;  /* r_s >= 0                                                */
  int32_t n_routed;     /* N_r in [1, 16]                                          */
  int32_t rank_routed;  /* r_r >= 0; r_s + N_r*r_r <= 512                          */
  int32_t routed_channels; /* k_c: 0 = dense routed experts (A_r[e] spans d_in).     */
                           /* k_c > 0 = cluster-sparse routed experts (Method,      */
                           /* "Routed Experts": each expert serves a cluster of     */
                           /* token-dependent channels): A_r[e] is nonzero only on  */
                           /* k_c channels, given to qe_pack_adapters_sparse.       */
                           /* Needs r_r > 0 and r_s <= 240; k_c <= d_in.           */
  int32_t w_scale_fp16;    /* 0: fp32 weight group scales; 1: fp16 scales (half the */
                           /* scale bytes; the codes are computed from the stored  */
                           /* fp16 scale)                                          */
} qe_layer_desc;

/*
 * Quantized weight storage (library-defined layouts; produced by
 * qe_quantize_weights, read by qe_linear_forward; safe to save and reload as
 * bytes on the same library version):
 *
 * w_packed (device, qe_packed_weight_bytes bytes): codes in blocks of
 *   128 output rows x 128 input channels. Block (n, b) with n = o/128 and
 *   b = k/128 starts at byte (n*ceil(d_in/128) + b) * block_bytes. Rows past
 *   d_out and channels past d_in hold zero codes.
 *   W4: block_bytes = 8192. Row r of a block is 64 bytes at r*64: four
 *     16-byte pieces i = 0..3. In piece i, byte 4w+b of 32-bit word w holds
 *     code (32i + 4w + b) in its low nibble and code (32i + 16 + 4w + b) in
 *     its high nibble. Codes are 4-bit two's complement in [-7, 7].
 *   W3: block_bytes = 6144. Row r of a block is 48 bytes at r*48. Codes are
 *     stored offset-binary as u = q + 4 in [1, 7]. Bytes 0..31 are eight
 *     32-bit words of 2-bit fields: word m holds the low two bits of u for
 *     code 16m + 2p at bits [2p, 2p+2), and for code 16m + 2p + 1 at bits
 *     [16+2p, 18+2p), p = 0..7. Bytes 32..47 are four 32-bit words of
 *     high bits: word h holds bit 2 of u for code 32h + 2p at bit p, and for
 *     code 32h + 2p + 1 at bit 16 + p, p = 0..15.
 * w_scale (device, [d_in/group][d_out], group-major, fp32; fp16 when
 *   desc->w_scale_fp16 = 1): the weight scale of (output row o, group j) is
 *   w_scale[j*d_out + o].
 * s_inv (device, fp32 [d_in]): 1/s, the reciprocal channel smoothing factor.
 * adapters (device, qe_adapter_packed_bytes bytes): produced by
 *   qe_pack_adapters from the natural-layout adapters and router.
 */
typedef struct {
  const void* w_packed;
  const float* w_scale;
  const float* s_inv;
  const void* adapters;
} qe_layer_weights;

/* ---------------------------------------------------------------- sizes */

/* Bytes of w_packed for this layer (0 on an invalid desc). */
QE_API size_t qe_packed_weight_bytes(const qe_layer_desc* desc);

/* Bytes of the packed adapter/router buffer for this layer (0 on an invalid desc). */
QE_API size_t qe_adapter_packed_bytes(const qe_layer_desc* desc);

/* Bytes of the caller-provided scratch that qe_linear_forward needs for T tokens. */
QE_API size_t qe_linear_workspace_bytes(const qe_layer_desc* desc, int32_t T);

/* ---------------------------------------------------------------- weight preparation */

/*
 * Channel-scaled symmetric group quantization of W (Method, "Shared Expert":
 * weights are multiplied by s; bit widths W4/W3 from Tables 1-3), plus the
 * importance statistic's weight term w = Meanrow(|W_f|) (Method: per input
 * channel, the mean over output rows of |W|).
 *   W        (device) [d_out, d_in], fp32 or bf16 (w_dtype)
 *   s        (device) fp32 [d_in] smoothing factor (the weights are multiplied by it)
 *   w_packed (device) out, qe_packed_weight_bytes(desc) bytes
 *   w_scale  (device) out, [d_in/group][d_out], fp32 (fp16 with desc->w_scale_fp16)
 *   w_mean   (device) out, fp32 [d_in], may be NULL
 *   w_colmax (device) out, fp32 [d_in] = max_o |W[o][k]|, may be NULL
 *   s_inv    (device) out, fp32 [d_in] = fl32(1/s[k]) (one IEEE division per
 *            channel): the stored factor qe_layer_weights.s_inv that the
 *            activations are multiplied by. May be NULL.
 * For each (o, group j): scale = fl32(max_k |fl32(W[o][k]*s[k])| / qmax) and
 * code = clamp(rint(fl32(fl32(W*s)/scale)), -qmax, qmax), with ties to
 * even. A zero scale gives zero codes. qmax = 7 (W4) or 3 (W3). w_mean
 * is summed in fp64 and rounded once. With fp16 scales, the scale is rounded
 * to fp16 (nearest even) before the codes are computed from it; a scale
 * above 65504 is stored as 65504 and reported through qe_device_error
 * (code 0x203).
 */
QE_API qe_status qe_quantize_weights(const qe_layer_desc* desc, const void* W, qe_dtype w_dtype, const float* s,
                              void* w_packed, float* w_scale, float* w_mean, float* w_colmax, float* s_inv,
                              void* stream);

/*
 * Packs the shared expert, the routed experts and the router into the
 * library's adapter layout.
 *   A_s (device) bf16 [d_in][r_s]      B_s (device) bf16 [r_s][d_out]
 *   A_r (device) bf16 [N_r][d_in][r_r] B_r (device) bf16 [N_r][r_r][d_out]
 *   G   (device) bf16 [d_in][N_r]      (router: logits = X.G)
 *   out (device) qe_adapter_packed_bytes(desc) bytes
 * A_s/B_s may be NULL when r_s = 0, and A_r/B_r may be NULL when r_r = 0.
 * The up-projections are kept as fp16 inside the packed buffer. Their magnitude
 * must stay below 65504: a larger value is saturated and reported through
 * qe_device_error (code 0x201).
 */
QE_API qe_status qe_pack_adapters(const qe_layer_desc* desc, const void* A_s, const void* B_s, const void* A_r,
                           const void* B_r, const void* G, void* out, void* stream);

/*
 * The same packing for cluster-sparse routed experts (desc->routed_channels = k_c > 0; the
 * cluster reading of Method, "Routed Experts": an expert's down-projection touches only the
 * token-dependent channels of its cluster):
 *   channels (device) int32 [N_r][k_c]: expert e's channels, distinct, in [0, d_in)
 *   A_r      (device) bf16 [N_r][k_c][r_r]: its down-projection over those channels, so that
 *            U_r[t] = sum_i x[t][channels[e][i]] * A_r[e][i][:] (equal to a dense A_r that is zero
 *            outside the channels)
 * A_s, B_s, B_r and G are as for qe_pack_adapters. The forward then leaves the routed columns
 * out of its adapter/router GEMM and gathers them per token. A channel outside [0, d_in) is
 * replaced by channel 0 with zero weights and reported through qe_device_error (code 0x202).
 * qe_pack_adapters accepts only routed_channels = 0 (QE_ERR_INVALID_ARG otherwise).
 */
QE_API qe_status qe_pack_adapters_sparse(const qe_layer_desc* desc, const void* A_s, const void* B_s,
                                  const int32_t* channels, const void* A_r, const void* B_r, const void* G,
                                  void* out, void* stream);

/* ---------------------------------------------------------------- the hot path */

/*
 * Token-aware importance statistic (Method: Top-k(|x_t| * w) per token with
 * w = Meanrow(|W_f|); the channel frequency is counted over tokens).
 *   X      (device) [T, d_in], fp32 or bf16
 *   w_mean (device) fp32 [d_in]
 *   idx    (device) out int32 [T, k]. The k channels with the largest
 *          score fl32(|x|*w_mean), ordered by (score desc, channel asc).
 *          Equal scores go to the lower channel.
 *   hist   (device) int32 [d_in]: hist[c] += number of tokens whose Top-k
 *          holds c. It is zeroed first unless accumulate_hist != 0. May be NULL.
 * 1 <= k <= min(d_in, 128). T = 0 is a no-op.
 */
QE_API qe_status qe_topk_importance(const void* X, qe_dtype x_dtype, const float* w_mean, int32_t T, int32_t d_in,
                             int32_t k, int32_t* idx, int32_t* hist, int32_t accumulate_hist, void* stream);

/*
 * Router and token buckets (Method, "Routed Experts": the router picks the
 * expert with the smallest predicted residual error; one routed expert
 * per token).
 *   X       (device) [T, d_in], fp32 or bf16
 *   G       (device) bf16 [d_in][n_routed]
 *   expert  (device) out int32 [T]: argmin_e fl32-accumulated (X.G)[t,e],
 *           ties -> lowest e
 *   perm    (device) out int32 [T]: token at sorted position p (stable by t)
 *   offsets (device) out int32 [n_routed+1]: expert e owns positions
 *           [offsets[e], offsets[e+1])
 *   logits  (device) out fp32 [T, n_routed], may be NULL
 * T <= 1<<20.
 */
QE_API qe_status qe_route(const void* X, qe_dtype x_dtype, const void* G, int32_t T, int32_t d_in, int32_t n_routed,
                   int32_t* expert, int32_t* perm, int32_t* offsets, float* logits, void* stream);

/*
 * The QE linear layer forward (the formula at the top of this file).
 *   X         (device) [T, d_in], fp32 or bf16 (x_dtype)
 *   Y         (device) out [T, d_out], fp32 or bf16 (y_dtype)
 *   workspace (device) scratch of at least qe_linear_workspace_bytes(desc, T)
 *             bytes. Contents on entry are ignored. Calls that share a
 *             workspace must not overlap on the GPU.
 * Steps (all on the GPU): one tensor-core GEMM for the adapter
 * down-projections and the router logits -> one cooperative launch for the
 * argmin routing, the per-token absmax and scale, the stable bucket sort,
 * and the per-token quantization and expert-masked adapter rows in bucket
 * order -> int8 tcgen05 GEMM with per-group scale promotion and the adapter
 * up-projection in its epilogue -> scatter to token order. With a_bits = 16
 * the main product is the weight-only path.
 * T = 0 is a no-op. T <= 1<<20 (else QE_ERR_INVALID_ARG); d_in <= 32768
 * (else QE_ERR_UNSUPPORTED: the cooperative launch keeps s_inv in shared
 * memory).
 */
QE_API qe_status qe_linear_forward(const qe_layer_desc* desc, const qe_layer_weights* weights, const void* X,
                            qe_dtype x_dtype, int32_t T, void* Y, qe_dtype y_dtype, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * The same forward split into its steps, for per-step timing: `stages` is a
 * bitmask of QE_STAGE_* run in the documented order. Running every stage in
 * separate calls on one stream, with the same workspace, computes exactly
 * what qe_linear_forward computes. A stage reads what earlier stages left in
 * the workspace. ROUTE and QUANT requested together run as one launch.
 * Unknown bits -> QE_ERR_INVALID_ARG.
 */
#define QE_STAGE_PROJECT 1 /* tensor-core GEMM: adapter down-projections + router logits                */
#define QE_STAGE_ROUTE 2   /* argmin routing, per-token absmax and scale, stable bucket sort          */
#define QE_STAGE_QUANT 4   /* per-token quantization and the expert-masked adapter rows, bucket order */
#define QE_STAGE_PRODUCT 8 /* main product with the adapter epilogue, scatter to Y                      */
#define QE_STAGE_ALL 15
QE_API qe_status qe_linear_forward_stages(const qe_layer_desc* desc, const qe_layer_weights* weights, const void* X,
                                          qe_dtype x_dtype, int32_t T, void* Y, qe_dtype y_dtype, void* workspace,
                                          size_t workspace_bytes, int32_t stages, void* stream);

/* Number of kernels one qe_linear_forward launches for this layer and T (-1 on an invalid desc). */
QE_API int32_t qe_linear_kernel_launches(const qe_layer_desc* desc, int32_t T, qe_dtype x_dtype);

/*
 * How qe_linear_forward runs this layer for T tokens (host only; no GPU call).
 *   product_tile_tokens  token positions per tile of the main product (16 .. 256)
 *   product_k_splits     K splits of the main product (> 1 adds a reduce launch)
 *   adapter_atoms        64-wide adapter atoms per unit (R_pad / 64; 0 without adapters)
 *   adapter_gemm_width   columns of the adapter/router GEMM (R_tot)
 *   adapter_gemm_tile    its columns per CTA
 *   adapter_gemm_splits  its K splits (partial slots; doubled for fp32 inputs)
 *   weight_only          1 for a_bits = 16 (the weight-only product)
 *   workspace_bytes      the scratch this call needs for this x_dtype (qe_linear_workspace_bytes
 *                        is the larger of the fp32 and bf16 needs)
 *   decode_product       1 when the product is the decode-batch kernel (T <= 16 and, with
 *                        adapters, R_pad <= 384): the (128-row tile, 128-channel block) sequence
 *                        split evenly over decode_ctas CTAs, at most decode_max_segments
 *                        pieces per output tile; 0 (and 0, 0) otherwise. The CTA count is
 *                        the current device's SM count (148 when no device is visible).
 * Returns QE_ERR_INVALID_ARG for a null pointer or T < 1, and check errors of desc.
 */
typedef struct {
  int32_t product_tile_tokens, product_k_splits, adapter_atoms, adapter_gemm_width, adapter_gemm_tile,
      adapter_gemm_splits, weight_only;
  int64_t workspace_bytes;
  int32_t decode_product, decode_ctas, decode_max_segments;
} qe_linear_plan_info;
QE_API qe_status qe_linear_plan(const qe_layer_desc* desc, int32_t T, qe_dtype x_dtype, qe_linear_plan_info* out);

/*
 * qe_linear_forward without a caller-provided workspace. (No counterpart in
 * the paper: this is a deployment convenience of this library.)
 *
 * Some host programs cannot allocate device memory for the layer. Examples:
 * a plugin whose host framework owns all device memory and exposes no
 * allocator to it, or a process that must not grow its device footprint
 * after start-up. For them, this entry point uses a fixed scratch array that
 * lives in the library's own device memory. It calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *
 * Limits and behaviour:
 * - The scratch is QE_NOALLOC_WORKSPACE_BYTES (32 MiB) on every GPU that
 *   loads the library, held until the process exits.
 * - A layer, T and input dtype whose scratch need exceeds that size are
 *   rejected with QE_ERR_WORKSPACE; qe_last_cuda_error() says how much was
 *   needed. qe_linear_workspace_bytes is an upper bound on the need. fp32
 *   inputs need two extra bf16 copies of X. For example, every Qwen2VL-2B
 *   projection fits at T = 2048 with bf16 inputs.
 * - The first call on a device looks up the array's device address for that
 *   device, then synchronizes the device once, because loading the array
 *   initializes it asynchronously. Make that first call before any stream
 *   capture. The lookup is repeated (with its synchronization) when the
 *   device's context has changed since, e.g. after cudaDeviceReset.
 * - All calls share the one array and it keeps the last call's contents.
 *   Calls whose kernels overlap on the GPU (different streams, or
 *   different host threads, without ordering) race on it. Order them.
 * - Arguments, outputs and errors are as for qe_linear_forward.
 */
#define QE_NOALLOC_WORKSPACE_BYTES (32u << 20)
QE_API qe_status qe_linear_forward_noalloc(const qe_layer_desc* desc, const qe_layer_weights* weights,
                                           const void* X, qe_dtype x_dtype, int32_t T, void* Y, qe_dtype y_dtype,
                                           void* stream);

/* ---------------------------------------------------------------- status */

QE_API const char* qe_status_string(qe_status s);
/* The last CUDA error string seen by a call that returned QE_ERR_CUDA (thread-local). */
QE_API const char* qe_last_cuda_error(void);
/*
 * Synchronizes `stream`, then reads the device error word. *code receives 0,
 * or the code of the first device wait that ran out. clear != 0 resets it.
 * Returns QE_ERR_TIMEOUT when a code was set, QE_OK otherwise.
 */
QE_API qe_status qe_device_error(void* stream, int32_t* code, int32_t clear);

/*
 * Split of the channels by calibration frequency ([DR]: Quant Experts, MCISLAB DeepRead summary,
 * Method: the k channels most often in a token's Top-k set are token-independent and go to the
 * shared expert; the next N_r * k are token-dependent and are clustered into routed experts).
 *   hist        (device) int32 [d_in]: per-channel Top-k counts (qe_topk_importance's histogram)
 *   k           number of token-independent channels (0 <= k <= 128)
 *   C           number of token-dependent channels (N_r * k; 1 <= C <= 4096)
 *   channel_pos (device) out int32 [d_in]: for the channel of rank r (higher count first, equal
 *               counts by lower channel index) r - k when k <= r < k + C, else -1.
 * One CTA, exact (integer compares only). Limits: 1 <= d_in <= 1<<24, else QE_ERR_INVALID_ARG.
 */
QE_API qe_status qe_split_channels(const int32_t* hist, int32_t d_in, int32_t k, int32_t C, int32_t* channel_pos,
                                   void* stream);

/*
 * Co-occurrence of the token-dependent channels and their NPMI similarity ([DR]: Quant Experts,
 * MCISLAB DeepRead summary, Method, routed experts: channels that are often important in the
 * same token are counted together, and NPMI measures how strongly a pair co-occurs).
 *   idx         (device) int32 [T][k]: each token's Top-k channels (as qe_topk_importance writes)
 *   channel_pos (device) int32 [d_in]: the position in [0, C) of each token-dependent channel,
 *               -1 for every other channel. Distinct channels need distinct positions.
 *   O           (device) out int32 [C][C]: O[i][j] = number of tokens whose set holds both
 *               channels i and j; O[i][i] = number of tokens holding channel i. Zeroed first.
 *   S           (device) out fp32 [C][C], may be NULL: NPMI with p(i) = O[i][i]/T and
 *               p(i,j) = O[i][j]/T, S = ln(p(i,j)/(p(i)p(j))) / (-ln p(i,j)), computed in fp64
 *               and rounded once; -1 where p(i,j) = 0 and 1 where p(i,j) = 1. With
 *               threshold > -1, entries below it become 0 (the pages suggest 0.2).
 * Each idx row must name distinct channels (a Top-k set does). Counts use integer atomics, so
 * the result is exact and does not depend on the schedule. Index values outside [0, d_in) and
 * positions outside [0, C) are ignored.
 * Limits: 1 <= k <= 128, 1 <= C <= 4096, 0 <= T <= 1<<20 (else QE_ERR_INVALID_ARG).
 */
QE_API qe_status qe_cooccurrence_npmi(const int32_t* idx, int32_t T, int32_t k, const int32_t* channel_pos,
                                      int32_t d_in, int32_t C, int32_t* O, float* S, float threshold,
                                      void* stream);

/*
 * Self-test of the bounded device waits (a library convenience; the paper has no counterpart).
 * Launches one thread that waits on a barrier nothing arrives on, for at most limit_us
 * microseconds (1 .. 1000000). The wait runs out, records code 0x107 in the device error word,
 * and the kernel returns normally, so the context stays usable and qe_device_error() then reports
 * QE_ERR_TIMEOUT. limit_us outside that range -> QE_ERR_INVALID_ARG.
 */
QE_API qe_status qe_selftest_wait_timeout(int32_t limit_us, void* stream);

/* ---------------------------------------------------------------- diagnostics (tests) */

/* Unpacks w_packed to int8 codes [d_out, d_in] (device), one code per byte. */
QE_API qe_status qe_unpack_weights(const qe_layer_desc* desc, const void* w_packed, int8_t* codes, void* stream);

/*
 * Per-token quantization alone, in token order: codes (device) int8 [T, d_in],
 * sa (device) fp32 [T]. a_bits 6 or 8.
 */
QE_API qe_status qe_act_quant(const void* X, qe_dtype x_dtype, const float* s_inv, int32_t T, int32_t d_in,
                       int32_t a_bits, int8_t* codes, float* sa, void* stream);

/*
 * qe_linear_forward with its intermediates exposed (a_bits 6/8 only):
 *   acc     (device) out int32 [T, d_out, d_in/group]: the exact int32 group
 *           accumulators sum_{k in group} xq[t][k]*wq[o][k], taken from TMEM.
 *           For small layers only (T*d_out*d_in/group*4 bytes).
 *   expert/perm (device) out int32 [T] (as qe_route); sa (device) out fp32 [T]
 *   in token order. Any of acc/expert/perm/sa may be NULL.
 */
QE_API qe_status qe_linear_forward_debug(const qe_layer_desc* desc, const qe_layer_weights* weights, const void* X,
                                  qe_dtype x_dtype, int32_t T, void* Y, qe_dtype y_dtype, void* workspace,
                                  size_t workspace_bytes, int32_t* acc, int32_t* expert, int32_t* perm, float* sa,
                                  void* stream);

#ifdef __cplusplus
}
#endif
#endif /* QE_H_ */
