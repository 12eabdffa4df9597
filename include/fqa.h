/*
 * fqa.h -- C ABI of the FP8 quantized attention library for B200 (sm_100a).
 *
 * The library computes the hot path of FLUX-style diffusion-transformer
 * inference: non-causal scaled dot-product attention over the joint
 * text + image (+ context-image) token sequence, with Q, K and V quantized to
 * FP8 E4M3 and the attention itself run in FP8, plus an unquantized BF16
 * comparison path.
 *
 * Sources (web pages, by title and section):
 *  [RTX-DE] "NVIDIA RTX AI optimiert FLUX.1 fuer Bilddaten mit niedriger
 *           Genauigkeit": the SDPA quantization paragraph (FP8 and FP4 schemes
 *           differ only in the precision of the Q, K, V projections;
 *           SageAttention named as the lineage) and the Table-1 paragraph
 *           (attention kept in FP8 for numerical stability; FP8 about 2x BF16).
 *  [RTX-KR] "NVIDIA RTX AI, 저정밀 양자화로 FLUX.1 Kontext 최적화": SDPA is about
 *           75% of the transformer's compute cost; quantizing it is the core
 *           of the work; Kontext concatenates context-image tokens (about 2x
 *           the sequence).
 *  [KLEIN]  "FLUX 3 Image Klein Base: 생성 3.46배, 8장 확장 병목", section
 *           "왜 이런 차이가 나나": VANILLA BF16 attention is about 60% of DiT
 *           kernel time on one B200; cuDNN FP8 and VC-Attention FP8 are the
 *           FP8 backends measured there.
 * The pages give no scale granularity, smoothing, rounding, P rule or API.
 * The readings used (stated again at each call): one FP32 absmax scale per
 * (batch, head, 64-token block) mapping onto the E4M3 maximum 448, K smoothed
 * by its per-channel mean, KV tiles of 128 keys with an exact running maximum,
 * P = E4M3(p * 448 * sv_J / sv_max), row sum of unquantized p.
 *
 * Conventions for every call:
 *  - Pointers named as tensors are DEVICE pointers owned by the caller; the
 *    library allocates no device memory, frees nothing and keeps no per-call
 *    state (a per-device cache of a status-word address and the driver's
 *    tensor-map encoder is built on first use, thread-safely).
 *  - All work is enqueued asynchronously on `cuda_stream` (a cudaStream_t;
 *    NULL = the legacy default stream).  No call synchronizes, except
 *    fqa_debug_status().
 *  - Layouts are row-major and contiguous: [B, H, N, d] with d innermost.
 *  - Limits: d == 128; any 1 <= N <= 65536 (real prompt lengths: the last
 *    64-token block and the last 128-key tile of a head may be short; see
 *    fqa_quantize and fqa_attention_fp8); B, H >= 1, B*H <= 65535,
 *    B*H*N < 2^31; device pointers
 *    16-byte aligned (the block-scale arrays and sv_max 4-byte aligned; k_mean
 *    16-byte aligned); a finite softmax_scale > 0; outputs must not overlap
 *    inputs.
 *  - Errors: arguments are checked on the host before anything is launched;
 *    an argument error returns a status and launches nothing.  A launch
 *    failure returns FQA_ERR_CUDA.  Non-finite input values are outside the
 *    contract (no error is reported; results are unspecified).
 *  - Device-side waits are bounded (about 1.5 s); a wait that gives up sets a
 *    bit in a device status word, abandons the tile and returns; read it with
 *    fqa_debug_status().  No kernel traps.
 */
#ifndef FQA_H
#define FQA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FQA_API __attribute__((visibility("default")))
#else
#define FQA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FQA_OK = 0,
  FQA_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad dtype, small workspace */
  FQA_ERR_UNSUPPORTED = 2,  /* d != 128, sizes beyond the limits */
  FQA_ERR_MISALIGNED = 3,   /* a pointer not aligned as required */
  FQA_ERR_CUDA = 4,         /* a CUDA runtime / driver call or launch failed */
  FQA_ERR_TIMEOUT = 5       /* a bounded device wait gave up (from fqa_debug_status) */
} fqa_status;

typedef enum {
  FQA_OUT_BF16 = 0,         /* production output, round to nearest even */
  FQA_OUT_F32 = 1           /* verification output: the FP32 values before BF16 rounding */
} fqa_out_dtype;

/* Library version, (major << 16) | minor. */
FQA_API int fqa_version(void);

/* Human-readable name of a status code (static storage). */
FQA_API const char* fqa_status_string(fqa_status status);

/*
 * Bytes of device workspace fqa_quantize() needs: B*H*ceil(N/64)*d*4 rounded
 * up to a multiple of 256 (the per-64-token-block partial sums of the K mean),
 * plus 256 (the launch's grid-barrier and work-queue counters).  Returns 0
 * for invalid sizes.
 */
FQA_API size_t fqa_quantize_workspace_bytes(int B, int H, int N, int d);

/*
 * fqa_quantize -- BF16 Q, K, V -> E4M3 codes and FP32 block scales.
 * [RTX-DE] SDPA quantization paragraph: Q, K and V are the quantized inputs.
 *
 * For each (b, h), with blocks of 64 tokens (the last one holds the
 * N - 64*(ceil(N/64)-1) remaining tokens):
 *   k_mean[c] = (sum over blocks j, ascending, of the sequential binary32 sum
 *               of K over the block's tokens) / N
 *               (pinned order, one round-to-nearest division);
 *   for each block and tensor X in {Q, K - k_mean, V} (the K difference is
 *   one binary32 subtraction per element):
 *     amax = max |X| over the block's tokens x 128 channels;
 *     scale = amax / 448, inv = 448 / amax (binary32 divisions; both 0 if amax = 0);
 *     code  = E4M3 round-to-nearest-even, saturating, of fl32(X * inv);
 *     tiny blocks: where inv overflows binary32 the code is that of
 *     fl32(X / scale), and where scale underflows to 0 the block is flushed
 *     (inv = 0, signed-zero codes) -- finite inputs never give NaN codes;
 *   sv_max = max over blocks of the V scales.
 * The results are bit-exact functions of the inputs (no atomics that change
 * values, no order dependence).
 *
 * q, k, v      in : BF16 [B,H,N,d]
 * q8, k8, v8   out: E4M3 codes, uint8 [B,H,N,d] (same layout as the inputs)
 * sq, sk, sv   out: FP32 [B,H,ceil(N/64)] block scales
 * sv_max       out: FP32 [B,H]
 * k_mean       out: FP32 [B,H,d]
 * workspace    scratch of at least fqa_quantize_workspace_bytes(B,H,N,d)
 *              bytes, 16-byte aligned; contents on entry are ignored.
 * Enqueues on cuda_stream a 24-byte memset of the workspace counters and one
 * cooperative kernel launch (V codes and K partial sums; K mean and V head
 * maxima; K codes -- phases separated by bounded grid barriers, with the Q
 * codes computed while each barrier completes; 64-token blocks handed out
 * through work queues).
 */
FQA_API fqa_status fqa_quantize(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                        void* q8, void* k8, void* v8, float* sq, float* sk, float* sv,
                        float* sv_max, float* k_mean, void* workspace, size_t workspace_bytes,
                        void* cuda_stream);

/*
 * fqa_quantize_keyerr -- fqa_quantize() that also writes each key's
 * quantization error, the selection metric of fqa_attention_fp8_corrected().
 * [KLEIN] section "왜 이런 차이가 나나" (VC-Attention FP8 corrects the tokens
 * with large error); the error measure is a reading:
 *   k_err[b,h,n] = sum over channels c of r_c^2, r_c = fl32(x_c - fl32(dec(k8_c) * sk)),
 *   x_c = fl32(k_c - k_mean[c]), each square rounded to binary32, summed in a
 *   pinned order: 16 groups of 8 consecutive channels summed sequentially,
 *   then g_i + g_i+8, then + the term 4 apart, 2 apart, 1 apart.
 * Same arguments and results as fqa_quantize() plus
 * k_err  out: FP32 [B,H,N] (4-byte aligned, not NULL).
 * Computed in the same launch (no extra pass over K).
 */
FQA_API fqa_status fqa_quantize_keyerr(const void* q, const void* k, const void* v, int B, int H, int N,
                                       int d, void* q8, void* k8, void* v8, float* sq, float* sk,
                                       float* sv, float* sv_max, float* k_mean, float* k_err,
                                       void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * fqa_quantize_noalloc -- fqa_quantize() without a workspace argument, for
 * callers that cannot allocate device memory at call time: for example an
 * operator running inside a host framework that owns all device memory and
 * forbids allocation while it executes, or a runtime whose device memory is
 * planned once up front.  (The pages have no counterpart; this is a library
 * convenience.)
 *
 * Same arguments, results and bit-exactness as fqa_quantize(), minus
 * workspace/workspace_bytes.  The scratch is a fixed array of
 * fqa_quantize_noalloc_max_workspace_bytes() = 8 MiB + 256 bytes inside the
 * library (8 MiB of K-mean partial sums, enough for B*H*ceil(N/64) <= 16384
 * blocks, plus the launch's counters), one per GPU that loads it, held until
 * the process exits.  Sizes whose scratch need,
 * fqa_quantize_workspace_bytes(B,H,N,d), exceeds that limit are rejected with
 * FQA_ERR_UNSUPPORTED before anything is launched.  Neither this call nor
 * its set-up allocates device memory (no cudaMalloc, cudaFree or allocating
 * library routine).
 *
 * The first call on a device looks up the device address of that device's
 * array (with that device current); make that first call before any stream
 * capture.  The address is cached only once the lookup succeeds, so a first
 * call that failed is retried by the next one.  Every call on a device shares the one array and
 * leaves its last contents there; nothing in it needs to start at zero.  Calls
 * that overlap on the GPU (e.g. on two streams at once) race on the array:
 * order them on one stream or synchronize between them.
 */
FQA_API fqa_status fqa_quantize_noalloc(const void* q, const void* k, const void* v, int B, int H,
                                        int N, int d, void* q8, void* k8, void* v8, float* sq,
                                        float* sk, float* sv, float* sv_max, float* k_mean,
                                        void* cuda_stream);

/* Size of the fixed scratch array fqa_quantize_noalloc() uses (8 MiB + 256 bytes). */
FQA_API size_t fqa_quantize_noalloc_max_workspace_bytes(void);

/*
 * fqa_attention_fp8 -- fused FP8 attention on fqa_quantize() outputs.
 * [RTX-DE] Table-1 paragraph (attention in FP8); [RTX-KR] SDPA paragraph.
 *
 * For query row i (64-token block I) over KV tiles of 128 keys, ascending:
 *   x_j  = (q8_i . k8_j) * sq_I * sk_J * softmax_scale * log2(e)   (J = j/64)
 *   m    = running max of x, updated exactly once per tile
 *   p_j  = 2^(x_j - m),  l = l * 2^(m_old - m_new) + sum p_j
 *   P_j  = E4M3(p_j * 448 * sv_J / sv_max)
 *   O    = O * 2^(m_old - m_new) + sum_j P_j * v8_j        (FP32 accumulate)
 *   out_i = O * (sv_max / 448) / l
 * Scores use the smoothed K codes; smoothing leaves softmax unchanged because
 * q . k_mean is constant along a row.  sv_max == 0 gives out = 0.
 * Evaluated in binary32: x = fl(S * a) rounded toward zero, then x - m, so
 * the row maximum gets p = 1 exactly; a P code whose binary32 value lies
 * within evaluation error of an E4M3 rounding midpoint may round either way.
 * Any N: the last tile holds the N % 128 remaining keys (when nonzero) and
 * keys past N take no part (no maximum, row-sum term or P code); the row
 * sum's correction for them is a binary32 subtraction, so l may differ from
 * a sum that never had them by a few ulp.
 * Enqueues one persistent kernel launch (one CTA per SM).
 *
 * out: [B,H,N,d] BF16 (FQA_OUT_BF16) or FP32 (FQA_OUT_F32).
 * softmax_scale: typically fl32(1/sqrt(d)).
 */
FQA_API fqa_status fqa_attention_fp8(const void* q8, const void* k8, const void* v8, const float* sq,
                             const float* sk, const float* sv, const float* sv_max, int B, int H,
                             int N, int d, float softmax_scale, void* out,
                             fqa_out_dtype out_dtype, void* cuda_stream);

/*
 * fqa_attention_bf16 -- the unquantized comparison path ([KLEIN], VANILLA
 * BF16 attention): softmax(Q K^T * softmax_scale) V with BF16 operands, FP32
 * accumulation and online softmax over 128-key tiles (the last one holds the
 * N % 128 remaining keys), P rounded to BF16 for the P.V product, out = O / l.
 *
 * q, k, v: BF16 [B,H,N,d]; out: [B,H,N,d] BF16 or FP32.
 */
FQA_API fqa_status fqa_attention_bf16(const void* q, const void* k, const void* v, int B, int H, int N,
                              int d, float softmax_scale, void* out, fqa_out_dtype out_dtype,
                              void* cuda_stream);

/*
 * Sequence-parallel (Ulysses) layouts.  [KLEIN] section "결과" and "고를 때
 * 기준": multi-GPU runs split the CFG pair across GPU groups and shard each
 * sequence over the GPUs of a group (Ulysses, degree 4 or 8), with an
 * all-to-all that turns a sequence shard into a head shard before attention
 * and back after it.  With P ranks in a group, rank r holding tokens
 * [r Nl, (r+1) Nl) of all H = P * Hl heads, the all-to-all delivers to rank
 * r its Hl heads for every token as P chunks: the layout
 *   [B, P, Hl, Nl, d]   (chunk p: tokens [p Nl, (p+1) Nl) of the Hl heads).
 * The two calls below read and write that layout directly, so no separate
 * pack or unpack pass runs around the collectives.  Nl must be a multiple of
 * 64 (no quantization block straddles two chunks); N = P * Nl.
 */

/* fqa_quantize() on inputs q, k, v in the layout [B, P, Hl, Nl, d]; every
 * output in the usual layouts for B, Hl heads and N = P * Nl tokens.  Codes
 * and scales are bit-identical to fqa_quantize() on the same tokens. */
FQA_API fqa_status fqa_quantize_a2a(const void* q, const void* k, const void* v, int B, int Hl, int P, int Nl,
                                    int d, void* q8, void* k8, void* v8, float* sq, float* sk, float* sv,
                                    float* sv_max, float* k_mean, void* workspace, size_t workspace_bytes,
                                    void* cuda_stream);

/* fqa_attention_fp8() for B, Hl heads and N = P * Nl tokens, with out written
 * in the layout [B, P, Hl, Nl, d] (ready for the return all-to-all);
 * bit-identical values to fqa_attention_fp8(). */
FQA_API fqa_status fqa_attention_fp8_a2a(const void* q8, const void* k8, const void* v8, const float* sq,
                                         const float* sk, const float* sv, const float* sv_max, int B, int Hl,
                                         int P, int Nl, int d, float softmax_scale, void* out,
                                         fqa_out_dtype out_dtype, void* cuda_stream);

/*
 * Error-corrected FP8 attention: FP8 attention that corrects only the tokens
 * with large error.  [KLEIN] section "왜 이런 차이가 나나": VC-Attention FP8
 * (rho = 0.005) is one of the B200 FP8 attention backends measured there; the
 * page gives the name, the idea and rho only.  Readings: the corrected tokens
 * are, per (b, h), the fqa_corrected_keys(N, rho) keys with the largest
 * k_err (ties to the lower index); their part of the softmax is computed
 * exactly from the BF16 inputs (scores on the smoothed keys,
 * (q . k - q . k_mean) * softmax_scale), the FP8 rule of fqa_attention_fp8()
 * runs over the other keys, and the two partial softmaxes are merged by their
 * maxima and row sums.
 */

/* Keys corrected per head: ceil(rho * N - 0.01) clamped to [0, N] (rho is
 * binary32, whose rounding moves rho * N by at most 0.004 for N <= 65536: a
 * product meant to be an integer stays that integer); -1 for N < 1 or rho
 * outside [0, 1]. */
FQA_API int fqa_corrected_keys(int N, float rho);

/*
 * fqa_select_keys -- the kc keys of each (b, h) with the largest k_err, ties
 * to the lower token index.  k_err: FP32 [B,H,N] (fqa_quantize_keyerr);
 * kmask out: uint32 [B,H,ceil(N/32)], bit k of word w set when key 32w + k
 * is selected; idx out: int32 [B,H,kc], the selected keys in ascending order.
 * 1 <= kc <= N.  One launch, one CTA per (b, h).
 */
FQA_API fqa_status fqa_select_keys(const float* k_err, int B, int H, int N, int kc, uint32_t* kmask,
                                   int* idx, void* cuda_stream);

/* Workspace bytes of fqa_attention_fp8_corrected(): the key mask, the
 * corrected indices, each row's FP8-part (m, l) and the FP8 part's FP32
 * output (B*H*N*512 bytes dominate); 0 for invalid sizes. */
FQA_API size_t fqa_attention_fp8_corrected_workspace_bytes(int B, int H, int N, int d, float rho);

/*
 * fqa_attention_fp8_corrected -- error-corrected FP8 attention.
 * q, k, v: the BF16 inputs [B,H,N,d]; q8 .. k_mean: the fqa_quantize_keyerr()
 * outputs for them; k_err: its key errors; rho in [0, 1] (0 = plain FP8
 * attention); out: [B,H,N,d] BF16 or FP32; workspace of at least
 * fqa_attention_fp8_corrected_workspace_bytes(), 16-byte aligned.
 * For query row i, with C the selected keys of its head:
 *   FP8 part over keys not in C (the fqa_attention_fp8() rule, keys in C
 *   taking no part): normalized output O1, maximum m1, row sum l1;
 *   exact part over C: s_j = (q_i . k_j - q_i . k_mean) * softmax_scale * log2(e),
 *   m2 = max s_j, p_j = 2^(s_j - m2), l2 = sum p_j, A2 = sum p_j v_j;
 *   out_i = (O1 l1 2^(m1 - M) + A2 2^(m2 - M)) / (l1 2^(m1 - M) + l2 2^(m2 - M)),
 *   M = max(m1, m2).
 * The exact part runs in FP32 on the tensor cores (BF16 operands, P split
 * into BF16 high and low parts).  Enqueues the selection, the FP8 attention
 * launch with the key mask, and the exact part and merge.
 */
FQA_API fqa_status fqa_attention_fp8_corrected(const void* q, const void* k, const void* v, const void* q8,
                                               const void* k8, const void* v8, const float* sq,
                                               const float* sk, const float* sv, const float* sv_max,
                                               const float* k_mean, const float* k_err, int B, int H, int N,
                                               int d, float softmax_scale, float rho, void* out,
                                               fqa_out_dtype out_dtype, void* workspace,
                                               size_t workspace_bytes, void* cuda_stream);

/*
 * fqa_quantize_nvfp4_qk -- Q and smoothed K in NVFP4 for the FP4 Q.K variant.
 * [RTX-DE] SDPA quantization paragraph: the FP8 and FP4 schemes differ only
 * in the precision of the Q, K, V projections; attention itself stays in FP8.
 * The element format (E2M1) and the 16-channel E4M3 group scale are the
 * NVFP4 reading of "FP4"; V keeps its FP8 codes and scales from fqa_quantize().
 * q, k: BF16 [B,H,N,d] (16-byte aligned); k_mean: FP32 [B,H,d], the channel
 * means fqa_quantize() wrote for the same k.  Outputs (device, caller-owned):
 *   q4, k4  : uint8 [B,H,N,d/2], two E2M1 codes per byte (element 2i in bits
 *             [0,4), 2i+1 in bits [4,8)); 4-byte aligned
 *   sfq, sfk: uint8 [B,H,N,d/16], one unsigned E4M3 scale per 16 channels
 *   sq1, sk1: FP32 [B,H,ceil(N/64)], one scale per 64-token block
 * Per 64-token block of x (= q, or fl32(k - k_mean) for K), in binary32:
 *   s1 = amax / 2688 (6 x 448, so group scales reach up to 448);
 *   per token and 16-channel group g: s2 = E4M3(amax_g / fl32(6 s1)) (round
 *   to nearest even, saturating), dg = fl32(s1 dec(s2)),
 *   code = E2M1(fl32(x / dg)) (nearest even, saturating to +-6; 0 if dg = 0).
 * amax = 0 flushes the block (s1 = 0, every scale and code 0).  Any N >= 1.
 */
FQA_API fqa_status fqa_quantize_nvfp4_qk(const void* q, const void* k, const float* k_mean, int B, int H,
                                         int N, int d, uint8_t* q4, uint8_t* k4, uint8_t* sfq,
                                         uint8_t* sfk, float* sq1, float* sk1, void* cuda_stream);

/*
 * fqa_attention_nvfp4 -- attention with Q.K^T on the block-scaled FP4 tensor
 * cores and P.V as in fqa_attention_fp8().  [RTX-DE] SDPA quantization
 * paragraph, as fqa_quantize_nvfp4_qk().  For query row i and key j:
 *   S_ij = sum over groups g of dec(sfq_ig) dec(sfk_jg) sum_c e2m1(q_ic) e2m1(k_jc)
 *   x_ij = S_ij * sq1_I * sk1_J * softmax_scale * log2(e)
 * then the fqa_attention_fp8() rule on x: exact running maximum over KV
 * tiles of 128 keys, P = E4M3(2^(x - m) * 448 * sv_J / sv_max), O += P.V in
 * FP32, out = O * (sv_max / 448) / l.
 * q4 .. sk1: fqa_quantize_nvfp4_qk() outputs; v8, sv, sv_max: fqa_quantize()
 * outputs.  q4, k4, v8 and out 16-byte aligned, sfq and sfk 8-byte aligned.
 * Any N >= 1: the last 128-key tile of a short sequence holds N % 128 keys
 * (keys past N take no part), as in fqa_attention_fp8().
 */
FQA_API fqa_status fqa_attention_nvfp4(const uint8_t* q4, const uint8_t* k4, const uint8_t* sfq,
                                       const uint8_t* sfk, const float* sq1, const float* sk1,
                                       const void* v8, const float* sv, const float* sv_max, int B, int H,
                                       int N, int d, float softmax_scale, void* out, fqa_out_dtype out_dtype,
                                       void* cuda_stream);

/*
 * fqa_e2m1_encode -- the library's binary32 -> E2M1 conversion (round to
 * nearest even, saturating to +-6), two values per byte as in
 * fqa_quantize_nvfp4_qk: out[i] = code(x[2i]) | code(x[2i+1]) << 4.
 * x: FP32 [2 npairs], 8-byte aligned; out: uint8 [npairs] (device).
 */
FQA_API fqa_status fqa_e2m1_encode(const float* x, uint8_t* out, size_t npairs, void* cuda_stream);

/*
 * fqa_exp2_error -- measures the exponential the attention kernels use for
 * p = 2^(x - m) and the rescale factors (the hardware ex2 approximation with
 * flush-to-zero) at every binary32 x in [lo, hi], -126 <= lo <= hi <= 0,
 * against binary64 exp2 (results of 2^x below 2^-126 are skipped: they flush
 * to zero by design).  *max_rel_bits (device, 4-byte aligned) receives the
 * bit pattern of the largest relative error as a binary32 value; it is
 * zeroed first.  A check of the error budget the parity tolerance assumes
 * for this step (2^-21), not part of the path.
 */
FQA_API fqa_status fqa_exp2_error(float lo, float hi, uint32_t* max_rel_bits, void* cuda_stream);

/*
 * fqa_e4m3_encode -- the library's binary32 -> E4M3 conversion (round to
 * nearest even, saturating to +-448, NaN -> 0x7F), exposed so that callers
 * can check the codec exhaustively.  x: FP32 [n], out: uint8 [n] (device).
 */
FQA_API fqa_status fqa_e4m3_encode(const float* x, uint8_t* out, size_t n, void* cuda_stream);

/*
 * fqa_debug_wait_timeout -- checks the bounded-wait path (no counterpart on
 * the pages): launches one thread that waits on an mbarrier nothing arrives
 * on; after limit_us microseconds (1 .. 2,000,000) the wait gives up, sets the
 * timeout bit of the device status word and the kernel returns, leaving the
 * context usable.  The next fqa_debug_status() then returns FQA_ERR_TIMEOUT.
 */
FQA_API fqa_status fqa_debug_wait_timeout(uint32_t limit_us, void* cuda_stream);

/*
 * fqa_debug_status -- synchronizes cuda_stream, reads and clears the
 * device status word of the current device.  Returns FQA_ERR_TIMEOUT if a
 * bounded device wait gave up since the last call, FQA_ERR_CUDA if the
 * synchronization failed, FQA_OK otherwise.  *flags_out (if not NULL)
 * receives the raw bits.
 */
FQA_API fqa_status fqa_debug_status(void* cuda_stream, uint32_t* flags_out);

#ifdef __cplusplus
}
#endif

#endif /* FQA_H */
