/*
 * qk4v8.h - C ABI of the QK4V8 mixed-precision attention library (libqk4v8.so).
 *
 * The method: the MpFA QK4V8 article (mhpn.cn, "MpFA免训练量化：QK4V8混合精度在
 * Blackwell上的推理加速实践").
 *   - Q and K are quantized to 4 bits and V to 8 bits (sections 1.1, 2.1, 2.2).
 *   - Scales are computed online, block by block, with no calibration
 *     (sections 1.2, 3.2).
 *   - Attention runs tile by tile with an FP32 online softmax and FP32
 *     accumulators (sections 2.3, 3.3).
 * The block format is OCP MX with one E8M0 scale per 32 values (MiMo FP4
 * article, wmrh.cn, section "MXFP4专家量化"):
 *   - MXFP4 (E2M1 elements) for Q and K, grouped along head_dim.
 *   - MXFP8 (E4M3 elements) for V, grouped along the token axis.
 *
 * Conventions shared by every entry point
 *   - head_dim d is 128.
 *   - bf16 activations are [B][T][H][128] with caller-given element strides for
 *     B, T and H. The channel stride is 1. Base and strides are 16-byte aligned.
 *   - Device pointers are owned by the caller. The library never allocates
 *     device memory, never synchronises, and only enqueues work on `stream`
 *     (a cudaStream_t passed as void*; NULL is the legacy default stream).
 *   - Return value: a qk4v8_status. Arguments are validated synchronously,
 *     before anything is enqueued. QK4V8_ERR_CUDA carries the CUDA error text,
 *     available from qk4v8_last_error() on the calling thread.
 *   - Device-side failures (a pipeline wait that exceeded its time limit) are
 *     written to *dev_status (device int32, optional) as QK4V8_ERR_TIMEOUT. The
 *     kernel then returns normally, so the CUDA context stays usable.
 *
 * Packed formats (produced by the quantize calls, consumed by attention)
 *   MXFP4 tensor (Q or K), token capacity `cap` (a multiple of 128):
 *     codes  uint8 [B][H][cap][64]      two E2M1 codes per byte; element 2i of a
 *                                        token's 128 channels is the low nibble
 *                                        of byte i.
 *     scales uint8 [B][H][cap/128][512] E8M0 (value 2^(byte-127)), one per 32
 *                                        channels. In block n (tokens 128n..128n+127)
 *                                        token t, group g (channels 32g..32g+31) is
 *                                        at byte (t%32)*16 + ((t%128)/32)*4 + g.
 *   MXFP8 V tensor, capacity `cap` (a multiple of 128):
 *     codes  uint8 [B][H][cap/128][128][128]  E4M3 in 128-token blocks: block n
 *                                        holds tokens 128n..128n+127 as 128
 *                                        channel rows of 128 bytes (token t at
 *                                        byte t%128 of its channel's row), each
 *                                        block 16 KiB contiguous.
 *     scales uint8 [B][H][cap/128][512] E8M0, one per channel per 32 tokens. In
 *                                        block n, channel c, group g (tokens
 *                                        128n+32g .. 128n+32g+31) is at byte
 *                                        (c%32)*16 + (c/32)*4 + g.
 *   Tokens at or past a sequence's length are padding. Their codes are 0, and
 *   scale bytes of groups with no valid token are 0. A V group that is only
 *   partly valid takes its amax over the valid tokens only.
 *
 * Quantization rule (OCP MX): per group of 32 values,
 *     X = floor(log2(max |x|)) - emax (E2M1: 2, E4M3: 8), clamped to [-127, 127],
 *         and X = -127 when the group is all zeros;
 *     code = round-to-nearest-even(x / 2^X) onto the element grid, saturating
 *            at +-6 (E2M1) or +-448 (E4M3). A value that rounds to zero keeps
 *            its sign bit.
 */
#ifndef QK4V8_H
#define QK4V8_H

#include <stddef.h>
#include <stdint.h>

#ifndef QK4V8_API
#define QK4V8_API __attribute__((visibility("default")))
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QK4V8_OK = 0,
    QK4V8_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad shape or stride, small workspace */
    QK4V8_ERR_UNSUPPORTED = 2,  /* the current device is not sm_100 (B200 class) */
    QK4V8_ERR_CUDA = 3,         /* a CUDA call failed; see qk4v8_last_error() */
    QK4V8_ERR_TIMEOUT = 4       /* written to *dev_status by a kernel whose wait expired */
} qk4v8_status;

/* Text for a status code (static storage). */
QK4V8_API const char *qk4v8_status_string(int status);

/* Text of the last QK4V8_ERR_CUDA or QK4V8_ERR_INVALID_ARG on this thread. */
QK4V8_API const char *qk4v8_last_error(void);

/* QK4V8_OK when `device` is an sm_100 GPU this library was built for. */
QK4V8_API int qk4v8_device_supported(int device);

/* Byte sizes of the packed buffers for B sequences, H heads, capacity cap. */
QK4V8_API size_t qk4v8_mxfp4_codes_bytes(int B, int H, int cap);
QK4V8_API size_t qk4v8_mxfp8_codes_bytes(int B, int H, int cap);
QK4V8_API size_t qk4v8_scales_bytes(int B, int H, int cap);

/*
 * MXFP4 quantization of Q or K (article section 3.2: scales computed while the
 * block is loaded; one E8M0 scale per 32 channels).
 *   x        bf16 [B][S][H][128] (device), strides in elements
 *   seqlens  int32 [B] (device, nullable): tokens t >= seqlens[b] become padding
 *   cap      token capacity of the output, a multiple of 128, >= S
 *   codes, scales  outputs in the MXFP4 layout above. Every token < cap is
 *            written: tokens >= S, or >= seqlens[b], as padding.
 */
QK4V8_API int qk4v8_quantize_qk(const void *x, int B, int S, int H, int d,
                      int64_t stride_b, int64_t stride_s, int64_t stride_h,
                      const int32_t *seqlens, int cap,
                      uint8_t *codes, uint8_t *scales, void *stream);

/*
 * MXFP4 quantization of Q or K after a Hadamard rotation of each row (MpFA
 * article, section 3.1, and the outlier discussion of section 2.1: a light
 * rotation ahead of the per-group 4-bit quantization spreads outlier channels
 * over the whole row). Each (token, head) row x of 128 channels becomes
 * y = x H / sqrt(128), H the Sylvester Hadamard matrix
 * (H[i][j] = (-1)^popcount(i & j)), computed in fp32 as the fast
 * Walsh-Hadamard transform (butterfly strides 1, 2, ..., 64) followed by one
 * multiply by the fp32 value nearest 2^-3.5; y is then quantized exactly as by
 * qk4v8_quantize_qk. The rotation is orthonormal, so quantizing both Q and K
 * this way leaves Q K^T, and the attention calls, unchanged: pass the rotated
 * packed Q and K to them as they are (V is not rotated). Arguments, layout and
 * errors as for qk4v8_quantize_qk.
 */
QK4V8_API int qk4v8_quantize_qk_hadamard(const void *x, int B, int S, int H, int d,
                               int64_t stride_b, int64_t stride_s, int64_t stride_h,
                               const int32_t *seqlens, int cap,
                               uint8_t *codes, uint8_t *scales, void *stream);

/*
 * MXFP8-E4M3 quantization of V, groups of 32 along the token axis (article
 * section 2.2: V stays at 8 bits).
 *   v        bf16 [B][S][H][128] (device), strides in elements
 *   seqlens  int32 [B] (device, nullable): valid tokens per sequence
 *   cap      capacity, multiple of 128, >= S
 *   codes, scales  outputs in the MXFP8 V layout above, fully written.
 */
QK4V8_API int qk4v8_quantize_v(const void *v, int B, int S, int H, int d,
                     int64_t stride_b, int64_t stride_s, int64_t stride_h,
                     const int32_t *seqlens, int cap,
                     uint8_t *codes, uint8_t *scales, void *stream);

/*
 * Q, K and V in one call and one launch on `stream` (the same bytes as the three
 * calls above): Q [B][Sq][Hq][128] into capacity q_cap, K and V
 * [B][Sk][Hkv][128] into capacity kv_cap. Contiguous [B][T][H][128] inputs;
 * seqlens_k (device, nullable) marks valid KV tokens. Errors as for the
 * separate calls; q_cap * Hq and kv_cap * Hkv below 2^30.
 */
QK4V8_API int qk4v8_quantize(const void *q, const void *k, const void *v,
                   int B, int Sq, int Sk, int Hq, int Hkv, int d,
                   const int32_t *seqlens_k, int q_cap, int kv_cap,
                   uint8_t *q_codes, uint8_t *q_scales,
                   uint8_t *k_codes, uint8_t *k_scales,
                   uint8_t *v_codes, uint8_t *v_scales, void *stream);

/*
 * QK4V8 attention for prefill (article sections 2.3 and 3.3: blockwise online
 * softmax in FP32, dequantization folded into the block-scaled tensor-core MMA).
 *   q_*      packed MXFP4 Q, [B][Hq][q_cap], Sq valid query tokens per sequence
 *   k_*, v_* packed MXFP4 K and MXFP8 V, [B][Hkv][kv_cap]
 *   seqlens_k int32 [B] (device, nullable: every sequence has Sk keys)
 *   causal   bottom-right aligned: query i attends keys j <= i + (L - Sq)
 *   softmax_scale  <= 0 selects 1/sqrt(128)
 *   out      bf16 [B][Sq][Hq][128]
 *   lse      float [B][Hq][Sq] natural-log log-sum-exp (nullable)
 *   dev_status int32 (device, nullable): receives QK4V8_ERR_TIMEOUT on a stall
 * Query head h reads KV head h / (Hq / Hkv). Rows with no allowed key output 0
 * with lse = -inf.
 */
QK4V8_API int qk4v8_attention_prefill(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int Sq, int q_cap,
                            const uint8_t *k_codes, const uint8_t *k_scales,
                            const uint8_t *v_codes, const uint8_t *v_scales, int Hkv, int Sk, int kv_cap,
                            const int32_t *seqlens_k, int causal, float softmax_scale,
                            void *out, float *lse, int32_t *dev_status, void *stream);

/*
 * Workspace bytes for qk4v8_attention_decode with these sizes: the split
 * partials float O[B][Hq][nq][splits][128], then float lse2[B][Hq][nq][splits],
 * then int32 [B][Hq] piece counts (the GQA decode kernel records there which
 * sequences it cut, for its merge launch).
 */
QK4V8_API size_t qk4v8_decode_workspace_bytes(int B, int Hq, int nq, int num_splits);

/*
 * The split count qk4v8_attention_decode picks when given num_splits = 0 for
 * B sequences of Hkv KV heads, (Hq / Hkv) * nq query rows per KV head and keys
 * up to max_seqlen: the count that minimises the modelled time of the waves of
 * CTAs on the current device (148 SMs when no device can be queried). Returns
 * 1 for invalid sizes.
 */
QK4V8_API int qk4v8_decode_default_splits(int B, int Hq, int Hkv, int nq, int max_seqlen);

/*
 * The two stages of qk4v8_attention_decode, as separate launches (MpFA
 * article, sections 1.3 and 3.3: the memory-bound decode attention with its
 * FP32 online softmax, here split over the KV length; the splits' partial
 * (max, sum, O) are combined afterwards).
 *
 * qk4v8_attention_decode_splitkv: for every (sequence, KV head, split) the
 * split kernel runs the tiled QK4V8 attention over the split's contiguous
 * slice of the cache. It writes the split's normalised partial output and
 * log2-sum-exp to `workspace`:
 *     float O[B][Hq][nq][splits][128], then float lse2[B][Hq][nq][splits].
 * A split with no key writes O = 0 and lse2 = -inf. Arguments as for
 * qk4v8_attention_decode.
 *
 * qk4v8_decode_merge: combines the splits of each query row,
 *     O = sum_s 2^(lse2_s - m) O_s / sum_s 2^(lse2_s - m),  m = max_s lse2_s,
 * into out bf16 [B][nq][Hq][128]. lse (nullable) receives the natural-log
 * log-sum-exp [B][Hq][nq]. num_splits must be the count the split-KV launch
 * used (qk4v8_decode_default_splits when it was given 0).
 */
QK4V8_API int qk4v8_attention_decode_splitkv(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int nq,
                                             int q_cap, const uint8_t *k_codes, const uint8_t *k_scales,
                                             const uint8_t *v_codes, const uint8_t *v_scales, int Hkv, int kv_cap,
                                             const int32_t *seqlens_k, int max_seqlen, int causal_in_block,
                                             float softmax_scale, int num_splits, void *workspace,
                                             size_t workspace_bytes, int32_t *dev_status, void *stream);

QK4V8_API int qk4v8_decode_merge(const void *workspace, size_t workspace_bytes, int B, int Hq, int nq,
                                 int num_splits, void *out, float *lse, void *stream);

/*
 * Split-KV decode and speculative block verify over a packed KV cache.
 * MpFA article, section 1.3: in decode, attention is memory bound, so the
 * packed cache (4-bit K, 8-bit V) is streamed once, split across CTAs, at HBM
 * rate. MiMo DFlash article, section on block-diffusion speculative decoding
 * (block_size 8): the backbone verifies a whole draft block in one forward,
 * hence up to nq = 8 query tokens per sequence, causal within the block.
 *   q_*      packed MXFP4 Q, [B][Hq][q_cap] with nq (1..8) query tokens
 *   k_*, v_* packed cache, [B][Hkv][kv_cap]
 *   seqlens_k int32 [B] (device, required), each <= kv_cap
 *   max_seqlen host upper bound on seqlens_k, used to plan the splits
 *   causal_in_block  query t of nq attends keys j <= L - nq + t
 *   num_splits  0 = qk4v8_decode_default_splits
 *   workspace  device scratch of qk4v8_decode_workspace_bytes(B, Hq, nq, splits);
 *            unused (and may be null) when the call runs one split with
 *            (Hq / Hkv) * nq <= 64, as the split kernel then writes out itself
 *   out      bf16 [B][nq][Hq][128]; lse float [B][Hq][nq] (nullable)
 * Requires (Hq / Hkv) * nq <= 128. Kernels by query rows per KV head:
 *   - up to 32: the swap-AB split kernel, then the merge (one launch when one
 *     split);
 *   - 33..64: the GQA decode kernel, one CTA per SM, which writes out and lse
 *     for every sequence it does not cut. When splits >= 2 and no sequence
 *     would be cut into more than `splits` pieces, it spreads the key tiles of
 *     all sequences evenly over the CTAs instead of cutting every sequence
 *     into `splits` equal parts; a sequence is then cut only where a CTA's
 *     share ends. With splits >= 2 a second, short launch merges the pieces of
 *     the cut sequences from the workspace.
 *   - 65..128: the 128-row split kernel, then the merge.
 */
QK4V8_API int qk4v8_attention_decode(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int nq, int q_cap,
                           const uint8_t *k_codes, const uint8_t *k_scales,
                           const uint8_t *v_codes, const uint8_t *v_scales, int Hkv, int kv_cap,
                           const int32_t *seqlens_k, int max_seqlen, int causal_in_block,
                           float softmax_scale, int num_splits, void *workspace, size_t workspace_bytes,
                           void *out, float *lse, int32_t *dev_status, void *stream);

/*
 * QK4V4: the comparison point of the MpFA article (section 2.2: V at 4 bits
 * costs about 0.8 perplexity against QK4V8; section 5.3: on long texts it
 * degrades further). V is quantized to MXFP4 (E2M1 codes, one E8M0 scale per
 * 32 tokens along the sequence, the same OCP MX rule with emax 2), halving
 * V's cache bytes (136 instead of 200 bytes per token and KV head with K).
 *   MXFP4 V tensor, capacity cap (a multiple of 128):
 *     codes  uint8 [B][H][cap/128][128][64]  the 128-token blocks of MXFP8 V,
 *                                        two E2M1 codes per byte along the token
 *                                        axis (even token in the low nibble), 64
 *                                        bytes per channel row of a block
 *                                        (qk4v8_mxfp4v_codes_bytes)
 *     scales uint8 [B][H][cap/128][512] as for MXFP8 V
 * qk4v8_quantize_v4: arguments as for qk4v8_quantize_v.
 * qk4v8_attention_decode_v4 / qk4v8_attention_decode_bf16_v4: the decode calls
 * (window included) over packed MXFP4 K and MXFP4 V, for up to 64 query rows
 * per KV head (the swap-AB and GQA decode kernels); V codes 32-byte aligned,
 * contiguous caches.
 * P stays two E4M3 terms; the block-scaled MMA takes V as its E2M1 operand.
 */
QK4V8_API size_t qk4v8_mxfp4v_codes_bytes(int B, int H, int cap);

QK4V8_API int qk4v8_quantize_v4(const void *v, int B, int S, int H, int d, int64_t stride_b, int64_t stride_s,
                                int64_t stride_h, const int32_t *seqlens, int cap, uint8_t *codes, uint8_t *scales,
                                void *stream);

QK4V8_API int qk4v8_attention_decode_v4(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int nq,
                                        int q_cap, const uint8_t *k_codes, const uint8_t *k_scales,
                                        const uint8_t *v_codes, const uint8_t *v_scales, int Hkv, int kv_cap,
                                        const int32_t *seqlens_k, int max_seqlen, int causal_in_block, int window,
                                        float softmax_scale, int num_splits, void *workspace,
                                        size_t workspace_bytes, void *out, float *lse, int32_t *dev_status,
                                        void *stream);

QK4V8_API int qk4v8_attention_decode_bf16_v4(const void *q, int B, int Hq, int nq, int64_t q_stride_b,
                                             int64_t q_stride_t, int64_t q_stride_h, const uint8_t *k_codes,
                                             const uint8_t *k_scales, const uint8_t *v_codes,
                                             const uint8_t *v_scales, int Hkv, int kv_cap, const int32_t *seqlens_k,
                                             int max_seqlen, int causal_in_block, int window, float softmax_scale,
                                             int num_splits, void *workspace, size_t workspace_bytes, void *out,
                                             float *lse, int32_t *dev_status, void *stream);

/*
 * Draft-block attention: decode with a sliding window (MiMo DFlash article,
 * section on block-diffusion speculative decoding: the draft model predicts a
 * block of 8 tokens in one forward; its attention sees the in-block positions
 * together with a sliding window over the most recent 1024 context tokens).
 * Reading taken: for a sequence of L keys whose last nq positions are the
 * query block, every query row sees keys j >= max(0, L - nq - window) (the
 * last `window` keys before the block, and the block), and, with
 * causal_in_block, only up to its own position; with causal_in_block = 0 the
 * block is non-causal, as in the draft model. window = 0 is plain decode.
 * Only the keys in the window are streamed: the splits cover the tiles from
 * the one holding the window's first key.
 *   window   >= 0; a window needs (Hq / Hkv) * nq <= 64 query rows per KV head
 *   other arguments, layouts and errors as for qk4v8_attention_decode (packed
 *   Q) and qk4v8_attention_decode_bf16 (bf16 Q, with its workspace rule);
 *   num_splits = 0 picks qk4v8_decode_default_splits_window.
 * qk4v8_decode_default_splits_window: the default split count for such a call
 * (qk4v8_decode_default_splits over the keys one block can see).
 */
QK4V8_API int qk4v8_attention_decode_window(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int nq,
                                            int q_cap, const uint8_t *k_codes, const uint8_t *k_scales,
                                            const uint8_t *v_codes, const uint8_t *v_scales, int Hkv, int kv_cap,
                                            const int32_t *seqlens_k, int max_seqlen, int causal_in_block,
                                            int window, float softmax_scale, int num_splits, void *workspace,
                                            size_t workspace_bytes, void *out, float *lse, int32_t *dev_status,
                                            void *stream);

QK4V8_API int qk4v8_attention_decode_bf16_window(const void *q, int B, int Hq, int nq, int64_t q_stride_b,
                                                 int64_t q_stride_t, int64_t q_stride_h, const uint8_t *k_codes,
                                                 const uint8_t *k_scales, const uint8_t *v_codes,
                                                 const uint8_t *v_scales, int Hkv, int kv_cap,
                                                 const int32_t *seqlens_k, int max_seqlen, int causal_in_block,
                                                 int window, float softmax_scale, int num_splits, void *workspace,
                                                 size_t workspace_bytes, void *out, float *lse, int32_t *dev_status,
                                                 void *stream);

QK4V8_API int qk4v8_decode_default_splits_window(int B, int Hq, int Hkv, int nq, int max_seqlen, int window);

/*
 * Split count for a decode call when the caller knows the sequence lengths on
 * the host (seqlens_host, int32 [B]; window as for the _window calls). For up
 * to 32 query rows per KV head it models each candidate split count with the
 * lengths as they are: CTAs start in launch order on the resident slots,
 * splits past a sequence's end cost nothing, and the running CTAs share the
 * memory bandwidth, so a last partial wave runs faster per CTA. It returns the
 * count with the least modelled time (a fixed split count assumes every
 * sequence has the longest length, and over-splits batches of mixed lengths).
 * For 33..64 rows it returns qk4v8_decode_default_splits_window (that kernel
 * balances its key tiles itself). Returns 1 for invalid sizes. Host only; no
 * device work.
 */
QK4V8_API int qk4v8_decode_plan_splits(int B, int Hq, int Hkv, int nq, const int32_t *seqlens_host, int window);

/*
 * Paged KV cache (MpFA article, section 6.1: the QK4V8 attention combined with
 * a quantized KV cache; section 3.2: block scales computed online as the data
 * arrives). The packed cache lives in pools of pages of 128 tokens; page p of
 * KV head h holds
 *   K codes  [num_pages][Hkv][128][64],  K scales [num_pages][Hkv][512]
 *   V codes  [num_pages][Hkv][128][128], V scales [num_pages][Hkv][512]
 * i.e. the packed layouts above with B = num_pages and cap = 128 (the size
 * helpers give the pool sizes: qk4v8_mxfp4_codes_bytes(num_pages, Hkv, 128)
 * and so on). block_table int32 [B][max_pages] (device) maps the n-th 128-token
 * block of sequence b to its page; sequences hold at most max_pages * 128
 * tokens. A block-table entry outside [0, num_pages) is not followed: the
 * kernels read page 0 instead (attention) or skip the token (append) and write
 * QK4V8_ERR_INVALID_ARG to *dev_status.
 *
 * qk4v8_kv_append: appends n_new tokens to every sequence. k_new and v_new are
 * bf16 [B][n_new][Hkv][128] with the given element strides (shared by both;
 * multiples of 8). Token t goes to position seqlens[b] + t (seqlens: device
 * int32 [B], the lengths before the call); seqlens_out (device, nullable, may
 * be seqlens) receives seqlens[b] + n_new once every kernel of the call has
 * read seqlens. K rows are quantized on their own (with hadamard_k, after the
 * rotation of qk4v8_quantize_qk_hadamard). V's 32-token groups change as
 * tokens arrive: every group the new tokens touch gets its E8M0 scale
 * recomputed from all of its tokens and all its codes rewritten, which needs
 * the bf16 values of the open (last, partly filled) group of each sequence and
 * head: v_tail, bf16 [B][Hkv][32][128] (qk4v8_kv_tail_bytes), owned by the
 * caller, read and refreshed by every append. So the bytes after any sequence
 * of appends equal those of qk4v8_quantize_qk / qk4v8_quantize_v over the whole
 * sequence. Build a sequence's cache by appending its prompt to an empty
 * sequence (seqlens 0, v_tail contents then unused). Codes of tokens past the
 * new length within the last V group are written as 0; other padding is left
 * as it was (the attention kernels ignore it). One launch on `stream`, two when
 * seqlens_out is seqlens (the in-place length update runs after every reader).
 *
 * qk4v8_attention_decode_paged / qk4v8_attention_decode_bf16_paged: the
 * decode calls (with the draft-block window) over such a pool, for up to 64
 * query rows per KV head; other arguments as for the non-paged calls.
 */
QK4V8_API size_t qk4v8_kv_tail_bytes(int B, int Hkv);

QK4V8_API int qk4v8_kv_append(const void *k_new, const void *v_new, int B, int n_new, int Hkv, int d,
                              int64_t stride_b, int64_t stride_t, int64_t stride_h, const int32_t *seqlens,
                              int32_t *seqlens_out, const int32_t *block_table, int max_pages, int num_pages,
                              uint8_t *k_codes, uint8_t *k_scales, uint8_t *v_codes, uint8_t *v_scales,
                              void *v_tail, int hadamard_k, int32_t *dev_status, void *stream);

QK4V8_API int qk4v8_attention_decode_paged(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int nq,
                                           int q_cap, const uint8_t *k_codes, const uint8_t *k_scales,
                                           const uint8_t *v_codes, const uint8_t *v_scales, int Hkv, int num_pages,
                                           const int32_t *block_table, int max_pages, const int32_t *seqlens_k,
                                           int max_seqlen, int causal_in_block, int window, float softmax_scale,
                                           int num_splits, void *workspace, size_t workspace_bytes, void *out,
                                           float *lse, int32_t *dev_status, void *stream);

QK4V8_API int qk4v8_attention_decode_bf16_paged(const void *q, int B, int Hq, int nq, int64_t q_stride_b,
                                                int64_t q_stride_t, int64_t q_stride_h, const uint8_t *k_codes,
                                                const uint8_t *k_scales, const uint8_t *v_codes,
                                                const uint8_t *v_scales, int Hkv, int num_pages,
                                                const int32_t *block_table, int max_pages, const int32_t *seqlens_k,
                                                int max_seqlen, int causal_in_block, int window,
                                                float softmax_scale, int num_splits, void *workspace,
                                                size_t workspace_bytes, void *out, float *lse, int32_t *dev_status,
                                                void *stream);

/*
 * Decode step from bf16 queries (MpFA QK4V8 article, section 3.2: the query's
 * MXFP4 scales are computed as it is loaded, inside the attention call).
 * Same result, bit for bit, as qk4v8_quantize_qk (capacity 128) followed by
 * qk4v8_attention_decode, in one call and usually one launch:
 *   - (Hq / Hkv) * nq <= 32: the split kernel reads the bf16 query rows and
 *     encodes them to MXFP4 itself; with one split it also writes out and lse
 *     directly, so there is no merge launch and no workspace.
 *   - 33..64: the nq query rows of each head are quantized into the front of
 *     the workspace (capacity 128 tokens), then the GQA decode kernel writes
 *     out and lse.
 *   - larger groups: the queries are quantized into the front of the
 *     workspace, then the 128-row split kernel and the merge run.
 *   q        bf16 [B][nq][Hq][128] (device), element strides q_stride_b,
 *            q_stride_t, q_stride_h, each a multiple of 8; channel stride 1;
 *            16-byte aligned
 *   workspace  device scratch of qk4v8_decode_bf16_workspace_bytes(B, Hq, Hkv,
 *            nq, splits) bytes (0: may be null), 16-byte aligned
 *   other arguments, out, lse and errors as for qk4v8_attention_decode.
 */
QK4V8_API size_t qk4v8_decode_bf16_workspace_bytes(int B, int Hq, int Hkv, int nq, int num_splits);

QK4V8_API int qk4v8_attention_decode_bf16(const void *q, int B, int Hq, int nq, int64_t q_stride_b,
                                          int64_t q_stride_t, int64_t q_stride_h, const uint8_t *k_codes,
                                          const uint8_t *k_scales, const uint8_t *v_codes, const uint8_t *v_scales,
                                          int Hkv, int kv_cap, const int32_t *seqlens_k, int max_seqlen,
                                          int causal_in_block, float softmax_scale, int num_splits, void *workspace,
                                          size_t workspace_bytes, void *out, float *lse, int32_t *dev_status,
                                          void *stream);

/*
 * Decode for callers that cannot allocate device memory: qk4v8_attention_decode
 * with the split-KV scratch taken from a fixed array inside the library
 * instead of a caller workspace. The paper has no counterpart; this is a
 * deployment convenience.
 *
 * Who needs it: code that may not call cudaMalloc, for example a plug-in whose
 * host application owns all device memory, or a latency-critical loop that
 * cannot afford cudaMalloc's implicit device synchronisation.
 *
 *   - The scratch is a device array of QK4V8_NOALLOC_SCRATCH_BYTES (8 MiB),
 *     present on every GPU that loads the library until the process exits.
 *     Requests that need more (qk4v8_decode_workspace_bytes(B, Hq, nq, splits)
 *     larger than that) fail with QK4V8_ERR_INVALID_ARG and a message naming
 *     the size.
 *   - The first call on each device looks up the array's device address, with
 *     that device current. Make that first call before any stream capture.
 *     The address is cached per device and CUDA context; after a
 *     cudaDeviceReset the next call looks it up again.
 *   - One split with up to 64 query rows per KV head needs no scratch, so such
 *     calls are never refused for size.
 *   - Every call shares the one array, and the array keeps the last call's
 *     contents. Nothing in it has to start at zero: the split kernels write
 *     every partial slot before a merge reads it. Calls that overlap on the GPU
 *     (different streams, or different host threads without ordering) race on
 *     the array; serialise them.
 *   - It allocates nothing (no cudaMalloc, no cudaFree, no allocating library
 *     call). Arguments and results as for qk4v8_attention_decode.
 */
#define QK4V8_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)

QK4V8_API int qk4v8_attention_decode_noalloc(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int nq,
                                             int q_cap, const uint8_t *k_codes, const uint8_t *k_scales,
                                             const uint8_t *v_codes, const uint8_t *v_scales, int Hkv, int kv_cap,
                                             const int32_t *seqlens_k, int max_seqlen, int causal_in_block,
                                             float softmax_scale, int num_splits, void *out, float *lse,
                                             int32_t *dev_status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* QK4V8_H */
