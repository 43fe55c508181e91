// Internal declarations shared by the CUDA translation units of libqk4v8.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace qk4v8 {

// Limit on any single pipeline wait inside a kernel before it gives up, sets
// the timeout status and unwinds (nanoseconds).
constexpr uint64_t kWaitTimeoutNs = 1000000000ull;

struct AttnParams {
    const uint8_t *q_codes;   // [B][Hq][q_cap][64]
    // Swap-AB decode only: when q_bf16 is set, the kernel quantizes the query
    // rows itself from bf16 [b][t][h][128] (element strides q_sb, q_st, q_sh)
    // and q_codes / q_scales are unused.
    const __nv_bfloat16 *q_bf16;
    int64_t q_sb, q_st, q_sh;
    const uint8_t *q_scales;  // [B][Hq][q_cap/128][512]
    const uint8_t *k_scales;  // [B][Hkv][kv_cap/128][512]
    const uint8_t *v_scales;  // [B][Hkv][kv_cap/128][512]
    const int32_t *seqlens;   // [B] or null
    int B, Hq, Hkv, G;
    int Sq;                   // query tokens per sequence (prefill length, or nq when decoding)
    int q_cap, kv_cap;
    int Lk;                   // KV length when seqlens is null
    int causal;
    // Decode only: > 0 limits every query row of a sequence of L keys to keys
    // j >= L - Sq - window (the last `window` keys before the Sq-token block, and
    // the block); 0: no lower bound.
    int window;
    // Decode only: paged K/V when non-null. Key tile t of sequence b is page
    // block_table[b * max_pages + t] of pools [num_pages][Hkv][128 tokens]
    // (kv_cap is then max_pages * 128); null: contiguous [B][Hkv][kv_cap].
    const int32_t *block_table;
    int max_pages, num_pages;
    // Decode only: V is MXFP4 (E2M1 codes [B][Hkv][128][kv_cap / 2], the QK4V4
    // comparison point) instead of MXFP8.
    int v_fp4;
    float scale_log2;         // softmax_scale * log2(e)
    int decode;               // 0: units (b, h_q, q tile); 1: units (b, h_kv, split)
    int n_qtiles;
    int num_splits, split_tiles;
    __nv_bfloat16 *out;       // prefill [B][Sq][Hq][128]
    float *lse;               // prefill [B][Hq][Sq] (natural log), nullable
    float *ws_o;              // decode partial outputs [B][Hq][nq][splits][128]
    float *ws_lse;            // decode partial log2-sum-exp [B][Hq][nq][splits]
    int direct_out;           // decode: write out [B][nq][Hq][128] and lse directly
    int32_t *piece_counts;    // GQA decode with splits: [B][Hkv] pieces of each sequence (0: written whole)
    int32_t *status;          // nullable
    int test_stall;           // test hook: the producer withholds the Q-ready signal
    float *test_dump_s;       // test hook: CTA 0 writes its first raw score tile [128 lanes][128 keys]
};

// pad_to_cap: write all `cap` token rows of each sequence (rows past the valid
// length get zero codes and scales); otherwise only the S input rows.
// rotate: quantize each row after its rotation by H / sqrt(128).
cudaError_t launch_quantize_qk(const void *x, int B, int S, int H, int64_t sb, int64_t ss, int64_t sh,
                               const int32_t *seqlens, int cap, uint8_t *codes, uint8_t *scales,
                               cudaStream_t stream, bool pad_to_cap = true, bool rotate = false);
cudaError_t launch_quantize_v(const void *v, int B, int S, int H, int64_t sb, int64_t ss, int64_t sh,
                              const int32_t *seqlens, int cap, uint8_t *codes, uint8_t *scales,
                              cudaStream_t stream);
cudaError_t launch_quantize_qkv(const void *q, const void *k, const void *v, int B, int Sq, int Sk, int Hq, int Hkv,
                                const int32_t *seqlens_k, int q_cap, int kv_cap, uint8_t *q_codes, uint8_t *q_scales,
                                uint8_t *k_codes, uint8_t *k_scales, uint8_t *v_codes, uint8_t *v_scales,
                                cudaStream_t stream);
cudaError_t launch_quantize_v4(const void *v, int B, int S, int H, int64_t sb, int64_t ss, int64_t sh,
                               const int32_t *seqlens, int cap, uint8_t *codes, uint8_t *scales,
                               cudaStream_t stream);
cudaError_t launch_attention(const CUtensorMap &tmap_k, const CUtensorMap &tmap_v, const AttnParams &p,
                             int grid, cudaStream_t stream);
// Prefill kernel (persistent: one CTA per SM over the (sequence, query head,
// 128-token query tile) units), and its QK^T-stage-only build over the same
// schedule. tmap_q maps the packed Q codes like tmap_k the K codes.
cudaError_t launch_prefill(const CUtensorMap &tmap_q, const CUtensorMap &tmap_k, const CUtensorMap &tmap_v,
                           const AttnParams &p, cudaStream_t stream);
cudaError_t launch_prefill_stage_qk(const CUtensorMap &tmap_q, const CUtensorMap &tmap_k, const CUtensorMap &tmap_v,
                                    const AttnParams &p, cudaStream_t stream);
// Tensor-pipe peak run of one block-scaled MMA shape (measurement aid).
cudaError_t launch_mma_peak(int kind, int ctas, int iters, int32_t *status, cudaStream_t stream);
// Swap-AB split-KV decode kernel; handles G*nq <= kDecodeMaxRows query rows.
constexpr int kDecodeMaxRows = 64;
cudaError_t launch_decode(const CUtensorMap &tmap_k, const CUtensorMap &tmap_v, const AttnParams &p, int grid,
                          cudaStream_t stream);
// GQA decode kernel for kGqaMinRows..kDecodeMaxRows query rows per KV head
// (persistent, one CTA per SM; packed MXFP4 queries), followed, for a
// direct-output call with splits, by the merge of the cut sequences.
constexpr int kGqaMinRows = 33;
cudaError_t launch_gqa_decode(const CUtensorMap &tmap_k, const CUtensorMap &tmap_v, const AttnParams &p,
                              cudaStream_t stream);
// Merge of the sequences a persistent decode kernel cut (direct output, splits >= 2,
// <= 64 rows per KV head), from the partials and the recorded piece counts.
cudaError_t launch_cut_merge(const AttnParams &p, cudaStream_t stream);
// Paged KV append (K and V of n_new tokens per sequence at positions
// seqlens[b] ..; V groups re-encoded from the staging buffer `tail`), then
// seqlens_out[b] = seqlens[b] + n_new (seqlens_out may be seqlens).
cudaError_t launch_kv_append(const void *k, const void *v, int B, int n_new, int H, int64_t sb, int64_t st,
                             int64_t sh, const int32_t *seqlens, const int32_t *block_table, int max_pages,
                             int num_pages, uint8_t *k_codes, uint8_t *k_scales, uint8_t *v_codes,
                             uint8_t *v_scales, void *tail, bool rotate_k, int32_t *seqlens_out, int32_t *status,
                             cudaStream_t stream);
cudaError_t launch_decode_merge(const float *ws_o, const float *ws_lse, int B, int Hq, int nq, int splits,
                                __nv_bfloat16 *out, float *lse, cudaStream_t stream);

}  // namespace qk4v8
