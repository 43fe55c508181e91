/*
 * qk4v8_test.h - test-only hooks of libqk4v8.so. Not part of the product API.
 */
#ifndef QK4V8_TEST_H
#define QK4V8_TEST_H

#ifndef QK4V8_API
#define QK4V8_API __attribute__((visibility("default")))
#endif

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * While `enable` is non-zero, every attention launch withholds its producer's
 * "Q tile ready" signal. The pipeline's bounded waits then expire after about
 * one second. The kernel writes QK4V8_ERR_TIMEOUT to *dev_status, unwinds,
 * frees its tensor memory and returns, so the CUDA context stays usable. The
 * outputs of such a launch are undefined. Host-side state, not thread safe;
 * call it with no launch in flight.
 */
QK4V8_API void qk4v8_test_set_stall(int enable);

/*
 * While dev_ptr is non-NULL, CTA 0 of every attention launch writes the raw
 * FP32 scores S = Q K^T of its first key tile (no softmax scale) to
 * dev_ptr[lane * 128 + key], for the 128 TMEM lanes (query rows) of that CTA.
 * dev_ptr is a device buffer of 128*128 floats owned by the caller.
 */
QK4V8_API void qk4v8_test_set_dump_scores(float *dev_ptr);

/*
 * While `enable` is non-zero, decode calls whose GQA group has 33..64 query
 * rows per KV head run on the swap-AB split kernel (the one that serves up to
 * 32 rows) instead of the GQA decode kernel, so that tests and measurements
 * can compare the two. Both compute the same attention. Host-side state, not
 * thread safe; workspace sizes do not depend on it.
 */
QK4V8_API void qk4v8_test_set_force_swap_ab(int enable);

/*
 * The QK^T stage of qk4v8_attention_prefill alone, for measurement: the same
 * prefill kernel built without exp, P and P V, over the same causal tile
 * schedule (Q and K loads with their scale atoms, the block-scaled FP4 MMAs,
 * and the TMEM drain of each score tile with its row maximum). Arguments as
 * for qk4v8_attention_prefill without V and out. row_max (device float
 * [B][Hq][Sq], nullable) receives each query row's largest allowed scaled
 * score, softmax_scale * log2(e) * max_j S[i][j], or -inf for a row with no
 * allowed key.
 */
QK4V8_API int qk4v8_test_prefill_stage_qk(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int Sq,
                                          int q_cap, const uint8_t *k_codes, const uint8_t *k_scales, int Hkv, int Sk,
                                          int kv_cap, const int32_t *seqlens_k, int causal, float softmax_scale,
                                          float *row_max, int32_t *dev_status, void *stream);

/*
 * Tensor-pipe peak of one block-scaled MMA shape, for the roofline's
 * denominator: `ctas` CTAs each issue `iters` tcgen05.mma instructions of one
 * shape into a TMEM accumulator from operands resident in shared memory, with
 * no loads and no other work. The caller times the launch on `stream`.
 *   kind 0: kind::mxf4 (E2M1), M=128 N=128 K=64 (the QK^T instruction)
 *   kind 1: kind::mxf8f6f4 (E4M3), M=128 N=144 K=32 (the P V instruction)
 *   kind 2: kind::mxf8f6f4, M=128 N=256 K=32
 *   kind 3: kind::mxf4, M=128 N=256 K=64
 * FLOPs per instruction: 2*M*N*K. dev_status (nullable) receives
 * QK4V8_ERR_TIMEOUT if the run did not drain within its wait limit.
 */
QK4V8_API int qk4v8_test_mma_peak(int kind, int ctas, int iters, int32_t *dev_status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* QK4V8_TEST_H */
