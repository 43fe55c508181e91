/*
 * qk4v8_test.h - test-only hooks of libqk4v8.so. Not part of the product API.
 */
#ifndef QK4V8_TEST_H
#define QK4V8_TEST_H

#ifndef QK4V8_API
#define QK4V8_API __attribute__((visibility("default")))
#endif

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

#ifdef __cplusplus
}
#endif

#endif /* QK4V8_TEST_H */
