// extern "C" entry points of libqk4v8.so: argument validation, TMA descriptor
// construction and kernel launches. See include/qk4v8.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <functional>
#include <mutex>
#include <queue>
#include <vector>

#include "../../include/qk4v8.h"
#include "../../include/qk4v8_test.h"
#include "qk4v8_internal.h"

namespace {

thread_local char g_last_error[512] = "";
int g_test_stall = 0;
float *g_test_dump_s = nullptr;
int g_test_force_swap_ab = 0;

int set_error(int status, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return status;
}

int cuda_error(cudaError_t e, const char *what) {
    return set_error(QK4V8_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// sm_100 check, cached per device.
int check_device() {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
    return qk4v8_device_supported(dev);
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// MXFP4 codes [B*H][cap][64] (K, or Q for prefill) as a 3-D uint8 tensor, 128-token x 64-byte boxes,
// 64-byte swizzle (one token row is exactly one swizzle span).
int make_k_map(CUtensorMap *map, const uint8_t *codes, int BH, int cap) {
    auto enc = get_encode_fn();
    if (!enc) return set_error(QK4V8_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(cap), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {64, static_cast<cuuint64_t>(cap) * 64};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(codes), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(QK4V8_ERR_CUDA, "cuTensorMapEncodeTiled(K) failed (%d)", int(r));
    return QK4V8_OK;
}

// V codes [B*Hkv][cap / 128][128][128] (a 128-token block of a channel row
// after another, each block's 16 KiB contiguous) as a 3-D uint8 tensor of
// B*Hkv*(cap/128) 128-channel x 128-token tiles: tile z = row * (cap / 128) +
// block, the index of its scale atom. 128-byte swizzle.
int make_v_map(CUtensorMap *map, const uint8_t *codes, int BH, int cap) {
    auto enc = get_encode_fn();
    if (!enc) return set_error(QK4V8_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[3] = {128, 128, static_cast<cuuint64_t>(BH) * static_cast<cuuint64_t>(cap / 128)};
    cuuint64_t strides[2] = {128, 128 * 128};
    cuuint32_t box[3] = {128, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(codes), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(QK4V8_ERR_CUDA, "cuTensorMapEncodeTiled(V) failed (%d)", int(r));
    return QK4V8_OK;
}

// MXFP4 V codes [B*Hkv][cap / 128][128][64] (the QK4V4 comparison point; the
// blocks as for MXFP8 V, 64 bytes per channel row of a block): loaded with the
// 16U4_ALIGN16B element type, which lands each 16 packed codes (8 bytes) in a
// 16-byte slot of shared memory, the layout the block-scaled f8f6f4 MMA reads
// for an E2M1 operand. A 128-token x 128-channel box then fills the same
// 128 x 128-byte, 128-byte-swizzled tile as an MXFP8 V box.
int make_v4_map(CUtensorMap *map, const uint8_t *codes, int BH, int cap) {
    auto enc = get_encode_fn();
    if (!enc) return set_error(QK4V8_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[3] = {128, 128, static_cast<cuuint64_t>(BH) * static_cast<cuuint64_t>(cap / 128)};
    cuuint64_t strides[2] = {64, 64 * 128};
    cuuint32_t box[3] = {128, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, const_cast<uint8_t *>(codes), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(QK4V8_ERR_CUDA, "cuTensorMapEncodeTiled(V, MXFP4) failed (%d)", int(r));
    return QK4V8_OK;
}

int validate_quant_args(const void *x, int B, int S, int H, int d, int64_t sb, int64_t ss, int64_t sh, int cap,
                        const uint8_t *codes, const uint8_t *scales) {
    if (!x || !codes || !scales) return set_error(QK4V8_ERR_INVALID_ARG, "null pointer");
    if (d != 128) return set_error(QK4V8_ERR_INVALID_ARG, "head_dim must be 128 (got %d)", d);
    if (B <= 0 || S < 0 || H <= 0) return set_error(QK4V8_ERR_INVALID_ARG, "bad shape B=%d S=%d H=%d", B, S, H);
    if (cap <= 0 || cap % 128 || cap < S)
        return set_error(QK4V8_ERR_INVALID_ARG, "cap must be a positive multiple of 128 and >= S (cap=%d S=%d)", cap,
                         S);
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales))
        return set_error(QK4V8_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    if (sb % 8 || ss % 8 || sh % 8 || sb < 0 || ss < 0 || sh < 0)
        return set_error(QK4V8_ERR_INVALID_ARG, "strides must be non-negative multiples of 8 elements");
    return QK4V8_OK;
}

int validate_packed(const uint8_t *codes, const uint8_t *scales, const char *what) {
    if (!codes || !scales) return set_error(QK4V8_ERR_INVALID_ARG, "null %s pointer", what);
    if (!aligned16(codes) || !aligned16(scales))
        return set_error(QK4V8_ERR_INVALID_ARG, "%s buffers must be 16-byte aligned", what);
    return QK4V8_OK;
}

float resolve_scale(float s) { return s > 0.f ? s : 1.0f / std::sqrt(128.0f); }

constexpr float kLog2e = 1.4426950408889634f;

}  // namespace

extern "C" {

const char *qk4v8_status_string(int status) {
    switch (status) {
        case QK4V8_OK: return "ok";
        case QK4V8_ERR_INVALID_ARG: return "invalid argument";
        case QK4V8_ERR_UNSUPPORTED: return "unsupported device (needs sm_100)";
        case QK4V8_ERR_CUDA: return "CUDA error";
        case QK4V8_ERR_TIMEOUT: return "device wait timed out";
        default: return "unknown status";
    }
}

const char *qk4v8_last_error(void) { return g_last_error; }

int qk4v8_device_supported(int device) {
    int major = 0, minor = 0;
    cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device);
    if (e != cudaSuccess) return cuda_error(e, "cudaDeviceGetAttribute");
    e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device);
    if (e != cudaSuccess) return cuda_error(e, "cudaDeviceGetAttribute");
    if (major != 10 || minor != 0)
        return set_error(QK4V8_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", device,
                         major, minor);
    return QK4V8_OK;
}

size_t qk4v8_mxfp4_codes_bytes(int B, int H, int cap) {
    return static_cast<size_t>(B) * H * cap * 64;
}
size_t qk4v8_mxfp8_codes_bytes(int B, int H, int cap) {
    return static_cast<size_t>(B) * H * 128 * cap;
}
size_t qk4v8_scales_bytes(int B, int H, int cap) {
    return static_cast<size_t>(B) * H * (cap / 128) * 512;
}

int qk4v8_quantize_qk(const void *x, int B, int S, int H, int d, int64_t stride_b, int64_t stride_s,
                      int64_t stride_h, const int32_t *seqlens, int cap, uint8_t *codes, uint8_t *scales,
                      void *stream) {
    int st = validate_quant_args(x, B, S, H, d, stride_b, stride_s, stride_h, cap, codes, scales);
    if (st) return st;
    if ((st = check_device())) return st;
    cudaError_t e = qk4v8::launch_quantize_qk(x, B, S, H, stride_b, stride_s, stride_h, seqlens, cap, codes, scales,
                                              static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? QK4V8_OK : cuda_error(e, "quantize_qk launch");
}

int qk4v8_quantize_qk_hadamard(const void *x, int B, int S, int H, int d, int64_t stride_b, int64_t stride_s,
                               int64_t stride_h, const int32_t *seqlens, int cap, uint8_t *codes, uint8_t *scales,
                               void *stream) {
    int st = validate_quant_args(x, B, S, H, d, stride_b, stride_s, stride_h, cap, codes, scales);
    if (st) return st;
    if ((st = check_device())) return st;
    cudaError_t e = qk4v8::launch_quantize_qk(x, B, S, H, stride_b, stride_s, stride_h, seqlens, cap, codes, scales,
                                              static_cast<cudaStream_t>(stream), /*pad_to_cap=*/true,
                                              /*rotate=*/true);
    return e == cudaSuccess ? QK4V8_OK : cuda_error(e, "quantize_qk_hadamard launch");
}

int qk4v8_quantize_v(const void *v, int B, int S, int H, int d, int64_t stride_b, int64_t stride_s,
                     int64_t stride_h, const int32_t *seqlens, int cap, uint8_t *codes, uint8_t *scales,
                     void *stream) {
    int st = validate_quant_args(v, B, S, H, d, stride_b, stride_s, stride_h, cap, codes, scales);
    if (st) return st;
    if ((st = check_device())) return st;
    cudaError_t e = qk4v8::launch_quantize_v(v, B, S, H, stride_b, stride_s, stride_h, seqlens, cap, codes, scales,
                                             static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? QK4V8_OK : cuda_error(e, "quantize_v launch");
}

size_t qk4v8_mxfp4v_codes_bytes(int B, int H, int cap) {
    return static_cast<size_t>(B) * H * 128 * (cap / 2);
}

int qk4v8_quantize_v4(const void *v, int B, int S, int H, int d, int64_t stride_b, int64_t stride_s,
                      int64_t stride_h, const int32_t *seqlens, int cap, uint8_t *codes, uint8_t *scales,
                      void *stream) {
    int st = validate_quant_args(v, B, S, H, d, stride_b, stride_s, stride_h, cap, codes, scales);
    if (st) return st;
    if ((st = check_device())) return st;
    cudaError_t e = qk4v8::launch_quantize_v4(v, B, S, H, stride_b, stride_s, stride_h, seqlens, cap, codes, scales,
                                              static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? QK4V8_OK : cuda_error(e, "quantize_v4 launch");
}

int qk4v8_quantize(const void *q, const void *k, const void *v, int B, int Sq, int Sk, int Hq, int Hkv, int d,
                   const int32_t *seqlens_k, int q_cap, int kv_cap, uint8_t *q_codes, uint8_t *q_scales,
                   uint8_t *k_codes, uint8_t *k_scales, uint8_t *v_codes, uint8_t *v_scales, void *stream) {
    const int64_t qs = static_cast<int64_t>(Hq) * 128, ks = static_cast<int64_t>(Hkv) * 128;
    int st = validate_quant_args(q, B, Sq, Hq, d, qs * Sq, qs, 128, q_cap, q_codes, q_scales);
    if (!st) st = validate_quant_args(k, B, Sk, Hkv, d, ks * Sk, ks, 128, kv_cap, k_codes, k_scales);
    if (!st) st = validate_quant_args(v, B, Sk, Hkv, d, ks * Sk, ks, 128, kv_cap, v_codes, v_scales);
    if (st) return st;
    if ((st = check_device())) return st;
    cudaError_t e = qk4v8::launch_quantize_qkv(q, k, v, B, Sq, Sk, Hq, Hkv, seqlens_k, q_cap, kv_cap, q_codes,
                                               q_scales, k_codes, k_scales, v_codes, v_scales,
                                               static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? QK4V8_OK : cuda_error(e, "quantize (Q, K, V) launch");
}

}  // extern "C"

namespace {

// Shared by the prefill entry point and its QK^T-stage test build.
int prefill_common(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int Sq, int q_cap,
                   const uint8_t *k_codes, const uint8_t *k_scales, const uint8_t *v_codes, const uint8_t *v_scales,
                   int Hkv, int Sk, int kv_cap, const int32_t *seqlens_k, int causal, float softmax_scale, void *out,
                   float *lse, int32_t *dev_status, void *stream, bool stage_qk) {
    int st;
    if ((st = validate_packed(q_codes, q_scales, "Q")) || (st = validate_packed(k_codes, k_scales, "K")))
        return st;
    if (!stage_qk && (st = validate_packed(v_codes, v_scales, "V"))) return st;
    if (!stage_qk && (!out || !aligned16(out)))
        return set_error(QK4V8_ERR_INVALID_ARG, "out must be a 16-byte aligned pointer");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv)
        return set_error(QK4V8_ERR_INVALID_ARG, "bad heads B=%d Hq=%d Hkv=%d", B, Hq, Hkv);
    if (Sq <= 0 || q_cap % 128 || q_cap < Sq || kv_cap <= 0 || kv_cap % 128 || Sk < 0 || Sk > kv_cap)
        return set_error(QK4V8_ERR_INVALID_ARG, "bad lengths Sq=%d q_cap=%d Sk=%d kv_cap=%d", Sq, q_cap, Sk, kv_cap);
    if ((st = check_device())) return st;
    CUtensorMap tq, tk, tv;
    if ((st = make_k_map(&tq, q_codes, B * Hq, q_cap)) || (st = make_k_map(&tk, k_codes, B * Hkv, kv_cap))) return st;
    if (stage_qk)
        tv = tk;  // unused by the QK^T stage
    else if ((st = make_v_map(&tv, v_codes, B * Hkv, kv_cap)))
        return st;
    qk4v8::AttnParams p{};
    p.q_codes = q_codes;
    p.q_scales = q_scales;
    p.k_scales = k_scales;
    p.v_scales = v_scales;
    p.seqlens = seqlens_k;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.G = Hq / Hkv;
    p.Sq = Sq;
    p.q_cap = q_cap;
    p.kv_cap = kv_cap;
    p.Lk = Sk;
    p.causal = causal ? 1 : 0;
    p.scale_log2 = resolve_scale(softmax_scale) * kLog2e;
    p.decode = 0;
    p.n_qtiles = (Sq + 127) / 128;
    p.num_splits = 1;
    p.split_tiles = 0;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    p.status = dev_status;
    p.test_stall = g_test_stall;
    p.test_dump_s = g_test_dump_s;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = stage_qk ? qk4v8::launch_prefill_stage_qk(tq, tk, tv, p, s) : qk4v8::launch_prefill(tq, tk, tv, p, s);
    return e == cudaSuccess ? QK4V8_OK : cuda_error(e, "attention (prefill) launch");
}

}  // namespace

extern "C" {

int qk4v8_attention_prefill(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int Sq, int q_cap,
                            const uint8_t *k_codes, const uint8_t *k_scales, const uint8_t *v_codes,
                            const uint8_t *v_scales, int Hkv, int Sk, int kv_cap, const int32_t *seqlens_k,
                            int causal, float softmax_scale, void *out, float *lse, int32_t *dev_status,
                            void *stream) {
    return prefill_common(q_codes, q_scales, B, Hq, Sq, q_cap, k_codes, k_scales, v_codes, v_scales, Hkv, Sk, kv_cap,
                          seqlens_k, causal, softmax_scale, out, lse, dev_status, stream, false);
}

int qk4v8_test_prefill_stage_qk(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int Sq, int q_cap,
                                const uint8_t *k_codes, const uint8_t *k_scales, int Hkv, int Sk, int kv_cap,
                                const int32_t *seqlens_k, int causal, float softmax_scale, float *row_max,
                                int32_t *dev_status, void *stream) {
    return prefill_common(q_codes, q_scales, B, Hq, Sq, q_cap, k_codes, k_scales, nullptr, nullptr, Hkv, Sk, kv_cap,
                          seqlens_k, causal, softmax_scale, nullptr, row_max, dev_status, stream, true);
}

size_t qk4v8_decode_workspace_bytes(int B, int Hq, int nq, int num_splits) {
    if (B <= 0 || Hq <= 0 || nq <= 0 || num_splits <= 0) return 0;
    const size_t rows = static_cast<size_t>(B) * Hq * nq * num_splits;
    // Split partials O [rows][128] and log2-sum-exp [rows], then the piece count
    // of each (sequence, head), which the GQA decode kernel records for its merge.
    return rows * 128 * sizeof(float) + rows * sizeof(float) + static_cast<size_t>(B) * Hq * sizeof(int32_t);
}

int qk4v8_decode_default_splits(int B, int Hq, int Hkv, int nq, int max_seqlen) {
    // For 33..64 query rows per KV head the GQA decode kernel is persistent and
    // can spread the key tiles of all sequences evenly over the CTAs; it does so
    // when no sequence would be cut into more pieces than there are splits.
    // With at most half as many sequences as CTAs (where whole sequences would
    // leave many CTAs idle), plan for that: for sequences of at least half the
    // maximum length each CTA's share is at least range/2 tiles (range = units
    // * tiles / slots), and a sequence meets at most ceil(tiles / (range/2)) + 1
    // shares. Otherwise (and for problems of less than two tiles per CTA, and
    // other group sizes) use the wave cost model: a launch of units * s CTAs
    // over `slots` resident CTA slots
    // takes ceil(units * s / slots) waves, each as long as one split
    // (ceil(tiles / s) key tiles of 128) plus a fixed cost of about
    // kSplitOverheadTiles tiles for the prologue, pipeline fill and epilogue;
    // the cheapest s, the smallest on ties.
    constexpr int kSplitOverheadTiles = 3;
    constexpr int kMaxSplits = 64;
    if (B <= 0 || Hkv <= 0 || Hq <= 0 || Hq % Hkv || nq <= 0) return 1;
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
        sms = 148;
        (void)cudaGetLastError();
    }
    const int rows = (Hq / Hkv) * nq;
    const int64_t slots = static_cast<int64_t>(sms) * (rows <= 16 ? 2 : 1);
    const int64_t units = static_cast<int64_t>(B) * Hkv;
    const int tiles = max_seqlen > 0 ? (max_seqlen + 127) / 128 : 1;
    if (rows >= qk4v8::kGqaMinRows && rows <= qk4v8::kDecodeMaxRows && 2 * units <= slots &&
        units * tiles >= 2 * slots) {
        const int64_t half = units * tiles / slots / 2;
        const int64_t s = (tiles + half - 1) / half + 1;
        return static_cast<int>(s < kMaxSplits ? s : kMaxSplits);
    }
    int best = 1;
    int64_t best_cost = INT64_MAX;
    for (int s = 1; s <= kMaxSplits && s <= tiles; ++s) {
        const int64_t waves = (units * s + slots - 1) / slots;
        const int64_t cost = waves * ((tiles + s - 1) / s + kSplitOverheadTiles);
        if (cost < best_cost) {
            best_cost = cost;
            best = s;
        }
    }
    return best;
}

}  // extern "C"

namespace {

// Largest number of keys one sequence's query block sees: max_seqlen, or with
// a window the window plus the block, plus up to 127 keys of the tile that
// holds the window's first key.
int window_span(int max_seqlen, int nq, int window) {
    if (window <= 0) return max_seqlen;
    const int64_t span = static_cast<int64_t>(window) + nq + 127;
    return span < max_seqlen ? static_cast<int>(span) : max_seqlen;
}

// Query of a decode call: packed MXFP4 (codes, scales, cap) or bf16 rows
// [b][t][h][128] with element strides, quantized inside the kernel.
struct DecodeQuery {
    const uint8_t *codes = nullptr;
    const uint8_t *scales = nullptr;
    int cap = 0;
    const __nv_bfloat16 *bf16 = nullptr;
    int64_t sb = 0, st = 0, sh = 0;
};

// Which split kernel serves a GQA group of G*nq query rows: the swap-AB kernel
// up to 32 rows (or up to 64 under the test hook), the GQA decode kernel for
// 33..64, the 128-row attention kernel above. The first two write the output
// directly when there is one split.
bool swap_ab_rows(int Hq, int Hkv, int nq) {
    const int rows = (Hq / Hkv) * nq;
    return rows < qk4v8::kGqaMinRows || (g_test_force_swap_ab && rows <= qk4v8::kDecodeMaxRows);
}
bool gqa_rows(int Hq, int Hkv, int nq) {
    return !swap_ab_rows(Hq, Hkv, nq) && (Hq / Hkv) * nq <= qk4v8::kDecodeMaxRows;
}

// Validates decode arguments, builds the tensor maps and launches the split-KV
// kernel. With `out` given and a single split on the swap-AB kernel, the kernel
// writes out (and lse) itself and *direct is set; otherwise it writes the split
// partials to the workspace and the caller runs the merge.
// How a decode call's cache is laid out: paged K/V pools (block_table null:
// contiguous caches), and the V element format (v_fp4: MXFP4, the QK4V4
// comparison point, contiguous caches only).
struct KvPages {
    const int32_t *block_table = nullptr;
    int max_pages = 0, num_pages = 0;
    bool v_fp4 = false;
};

int decode_splitkv(const DecodeQuery &q, int B, int Hq, int nq, const uint8_t *k_codes, const uint8_t *k_scales,
                   const uint8_t *v_codes, const uint8_t *v_scales, int Hkv, int kv_cap, const KvPages &pages,
                   const int32_t *seqlens_k, int max_seqlen, int causal_in_block, int window, float softmax_scale,
                   int num_splits, void *workspace, size_t workspace_bytes, void *out, float *lse,
                   int32_t *dev_status, cudaStream_t stream, int *splits_used, bool *direct) {
    int st;
    if (q.bf16) {
        if (!aligned16(q.bf16) || q.sb % 8 || q.st % 8 || q.sh % 8 || q.sb < 0 || q.st < 0 || q.sh < 0)
            return set_error(QK4V8_ERR_INVALID_ARG, "bf16 Q must be 16-byte aligned with strides of whole 8-element "
                                                    "(16-byte) units");
    } else if ((st = validate_packed(q.codes, q.scales, "Q"))) {
        return st;
    }
    if ((st = validate_packed(k_codes, k_scales, "K")) || (st = validate_packed(v_codes, v_scales, "V"))) return st;
    if (!seqlens_k) return set_error(QK4V8_ERR_INVALID_ARG, "decode needs seqlens_k");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv)
        return set_error(QK4V8_ERR_INVALID_ARG, "bad heads B=%d Hq=%d Hkv=%d", B, Hq, Hkv);
    if (nq < 1 || nq > 8 || (Hq / Hkv) * nq > 128)
        return set_error(QK4V8_ERR_INVALID_ARG, "need 1 <= nq <= 8 and (Hq/Hkv)*nq <= 128 (nq=%d G=%d)", nq,
                         Hq / Hkv);
    if ((!q.bf16 && (q.cap <= 0 || q.cap % 128 || q.cap < nq)) || kv_cap <= 0 || kv_cap % 128 || max_seqlen < 0 ||
        max_seqlen > kv_cap)
        return set_error(QK4V8_ERR_INVALID_ARG, "bad lengths q_cap=%d kv_cap=%d max_seqlen=%d", q.cap, kv_cap,
                         max_seqlen);
    // MXFP4 V runs on the swap-AB and GQA decode kernels, up to 64 query rows per KV head.
    const bool use_swap = swap_ab_rows(Hq, Hkv, nq);
    const bool use_gqa = !use_swap && gqa_rows(Hq, Hkv, nq);
    if (q.bf16 && !use_swap)
        return set_error(QK4V8_ERR_INVALID_ARG, "bf16 Q in the split kernel needs (Hq/Hkv)*nq < %d",
                         qk4v8::kGqaMinRows);
    if (pages.v_fp4 && ((Hq / Hkv) * nq > qk4v8::kDecodeMaxRows || pages.block_table ||
                        (reinterpret_cast<uintptr_t>(v_codes) & 31)))
        return set_error(QK4V8_ERR_INVALID_ARG, "MXFP4 V needs (Hq/Hkv)*nq <= %d, a contiguous cache and 32-byte "
                                                "aligned V codes", qk4v8::kDecodeMaxRows);
    if (num_splits < 0) return set_error(QK4V8_ERR_INVALID_ARG, "num_splits must be >= 0");
    if (window < 0) return set_error(QK4V8_ERR_INVALID_ARG, "window must be >= 0 (0: none)");
    if (pages.block_table) {
        if (pages.max_pages <= 0 || pages.num_pages <= 0 ||
            static_cast<int64_t>(pages.num_pages) * Hkv >= (int64_t{1} << 31) ||
            static_cast<int64_t>(pages.max_pages) * 128 >= (int64_t{1} << 31))
            return set_error(QK4V8_ERR_INVALID_ARG, "bad page pool: num_pages=%d max_pages=%d", pages.num_pages,
                             pages.max_pages);
        if ((Hq / Hkv) * nq > qk4v8::kDecodeMaxRows)
            return set_error(QK4V8_ERR_INVALID_ARG, "a paged cache needs (Hq/Hkv)*nq <= %d query rows per KV head",
                             qk4v8::kDecodeMaxRows);
    }
    if (window > 0 && (Hq / Hkv) * nq > qk4v8::kDecodeMaxRows)
        return set_error(QK4V8_ERR_INVALID_ARG, "a window needs (Hq/Hkv)*nq <= %d query rows per KV head",
                         qk4v8::kDecodeMaxRows);
    // Keys a sequence's query block can see, for planning the splits.
    const int span = window_span(max_seqlen, nq, window);
    const int splits = num_splits > 0 ? num_splits : qk4v8_decode_default_splits(B, Hq, Hkv, nq, span);
    // Direct output: the swap-AB kernel with one split, and the GQA decode kernel
    // always (with splits, its own merge launch finishes the cut sequences).
    const bool direct_out = out && ((splits == 1 && use_swap) || use_gqa);
    if (out && !aligned16(out)) return set_error(QK4V8_ERR_INVALID_ARG, "out must be a 16-byte aligned pointer");
    const size_t need = (direct_out && splits == 1) ? 0 : qk4v8_decode_workspace_bytes(B, Hq, nq, splits);
    if (need && (!workspace || !aligned16(workspace) || workspace_bytes < need))
        return set_error(QK4V8_ERR_INVALID_ARG, "workspace must be 16-byte aligned and >= %zu bytes", need);
    if ((st = check_device())) return st;
    CUtensorMap tk, tv;
    // A paged pool is the contiguous layout with num_pages rows of capacity 128.
    const int map_rows = pages.block_table ? pages.num_pages * Hkv : B * Hkv;
    const int map_cap = pages.block_table ? 128 : kv_cap;
    if ((st = make_k_map(&tk, k_codes, map_rows, map_cap)) ||
        (st = pages.v_fp4 ? make_v4_map(&tv, v_codes, map_rows, map_cap) : make_v_map(&tv, v_codes, map_rows, map_cap)))
        return st;
    const int tiles = (span + 127) / 128;
    qk4v8::AttnParams p{};
    p.q_codes = q.codes;
    p.q_scales = q.scales;
    p.q_bf16 = q.bf16;
    p.q_sb = q.sb;
    p.q_st = q.st;
    p.q_sh = q.sh;
    p.k_scales = k_scales;
    p.v_scales = v_scales;
    p.seqlens = seqlens_k;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.G = Hq / Hkv;
    p.Sq = nq;
    p.q_cap = q.cap;
    p.kv_cap = kv_cap;
    p.Lk = max_seqlen;
    p.causal = causal_in_block ? 1 : 0;
    p.window = window;
    p.block_table = pages.block_table;
    p.max_pages = pages.max_pages;
    p.num_pages = pages.num_pages;
    p.v_fp4 = pages.v_fp4 ? 1 : 0;
    p.scale_log2 = resolve_scale(softmax_scale) * kLog2e;
    p.decode = 1;
    p.n_qtiles = 1;
    p.num_splits = splits;
    p.split_tiles = tiles > 0 ? (tiles + splits - 1) / splits : 1;
    if (direct_out) {
        p.direct_out = 1;
        p.out = static_cast<__nv_bfloat16 *>(out);
        p.lse = lse;
    }
    if (need) {
        const size_t rows = static_cast<size_t>(B) * Hq * nq * splits;
        p.ws_o = static_cast<float *>(workspace);
        p.ws_lse = p.ws_o + rows * 128;
        p.piece_counts = reinterpret_cast<int32_t *>(p.ws_lse + rows);
    }
    p.status = dev_status;
    p.test_stall = g_test_stall;
    p.test_dump_s = g_test_dump_s;
    // G*nq <= 32 query rows: the swap-AB decode kernel; 33..64: the GQA decode
    // kernel; larger groups use the 128-row attention kernel in its decode
    // instantiation.
    cudaError_t e = use_swap  ? qk4v8::launch_decode(tk, tv, p, B * Hkv * splits, stream)
                    : use_gqa ? qk4v8::launch_gqa_decode(tk, tv, p, stream)
                              : qk4v8::launch_attention(tk, tv, p, B * Hkv * splits, stream);
    if (e != cudaSuccess) return cuda_error(e, "attention (decode) launch");
    *splits_used = splits;
    *direct = direct_out;
    return QK4V8_OK;
}

}  // namespace

extern "C" {

int qk4v8_attention_decode_splitkv(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int nq, int q_cap,
                                   const uint8_t *k_codes, const uint8_t *k_scales, const uint8_t *v_codes,
                                   const uint8_t *v_scales, int Hkv, int kv_cap, const int32_t *seqlens_k,
                                   int max_seqlen, int causal_in_block, float softmax_scale, int num_splits,
                                   void *workspace, size_t workspace_bytes, int32_t *dev_status, void *stream) {
    int splits = 0;
    bool direct = false;
    DecodeQuery q;
    q.codes = q_codes;
    q.scales = q_scales;
    q.cap = q_cap;
    return decode_splitkv(q, B, Hq, nq, k_codes, k_scales, v_codes, v_scales, Hkv, kv_cap, KvPages{}, seqlens_k,
                          max_seqlen, causal_in_block, 0, softmax_scale, num_splits, workspace, workspace_bytes,
                          nullptr, nullptr, dev_status, static_cast<cudaStream_t>(stream), &splits, &direct);
}

int qk4v8_decode_merge(const void *workspace, size_t workspace_bytes, int B, int Hq, int nq, int num_splits,
                       void *out, float *lse, void *stream) {
    if (!workspace || !aligned16(workspace) || !out || !aligned16(out))
        return set_error(QK4V8_ERR_INVALID_ARG, "workspace and out must be 16-byte aligned pointers");
    if (B <= 0 || Hq <= 0 || nq < 1 || nq > 8 || num_splits < 1)
        return set_error(QK4V8_ERR_INVALID_ARG, "bad merge sizes B=%d Hq=%d nq=%d splits=%d", B, Hq, nq,
                         num_splits);
    if (workspace_bytes < qk4v8_decode_workspace_bytes(B, Hq, nq, num_splits))
        return set_error(QK4V8_ERR_INVALID_ARG, "workspace smaller than %zu bytes",
                         qk4v8_decode_workspace_bytes(B, Hq, nq, num_splits));
    int st;
    if ((st = check_device())) return st;
    const size_t rows = static_cast<size_t>(B) * Hq * nq * num_splits;
    const float *ws_o = static_cast<const float *>(workspace);
    cudaError_t e = qk4v8::launch_decode_merge(ws_o, ws_o + rows * 128, B, Hq, nq, num_splits,
                                               static_cast<__nv_bfloat16 *>(out), lse,
                                               static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? QK4V8_OK : cuda_error(e, "decode merge launch");
}

}  // extern "C"

namespace {

int decode_packed(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int nq, int q_cap,
                  const uint8_t *k_codes, const uint8_t *k_scales, const uint8_t *v_codes, const uint8_t *v_scales,
                  int Hkv, int kv_cap, const KvPages &pages, const int32_t *seqlens_k, int max_seqlen,
                  int causal_in_block, int window, float softmax_scale, int num_splits, void *workspace,
                  size_t workspace_bytes, void *out, float *lse, int32_t *dev_status, void *stream) {
    if (!out || !aligned16(out)) return set_error(QK4V8_ERR_INVALID_ARG, "out must be a 16-byte aligned pointer");
    int splits = 0;
    bool direct = false;
    DecodeQuery q;
    q.codes = q_codes;
    q.scales = q_scales;
    q.cap = q_cap;
    int st = decode_splitkv(q, B, Hq, nq, k_codes, k_scales, v_codes, v_scales, Hkv, kv_cap, pages, seqlens_k,
                            max_seqlen, causal_in_block, window, softmax_scale, num_splits, workspace,
                            workspace_bytes, out, lse, dev_status, static_cast<cudaStream_t>(stream), &splits,
                            &direct);
    if (st || direct) return st;
    return qk4v8_decode_merge(workspace, workspace_bytes, B, Hq, nq, splits, out, lse, stream);
}

}  // namespace

extern "C" {

int qk4v8_attention_decode_window(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int nq,
                                  int q_cap, const uint8_t *k_codes, const uint8_t *k_scales, const uint8_t *v_codes,
                                  const uint8_t *v_scales, int Hkv, int kv_cap, const int32_t *seqlens_k,
                                  int max_seqlen, int causal_in_block, int window, float softmax_scale,
                                  int num_splits, void *workspace, size_t workspace_bytes, void *out, float *lse,
                                  int32_t *dev_status, void *stream) {
    return decode_packed(q_codes, q_scales, B, Hq, nq, q_cap, k_codes, k_scales, v_codes, v_scales, Hkv, kv_cap,
                         KvPages{}, seqlens_k, max_seqlen, causal_in_block, window, softmax_scale, num_splits,
                         workspace, workspace_bytes, out, lse, dev_status, stream);
}

int qk4v8_attention_decode_paged(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int nq, int q_cap,
                                 const uint8_t *k_codes, const uint8_t *k_scales, const uint8_t *v_codes,
                                 const uint8_t *v_scales, int Hkv, int num_pages, const int32_t *block_table,
                                 int max_pages, const int32_t *seqlens_k, int max_seqlen, int causal_in_block,
                                 int window, float softmax_scale, int num_splits, void *workspace,
                                 size_t workspace_bytes, void *out, float *lse, int32_t *dev_status, void *stream) {
    if (!block_table) return set_error(QK4V8_ERR_INVALID_ARG, "block_table is null");
    if (max_pages <= 0 || max_pages >= (1 << 24))
        return set_error(QK4V8_ERR_INVALID_ARG, "bad max_pages %d", max_pages);
    KvPages pages;
    pages.block_table = block_table;
    pages.max_pages = max_pages;
    pages.num_pages = num_pages;
    return decode_packed(q_codes, q_scales, B, Hq, nq, q_cap, k_codes, k_scales, v_codes, v_scales, Hkv,
                         max_pages * 128, pages, seqlens_k, max_seqlen, causal_in_block, window, softmax_scale,
                         num_splits, workspace, workspace_bytes, out, lse, dev_status, stream);
}

int qk4v8_attention_decode_v4(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int nq, int q_cap,
                              const uint8_t *k_codes, const uint8_t *k_scales, const uint8_t *v_codes,
                              const uint8_t *v_scales, int Hkv, int kv_cap, const int32_t *seqlens_k, int max_seqlen,
                              int causal_in_block, int window, float softmax_scale, int num_splits, void *workspace,
                              size_t workspace_bytes, void *out, float *lse, int32_t *dev_status, void *stream) {
    KvPages layout;
    layout.v_fp4 = true;
    return decode_packed(q_codes, q_scales, B, Hq, nq, q_cap, k_codes, k_scales, v_codes, v_scales, Hkv, kv_cap,
                         layout, seqlens_k, max_seqlen, causal_in_block, window, softmax_scale, num_splits, workspace,
                         workspace_bytes, out, lse, dev_status, stream);
}

int qk4v8_attention_decode(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int nq, int q_cap,
                           const uint8_t *k_codes, const uint8_t *k_scales, const uint8_t *v_codes,
                           const uint8_t *v_scales, int Hkv, int kv_cap, const int32_t *seqlens_k, int max_seqlen,
                           int causal_in_block, float softmax_scale, int num_splits, void *workspace,
                           size_t workspace_bytes, void *out, float *lse, int32_t *dev_status, void *stream) {
    return qk4v8_attention_decode_window(q_codes, q_scales, B, Hq, nq, q_cap, k_codes, k_scales, v_codes, v_scales,
                                         Hkv, kv_cap, seqlens_k, max_seqlen, causal_in_block, 0, softmax_scale,
                                         num_splits, workspace, workspace_bytes, out, lse, dev_status, stream);
}

int qk4v8_decode_default_splits_window(int B, int Hq, int Hkv, int nq, int max_seqlen, int window) {
    return qk4v8_decode_default_splits(B, Hq, Hkv, nq, window_span(max_seqlen, nq, window));
}

}  // extern "C"

namespace {

// Modelled time of a split-KV launch over sequences of `tiles` key tiles each
// (times Hkv heads), `s` splits of `st` tiles: the CTAs start in launch order
// (sequence, head, split) on `slots` resident slots, empty splits cost nothing,
// and the active CTAs share the memory bandwidth: each streams min(kBoost,
// slots / active) tiles per unit of time (1 when every slot is busy). Plus a
// fixed cost per launch and the merge launch when s > 1. The constants were
// fitted to measured split sweeps of the long-context decode workload (one
// time unit is one tile at full occupancy).
double model_split_time(const std::vector<int> &tiles, int Hkv, int s, int st, int slots) {
    constexpr double kBoost = 1.5, kLaunch = 17.0, kMerge = 4.0;
    std::priority_queue<double, std::vector<double>, std::greater<double>> fin;  // virtual finish times
    double v = 0.0, t = 0.0;
    auto advance = [&]() {
        const double vf = fin.top();
        const double n = static_cast<double>(fin.size());
        const double rate = std::min(kBoost, static_cast<double>(slots) / n);
        t += (vf - v) / rate;
        v = vf;
        fin.pop();
    };
    for (int tb : tiles)
        for (int h = 0; h < Hkv; ++h)
            for (int j = 0; j < s; ++j) {
                const int w = std::min(st, tb - j * st);
                if (w <= 0) break;
                if (static_cast<int>(fin.size()) == slots) advance();
                fin.push(v + w);
            }
    while (!fin.empty()) advance();
    return t + kLaunch + (s > 1 ? kMerge : 0.0);
}

}  // namespace

extern "C" {

int qk4v8_decode_plan_splits(int B, int Hq, int Hkv, int nq, const int32_t *seqlens_host, int window) {
    if (B <= 0 || Hkv <= 0 || Hq <= 0 || Hq % Hkv || nq <= 0 || !seqlens_host || window < 0) return 1;
    int max_len = 0;
    for (int b = 0; b < B; ++b) max_len = std::max(max_len, seqlens_host[b]);
    const int rows = (Hq / Hkv) * nq;
    // Groups of 33..64 rows: the GQA decode kernel balances the key tiles itself.
    if (rows >= qk4v8::kGqaMinRows || static_cast<int64_t>(B) * Hkv > 4096)
        return qk4v8_decode_default_splits_window(B, Hq, Hkv, nq, max_len, window);
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
        sms = 148;
        (void)cudaGetLastError();
    }
    const int slots = sms * (rows <= 16 ? 2 : 1);
    std::vector<int> tiles(static_cast<size_t>(B));
    int tmax = 1;
    for (int b = 0; b < B; ++b) {
        const int L = std::max(0, seqlens_host[b]);
        const int lo = window > 0 ? std::max(0, L - nq - window) : 0;
        tiles[b] = (L + 127) / 128 - lo / 128;
        tmax = std::max(tmax, tiles[b]);
    }
    int best = 1;
    double best_t = 0.0;
    for (int s = 1; s <= 64 && s <= tmax; ++s) {
        const int st = (tmax + s - 1) / s;
        if (s > 1 && (tmax + st - 1) / st < s) continue;  // the same plan as a smaller s
        const double t = model_split_time(tiles, Hkv, s, st, slots);
        if (s == 1 || t < best_t) {
            best_t = t;
            best = s;
        }
    }
    return best;
}

size_t qk4v8_decode_bf16_workspace_bytes(int B, int Hq, int Hkv, int nq, int num_splits) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || nq <= 0 || num_splits <= 0) return 0;
    // Sized by the row count alone (the test hook that moves groups of 33..64
    // rows to the swap-AB kernel only lowers the need). Up to 32 rows the
    // swap-AB kernel quantizes the queries itself and writes the output directly
    // from one split.
    const int rows = (Hq / Hkv) * nq;
    if (rows < qk4v8::kGqaMinRows) return num_splits == 1 ? 0 : qk4v8_decode_workspace_bytes(B, Hq, nq, num_splits);
    // Larger groups: the queries are quantized into the front of the workspace
    // (capacity 128 tokens), then the split partials follow (none when the GQA
    // decode kernel writes the output directly from one split).
    const size_t packed = qk4v8_mxfp4_codes_bytes(B, Hq, 128) + qk4v8_scales_bytes(B, Hq, 128);
    if (rows <= qk4v8::kDecodeMaxRows && num_splits == 1) return packed;
    return packed + qk4v8_decode_workspace_bytes(B, Hq, nq, num_splits);
}

int qk4v8_attention_decode_bf16(const void *q, int B, int Hq, int nq, int64_t q_stride_b, int64_t q_stride_t,
                                int64_t q_stride_h, const uint8_t *k_codes, const uint8_t *k_scales,
                                const uint8_t *v_codes, const uint8_t *v_scales, int Hkv, int kv_cap,
                                const int32_t *seqlens_k, int max_seqlen, int causal_in_block, float softmax_scale,
                                int num_splits, void *workspace, size_t workspace_bytes, void *out, float *lse,
                                int32_t *dev_status, void *stream) {
    return qk4v8_attention_decode_bf16_window(q, B, Hq, nq, q_stride_b, q_stride_t, q_stride_h, k_codes, k_scales,
                                              v_codes, v_scales, Hkv, kv_cap, seqlens_k, max_seqlen, causal_in_block,
                                              0, softmax_scale, num_splits, workspace, workspace_bytes, out, lse,
                                              dev_status, stream);
}

}  // extern "C"

namespace {

int decode_bf16(const void *q, int B, int Hq, int nq, int64_t q_stride_b, int64_t q_stride_t, int64_t q_stride_h,
                const uint8_t *k_codes, const uint8_t *k_scales, const uint8_t *v_codes, const uint8_t *v_scales,
                int Hkv, int kv_cap, const KvPages &pages, const int32_t *seqlens_k, int max_seqlen,
                int causal_in_block, int window, float softmax_scale, int num_splits, void *workspace,
                size_t workspace_bytes, void *out, float *lse, int32_t *dev_status, void *stream) {
    if (!q) return set_error(QK4V8_ERR_INVALID_ARG, "q is null");
    if (!out || !aligned16(out)) return set_error(QK4V8_ERR_INVALID_ARG, "out must be a 16-byte aligned pointer");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || nq < 1 || nq > 8 || (Hq / Hkv) * nq > 128)
        return set_error(QK4V8_ERR_INVALID_ARG, "bad sizes B=%d Hq=%d Hkv=%d nq=%d", B, Hq, Hkv, nq);
    if (num_splits < 0) return set_error(QK4V8_ERR_INVALID_ARG, "num_splits must be >= 0");
    if (window < 0 || (window > 0 && (Hq / Hkv) * nq > qk4v8::kDecodeMaxRows))
        return set_error(QK4V8_ERR_INVALID_ARG, "window must be >= 0, and > 0 only with (Hq/Hkv)*nq <= %d",
                         qk4v8::kDecodeMaxRows);
    const int splits =
        num_splits > 0 ? num_splits : qk4v8_decode_default_splits(B, Hq, Hkv, nq, window_span(max_seqlen, nq, window));
    const size_t need = qk4v8_decode_bf16_workspace_bytes(B, Hq, Hkv, nq, splits);
    if (need && (!workspace || !aligned16(workspace) || workspace_bytes < need))
        return set_error(QK4V8_ERR_INVALID_ARG, "workspace must be 16-byte aligned and >= %zu bytes", need);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int used = 0;
    bool direct = false;
    DecodeQuery dq;
    if (swap_ab_rows(Hq, Hkv, nq)) {
        dq.bf16 = static_cast<const __nv_bfloat16 *>(q);
        dq.sb = q_stride_b;
        dq.st = q_stride_t;
        dq.sh = q_stride_h;
        int st = decode_splitkv(dq, B, Hq, nq, k_codes, k_scales, v_codes, v_scales, Hkv, kv_cap, pages, seqlens_k,
                                max_seqlen, causal_in_block, window, softmax_scale, splits, workspace,
                                workspace_bytes, out, lse, dev_status, s, &used, &direct);
        if (st || direct) return st;
        return qk4v8_decode_merge(workspace, workspace_bytes, B, Hq, nq, used, out, lse, stream);
    }
    // More than 32 query rows per KV head: quantize Q into the front of the
    // workspace (capacity 128 tokens). The GQA decode kernel (up to 64 rows)
    // reads only the nq rows of each head, so only those are written; the
    // 128-row kernel gets the whole capacity.
    uint8_t *qc = static_cast<uint8_t *>(workspace);
    uint8_t *qs = qc + qk4v8_mxfp4_codes_bytes(B, Hq, 128);
    uint8_t *rest = qs + qk4v8_scales_bytes(B, Hq, 128);
    const size_t rest_bytes = workspace_bytes - static_cast<size_t>(rest - qc);
    const bool gqa = gqa_rows(Hq, Hkv, nq);
    int st;
    if (gqa) {
        if (!aligned16(q) || q_stride_b % 8 || q_stride_t % 8 || q_stride_h % 8 || q_stride_b < 0 || q_stride_t < 0 ||
            q_stride_h < 0)
            return set_error(QK4V8_ERR_INVALID_ARG, "bf16 Q must be 16-byte aligned with strides of whole 8-element "
                                                    "(16-byte) units");
        if ((st = check_device())) return st;
        cudaError_t e = qk4v8::launch_quantize_qk(q, B, nq, Hq, q_stride_b, q_stride_t, q_stride_h, nullptr, 128, qc,
                                                  qs, s, /*pad_to_cap=*/false);
        if (e != cudaSuccess) return cuda_error(e, "quantize (decode queries) launch");
    } else if ((st = qk4v8_quantize_qk(q, B, nq, Hq, 128, q_stride_b, q_stride_t, q_stride_h, nullptr, 128, qc, qs,
                                       stream))) {
        return st;
    }
    dq.codes = qc;
    dq.scales = qs;
    dq.cap = 128;
    st = decode_splitkv(dq, B, Hq, nq, k_codes, k_scales, v_codes, v_scales, Hkv, kv_cap, pages, seqlens_k,
                        max_seqlen, causal_in_block, window, softmax_scale, splits, rest, rest_bytes,
                        gqa ? out : nullptr, gqa ? lse : nullptr, dev_status, s, &used, &direct);
    if (st || direct) return st;
    return qk4v8_decode_merge(rest, rest_bytes, B, Hq, nq, used, out, lse, stream);
}

}  // namespace

extern "C" {

int qk4v8_attention_decode_bf16_window(const void *q, int B, int Hq, int nq, int64_t q_stride_b,
                                       int64_t q_stride_t, int64_t q_stride_h, const uint8_t *k_codes,
                                       const uint8_t *k_scales, const uint8_t *v_codes, const uint8_t *v_scales,
                                       int Hkv, int kv_cap, const int32_t *seqlens_k, int max_seqlen,
                                       int causal_in_block, int window, float softmax_scale, int num_splits,
                                       void *workspace, size_t workspace_bytes, void *out, float *lse,
                                       int32_t *dev_status, void *stream) {
    return decode_bf16(q, B, Hq, nq, q_stride_b, q_stride_t, q_stride_h, k_codes, k_scales, v_codes, v_scales, Hkv,
                       kv_cap, KvPages{}, seqlens_k, max_seqlen, causal_in_block, window, softmax_scale, num_splits,
                       workspace, workspace_bytes, out, lse, dev_status, stream);
}

int qk4v8_attention_decode_bf16_paged(const void *q, int B, int Hq, int nq, int64_t q_stride_b, int64_t q_stride_t,
                                      int64_t q_stride_h, const uint8_t *k_codes, const uint8_t *k_scales,
                                      const uint8_t *v_codes, const uint8_t *v_scales, int Hkv, int num_pages,
                                      const int32_t *block_table, int max_pages, const int32_t *seqlens_k,
                                      int max_seqlen, int causal_in_block, int window, float softmax_scale,
                                      int num_splits, void *workspace, size_t workspace_bytes, void *out, float *lse,
                                      int32_t *dev_status, void *stream) {
    if (!block_table) return set_error(QK4V8_ERR_INVALID_ARG, "block_table is null");
    if (max_pages <= 0 || max_pages >= (1 << 24))
        return set_error(QK4V8_ERR_INVALID_ARG, "bad max_pages %d", max_pages);
    KvPages pages;
    pages.block_table = block_table;
    pages.max_pages = max_pages;
    pages.num_pages = num_pages;
    return decode_bf16(q, B, Hq, nq, q_stride_b, q_stride_t, q_stride_h, k_codes, k_scales, v_codes, v_scales, Hkv,
                       max_pages * 128, pages, seqlens_k, max_seqlen, causal_in_block, window, softmax_scale,
                       num_splits, workspace, workspace_bytes, out, lse, dev_status, stream);
}

int qk4v8_attention_decode_bf16_v4(const void *q, int B, int Hq, int nq, int64_t q_stride_b, int64_t q_stride_t,
                                   int64_t q_stride_h, const uint8_t *k_codes, const uint8_t *k_scales,
                                   const uint8_t *v_codes, const uint8_t *v_scales, int Hkv, int kv_cap,
                                   const int32_t *seqlens_k, int max_seqlen, int causal_in_block, int window,
                                   float softmax_scale, int num_splits, void *workspace, size_t workspace_bytes,
                                   void *out, float *lse, int32_t *dev_status, void *stream) {
    KvPages layout;
    layout.v_fp4 = true;
    return decode_bf16(q, B, Hq, nq, q_stride_b, q_stride_t, q_stride_h, k_codes, k_scales, v_codes, v_scales, Hkv,
                       kv_cap, layout, seqlens_k, max_seqlen, causal_in_block, window, softmax_scale, num_splits,
                       workspace, workspace_bytes, out, lse, dev_status, stream);
}

size_t qk4v8_kv_tail_bytes(int B, int Hkv) {
    if (B <= 0 || Hkv <= 0) return 0;
    return static_cast<size_t>(B) * Hkv * 32 * 128 * 2;
}

int qk4v8_kv_append(const void *k_new, const void *v_new, int B, int n_new, int Hkv, int d, int64_t stride_b,
                    int64_t stride_t, int64_t stride_h, const int32_t *seqlens, int32_t *seqlens_out,
                    const int32_t *block_table, int max_pages, int num_pages, uint8_t *k_codes, uint8_t *k_scales,
                    uint8_t *v_codes, uint8_t *v_scales, void *v_tail, int hadamard_k, int32_t *dev_status,
                    void *stream) {
    if (!k_new || !v_new || !seqlens || !block_table || !k_codes || !k_scales || !v_codes || !v_scales || !v_tail)
        return set_error(QK4V8_ERR_INVALID_ARG, "null pointer");
    if (d != 128) return set_error(QK4V8_ERR_INVALID_ARG, "head_dim must be 128 (got %d)", d);
    if (B <= 0 || n_new <= 0 || Hkv <= 0 || max_pages <= 0 || num_pages <= 0 ||
        static_cast<int64_t>(num_pages) * Hkv >= (int64_t{1} << 31) || max_pages >= (1 << 24))
        return set_error(QK4V8_ERR_INVALID_ARG, "bad sizes B=%d n_new=%d Hkv=%d max_pages=%d num_pages=%d", B, n_new,
                         Hkv, max_pages, num_pages);
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_codes) || !aligned16(v_codes) || !aligned16(v_tail))
        return set_error(QK4V8_ERR_INVALID_ARG, "K/V inputs, code pools and v_tail must be 16-byte aligned");
    if (stride_b % 8 || stride_t % 8 || stride_h % 8 || stride_b < 0 || stride_t < 0 || stride_h < 0)
        return set_error(QK4V8_ERR_INVALID_ARG, "strides must be non-negative multiples of 8 elements");
    int st;
    if ((st = check_device())) return st;
    cudaError_t e = qk4v8::launch_kv_append(k_new, v_new, B, n_new, Hkv, stride_b, stride_t, stride_h, seqlens,
                                            block_table, max_pages, num_pages, k_codes, k_scales, v_codes, v_scales,
                                            v_tail, hadamard_k != 0, seqlens_out, dev_status,
                                            static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? QK4V8_OK : cuda_error(e, "kv append launch");
}

// Test hook (declared in include/qk4v8_test.h): while enabled, attention
// launches withhold the producer's Q-ready signal so the pipeline's bounded
// waits expire and report QK4V8_ERR_TIMEOUT through dev_status.
void qk4v8_test_set_stall(int enable) { g_test_stall = enable ? 1 : 0; }

// Test hook (declared in include/qk4v8_test.h): while set, CTA 0 of each
// attention launch writes its first raw score tile to `dev_ptr`.
void qk4v8_test_set_dump_scores(float *dev_ptr) { g_test_dump_s = dev_ptr; }

// Test hook (declared in include/qk4v8_test.h): while enabled, decode groups of
// 33..64 query rows run on the swap-AB kernel instead of the GQA decode kernel.
void qk4v8_test_set_force_swap_ab(int enable) { g_test_force_swap_ab = enable ? 1 : 0; }

int qk4v8_test_mma_peak(int kind, int ctas, int iters, int32_t *dev_status, void *stream) {
    if (kind < 0 || kind > 3 || ctas <= 0 || ctas > 65535 || iters <= 0 || iters > (1 << 24))
        return set_error(QK4V8_ERR_INVALID_ARG, "bad MMA peak run kind=%d ctas=%d iters=%d", kind, ctas, iters);
    int st;
    if ((st = check_device())) return st;
    cudaError_t e = qk4v8::launch_mma_peak(kind, ctas, iters, dev_status, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? QK4V8_OK : cuda_error(e, "MMA peak launch");
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode without any allocation by the caller.
//
// Some callers cannot call cudaMalloc. Examples are a plug-in running inside a
// host application that owns and budgets all device memory (an inference
// server's pre-reserved pool), and a latency-critical loop where cudaMalloc's
// implicit device synchronisation is not acceptable. For them, the split-KV
// scratch lives in this fixed, file-scope device array. Every GPU that loads
// the library holds it until the process exits.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char qk4v8_noalloc_scratch[QK4V8_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_noalloc_mu;
constexpr int kNoAllocMaxDevices = 64;
void *g_noalloc_ptr[kNoAllocMaxDevices] = {};
unsigned long long g_noalloc_ctx[kNoAllocMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Unique id of the current CUDA context (0 when it cannot be had). A context
// destroyed by cudaDeviceReset and created again gets a new id, even if its
// handle value is reused, so a cached device address is looked up again.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of the scratch array on the current device. In host code the
// array's name only stands in for the symbol and is not a device address, so
// the address is looked up with the device current, once per device and
// context (again after a cudaDeviceReset, which reloads the module).
int noalloc_scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
    if (dev < 0 || dev >= kNoAllocMaxDevices) return set_error(QK4V8_ERR_UNSUPPORTED, "device index %d too large", dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    const unsigned long long ctx = current_context_id();
    if (!g_noalloc_ptr[dev] || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, qk4v8_noalloc_scratch);
        if (e != cudaSuccess) return cuda_error(e, "cudaGetSymbolAddress(decode scratch)");
        g_noalloc_ptr[dev] = ptr;
        // The id is read again: the symbol lookup may have created the context.
        g_noalloc_ctx[dev] = current_context_id();
    }
    *out = g_noalloc_ptr[dev];
    return QK4V8_OK;
}

}  // namespace

extern "C" {

int qk4v8_attention_decode_noalloc(const uint8_t *q_codes, const uint8_t *q_scales, int B, int Hq, int nq,
                                   int q_cap, const uint8_t *k_codes, const uint8_t *k_scales,
                                   const uint8_t *v_codes, const uint8_t *v_scales, int Hkv, int kv_cap,
                                   const int32_t *seqlens_k, int max_seqlen, int causal_in_block,
                                   float softmax_scale, int num_splits, void *out, float *lse, int32_t *dev_status,
                                   void *stream) {
    if (num_splits < 0) return set_error(QK4V8_ERR_INVALID_ARG, "num_splits must be >= 0");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || nq < 1 || nq > 8 || (Hq / Hkv) * nq > 128)
        return set_error(QK4V8_ERR_INVALID_ARG, "bad sizes B=%d Hq=%d Hkv=%d nq=%d", B, Hq, Hkv, nq);
    const int splits = num_splits > 0 ? num_splits : qk4v8_decode_default_splits(B, Hq, Hkv, nq, max_seqlen);
    // One split with up to 64 query rows per KV head: the split kernel writes
    // the output itself and needs no scratch (qk4v8_attention_decode's rule).
    const bool direct = splits == 1 && (Hq / Hkv) * nq <= qk4v8::kDecodeMaxRows;
    const size_t need = direct ? 0 : qk4v8_decode_workspace_bytes(B, Hq, nq, splits);
    if (need > QK4V8_NOALLOC_SCRATCH_BYTES)
        return set_error(QK4V8_ERR_INVALID_ARG,
                         "decode scratch of %zu bytes (B=%d Hq=%d nq=%d splits=%d) exceeds the fixed %zu-byte "
                         "array of qk4v8_attention_decode_noalloc; use qk4v8_attention_decode with a workspace",
                         need, B, Hq, nq, splits, static_cast<size_t>(QK4V8_NOALLOC_SCRATCH_BYTES));
    void *scratch = nullptr;
    int st = noalloc_scratch_address(&scratch);
    if (st) return st;
    return qk4v8_attention_decode(q_codes, q_scales, B, Hq, nq, q_cap, k_codes, k_scales, v_codes, v_scales, Hkv,
                                  kv_cap, seqlens_k, max_seqlen, causal_in_block, softmax_scale, splits, scratch,
                                  QK4V8_NOALLOC_SCRATCH_BYTES, out, lse, dev_status, stream);
}

}  // extern "C"
