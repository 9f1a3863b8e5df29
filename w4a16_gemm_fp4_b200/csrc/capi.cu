// capi.cu -- the extern "C" entry points of libfp4w4a16.so: argument
// validation (before anything is launched), the per-format value tables,
// engine dispatch and the per-device status word.  See include/fp4w4a16.h
// for the contract of each call.
#include <math.h>
#include <stdio.h>

#include "common.cuh"

#include <cmath>
#include <cstring>

namespace fp4 {
// kernels (quantize.cu, preshift.cu, gemm_decode.cu, gemm_tc.cu)
size_t quantize_ws_bytes(long long total, bool search, bool want_sse);
cudaError_t launch_quantize(const float* W, int N, int K, int group, int fmt, int bias_search,
                            const int8_t* shift, int sdt, uint8_t* packed, void* scales, int32_t* choice,
                            double* sse, void* ws, const FmtTables& tabs, int* status, cudaStream_t st);
cudaError_t launch_dequantize(const uint8_t* packed, const void* scales, int sdt, const FmtTable& t, int N, int K,
                              int group, float* out, cudaStream_t st);
size_t preshift_ws_bytes(int M, int K);
cudaError_t launch_calibrate(const uint16_t* X, int M, int K, int8_t* shift, float* rho, void* ws, int* status,
                             cudaStream_t st);
cudaError_t launch_apply(const uint16_t* X, int M, int K, const int8_t* shift, const float* rho, uint16_t* Xt,
                         cudaStream_t st);
cudaError_t launch_gemm_decode(const uint16_t* X, const uint8_t* packed, const void* scales, int sdt,
                               const FmtTable& t, int M, int N, int K, int group, const float* x_scale, uint16_t* Y,
                               int act, cudaStream_t st);
int decode_max_m_lut();
cudaError_t launch_gemm_ts(const uint16_t* X, void* ws, size_t ws_bytes, const uint8_t* packed, const void* scales,
                           int sdt, int fmt, int M, int N, int K, const float* x_scale, uint16_t* Y, int act,
                           int ctas, int* status, unsigned long long timeout_ns, cudaStream_t st);
size_t ts_ws_bytes(int M, int N, int K);
cudaError_t launch_gemm_skinny(const uint16_t* X, int* cnt, void* ws, size_t ws_bytes, const uint8_t* packed,
                               const void* scales, int sdt, int fmt, int M, int N, int K, const float* x_scale,
                               uint16_t* Y, int act, int ctas, int* status, unsigned long long timeout_ns,
                               cudaStream_t st);
size_t skinny_ws_bytes(int M, int N, int K);
int skinny_max_m();
int skinny_max_tiles();
int skinny_tiles(int N, int K);
cudaError_t launch_gemm_rowblk(const uint16_t* X, const uint8_t* packed, const void* scales, int sdt, int fmt,
                               int M, int N, int K, const float* x_scale, uint16_t* Y, int act, int* status,
                               unsigned long long timeout_ns, cudaStream_t st);
bool rowblk_fits(int M, int K);
bool rowblk_preferred(int M, int K);
size_t tc_ws_bytes(int M, int N, int K);
cudaError_t launch_gemm_tc(const uint16_t* X, const uint8_t* packed, const void* scales, int sdt, const FmtTable& t,
                           bool e2m1, int M, int N, int K, int group, const float* x_scale, uint16_t* Y, int act,
                           void* ws, size_t ws_bytes, int splits, int* status, unsigned long long timeout_ns,
                           cudaStream_t st);
cudaError_t launch_bounded_wait_probe(int* status, unsigned long long timeout_ns, cudaStream_t st);
size_t quantize_blocks_ws_bytes(int N, int K, int group, int gran, int heads, bool search);
cudaError_t launch_quantize_blocks(const float* W, int N, int K, int group, int gran, int heads, int fmt, int j,
                                   const int8_t* shift, int sdt, uint8_t* packed, void* scales, int8_t* jmap,
                                   void* ws, const FmtTables& tabs, int* status, cudaStream_t st);
cudaError_t launch_act_quantize(const uint16_t* X, int M, int K, const int8_t* shift, const float* rho,
                                const FmtTables& tabs, int fmt, int j, uint8_t* packed, float* a_scale, int* status,
                                cudaStream_t st);
cudaError_t launch_act_expand(const uint8_t* codes, long long count, const FmtTable& t, uint16_t* out,
                              cudaStream_t st);
bool w4a4_native_fits(int afmt, int fmt, int M, int N, int K, int group, const void* apacked, const void* packed);
cudaError_t launch_gemm_w4a4(const uint8_t* apacked, const float* a_scale, const uint8_t* packed, const void* scales,
                             int sdt, int M, int N, int K, uint16_t* Y, int act, int* status,
                             unsigned long long timeout_ns, cudaStream_t st);
int noalloc_max_k();
cudaError_t launch_calibrate_noalloc(const uint16_t* X, int M, int K, int8_t* shift, float* rho, int* status,
                                     cudaStream_t st);
}  // namespace fp4

using namespace fp4;

// The status word lives in this module; each device holds its own copy.
__device__ int g_fp4_status;

namespace {

// Largest M of the decode engine: the tensor-memory engine at group 128,
// the per-lane-LUT kernel at groups 32 and 64.
constexpr int kDecodeMaxM128 = 64;     // decode engine on request (group 128)
constexpr int kAutoDecodeMaxM128 = 8;  // decode engine by default (group 128)
constexpr int kMaxDevices = 64;

int decode_max_m(int group) { return group == 128 ? kDecodeMaxM128 : decode_max_m_lut(); }
long long g_timeout_us = 2000000;

// Value of magnitude index i (code & 7) of the format with e exponent and m
// mantissa bits and bias b = 2^(e-1) - 1: exponent field p = i >> m,
// mantissa d = i & (2^m - 1); p == 0 is the subnormal binade.
float magnitude(int e, int m, int i) {
    const int b = (1 << (e - 1)) - 1;
    const int p = i >> m, d = i & ((1 << m) - 1);
    if (p == 0) return ldexpf((float)d, 1 - b - m);
    return ldexpf((float)((1 << m) + d), p - b - m);
}

const FmtTables& tables() {
    static FmtTables T;
    static bool init = false;
    if (!init) {
        const int em[3][2] = {{1, 2}, {2, 1}, {3, 0}};
        for (int f = 0; f < 3; ++f) {
            for (int i = 0; i < 8; ++i) T.f[f].mag[i] = magnitude(em[f][0], em[f][1], i);
            for (int i = 0; i < 7; ++i) T.f[f].mid[i] = 0.5f * (T.f[f].mag[i] + T.f[f].mag[i + 1]);
            T.f[f].qmax = T.f[f].mag[7];
            // Test i decides index >= i+1.  For even i it is fl32(y) > mid[i]
            // (a tie at mid[i] stays on the even index i): fl32(y) exceeds m
            // exactly when y lies above the rounding boundary between m and
            // its successor m+, or on it when round-to-even picks m+.  For
            // odd i it is fl32(y) >= mid[i] (a tie goes up to the even i+1):
            // the boundary between m's predecessor m- and m, passed on the
            // boundary when m is the even one.
            T.tie_up[f] = 0;
            for (int i = 0; i < 7; ++i) {
                const float m = T.f[f].mid[i];
                float lo, hi;
                if ((i & 1) == 0) {
                    lo = m;
                    hi = std::nextafter(m, INFINITY);
                } else {
                    lo = std::nextafter(m, 0.f);
                    hi = m;
                }
                T.hb[f][i] = 0.5 * ((double)lo + (double)hi);
                uint32_t hbits;
                std::memcpy(&hbits, &hi, 4);
                if ((hbits & 1u) == 0) T.tie_up[f] |= 1u << i;
            }
        }
        for (int j = 0; j < 8; ++j) T.cj[j] = (float)exp2(-(double)j / 8.0);
        init = true;
    }
    return T;
}

int* status_ptr() {
    static int* ptrs[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    if (!ptrs[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_fp4_status) != cudaSuccess) return nullptr;
        ptrs[dev] = reinterpret_cast<int*>(p);
    }
    return ptrs[dev];
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

fp4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA; }

fp4_status check_group(int K, int group) {
    if (group != 32 && group != 64 && group != 128) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (K % group != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
    return FP4_OK;
}

fp4_status check_weights(const uint8_t* packed, const void* scales, fp4_scale_dtype sdt, fp4_format fmt, int N,
                         int K, int group) {
    if (N < 0 || K < 0) return FP4_ERR_INVALID_ARG;
    if (fmt < FP4_E1M2 || fmt > FP4_E3M0) return FP4_ERR_INVALID_ARG;
    if (sdt != FP4_SCALE_F32 && sdt != FP4_SCALE_F16) return FP4_ERR_INVALID_ARG;
    fp4_status s = check_group(K, group);
    if (s != FP4_OK) return s;
    if ((long long)N * K > 0) {
        if (!packed || !scales) return FP4_ERR_INVALID_ARG;
        if (!aligned(packed, 16) || !aligned(scales, 4)) return FP4_ERR_MISALIGNED;
    }
    return FP4_OK;
}

}  // namespace

extern "C" {

int fp4_abi_version(void) { return 100; }

const char* fp4_status_string(fp4_status s) {
    switch (s) {
        case FP4_OK: return "ok";
        case FP4_ERR_INVALID_ARG: return "invalid argument";
        case FP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape (group must be 32/64/128 and divide K)";
        case FP4_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
        case FP4_ERR_WORKSPACE: return "workspace missing or too small";
        case FP4_ERR_CUDA: return "CUDA error";
        case FP4_ERR_DEVICE_STATUS: return "device status flag set";
    }
    return "unknown status";
}

void fp4_set_wait_timeout_us(long long us) { g_timeout_us = us < 1 ? 2000000 : us; }

size_t fp4_quantize_workspace_size(int N, int K, int group, fp4_format fmt, int bias_search) {
    (void)group;
    if (N <= 0 || K <= 0) return 0;
    const bool search = fmt == FP4_FMT_AUTO || bias_search != 0;
    return quantize_ws_bytes((long long)N * K, search, true);
}

fp4_status fp4_quantize(const float* W, int N, int K, int group, fp4_format fmt, int bias_search,
                        const int8_t* chan_shift, fp4_scale_dtype sdt, uint8_t* packed, void* scales,
                        int32_t* choice, double* sse, void* workspace, size_t ws_bytes, cudaStream_t stream) {
    if (N < 0 || K < 0) return FP4_ERR_INVALID_ARG;
    if (fmt < FP4_FMT_AUTO || fmt > FP4_E3M0) return FP4_ERR_INVALID_ARG;
    if (sdt != FP4_SCALE_F32 && sdt != FP4_SCALE_F16) return FP4_ERR_INVALID_ARG;
    fp4_status s = check_group(K, group);
    if (s != FP4_OK) return s;
    if (!choice) return FP4_ERR_INVALID_ARG;
    if (!aligned(choice, 4) || (sse && !aligned(sse, 8))) return FP4_ERR_MISALIGNED;
    const long long total = (long long)N * K;
    const bool search = fmt == FP4_FMT_AUTO || bias_search != 0;
    if (total > 0) {
        if (!W || !packed || !scales) return FP4_ERR_INVALID_ARG;
        if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(scales, 4)) return FP4_ERR_MISALIGNED;
        if (chan_shift && !aligned(chan_shift, 16)) return FP4_ERR_MISALIGNED;
        const size_t need = quantize_ws_bytes(total, search, sse != nullptr);
        if (need > 0 && (!workspace || ws_bytes < need)) return FP4_ERR_WORKSPACE;
        if (workspace && !aligned(workspace, 16)) return FP4_ERR_MISALIGNED;
    }
    int* st = status_ptr();
    if (!st) return FP4_ERR_CUDA;
    if (total == 0) {
        // nothing to quantize: every candidate has SSE 0, the first one wins
        const int f = fmt == FP4_FMT_AUTO ? 0 : (int)fmt;
        const int32_t host_choice[2] = {f, 0};
        cudaError_t e = cudaMemcpyAsync(choice, host_choice, sizeof(host_choice), cudaMemcpyHostToDevice, stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
        if (e == cudaSuccess && sse) {
            double host_sse[24];
            const int f1 = fmt == FP4_FMT_AUTO ? 2 : f;
            const int jn = bias_search ? 8 : 1;
            for (int ff = 0; ff < 3; ++ff)
                for (int j = 0; j < 8; ++j) host_sse[ff * 8 + j] = (ff >= f && ff <= f1 && j < jn) ? 0.0 : NAN;
            e = cudaMemcpyAsync(sse, host_sse, sizeof(host_sse), cudaMemcpyHostToDevice, stream);
            if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
        }
        return cuda_status(e);
    }
    return cuda_status(launch_quantize(W, N, K, group, (int)fmt, bias_search, chan_shift, (int)sdt, packed, scales,
                                       choice, sse, workspace, tables(), st, stream));
}

static bool blocks_shape_ok(int N, int K, fp4_granularity gran, int heads) {
    if (gran == FP4_GRAN_GROUP) return true;
    if (K % 128 != 0) return false;
    return gran == FP4_GRAN_CHANNEL || (heads > 0 && N % heads == 0);
}

size_t fp4_quantize_blocks_workspace_size(int N, int K, int group, fp4_granularity gran, int heads, int bias_index) {
    if (N <= 0 || K <= 0 || group <= 0 || K % group != 0) return 0;
    if (gran < FP4_GRAN_GROUP || gran > FP4_GRAN_HEAD || !blocks_shape_ok(N, K, gran, heads)) return 0;
    return quantize_blocks_ws_bytes(N, K, group, (int)gran, heads, bias_index < 0);
}

fp4_status fp4_quantize_blocks(const float* W, int N, int K, int group, fp4_granularity gran, int heads,
                               fp4_format fmt, int bias_index, const int8_t* chan_shift, fp4_scale_dtype sdt,
                               uint8_t* packed, void* scales, int8_t* jmap, void* workspace, size_t ws_bytes,
                               cudaStream_t stream) {
    if (N < 0 || K < 0) return FP4_ERR_INVALID_ARG;
    if (fmt < FP4_E1M2 || fmt > FP4_E3M0) return FP4_ERR_INVALID_ARG;
    if (sdt != FP4_SCALE_F32 && sdt != FP4_SCALE_F16) return FP4_ERR_INVALID_ARG;
    if (bias_index < -1 || bias_index > 7) return FP4_ERR_INVALID_ARG;
    if (gran < FP4_GRAN_GROUP || gran > FP4_GRAN_HEAD) return FP4_ERR_INVALID_ARG;
    if (gran == FP4_GRAN_HEAD && heads <= 0) return FP4_ERR_INVALID_ARG;
    fp4_status s = check_group(K, group);
    if (s != FP4_OK) return s;
    if (!blocks_shape_ok(N, K, gran, heads)) return FP4_ERR_UNSUPPORTED_SHAPE;
    if ((long long)N * K == 0) return FP4_OK;
    if (!W || !packed || !scales) return FP4_ERR_INVALID_ARG;
    if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(scales, 4)) return FP4_ERR_MISALIGNED;
    if (chan_shift && !aligned(chan_shift, 16)) return FP4_ERR_MISALIGNED;
    const size_t need = quantize_blocks_ws_bytes(N, K, group, (int)gran, heads, bias_index < 0);
    if (need > 0 && (!workspace || ws_bytes < need)) return FP4_ERR_WORKSPACE;
    if (workspace && !aligned(workspace, 16)) return FP4_ERR_MISALIGNED;
    int* st = status_ptr();
    if (!st) return FP4_ERR_CUDA;
    return cuda_status(launch_quantize_blocks(W, N, K, group, (int)gran, heads, (int)fmt, bias_index, chan_shift,
                                              (int)sdt, packed, scales, jmap, workspace, tables(), st, stream));
}

fp4_status fp4_act_quantize(const uint16_t* X, int M, int K, const int8_t* shift, const float* rho, fp4_format fmt,
                            int j, uint8_t* packed, float* a_scale, cudaStream_t stream) {
    if (M < 0 || K < 0) return FP4_ERR_INVALID_ARG;
    if (fmt < FP4_E1M2 || fmt > FP4_E3M0 || j < 0 || j > 7) return FP4_ERR_INVALID_ARG;
    if (K % 8 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (!rho || !a_scale) return FP4_ERR_INVALID_ARG;
    if (!aligned(rho, 4) || !aligned(a_scale, 4)) return FP4_ERR_MISALIGNED;
    if ((long long)M * K > 0) {
        if (!X || !packed) return FP4_ERR_INVALID_ARG;
        if (!aligned(X, 16) || !aligned(packed, 16)) return FP4_ERR_MISALIGNED;
        if (shift && !aligned(shift, 16)) return FP4_ERR_MISALIGNED;
    }
    int* st = status_ptr();
    if (!st) return FP4_ERR_CUDA;
    return cuda_status(launch_act_quantize(X, M, K, shift, rho, tables(), (int)fmt, j, packed, a_scale, st, stream));
}

// The W4A4 workspace: the GEMM's own (counter block first), then the
// expanded activations [M][K] bf16.
static size_t w4a4_gemm_part(int M, int N, int K) { return (fp4_gemm_workspace_size(M, N, K) + 255) & ~(size_t)255; }

size_t fp4_gemm_w4a4_workspace_size(int M, int N, int K) {
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    return w4a4_gemm_part(M, N, K) + (((size_t)M * K * 2 + 255) & ~(size_t)255);
}

fp4_status fp4_gemm_w4a4(const uint8_t* apacked, fp4_format afmt, const float* a_scale, const uint8_t* packed,
                         const void* scales, fp4_scale_dtype sdt, fp4_format fmt, int M, int N, int K, int group,
                         fp4_act act, uint16_t* Y, void* workspace, size_t ws_bytes, cudaStream_t stream) {
    if (M < 0) return FP4_ERR_INVALID_ARG;
    if (afmt < FP4_E1M2 || afmt > FP4_E3M0) return FP4_ERR_INVALID_ARG;
    if (act != FP4_ACT_NONE && act != FP4_ACT_SILU && act != FP4_ACT_GELU && act != FP4_ACT_SILU_GATE)
        return FP4_ERR_INVALID_ARG;
    fp4_status s = check_weights(packed, scales, sdt, fmt, N, K, group);
    if (s != FP4_OK) return s;
    if ((long long)M * N * K == 0)  // K == 0 (or nothing to write): fp4_gemm_act's own rules
        return fp4_gemm_act(nullptr, packed, scales, sdt, fmt, M, N, K, group, a_scale, act, Y, workspace, ws_bytes,
                            FP4_ENGINE_AUTO, 0, stream);
    if (!apacked || !a_scale || !Y) return FP4_ERR_INVALID_ARG;
    if (!aligned(apacked, 16) || !aligned(a_scale, 4)) return FP4_ERR_MISALIGNED;
    if (!workspace || ws_bytes < fp4_gemm_w4a4_workspace_size(M, N, K)) return FP4_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return FP4_ERR_MISALIGNED;
    if ((const void*)Y == (const void*)apacked) return FP4_ERR_INVALID_ARG;
    if (act == FP4_ACT_SILU_GATE && (N % 2 != 0 || group != 128)) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (w4a4_native_fits((int)afmt, (int)fmt, M, N, K, group, apacked, packed)) {
        // E2M1 x E2M1 from M = 65: both code tiles straight into kind::f8f6f4 MMAs
        int* st = status_ptr();
        if (!st) return FP4_ERR_CUDA;
        return cuda_status(launch_gemm_w4a4(apacked, a_scale, packed, scales, (int)sdt, M, N, K, Y, (int)act, st,
                                            (unsigned long long)g_timeout_us * 1000ull, stream));
    }
    const size_t gpart = w4a4_gemm_part(M, N, K);
    uint16_t* Xv = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(workspace) + gpart);
    cudaError_t e = launch_act_expand(apacked, (long long)M * K, tables().f[afmt], Xv, stream);
    if (e != cudaSuccess) return FP4_ERR_CUDA;
    return fp4_gemm_act(Xv, packed, scales, sdt, fmt, M, N, K, group, a_scale, act, Y, workspace, gpart,
                        FP4_ENGINE_AUTO, 0, stream);
}

fp4_status fp4_dequantize(const uint8_t* packed, const void* scales, fp4_scale_dtype sdt, fp4_format fmt, int N,
                          int K, int group, float* W_hat, cudaStream_t stream) {
    fp4_status s = check_weights(packed, scales, sdt, fmt, N, K, group);
    if (s != FP4_OK) return s;
    if ((long long)N * K == 0) return FP4_OK;
    if (!W_hat) return FP4_ERR_INVALID_ARG;
    if (!aligned(W_hat, 16)) return FP4_ERR_MISALIGNED;
    return cuda_status(launch_dequantize(packed, scales, (int)sdt, tables().f[fmt], N, K, group, W_hat, stream));
}

size_t fp4_preshift_workspace_size(int M, int K) {
    if (M <= 0 || K <= 0) return 0;
    return preshift_ws_bytes(M, K);
}

fp4_status fp4_preshift_calibrate(const uint16_t* X, int M, int K, int8_t* shift, float* rho, void* workspace,
                                  size_t ws_bytes, cudaStream_t stream) {
    if (M < 0 || K < 0) return FP4_ERR_INVALID_ARG;
    if (K % 8 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (!rho || (K > 0 && !shift)) return FP4_ERR_INVALID_ARG;
    if (!aligned(rho, 4) || (shift && !aligned(shift, 16))) return FP4_ERR_MISALIGNED;
    if ((long long)M * K == 0) {
        // rho = 1, every shift 0
        const float one = 1.0f;
        cudaError_t e = cudaMemcpyAsync(rho, &one, sizeof(one), cudaMemcpyHostToDevice, stream);
        if (e == cudaSuccess && K > 0) e = cudaMemsetAsync(shift, 0, (size_t)K, stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
        return cuda_status(e);
    }
    if (!X) return FP4_ERR_INVALID_ARG;
    if (!aligned(X, 16)) return FP4_ERR_MISALIGNED;
    const size_t need = preshift_ws_bytes(M, K);
    if (!workspace || ws_bytes < need) return FP4_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return FP4_ERR_MISALIGNED;
    int* st = status_ptr();
    if (!st) return FP4_ERR_CUDA;
    return cuda_status(launch_calibrate(X, M, K, shift, rho, workspace, st, stream));
}

fp4_status fp4_preshift_calibrate_noalloc(const uint16_t* X, int M, int K, int8_t* shift, float* rho,
                                          cudaStream_t stream) {
    if (M < 0 || K < 0) return FP4_ERR_INVALID_ARG;
    if (K % 8 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
    if (K > noalloc_max_k()) return FP4_ERR_WORKSPACE;  // the built-in buffer holds K <= 65536 columns
    if (!rho || (K > 0 && !shift)) return FP4_ERR_INVALID_ARG;
    if (!aligned(rho, 4) || (shift && !aligned(shift, 16))) return FP4_ERR_MISALIGNED;
    if ((long long)M * K == 0) {
        const float one = 1.0f;
        cudaError_t e = cudaMemcpyAsync(rho, &one, sizeof(one), cudaMemcpyHostToDevice, stream);
        if (e == cudaSuccess && K > 0) e = cudaMemsetAsync(shift, 0, (size_t)K, stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
        return cuda_status(e);
    }
    if (!X) return FP4_ERR_INVALID_ARG;
    if (!aligned(X, 16)) return FP4_ERR_MISALIGNED;
    int* st = status_ptr();
    if (!st) return FP4_ERR_CUDA;
    return cuda_status(launch_calibrate_noalloc(X, M, K, shift, rho, st, stream));
}

fp4_status fp4_preshift_apply(const uint16_t* X, int M, int K, const int8_t* shift, const float* rho, uint16_t* Xt,
                              cudaStream_t stream) {
    if (M < 0 || K < 0) return FP4_ERR_INVALID_ARG;
    if (K % 8 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
    if ((long long)M * K == 0) return FP4_OK;
    if (!X || !shift || !rho || !Xt || X == Xt) return FP4_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(Xt, 16) || !aligned(shift, 16) || !aligned(rho, 4)) return FP4_ERR_MISALIGNED;
    return cuda_status(launch_apply(X, M, K, shift, rho, Xt, stream));
}

// Every GEMM workspace starts with a block of tile counters that is zero
// between calls (the skinny kernel's split tiles); the engines' own data
// follows it.
constexpr size_t kCounterBlock = 65536;

static bool skinny_fits(int M, int N, int K) {
    return M <= skinny_max_m() && K % 128 == 0 && skinny_tiles(N, K) <= skinny_max_tiles();
}

size_t fp4_gemm_workspace_size(int M, int N, int K) {
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    if (skinny_fits(M, N, K)) return kCounterBlock + skinny_ws_bytes(M, N, K);
    if (M <= kDecodeMaxM128) return kCounterBlock + ts_ws_bytes(M, N, K);
    return kCounterBlock + tc_ws_bytes(M, N, K);
}

// Workspace bytes (counter block included) the group-128 decode engine needs.
static size_t decode_ws_bytes(int M, int N, int K) {
    return kCounterBlock + (skinny_fits(M, N, K) ? skinny_ws_bytes(M, N, K) : ts_ws_bytes(M, N, K));
}

fp4_status fp4_gemm_act(const uint16_t* X, const uint8_t* packed, const void* scales, fp4_scale_dtype sdt,
                        fp4_format fmt, int M, int N, int K, int group, const float* x_scale, fp4_act act,
                        uint16_t* Y, void* workspace, size_t ws_bytes, fp4_engine engine, int splits,
                        cudaStream_t stream) {
    if (M < 0) return FP4_ERR_INVALID_ARG;
    if (act != FP4_ACT_NONE && act != FP4_ACT_SILU && act != FP4_ACT_GELU && act != FP4_ACT_SILU_GATE)
        return FP4_ERR_INVALID_ARG;
    fp4_status s = check_weights(packed, scales, sdt, fmt, N, K, group);
    if (s != FP4_OK) return s;
    if (engine != FP4_ENGINE_AUTO && engine != FP4_ENGINE_DECODE && engine != FP4_ENGINE_TENSOR)
        return FP4_ERR_INVALID_ARG;
    if (splits < 0) return FP4_ERR_INVALID_ARG;
    if ((long long)M * N == 0) return FP4_OK;
    if (!Y) return FP4_ERR_INVALID_ARG;
    if (!aligned(Y, 16)) return FP4_ERR_MISALIGNED;
    if (x_scale && !aligned(x_scale, 4)) return FP4_ERR_MISALIGNED;
    if (workspace && !aligned(workspace, 16)) return FP4_ERR_MISALIGNED;
    // gate/up pairs: interleaved rows (N even), group-128 kernels; Y has N/2 columns
    const bool gated = act == FP4_ACT_SILU_GATE;
    if (gated && (N % 2 != 0 || group != 128)) return FP4_ERR_UNSUPPORTED_SHAPE;
    // K = 0: every output is act(0) = 0 for the supported activations
    if (K == 0)
        return cuda_status(cudaMemsetAsync(Y, 0, (size_t)M * (gated ? N / 2 : N) * sizeof(uint16_t), stream));
    if (!X) return FP4_ERR_INVALID_ARG;
    if (!aligned(X, 16)) return FP4_ERR_MISALIGNED;
    if ((const void*)Y == (const void*)X || (const void*)Y == (const void*)packed) return FP4_ERR_INVALID_ARG;
    const bool auto_engine = engine == FP4_ENGINE_AUTO;
    if (auto_engine) engine = fp4_gemm_engine_for(M, N, K, group);
    if (engine == FP4_ENGINE_DECODE && M > decode_max_m(group)) return FP4_ERR_UNSUPPORTED_SHAPE;
    // group 128, M <= 16: the row-block kernel (no workspace) unless a CTA
    // count is asked for or the activations do not fit it; else the
    // streaming kernels, which keep tile counters and partials in the
    // workspace
    const bool rowblk = engine == FP4_ENGINE_DECODE && group == 128 && splits == 0 && rowblk_fits(M, K);
    if (engine == FP4_ENGINE_DECODE && group == 128 && !rowblk &&
        (!workspace || ws_bytes < decode_ws_bytes(M, N, K))) {
        // the group-128 decode engine keeps its tile counters and partial
        // tiles in the workspace; without one the automatic choice takes the
        // tensor engine
        if (!auto_engine) return FP4_ERR_WORKSPACE;
        engine = FP4_ENGINE_TENSOR;
    }
    const FmtTable& t = tables().f[fmt];
    // the engines' part of the workspace follows the counter block
    void* eng_ws = workspace && ws_bytes > kCounterBlock ? static_cast<uint8_t*>(workspace) + kCounterBlock : nullptr;
    const size_t eng_bytes = eng_ws ? ws_bytes - kCounterBlock : 0;
    int* st = status_ptr();
    if (!st) return FP4_ERR_CUDA;
    const unsigned long long to_ns = (unsigned long long)g_timeout_us * 1000ull;
    if (engine == FP4_ENGINE_DECODE) {
        if (rowblk)
            return cuda_status(launch_gemm_rowblk(X, packed, scales, (int)sdt, (int)fmt, M, N, K, x_scale, Y,
                                                  (int)act, st, to_ns, stream));
        if (group == 128 && skinny_fits(M, N, K))
            return cuda_status(launch_gemm_skinny(X, static_cast<int*>(workspace), eng_ws, eng_bytes, packed, scales,
                                                  (int)sdt, (int)fmt, M, N, K, x_scale, Y, (int)act, splits, st,
                                                  to_ns, stream));
        if (group == 128)
            return cuda_status(launch_gemm_ts(X, eng_ws, eng_bytes, packed, scales, (int)sdt, (int)fmt, M, N, K,
                                              x_scale, Y, (int)act, splits, st, to_ns, stream));
        return cuda_status(
            launch_gemm_decode(X, packed, scales, (int)sdt, t, M, N, K, group, x_scale, Y, (int)act, stream));
    }
    return cuda_status(launch_gemm_tc(X, packed, scales, (int)sdt, t, fmt == FP4_E2M1, M, N, K, group, x_scale, Y,
                                      (int)act, eng_ws, eng_bytes, splits, st, to_ns, stream));
}

fp4_status fp4_gemm_ex(const uint16_t* X, const uint8_t* packed, const void* scales, fp4_scale_dtype sdt,
                       fp4_format fmt, int M, int N, int K, int group, const float* x_scale, uint16_t* Y,
                       void* workspace, size_t ws_bytes, fp4_engine engine, int splits, cudaStream_t stream) {
    return fp4_gemm_act(X, packed, scales, sdt, fmt, M, N, K, group, x_scale, FP4_ACT_NONE, Y, workspace, ws_bytes,
                        engine, splits, stream);
}

fp4_engine fp4_gemm_engine_for(int M, int N, int K, int group) {
    if (M <= 0 || N <= 0 || K <= 0) return FP4_ENGINE_AUTO;
    if (group != 32 && group != 64 && group != 128) return FP4_ENGINE_AUTO;
    // group 128: the decode engine up to 8 tokens, and up to 16 where the
    // row-block kernel runs with two block buffers; otherwise the tensor
    // engine's small token tiles measure faster (the decode engine stays
    // available on request up to 64 tokens)
    if (group == 128)
        return M <= kAutoDecodeMaxM128 || (M <= 16 && rowblk_preferred(M, K)) ? FP4_ENGINE_DECODE
                                                                                : FP4_ENGINE_TENSOR;
    return M <= decode_max_m(group) ? FP4_ENGINE_DECODE : FP4_ENGINE_TENSOR;
}

fp4_status fp4_gemm(const uint16_t* X, const uint8_t* packed, const void* scales, fp4_scale_dtype sdt,
                    fp4_format fmt, int M, int N, int K, int group, const float* x_scale, uint16_t* Y,
                    void* workspace, size_t ws_bytes, cudaStream_t stream) {
    return fp4_gemm_ex(X, packed, scales, sdt, fmt, M, N, K, group, x_scale, Y, workspace, ws_bytes,
                       FP4_ENGINE_AUTO, 0, stream);
}

fp4_status fp4_get_device_status(int32_t* host_code, int clear, cudaStream_t stream) {
    if (!host_code) return FP4_ERR_INVALID_ARG;
    int* st = status_ptr();
    if (!st) return FP4_ERR_CUDA;
    int v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, st, sizeof(int), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && clear) {
        e = cudaMemsetAsync(st, 0, sizeof(int), stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    }
    if (e != cudaSuccess) return FP4_ERR_CUDA;
    *host_code = v;
    return v ? FP4_ERR_DEVICE_STATUS : FP4_OK;
}

fp4_status fp4_selftest_bounded_wait(long long timeout_us, cudaStream_t stream) {
    if (timeout_us < 1 || timeout_us > 10000000) return FP4_ERR_INVALID_ARG;
    int* st = status_ptr();
    if (!st) return FP4_ERR_CUDA;
    return cuda_status(launch_bounded_wait_probe(st, (unsigned long long)timeout_us * 1000ull, stream));
}

}  // extern "C"
