// api.cu -- the C ABI of libfp8bw (declared in include/fp8bw.h): argument checks,
// per-device properties, and dispatch to the quantizer and GEMM launchers.
#include <atomic>
#include <initializer_list>
#include <cstdint>
#include <cuda_runtime.h>

#include "fp8bw.h"
#include "quant.cuh"

namespace {

constexpr int kMaxDevices = 64;
std::atomic<int> g_sms[kMaxDevices];    // 0 = not queried yet, -1 = not sm_100
std::atomic<int> g_major[kMaxDevices];

// Returns the SM count of the calling thread's current device, or -1 with *status
// set.  Every pointer must be device (or managed) memory of the current device: a
// host pointer would fault the kernel and another device's buffer would not match
// the caller's stream, so both are rejected here (FP8BW_EINVAL).  The current
// device is never changed.
int device_sms(std::initializer_list<const void *> ptrs, int *status)
{
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) {
        *status = FP8BW_ECUDA;
        return -1;
    }
    for (const void *p : ptrs) {
        if (!p)
            continue;
        cudaPointerAttributes at;
        if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
            cudaGetLastError();
            *status = FP8BW_ECUDA;
            return -1;
        }
        if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged) {
            *status = FP8BW_EINVAL;
            return -1;
        }
        if (at.type == cudaMemoryTypeDevice && at.device != cur) {
            *status = FP8BW_EINVAL;
            return -1;
        }
    }
    const int dev = cur;
    if (dev >= kMaxDevices) {
        *status = FP8BW_ECUDA;
        return -1;
    }
    int sms = g_sms[dev].load(std::memory_order_acquire);
    if (sms == 0) {
        int major = 0, count = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            *status = FP8BW_ECUDA;
            return -1;
        }
        g_major[dev].store(major, std::memory_order_relaxed);
        sms = (major == 10) ? count : -1;
        g_sms[dev].store(sms, std::memory_order_release);
    }
    if (sms < 0) {
        *status = FP8BW_EUNSUPPORTED;
        return -1;
    }
    *status = FP8BW_OK;
    return sms;
}

bool aligned16(const void *p)
{
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

bool dim_ok(int64_t d)
{
    return d > 0 && d <= FP8BW_MAX_DIM && (d % 128) == 0;
}

// A token count: the M of the activation quantizers and of FPROP/DGRAD, the
// reduction K of WGRAD.  Its last group of 128 may be partial; it must be a multiple
// of 16, the 16-byte row stride of the token-major codes and TMA's coordinate rule.
bool tok_ok(int64_t d)
{
    return d > 0 && d <= FP8BW_MAX_DIM && (d % 16) == 0;
}

int from_cuda(cudaError_t e)
{
    return e == cudaSuccess ? FP8BW_OK : FP8BW_ECUDA;
}

} // namespace

extern "C" {

int fp8_quant_act(const void *x_bf16, int64_t M, int64_t K, uint8_t *q, float *s, void *stream)
{
    if (!x_bf16 || !q || !s)
        return FP8BW_EINVAL;
    if (!tok_ok(M) || !dim_ok(K))
        return FP8BW_ESHAPE;
    if (!aligned16(x_bf16) || !aligned16(q) || !aligned16(s))
        return FP8BW_EALIGN;
    int st;
    const int sms = device_sms({x_bf16, q, s}, &st);
    if (sms < 0)
        return st;
    return from_cuda(fp8bw::launch_quant_act(x_bf16, M, K, q, s,
                                             static_cast<cudaStream_t>(stream), sms));
}

int fp8_quant_act_t(const void *x_bf16, int64_t M, int64_t K, uint8_t *qt, float *st_,
                    void *stream)
{
    if (!x_bf16 || !qt || !st_)
        return FP8BW_EINVAL;
    if (!tok_ok(M) || !dim_ok(K))
        return FP8BW_ESHAPE;
    if (!aligned16(x_bf16) || !aligned16(qt) || !aligned16(st_))
        return FP8BW_EALIGN;
    int st;
    if (device_sms({x_bf16, qt, st_}, &st) < 0)
        return st;
    return from_cuda(
        fp8bw::launch_quant_act_t(x_bf16, M, K, qt, st_, static_cast<cudaStream_t>(stream)));
}

int fp8_quant_act_dual(const void *x_bf16, int64_t M, int64_t K, uint8_t *q, float *s,
                       uint8_t *qt, float *st_, void *stream)
{
    if (!x_bf16 || !q || !s || !qt || !st_)
        return FP8BW_EINVAL;
    if (!tok_ok(M) || !dim_ok(K))
        return FP8BW_ESHAPE;
    if (!aligned16(x_bf16) || !aligned16(q) || !aligned16(s) || !aligned16(qt) || !aligned16(st_))
        return FP8BW_EALIGN;
    int st;
    if (device_sms({x_bf16, q, s, qt, st_}, &st) < 0)
        return st;
    return from_cuda(fp8bw::launch_quant_dual(x_bf16, M, K, q, s, qt, st_,
                                              static_cast<cudaStream_t>(stream)));
}

int fp8_quant_weight(const void *w_bf16, int64_t N, int64_t K, uint8_t *q, float *s,
                     uint8_t *qt_or_null, void *stream)
{
    if (!w_bf16 || !q || !s)
        return FP8BW_EINVAL;
    if (!dim_ok(N) || !dim_ok(K))
        return FP8BW_ESHAPE;
    if (!aligned16(w_bf16) || !aligned16(q) || !aligned16(s) ||
        (qt_or_null && !aligned16(qt_or_null)))
        return FP8BW_EALIGN;
    int st;
    if (device_sms({w_bf16, q, s, qt_or_null}, &st) < 0)
        return st;
    return from_cuda(fp8bw::launch_quant_weight(w_bf16, N, K, q, s, qt_or_null,
                                                static_cast<cudaStream_t>(stream)));
}

// ---- power-of-two (E8M0) scale variants: same layouts, uint8 scale codes ----

static int quant_e8m0(int which, const void *x, int64_t M, int64_t K, uint8_t *q, uint8_t *s,
                      uint8_t *qt, uint8_t *st, void *stream)
{
    if (!dim_ok(M) || !dim_ok(K))
        return FP8BW_ESHAPE;
    if (!aligned16(x) || (q && !aligned16(q)) || (s && !aligned16(s)) ||
        (qt && !aligned16(qt)) || (st && !aligned16(st)))
        return FP8BW_EALIGN;
    int status;
    if (device_sms({x, q, s, qt, st}, &status) < 0)
        return status;
    return from_cuda(fp8bw::launch_quant_e8m0(which, x, M, K, q, s, qt, st,
                                              static_cast<cudaStream_t>(stream)));
}

int fp8_quant_act_e8m0(const void *x_bf16, int64_t M, int64_t K, uint8_t *q, uint8_t *s_e8m0,
                       void *stream)
{
    if (!x_bf16 || !q || !s_e8m0)
        return FP8BW_EINVAL;
    return quant_e8m0(0, x_bf16, M, K, q, s_e8m0, nullptr, nullptr, stream);
}

int fp8_quant_act_t_e8m0(const void *x_bf16, int64_t M, int64_t K, uint8_t *qt,
                         uint8_t *st_e8m0, void *stream)
{
    if (!x_bf16 || !qt || !st_e8m0)
        return FP8BW_EINVAL;
    return quant_e8m0(1, x_bf16, M, K, nullptr, nullptr, qt, st_e8m0, stream);
}

int fp8_quant_act_dual_e8m0(const void *x_bf16, int64_t M, int64_t K, uint8_t *q,
                            uint8_t *s_e8m0, uint8_t *qt, uint8_t *st_e8m0, void *stream)
{
    if (!x_bf16 || !q || !s_e8m0 || !qt || !st_e8m0)
        return FP8BW_EINVAL;
    return quant_e8m0(2, x_bf16, M, K, q, s_e8m0, qt, st_e8m0, stream);
}

int fp8_quant_weight_e8m0(const void *w_bf16, int64_t N, int64_t K, uint8_t *q,
                          uint8_t *s_e8m0, uint8_t *qt_or_null, void *stream)
{
    if (!w_bf16 || !q || !s_e8m0)
        return FP8BW_EINVAL;
    return quant_e8m0(3, w_bf16, N, K, q, s_e8m0, qt_or_null, nullptr, stream);
}

int fp8_gemm_blockwise_e8m0(int mode, const uint8_t *a, const uint8_t *sa_e8m0,
                            const uint8_t *b, const uint8_t *sb_e8m0, void *d_bf16, int64_t M,
                            int64_t N, int64_t K, void *stream)
{
    if (mode < FP8BW_FPROP || mode > FP8BW_WGRAD || !a || !sa_e8m0 || !b || !sb_e8m0 || !d_bf16)
        return FP8BW_EINVAL;
    if (!dim_ok(M) || !dim_ok(N) || !dim_ok(K))
        return FP8BW_ESHAPE;
    if (!aligned16(a) || !aligned16(sa_e8m0) || !aligned16(b) || !aligned16(sb_e8m0) ||
        !aligned16(d_bf16))
        return FP8BW_EALIGN;
    int st;
    const int sms = device_sms({a, sa_e8m0, b, sb_e8m0, d_bf16}, &st);
    if (sms < 0)
        return st;
    return from_cuda(fp8bw::launch_gemm_mx(mode, a, sa_e8m0, b, sb_e8m0, d_bf16, M, N, K,
                                           static_cast<cudaStream_t>(stream), sms));
}

int fp8_gemm_blockwise(int mode, const uint8_t *a, const float *sa, const uint8_t *b,
                       const float *sb, void *d_bf16, int64_t M, int64_t N, int64_t K,
                       void *stream)
{
    if (mode < FP8BW_FPROP || mode > FP8BW_WGRAD || !a || !sa || !b || !sb || !d_bf16)
        return FP8BW_EINVAL;
    // the token count is M for FPROP/DGRAD and the reduction K for WGRAD
    if (!dim_ok(N) || (mode == FP8BW_WGRAD ? !dim_ok(M) || !tok_ok(K) : !tok_ok(M) || !dim_ok(K)))
        return FP8BW_ESHAPE;
    if (!aligned16(a) || !aligned16(sa) || !aligned16(b) || !aligned16(sb) || !aligned16(d_bf16))
        return FP8BW_EALIGN;
    int st;
    const int sms = device_sms({a, sa, b, sb, d_bf16}, &st);
    if (sms < 0)
        return st;
    return from_cuda(fp8bw::launch_gemm(mode, a, sa, b, sb, d_bf16, M, N, K,
                                        static_cast<cudaStream_t>(stream), sms));
}

int fp8_gemm_wgrad_acc32(const uint8_t *a, const float *sa, const uint8_t *b, const float *sb,
                         float *dw32, int64_t M, int64_t N, int64_t K, void *stream)
{
    if (!a || !sa || !b || !sb || !dw32)
        return FP8BW_EINVAL;
    if (!dim_ok(M) || !dim_ok(N) || !tok_ok(K))  // K: tokens
        return FP8BW_ESHAPE;
    if (!aligned16(a) || !aligned16(sa) || !aligned16(b) || !aligned16(sb) || !aligned16(dw32))
        return FP8BW_EALIGN;
    int st;
    const int sms = device_sms({a, sa, b, sb, dw32}, &st);
    if (sms < 0)
        return st;
    return from_cuda(fp8bw::launch_gemm_wgrad_acc32(a, sa, b, sb, dw32, M, N, K,
                                                    static_cast<cudaStream_t>(stream), sms));
}

const char *fp8bw_status_string(int status)
{
    switch (status) {
    case FP8BW_OK: return "FP8BW_OK";
    case FP8BW_EINVAL: return "FP8BW_EINVAL: null pointer or invalid mode";
    case FP8BW_EALIGN: return "FP8BW_EALIGN: pointer not 16-byte aligned";
    case FP8BW_ESHAPE:
        return "FP8BW_ESHAPE: size not a positive multiple of 128 (16 for a token count), or too large";
    case FP8BW_ECUDA: return "FP8BW_ECUDA: CUDA runtime error";
    case FP8BW_ETIMEOUT: return "FP8BW_ETIMEOUT: a bounded in-kernel wait ran out";
    case FP8BW_EUNSUPPORTED: return "FP8BW_EUNSUPPORTED: device is not sm_100";
    default: return "unknown fp8bw status";
    }
}

int fp8bw_last_device_error(void *stream)
{
    int st;
    if (device_sms({}, &st) < 0)
        return st;
    int v = 0, w = 0, u = 0;
    if (fp8bw::read_and_clear_device_error(static_cast<cudaStream_t>(stream), &v) != cudaSuccess ||
        fp8bw::read_and_clear_mx_error(&w) != cudaSuccess ||
        fp8bw::read_and_clear_quant_error(&u) != cudaSuccess)
        return FP8BW_ECUDA;
    return (v || w || u) ? FP8BW_ETIMEOUT : FP8BW_OK;
}

int fp8bw_selftest_wait_timeout(int64_t limit_us, void *stream)
{
    if (limit_us < 1 || limit_us > 1000000)
        return FP8BW_EINVAL;
    int st;
    if (device_sms({}, &st) < 0)
        return st;
    return from_cuda(fp8bw::launch_selftest_wait(uint64_t(limit_us) * 1000u,
                                                 static_cast<cudaStream_t>(stream)));
}

const char *fp8bw_version(void)
{
    return "fp8bw 0.1 sm_100a";
}

} // extern "C"
