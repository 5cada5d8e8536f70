// quant.cuh -- launchers of the quantizer kernels (internal to libfp8bw).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fp8bw {

cudaError_t launch_quant_act(const void *x, int64_t M, int64_t K, uint8_t *q, float *s,
                             cudaStream_t stream, int num_sms);
cudaError_t launch_quant_act_t(const void *x, int64_t M, int64_t K, uint8_t *qt, float *st,
                               cudaStream_t stream);
cudaError_t launch_quant_dual(const void *x, int64_t M, int64_t K, uint8_t *q, float *s,
                              uint8_t *qt, float *st, cudaStream_t stream);
// Power-of-two (E8M0) scale quantizers (which: 0 rows, 1 token groups, 2 both,
// 3 weight blocks with rows = M); scales are uint8 E8M0 codes in the FP32 layouts.
cudaError_t launch_quant_e8m0(int which, const void *x, int64_t M, int64_t K, uint8_t *q,
                              uint8_t *s, uint8_t *qt, uint8_t *st, cudaStream_t stream);

// Error word of the quantizers' bounded waits (read and cleared; caller synchronizes).
cudaError_t read_and_clear_quant_error(int *value);

cudaError_t launch_quant_weight(const void *w, int64_t N, int64_t K, uint8_t *q, float *s,
                                uint8_t *qt, cudaStream_t stream);

// GEMM: D[M][N] bf16 from FP8 operands with blockwise scales (mode 0/1/2 =
// fprop/dgrad/wgrad).  Arguments already validated.
cudaError_t launch_gemm(int mode, const uint8_t *a, const float *sa, const uint8_t *b,
                        const float *sb, void *d, int64_t M, int64_t N, int64_t K,
                        cudaStream_t stream, int num_sms);

// wgrad with FP32 main-grad accumulation: d32[M][N] += sum (no BF16 rounding).
cudaError_t launch_gemm_wgrad_acc32(const uint8_t *a, const float *sa, const uint8_t *b,
                                    const float *sb, float *d32, int64_t M, int64_t N, int64_t K,
                                    cudaStream_t stream, int num_sms);

// GEMM with power-of-two (E8M0) scale codes (uint8, the layouts of the FP32 scales),
// promoted inside the block-scaled MMA.  Arguments already validated.
cudaError_t launch_gemm_mx(int mode, const uint8_t *a, const uint8_t *sa, const uint8_t *b,
                           const uint8_t *sb, void *d, int64_t M, int64_t N, int64_t K,
                           cudaStream_t stream, int num_sms);

// Error word of the E8M0 GEMM's bounded waits (read and cleared; caller synchronizes).
cudaError_t read_and_clear_mx_error(int *value);

// Bounded-wait self-test (records a timeout in the error word, no fault).
cudaError_t launch_selftest_wait(uint64_t limit_ns, cudaStream_t stream);

// Per-device error word written by bounded in-kernel waits.
cudaError_t read_and_clear_device_error(cudaStream_t stream, int *value);

} // namespace fp8bw
