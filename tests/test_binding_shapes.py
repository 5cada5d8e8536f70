"""The Python binding checks every tensor's shape against the sizes it hands to the C
ABI, and raises before any launch.  A mismatch that reached the library would make a
kernel (or a TMA map built from M, N, K) read or write past an allocation, so these
checks run on the CPU, with CPU tensors: shapes are checked before anything else."""
import pytest
import torch

import blockwise_fp8_linear_b200 as fb

bf16, u8, f32 = torch.bfloat16, torch.uint8, torch.float32


def z(*shape, dtype=u8):
    return torch.zeros(*shape, dtype=dtype)


X = z(256, 384, dtype=bf16)  # M=256 tokens, K=384


@pytest.mark.parametrize("call", [
    lambda: fb.fp8_quant_act(X, q=z(256, 256)),
    lambda: fb.fp8_quant_act(X, s=z(2, 256, dtype=f32)),
    lambda: fb.fp8_quant_act_t(X, qt=z(256, 384)),
    lambda: fb.fp8_quant_act_t(X, st=z(3, 384, dtype=f32)),
    lambda: fb.fp8_quant_act_dual(X, st=z(2, 256, dtype=f32)),
    lambda: fb.fp8_quant_act_dual(X, qt=z(384, 128)),
    lambda: fb.fp8_quant_weight(X, q=z(384, 256)),
    lambda: fb.fp8_quant_weight(X, s=z(3, 2, dtype=f32)),
    lambda: fb.fp8_quant_weight(X, want_t=True, qt=z(256, 384)),
    lambda: fb.fp8_quant_act_e8m0(X, s=z(2, 3 * 128)),
    lambda: fb.fp8_quant_act_t_e8m0(X, st=z(2, 3 * 512)),
    lambda: fb.fp8_quant_act_dual_e8m0(X, q=z(128, 384)),
    lambda: fb.fp8_quant_weight_e8m0(X, s=z(3, 2 * 512)),
    lambda: fb.fp8_quant_act(z(200, 384, dtype=bf16)),   # not a multiple of 128
    lambda: fb.fp8_quant_act(z(256, dtype=bf16)),        # not 2-D
], ids=lambda c: "")
def test_quantizers_reject_mismatched_shapes(call):
    with pytest.raises(ValueError):
        call()


M, N, K = 256, 384, 512


def gemm_args(mode, e8m0=False):
    a, sa, b, sb = fb._gemm_shapes(mode, M, N, K, e8m0)
    sdt = u8 if e8m0 else f32
    return z(*a), z(*sa, dtype=sdt), z(*b), z(*sb, dtype=sdt)


def test_gemm_operand_shapes_follow_the_header():
    # include/fp8bw.h: FPROP b = Qw[N][K], sb = [N/128][K/128]; DGRAD b = Qw[K][N],
    # sb = [K/128][N/128]; WGRAD b = Qx^T[N][K], sb = [K/128][N]; sa = [K/128][M]
    assert fb._gemm_shapes(fb.FPROP, M, N, K) == ((M, K), (K // 128, M), (N, K), (N // 128, K // 128))
    assert fb._gemm_shapes(fb.DGRAD, M, N, K) == ((M, K), (K // 128, M), (K, N), (K // 128, N // 128))
    assert fb._gemm_shapes(fb.WGRAD, M, N, K) == ((M, K), (K // 128, M), (N, K), (K // 128, N))
    assert fb._gemm_shapes(fb.FPROP, M, N, K, True)[1] == (M // 128, (K // 128) * 512)
    assert fb._gemm_shapes(fb.DGRAD, M, N, K, True)[3] == (K // 128, (N // 128) * 512)


@pytest.mark.parametrize("mode", [fb.FPROP, fb.DGRAD, fb.WGRAD])
@pytest.mark.parametrize("e8m0", [False, True])
@pytest.mark.parametrize("which", range(5))
def test_gemm_rejects_each_mismatched_operand(mode, e8m0, which):
    args = list(gemm_args(mode, e8m0))
    fn = fb.fp8_gemm_blockwise_e8m0 if e8m0 else fb.fp8_gemm_blockwise
    out = None
    if which < 4:
        t = args[which]
        args[which] = torch.zeros(t.shape[0], t.shape[1] + 128, dtype=t.dtype)  # one size off
    else:
        out = z(M, N + 128, dtype=bf16)
    with pytest.raises(ValueError):
        fn(mode, *args, M, N, K, out=out)
    # the correct shapes pass the shape checks and stop at the device check
    with pytest.raises(TypeError):
        fn(mode, *gemm_args(mode, e8m0), M, N, K)


@pytest.mark.parametrize("mnk", [(M + 128, N, K), (M, N - 128, K), (M, N, K + 128), (M, N, 200)])
def test_gemm_rejects_sizes_that_disagree_with_tensors(mnk):
    a, sa, b, sb = gemm_args(fb.FPROP)
    with pytest.raises(ValueError):
        fb.fp8_gemm_blockwise(fb.FPROP, a, sa, b, sb, *mnk)


def test_wgrad_acc32_checks_the_fp32_buffer():
    a, sa, b, sb = gemm_args(fb.WGRAD)
    with pytest.raises(ValueError):
        fb.fp8_gemm_wgrad_acc32(a, sa, b, sb, M, N, K, z(M, N + 128, dtype=f32))
    with pytest.raises(TypeError):
        fb.fp8_gemm_wgrad_acc32(a, sa, b, sb, M, N, K, z(M, N, dtype=bf16))
    with pytest.raises(TypeError):
        fb.fp8_gemm_wgrad_acc32(a, sa, b, sb, M, N, K, None)


def test_bad_mode_is_rejected():
    with pytest.raises(ValueError):
        fb.fp8_gemm_blockwise(3, *gemm_args(fb.FPROP), M, N, K)


# ---- token counts that are not a multiple of 128 ----

def test_ragged_token_shapes():
    """A token count only needs to be a multiple of 16; token-wise scale arrays then
    have ceil(tokens/128) rows, and the feature dimensions stay multiples of 128."""
    T = 144
    assert fb._gemm_shapes(fb.FPROP, T, N, K) == ((T, K), (K // 128, T), (N, K), (N // 128, K // 128))
    assert fb._gemm_shapes(fb.WGRAD, M, N, T) == ((M, T), (2, M), (N, T), (2, N))
    with pytest.raises(ValueError):
        fb._gemm_shapes(fb.FPROP, 136, N, K)          # not a multiple of 16
    with pytest.raises(ValueError):
        fb._gemm_shapes(fb.FPROP, T, N, 144)          # FPROP reduction = features
    with pytest.raises(ValueError):
        fb._gemm_shapes(fb.WGRAD, 144, N, T)          # WGRAD M = features
    with pytest.raises(ValueError):
        fb._gemm_shapes(fb.FPROP, T, N, K, True)      # E8M0 keeps whole groups
    xr = z(T, 384, dtype=bf16)
    with pytest.raises(ValueError):   # st must have ceil(144/128) = 2 rows
        fb.fp8_quant_act_t(xr, st=z(1, 384, dtype=f32))
    with pytest.raises(ValueError):
        fb.fp8_quant_act_dual(xr, st=z(1, 384, dtype=f32))
    with pytest.raises(TypeError):    # the right shapes pass and stop at the device check
        fb.fp8_quant_act_t(xr, qt=z(384, T), st=z(2, 384, dtype=f32))
    with pytest.raises(ValueError):   # weights stay whole blocks
        fb.fp8_quant_weight(xr)
