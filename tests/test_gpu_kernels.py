"""Kernel-level parity on the GPU, through the C ABI: the tcgen05 linear layer
and its epilogues, LayerNorm and window attention against the oracle's
definitions on the same bf16 inputs; the bounded-wait timeout status."""
import numpy as np
import pytest

import aut_synth as S
import oracle as O
from gpu_util import assert_f16_output_close, assert_bf16_output_close, assert_rows_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from audio_encoder_aut_b200 import _lib as A  # noqa: E402


def _dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda").to(dtype)


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _rand(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return S.round_bf16(rng.standard_normal(shape).astype(np.float32) * scale)


SHAPES = [(1, 64, 64), (31, 192, 64), (128, 256, 256), (300, 1280, 1280), (1000, 3840, 1280),
          (257, 2688, 896), (390, 3584, 896), (77, 16, 64), (129, 240, 7680), (4000, 5120, 1280),
          (3000, 1280, 5120), (513, 2048, 1280), (45, 1024, 896),
          # K = 64: one k-block per tile, so a CTA drains one tile while it
          # preloads the residual of its next - the two must not overlap columns
          (8192, 1280, 64), (2000, 512, 64)]


@pytest.mark.parametrize("flags", [0, A.LINEAR_SINGLE_CTA], ids=["auto", "single_cta"])
@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("epi", [A.EPI_BF16, A.EPI_BF16_GELU, A.EPI_RESID_F32])
def test_linear_matches_definition(M, N, K, epi, flags):
    x = _rand((M, K), 1)
    w = _rand((N, K), 2, 0.05)
    b = _rand((N,), 3, 0.1)
    ref = x.astype(np.float64) @ w.astype(np.float64).T + b
    xd, wd, bd = _dev(x, torch.bfloat16), _dev(w, torch.bfloat16), _dev(b, torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    if epi == A.EPI_RESID_F32:
        y0 = np.random.default_rng(4).standard_normal((M, N)).astype(np.float32)
        yd = _dev(y0, torch.float32)
        ref = ref + y0
    else:
        yd = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        if epi == A.EPI_BF16_GELU:
            ref = O.gelu(ref)
    st = A.aut_linear(xd.data_ptr(), wd.data_ptr(), bd.data_ptr(), yd.data_ptr(), M, N, K, epi,
                      status.data_ptr(), 0, flags, _stream())
    assert st == A.AUT_OK
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = yd.float().cpu().numpy()
    if epi == A.EPI_RESID_F32:
        # fp32 output: only accumulation-order error
        np.testing.assert_allclose(got, ref, rtol=0, atol=2e-3 * np.sqrt(K / 64))
    else:
        assert_bf16_output_close(got, ref, f"linear {M}x{N}x{K} epi {epi}")
        assert_rows_close(got, ref, f"linear {M}x{N}x{K} epi {epi}", rel_max=3e-2)


@pytest.mark.parametrize("M,N,K", [(300, 1280, 1280), (31, 2048, 1280), (4000, 1024, 896)])
def test_linear_fp32_output(M, N, K):
    x = _rand((M, K), 1)
    w = _rand((N, K), 2, 0.05)
    b = _rand((N,), 3, 0.1)
    ref = x.astype(np.float64) @ w.astype(np.float64).T + b
    xd, wd, bd = _dev(x, torch.bfloat16), _dev(w, torch.bfloat16), _dev(b, torch.bfloat16)
    yd = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    st = A.aut_linear(xd.data_ptr(), wd.data_ptr(), bd.data_ptr(), yd.data_ptr(), M, N, K,
                      A.EPI_F32, None, 0, 0, _stream())
    assert st == A.AUT_OK
    torch.cuda.synchronize()
    np.testing.assert_allclose(yd.cpu().numpy(), ref, rtol=0, atol=2e-3 * np.sqrt(K / 64))


@pytest.mark.parametrize("flags", [A.LINEAR_F16, A.LINEAR_F16 | A.LINEAR_SINGLE_CTA],
                         ids=["auto", "single_cta"])
@pytest.mark.parametrize("M,N,K", [(3253, 1280, 1280), (300, 896, 896), (77, 256, 128)])
def test_linear_fp16_operands(M, N, K, flags):
    """The o_proj form: fp16 x and w (values with 11 significant bits, which a
    bf16 reading of the same bytes would get badly wrong), fp32 residual add."""
    rng = np.random.default_rng(7)
    x = rng.standard_normal((M, K)).astype(np.float16)
    w = (rng.standard_normal((N, K)) * 0.05).astype(np.float16)
    b = _rand((N,), 3, 0.1)
    y0 = rng.standard_normal((M, N)).astype(np.float32)
    ref = x.astype(np.float64) @ w.astype(np.float64).T + b + y0
    xd, wd, bd = _dev(x, torch.float16), _dev(w, torch.float16), _dev(b, torch.bfloat16)
    yd = _dev(y0, torch.float32)
    st = A.aut_linear(xd.data_ptr(), wd.data_ptr(), bd.data_ptr(), yd.data_ptr(), M, N, K,
                      A.EPI_RESID_F32, None, 0, flags, _stream())
    assert st == A.AUT_OK
    torch.cuda.synchronize()
    np.testing.assert_allclose(yd.cpu().numpy(), ref, rtol=0, atol=2e-3 * np.sqrt(K / 64))


@pytest.mark.parametrize("M,N,K,flags", [(128, 256, 256, 0), (512, 256, 256, 0),
                                         (512, 256, 256, A.LINEAR_SINGLE_CTA), (300, 240, 128, 0)])
def test_linear_no_bias_and_structured_inputs(M, N, K, flags):
    """Identity-like A picks out rows of W: checks operand layout and K order exactly."""
    x = np.zeros((M, K), np.float32)
    for i in range(M):
        x[i, (3 * i) % K] = 1.0
    w = _rand((N, K), 5)
    xd, wd = _dev(x, torch.bfloat16), _dev(w, torch.bfloat16)
    yd = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    st = A.aut_linear(xd.data_ptr(), wd.data_ptr(), None, yd.data_ptr(), M, N, K, A.EPI_BF16,
                      None, 0, flags, _stream())
    assert st == A.AUT_OK
    torch.cuda.synchronize()
    ref = np.stack([w[:, (3 * i) % K] for i in range(M)])
    np.testing.assert_array_equal(yd.float().cpu().numpy(), ref)


@pytest.mark.parametrize("T,d", [(1, 64), (31, 64), (390, 896), (3200, 1280), (17, 2048)])
def test_layernorm_matches_oracle(T, d):
    rng = np.random.default_rng(T)
    x = (rng.standard_normal((T, d)) * 2 + 0.5).astype(np.float32)
    g = S.round_bf16(1 + 0.1 * rng.standard_normal(d).astype(np.float32))
    b = S.round_bf16(0.1 * rng.standard_normal(d).astype(np.float32))
    y = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    xd, gd, bd = _dev(x, torch.float32), _dev(g, torch.bfloat16), _dev(b, torch.bfloat16)
    st = A.aut_layernorm(xd.data_ptr(), gd.data_ptr(), bd.data_ptr(), y.data_ptr(), T, d, 1e-5,
                         _stream())
    assert st == A.AUT_OK
    torch.cuda.synchronize()
    ref = O.layer_norm(x.astype(np.float64), g, b, 1e-5)
    assert_bf16_output_close(y.float().cpu().numpy(), ref, "layernorm")


ATTN_CASES = [
    (4, 16, [26, 5]),
    (20, 64, [104, 104, 1, 17, 128, 50, 104, 3]),
    (14, 64, [104, 104, 104, 78]),
    (2, 32, [7, 64, 33]),
    (2, 128, [100, 1, 128]),
    # empty windows between full ones
    (20, 64, [0, 104, 0, 5, 128, 0]),
    # 64 windows x 16 heads = 1024 tiles: every CTA of the persistent kernel
    # walks several tiles and reuses its pipeline stages
    (16, 64, [int(n) for n in np.random.default_rng(5).integers(1, 129, 64)]),
]


@pytest.mark.parametrize("heads,hd,lens", ATTN_CASES)
def test_window_attention_matches_oracle(heads, hd, lens):
    d = heads * hd
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    T = cu[-1]
    qkv = _rand((T, 3 * d), 11, 1.0)
    out = torch.empty((T, d), dtype=torch.float16, device="cuda")
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    qd = _dev(qkv, torch.bfloat16)
    st = A.aut_window_attention(qd.data_ptr(), out.data_ptr(), T, d, heads, cu, ws.data_ptr(),
                                ws.numel(), _stream())
    assert st == A.AUT_OK
    torch.cuda.synchronize()
    ref = O.window_attention(qkv.astype(np.float64), cu, heads)
    o = out.float().cpu().numpy().astype(np.float64)
    # fp16 rounding of O (2^-11 |o|) on top of a near-exact O: P enters as fp16
    # (head_dim 64: relative rounding 2^-11 per element, averaging out over the
    # window's keys) or as two bf16 terms (~2^-16), with fp32 accumulation.
    vmax = np.abs(qkv[:, 2 * d:]).max()
    assert_f16_output_close(o, ref, "window attention", atol=2e-4 * vmax)


@pytest.mark.parametrize("mode", [0, A.LINEAR_SINGLE_CTA], ids=["cta_pair", "single_cta"])
def test_pipeline_wait_timeout_returns_status_and_gpu_stays_usable(mode):
    """A GEMM whose first block never receives its first operand tile: the
    consumer's bounded wait runs out, the kernel records AUT_ERR_TIMEOUT and
    returns; the next launch on the same context works.  In CTA-pair mode the
    skipped stage is the even CTA's, so the odd CTA's wait for that stage to be
    armed runs out as well, and the pair still leaves through its cluster
    barrier."""
    M, N, K = 256, 128, 128
    x = _dev(_rand((M, K), 1), torch.bfloat16)
    w = _dev(_rand((N, K), 2, 0.05), torch.bfloat16)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = A.aut_linear(x.data_ptr(), w.data_ptr(), None, y.data_ptr(), M, N, K, A.EPI_BF16,
                      status.data_ptr(), 200, A.LINEAR_FAULT_INJECT | mode, _stream())
    assert st == A.AUT_OK
    torch.cuda.synchronize()
    assert A.aut_check_status_word(status.data_ptr()) == A.AUT_ERR_TIMEOUT
    assert int(status.item()) == 0  # cleared by the check
    st = A.aut_linear(x.data_ptr(), w.data_ptr(), None, y.data_ptr(), M, N, K, A.EPI_BF16,
                      status.data_ptr(), 0, mode, _stream())
    torch.cuda.synchronize()
    assert st == A.AUT_OK and A.aut_check_status_word(status.data_ptr()) == A.AUT_OK
    ref = x.float().cpu().numpy().astype(np.float64) @ w.float().cpu().numpy().astype(np.float64).T
    assert_rows_close(y.float().cpu().numpy(), ref, "linear after timeout")


def test_attention_wait_timeout_returns_status_and_gpu_stays_usable():
    """The tensor-core attention with its first block's first operand stage
    never filled: the MMA's bounded wait runs out, the softmax groups and the
    producer leave on the abort flag, the kernel writes AUT_ERR_TIMEOUT to the
    workspace's status word and returns; the next launch on the same context
    computes the right result."""
    heads, hd, lens = 20, 64, [104, 104, 50, 77]
    d = heads * hd
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    T = cu[-1]
    qkv = _rand((T, 3 * d), 13, 1.0)
    qd = _dev(qkv, torch.bfloat16)
    out = torch.empty((T, d), dtype=torch.float16, device="cuda")
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    st = A.aut_window_attention_ex(qd.data_ptr(), out.data_ptr(), T, d, heads, cu, ws.data_ptr(),
                                   ws.numel(), 200, A.ATTN_FAULT_INJECT, _stream())
    assert st == A.AUT_OK
    torch.cuda.synchronize()
    assert A.aut_check(ws.data_ptr()) == A.AUT_ERR_TIMEOUT
    st = A.aut_window_attention_ex(qd.data_ptr(), out.data_ptr(), T, d, heads, cu, ws.data_ptr(),
                                   ws.numel(), 0, 0, _stream())
    torch.cuda.synchronize()
    assert st == A.AUT_OK and A.aut_check(ws.data_ptr()) == A.AUT_OK
    ref = O.window_attention(qkv.astype(np.float64), cu, heads)
    vmax = np.abs(qkv[:, 2 * d:]).max()
    assert_f16_output_close(out.float().cpu().numpy().astype(np.float64), ref,
                            "attention after timeout", atol=2e-4 * vmax)
