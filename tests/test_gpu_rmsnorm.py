"""RMSNorm front end (the guide's SparseBitLinear module normalises x before the
absmax) on the GPU against the CPU oracle: x_q and s_tok bit-exact, the
accumulators bit-exact and y within the fp32 / bf16 tolerances on every path."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_bf16_close, assert_fp32_close, layer_inputs, to_dev, x_dev
from sparse_linear_layers_b200 import synthetic

pytestmark = pytest.mark.gpu

EPS_TORCH = 2.0 ** -23


@pytest.fixture(scope="module")
def sbl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_linear_layers_b200 as m
    return m


def _g(K, seed=0):
    return np.random.default_rng(seed).uniform(0.5, 1.5, K).astype(np.float32)


@pytest.mark.parametrize("T,K", [(37, 256), (5, 896), (3, 4864), (2, 7168), (1, 16), (64, 2048), (9, 48)])
@pytest.mark.parametrize("eps", [EPS_TORCH, 1e-5, 0.0])
def test_rmsnorm_quant_bit_exact(sbl, T, K, eps):
    """Registers-only rows (K <= 2048), rows read again past four blocks per lane
    (K = 4864, 7168), a single block (K = 16) and a partial last block set."""
    _, xbits, xval = layer_inputs(8, K, T, seed=3, outlier_p=0.01)
    g = _g(K)
    xq_ref, s_ref = oracle.rmsnorm_quant_act(xval, g, eps)
    xq, s = sbl.sbl_rmsnorm_quant_act(x_dev(xbits), to_dev(g), eps)
    assert sbl.sbl_device_status() == 0
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def _bf16(v):
    return synthetic.bf16_bits_to_f32(synthetic.f32_to_bf16_bits(np.asarray(v, np.float32)))


def _exact_sum_tokens(K):
    """Tokens that reach every branch of the kernel's exact sum of squares:
    ordinary draws (one integer window), a value 2^-25 or 2^-60 below the rest
    (two windows / the limb columns), rows of tiny, subnormal or huge values,
    a double-rounding trap and a tie at float32 rounding boundaries."""
    rows = _bf16(synthetic.activations(12, K, seed=9)[1])
    rows[1, K // 2] = 2.0 ** -25
    rows[2, K // 3] = -(2.0 ** -60)
    rows[3] = _bf16(rows[3] * np.float32(2.0 ** -110))  # squares below float32: sum 0
    rows[4] = 0.0
    rows[4, :3] = [4096.0, 1.0, 2.0 ** -30]          # 2^24 + 1 + 2^-60 -> 16777218
    rows[5] = 0.0
    rows[5, 0], rows[5, 1:16] = 4096.0, 1.0           # 16777231, a tie -> 16777232
    rows[6] = _bf16(rows[6] * np.float32(2.0 ** -66))  # float32-subnormal sum
    rows[6, ::5] = 3 * 2.0 ** -133                    # bf16 subnormals
    rows[7, 0] = 1.5 * 2.0 ** 63                      # sum just below 2^127 * 1.2
    rows[8, K - 1] = 2.0 ** -20
    rows[9] = _bf16(rows[9] * np.float32(2.0 ** 50))
    rows[10] = 3.0
    rows[10, 1::2] = -3.0
    rows[11] = 0.0
    rows[11, K - 5] = -0.75
    bits = synthetic.f32_to_bf16_bits(rows)
    assert np.array_equal(synthetic.bf16_bits_to_f32(bits), rows)
    return bits, rows


@pytest.mark.parametrize("K", [16, 64, 512, 896, 2048, 4864, 7168, 16384])
def test_rmsnorm_exact_sum_branches(sbl, K):
    """x_q and s_tok bit-exact on tokens built to take each way the kernel forms
    the exact sum of squares, at row lengths held in registers (K <= 8192)
    and read again (K = 16384)."""
    bits, rows = _exact_sum_tokens(K)
    g = _g(K, seed=2)
    xq_ref, s_ref = oracle.rmsnorm_quant_act(rows, g, EPS_TORCH)
    xq, s = sbl.sbl_rmsnorm_quant_act(x_dev(bits), to_dev(g), EPS_TORCH)
    assert sbl.sbl_device_status() == 0
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(xq.cpu().numpy(), xq_ref)


def test_rmsnorm_overflowing_sum(sbl):
    """A sum of squares past the float32 range is +inf: every normalised value
    is 0 (as in the oracle) and the token is flagged."""
    K = 64
    rows = np.zeros((2, K), np.float32)
    rows[:, 0] = rows[:, 1] = 1.5 * 2.0 ** 63
    rows[1, 1] = 1.0
    bits = synthetic.f32_to_bf16_bits(rows)
    g = np.ones(K, np.float32)
    xq_ref, s_ref = oracle.rmsnorm_quant_act(rows, g, 0.0)
    xq, s = sbl.sbl_rmsnorm_quant_act(x_dev(bits), to_dev(g), 0.0)
    assert sbl.sbl_device_status() == 3
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(xq.cpu().numpy(), xq_ref)


def test_rmsnorm_constant_rows(sbl):
    """Constant rows normalise to +-1, so every code is +-127 and s = 127."""
    K = 64
    x = np.full((2, K), 3.0, np.float32)
    x[1, 1::2] = -3.0
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    xq, s = sbl.sbl_rmsnorm_quant_act(x_dev(bits), to_dev(np.ones(K, np.float32)), 0.0)
    assert xq.cpu().numpy()[0].tolist() == [127] * K
    assert xq.cpu().numpy()[1].tolist() == [127, -127] * (K // 2)
    assert np.all(s.cpu().numpy() == np.float32(127.0))


CASES = [
    # (O, K, T, n, m, path)
    (512, 256, 1, 2, 4, "decode"),
    (200, 448, 3, 3, 4, "decode"),
    (7168, 2048, 16, 2, 4, "decode"),
    (896, 896, 130, 3, 4, "prefill_1cta"),
    (896, 896, 300, 6, 8, "prefill_pair"),
    (384, 1024, 200, 2, 4, "prefill_sparse"),
    (512, 4096, 40, 2, 4, "auto"),        # one-CTA prefill split along k
    (4864, 896, 2048, 3, 4, "auto"),
]


@pytest.mark.parametrize("O,K,T,n,m,path", CASES)
def test_linear_rmsnorm_parity(sbl, O, K, T, n, m, path):
    W, xbits, xval = layer_inputs(O, K, T, seed=4, outlier_p=0.01)
    g = _g(K, seed=1)
    _, scale, _, Wt = oracle.prepare_weights(W, n, m)
    y_ref, acc_ref, _, _ = oracle.linear(xval, Wt, scale, g=g, eps=EPS_TORCH)
    w = sbl.sbl_prepare_weights(to_dev(W), n, m)
    gd = to_dev(g)
    acc = torch.empty((T, O), dtype=torch.int32, device="cuda")
    y = sbl.sbl_linear_rmsnorm(x_dev(xbits), w, gd, EPS_TORCH, acc_out=acc, path=path)
    assert sbl.sbl_device_status() == 0
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_fp32_close(y.cpu().numpy(), y_ref)
    yb = sbl.sbl_linear_rmsnorm(x_dev(xbits), w, gd, EPS_TORCH, out_dtype=torch.bfloat16, path=path)
    assert_bf16_close(yb.cpu().view(torch.int16).numpy(), y_ref)


def test_linear_rmsnorm_decode_needs_k_multiple_of_64(sbl):
    W, xbits, _ = layer_inputs(64, 48, 2, seed=5)
    w = sbl.sbl_prepare_weights(to_dev(W), 2, 4)
    with pytest.raises(sbl.SblError):
        sbl.sbl_linear_rmsnorm(x_dev(xbits), w, to_dev(np.ones(48, np.float32)))


def test_rmsnorm_nonfinite_sets_status(sbl):
    K = 64
    _, xbits, _ = layer_inputs(8, K, 3, seed=6)
    xbits = xbits.copy()
    xbits[1, 5] = 0x7F80  # +inf
    sbl.sbl_rmsnorm_quant_act(x_dev(xbits), to_dev(np.ones(K, np.float32)))
    assert sbl.sbl_device_status() == 3
    zeros = np.zeros((2, K), np.uint16)  # an all-zero token with eps = 0 divides by zero
    sbl.sbl_rmsnorm_quant_act(x_dev(zeros), to_dev(np.ones(K, np.float32)), 0.0)
    assert sbl.sbl_device_status() == 3
    xq, s = sbl.sbl_rmsnorm_quant_act(x_dev(zeros), to_dev(np.ones(K, np.float32)), 1e-6)
    assert sbl.sbl_device_status() == 0
    assert not xq.cpu().numpy().any()
