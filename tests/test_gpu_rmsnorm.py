"""RMSNorm front end (the guide's SparseBitLinear module normalises x before the
absmax) on the GPU against the CPU oracle: x_q and s_tok bit-exact, the
accumulators bit-exact and y within the fp32 / bf16 tolerances on every path."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_bf16_close, assert_fp32_close, layer_inputs, to_dev, x_dev

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
