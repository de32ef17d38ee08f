"""Parity on the full-size workloads: the N:M x token-count sweep on the
2048->7168 and 7168->2048 layers (seeds 0-2) and the hidden-2048 / FFN-7168
stack at T = 4096.  Weights (packed codes, mask bits, row scales) are compared
bit for bit; every accumulator bit for bit, every fp32 output within 1e-5
relative and, from T = 512 on, every bf16 output within 2 ulps.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_layer_outputs, layer_inputs, to_dev, x_dev

pytestmark = pytest.mark.gpu

SWEEP_LAYERS = [(2048, 7168), (7168, 2048)]
PATTERNS = [(2, 4), (3, 4), (6, 8)]
TOKENS = [1, 8, 64, 512, 4096]
BF16_FROM = 512


@pytest.fixture(scope="module")
def sbl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_linear_layers_b200 as m
    return m


_prep_cache = {}


def _prepared(sbl, K, O, n, m, seed):
    key = (K, O, n, m, seed)
    if key not in _prep_cache:
        _prep_cache.clear()  # one layer at a time keeps host memory small
        W, _, _ = layer_inputs(O, K, 1, seed=seed, tag="sweep")
        packed, scale, mbits, Wt = oracle.prepare_weights(W, n, m)
        w = sbl.sbl_prepare_weights(to_dev(W), n, m, with_mask=True)
        torch.cuda.synchronize()
        assert np.array_equal(w.packed.cpu().numpy(), packed)
        assert np.array_equal(w.row_scale.cpu().numpy().view(np.uint32), scale.view(np.uint32))
        assert np.array_equal(w.mask_bits.cpu().numpy(), mbits)
        _prep_cache[key] = (w, scale, Wt)
    return _prep_cache[key]


def _check(sbl, w, scale, Wt, T, K, O, seed, outlier_p=0.0, tag="sweep"):
    _, xbits, xval = layer_inputs(O, K, T, seed=seed, tag=tag, outlier_p=outlier_p)
    xq, s = oracle.quant_act(xval)
    x = x_dev(xbits)
    acc = torch.empty((T, O), dtype=torch.int32, device="cuda")
    y = sbl.sbl_linear(x, w, acc_out=acc)
    yb = sbl.sbl_linear(x, w, out_dtype=torch.bfloat16) if T >= BF16_FROM else None
    assert sbl.sbl_device_status() == 0
    assert_layer_outputs(acc.cpu().numpy(), y.cpu().numpy(), None if yb is None else yb.cpu().view(torch.int16).numpy(),
                         xq, s, Wt, scale, what=f"{K}->{O} T={T}")


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("n,m", PATTERNS)
@pytest.mark.parametrize("K,O", SWEEP_LAYERS)
def test_sweep(sbl, K, O, n, m, seed):
    w, scale, Wt = _prepared(sbl, K, O, n, m, seed)
    for T in TOKENS:
        _check(sbl, w, scale, Wt, T, K, O, seed)


def test_h2048_stack_t4096(sbl):
    from sparse_linear_layers_b200.synthetic import H2048_STACK
    for name, K, O in H2048_STACK:
        w, scale, Wt = _prepared(sbl, K, O, 2, 4, 0)
        _check(sbl, w, scale, Wt, 4096, K, O, 0, tag=f"h2048-{name}")
