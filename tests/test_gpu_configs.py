"""Parity on the full-size workloads: the N:M x token-count sweep on the
2048->7168 and 7168->2048 layers (seeds 0-2) and the hidden-2048 / FFN-7168
stack at T = 4096.  Weights (packed codes, mask bits, row scales) are compared
bit for bit; accumulators are compared in full up to T = 512 and on sampled
(t, o) entries, each computed by the oracle as its own dot product, above.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_fp32_close, layer_inputs, to_dev, x_dev

pytestmark = pytest.mark.gpu

SWEEP_LAYERS = [(2048, 7168), (7168, 2048)]
PATTERNS = [(2, 4), (3, 4), (6, 8)]
TOKENS = [1, 8, 64, 512, 4096]
FULL_LIMIT = 512
SAMPLES = 3000


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
    acc = torch.empty((T, O), dtype=torch.int32, device="cuda")
    y = sbl.sbl_linear(x_dev(xbits), w, acc_out=acc)
    assert sbl.sbl_device_status() == 0
    acc_h = acc.cpu().numpy()
    y_h = y.cpu().numpy()
    if T <= FULL_LIMIT:
        ref = oracle.int_contract(xq, Wt)
        assert np.array_equal(acc_h, ref)
        assert_fp32_close(y_h, oracle.dequant(ref, scale, s))
    else:
        rng = np.random.default_rng(seed)
        ti = rng.integers(0, T, SAMPLES)
        oi = rng.integers(0, O, SAMPLES)
        ti[:4] = [0, 0, T - 1, T - 1]
        oi[:4] = [0, O - 1, 0, O - 1]
        ref = oracle.acc_entries(xq, Wt, ti, oi)
        assert np.array_equal(acc_h[ti, oi].astype(np.int64), ref)
        assert_fp32_close(y_h[ti, oi], ref * scale.astype(np.float64)[oi] / s.astype(np.float64)[ti])


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
