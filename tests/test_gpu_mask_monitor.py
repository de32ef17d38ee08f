"""Mask change rate and mask verification on the GPU against the CPU oracle:
totals and per-row counts exact, on masks made by the weight preparation and
on arbitrary bitmaps, for every row-pitch width the kernel takes."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import layer_inputs, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sbl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_linear_layers_b200 as m
    return m


# K = 1024 (16-byte words), 96 (4-byte words), 48 (2-byte words); ragged row counts
@pytest.mark.parametrize("O,K", [(333, 1024), (70, 96), (9, 48), (4864, 896), (1, 16)])
@pytest.mark.parametrize("n,m", [(2, 4), (3, 4), (6, 8), (4, 8)])
def test_mask_monitor_random_bitmaps(sbl, O, K, n, m):
    rng = np.random.default_rng(O * 7 + K + n)
    a = rng.integers(0, 256, (O, K // 8), dtype=np.uint8)
    b = rng.integers(0, 256, (O, K // 8), dtype=np.uint8)
    ch, bad, rows = oracle.mask_monitor(a, b, K, n, m)
    totals, r = sbl.sbl_mask_monitor(to_dev(a), to_dev(b), K, n, m, per_row=True)
    assert totals.cpu().tolist() == [ch, bad]
    assert np.array_equal(r.cpu().numpy().astype(np.int64), rows)


@pytest.mark.parametrize("n,m", [(2, 4), (3, 4), (6, 8)])
def test_mask_monitor_between_two_preparations(sbl, n, m):
    """Masks of the latent weights before and after a small update: the change
    count matches the oracle and both masks verify (every group keeps N)."""
    O, K = 512, 896
    W, _, _ = layer_inputs(O, K, 1, seed=8)
    W2 = W + np.random.default_rng(3).normal(0, 0.004, W.shape).astype(np.float32)
    w1 = sbl.sbl_prepare_weights(to_dev(W), n, m, with_mask=True)
    w2 = sbl.sbl_prepare_weights(to_dev(W2), n, m, with_mask=True)
    m1, m2 = w1.mask_bits.cpu().numpy(), w2.mask_bits.cpu().numpy()
    ch, bad, rows = oracle.mask_monitor(m1, m2, K, n, m)
    assert bad == 0 and ch > 0
    totals, r = sbl.sbl_mask_monitor(w1.mask_bits, w2.mask_bits, K, n, m, per_row=True)
    assert totals.cpu().tolist() == [ch, 0]
    assert np.array_equal(r.cpu().numpy().astype(np.int64), rows)
    totals, _ = sbl.sbl_mask_monitor(w1.mask_bits, w1.mask_bits, K, n, m)
    assert totals.cpu().tolist() == [0, 0]


def test_mask_monitor_empty(sbl):
    z = torch.empty((0, 8), dtype=torch.uint8, device="cuda")
    totals, _ = sbl.sbl_mask_monitor(z, z, 64, 2, 4)
    assert totals.cpu().tolist() == [0, 0]
