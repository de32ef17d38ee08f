"""Straight-through backward (the training path) on the GPU against the CPU oracle.

dX and dW are fp32 contractions whose summation order is the kernel's, so the
bar is the bound that fp32 arithmetic guarantees for any order: within
(n + 3) * 2^-24 * sum |terms| of the oracle's float64 value, n the reduction
length (O for dX, T for dW).  On inputs whose every partial sum is a float
(integer loss gradients, power-of-two scales) the result is exact, and there
the comparison is bit for bit.  Shapes span several 128 x 128 tiles with
ragged edges in every dimension; the hot-path sizes are checked on sampled
entries; empty reductions write zeros.  Every test runs on both paths: the
tcgen05 tensor cores (bf16 parts of the fp32 factor, fp32 accumulation in
tensor memory) and the CUDA cores (fp32 fused multiply-adds)."""
import functools

import numpy as np
import pytest
import torch

import oracle
from parity_util import layer_inputs, to_dev, x_dev
from sparse_linear_layers_b200 import synthetic

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


@pytest.fixture(scope="module")
def sbl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_linear_layers_b200 as m
    return m


@pytest.fixture(params=[True, False], ids=["tcgen05", "cuda_cores"])
def bwd(request, sbl):
    """sbl_linear_backward on the tensor cores (with a workspace) and on the
    CUDA cores: both must meet the same bar."""
    return functools.partial(sbl.sbl_linear_backward, tensor_cores=request.param)


@functools.lru_cache(maxsize=2)
def _layer_cached(O, K, T, n, m, seed):
    import sparse_linear_layers_b200 as sbl
    return _layer_uncached(sbl, O, K, T, n, m, seed)


def _layer(sbl, O, K, T, n, m, seed):
    return _layer_cached(O, K, T, n, m, seed)


def _layer_uncached(sbl, O, K, T, n, m, seed):
    """GPU-prepared weights and GPU-quantised activations (checked equal to the oracle's)."""
    W, xbits, xval = layer_inputs(O, K, T, seed=seed, tag="bwd")
    packed, scale, _, Wt = oracle.prepare_weights(W, n, m)
    xq, s = oracle.quant_act(xval)
    w = sbl.sbl_prepare_weights(to_dev(W), n, m)
    xq_d, s_d = sbl.sbl_quant_act(x_dev(xbits))
    assert np.array_equal(w.packed.cpu().numpy(), packed)
    assert np.array_equal(w.row_scale.cpu().numpy().view(np.uint32), scale.view(np.uint32))
    assert np.array_equal(xq_d.cpu().numpy(), xq) and np.array_equal(s_d.cpu().numpy(), s)
    return w, xq_d, s_d, Wt, scale, xq, s


def _assert_within_bound(got, ref, absref, n, what):
    err = np.abs(np.asarray(got, np.float64) - ref)
    lim = (n + 3) * U * absref + 1e-37
    bad = err > lim
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {bad.sum()} entries beyond (n+3)u*sum|terms|; first at {i}: "
                             f"gpu {got[i]!r} ref {ref[i]!r} bound {lim[i]!r}")


# (O, K, T): tiles of 128 with ragged rows, columns and reduction in every dimension
SHAPES = [(512, 256, 16, 2, 4), (896, 896, 300, 3, 4), (160, 80, 129, 6, 8), (36, 48, 7, 4, 8),
          (2048, 2048, 257, 2, 4), (130, 144, 1, 3, 4)]


@pytest.mark.parametrize("O,K,T,n,m", SHAPES)
def test_backward_random(sbl, bwd, O, K, T, n, m):
    w, xq_d, s_d, Wt, scale, xq, s = _layer(sbl, O, K, T, n, m, seed=O + T)
    dY = synthetic.output_grads(T, O, seed=O * 3 + T)
    dX_ref, dW_ref = oracle.ste_backward(dY, xq, s, Wt, scale)
    _, dWt_ref = oracle.ste_backward(dY, xq, s, Wt, scale, dw_ternary=True)
    a = np.abs(dY).astype(np.float64)
    absx = (a * scale.astype(np.float64)[None, :]) @ np.abs(Wt).astype(np.float64)
    absw = a.T @ (np.abs(xq).astype(np.float64) / s.astype(np.float64)[:, None])
    dY_d = to_dev(dY)
    dX, dW = bwd(dY_d, xq_d, s_d, w)
    _assert_within_bound(dX.cpu().numpy(), dX_ref, absx, O, "dX")
    _assert_within_bound(dW.cpu().numpy(), dW_ref, absw, T, "dW")
    _, dWt = bwd(dY_d, xq_d, s_d, w, need_dx=False, dw_ternary=True)
    _assert_within_bound(dWt.cpu().numpy(), dWt_ref, absw * scale.astype(np.float64)[:, None], T + 1, "dW ternary")
    # one output at a time gives the same bits
    dX1, none = bwd(dY_d, xq_d, s_d, w, need_dw=False)
    assert none is None and torch.equal(dX1, dX)
    none, dW1 = bwd(dY_d, xq_d, s_d, w, need_dx=False)
    assert none is None and torch.equal(dW1, dW)


def _exact_inputs(sbl, O, K, T, n, m, seed):
    """Integer loss gradients in [-2, 2], row scales 2^-3..2^3 and token scales
    2^0..2^3: every product and partial sum is a multiple of 2^-3 well inside
    float's 24 bits, so the fp32 result equals the exact one."""
    from sparse_linear_layers_b200.api import PreparedWeights
    w, xq_d, _, Wt, _, xq, _ = _layer(sbl, O, K, T, n, m, seed)
    rng = np.random.default_rng(seed)
    dY = rng.integers(-2, 3, (T, O)).astype(np.float32)
    scale = np.ldexp(1.0, rng.integers(-3, 4, O)).astype(np.float32)
    s = np.ldexp(1.0, rng.integers(0, 4, T)).astype(np.float32)
    assert 2 * 8 * O * 8 < 2 ** 24 and 254 * T * 8 < 2 ** 24   # in units of 2^-3
    w2 = PreparedWeights(w.packed, to_dev(scale), n, m, K)
    return w2, xq_d, to_dev(s), to_dev(dY), dY, Wt, scale, xq, s


@pytest.mark.parametrize("O,K,T,n,m", [(896, 896, 300, 3, 4), (160, 80, 129, 2, 4), (36, 48, 7, 6, 8)])
def test_backward_exact(sbl, bwd, O, K, T, n, m):
    w, xq_d, s_d, dY_d, dY, Wt, scale, xq, s = _exact_inputs(sbl, O, K, T, n, m, seed=O + 1)
    dX_ref, dW_ref = oracle.ste_backward(dY, xq, s, Wt, scale)
    _, dWt_ref = oracle.ste_backward(dY, xq, s, Wt, scale, dw_ternary=True)
    for ref in (dX_ref, dW_ref, dWt_ref):
        assert np.array_equal(ref.astype(np.float32).astype(np.float64), ref)
    dX, dW = bwd(dY_d, xq_d, s_d, w)
    assert np.array_equal(dX.cpu().numpy(), dX_ref.astype(np.float32))
    assert np.array_equal(dW.cpu().numpy(), dW_ref.astype(np.float32))
    _, dWt = bwd(dY_d, xq_d, s_d, w, need_dx=False, dw_ternary=True)
    assert np.array_equal(dWt.cpu().numpy(), dWt_ref.astype(np.float32))


# The hidden-2048 stack's down (7168 -> 2048) and gate (2048 -> 7168)
# projections at 4096 tokens: the sizes the benchmark times.
@pytest.mark.parametrize("K,O", [(7168, 2048), (2048, 7168)])
def test_backward_full_size_sampled(sbl, bwd, K, O):
    T, n, m = 4096, 2, 4
    w, xq_d, s_d, Wt, scale, xq, s = _layer(sbl, O, K, T, n, m, seed=9)
    dY = synthetic.output_grads(T, O, seed=5)
    dX, dW = bwd(to_dev(dY), xq_d, s_d, w)
    dX, dW = dX.cpu().numpy(), dW.cpu().numpy()
    rng = np.random.default_rng(6)
    dY64, Wt64, sc64 = dY.astype(np.float64), Wt.astype(np.float64), scale.astype(np.float64)
    xh = xq.astype(np.float64) / s.astype(np.float64)[:, None]
    for t, k in zip(rng.integers(0, T, 256), rng.integers(0, K, 256)):
        terms = dY64[t] * sc64 * Wt64[:, k]
        assert abs(dX[t, k] - terms.sum()) <= (O + 3) * U * np.abs(terms).sum() + 1e-37
    for o, k in zip(rng.integers(0, O, 256), rng.integers(0, K, 256)):
        terms = dY64[:, o] * xh[:, k]
        assert abs(dW[o, k] - terms.sum()) <= (T + 3) * U * np.abs(terms).sum() + 1e-37
    # the last tile in each dimension too
    t, o, k = T - 1, O - 1, K - 1
    assert abs(dX[t, k] - (dY64[t] * sc64 * Wt64[:, k]).sum()) <= (O + 3) * U * np.abs(dY64[t]).sum() * sc64.max()
    assert abs(dW[o, k] - (dY64[:, o] * xh[:, k]).sum()) <= (T + 3) * U * np.abs(dY64[:, o] * xh[:, k]).sum() + 1e-37


def test_backward_full_size_exact(sbl, bwd):
    O, K, T = 2048, 7168, 4096
    w, xq_d, s_d, dY_d, dY, Wt, scale, xq, s = _exact_inputs(sbl, O, K, T, 2, 4, seed=9)
    dX, dW = bwd(dY_d, xq_d, s_d, w)
    dX_ref, dW_ref = oracle.ste_backward(dY, xq, s, Wt, scale)
    assert np.array_equal(dX.cpu().numpy(), dX_ref.astype(np.float32))
    assert np.array_equal(dW.cpu().numpy(), dW_ref.astype(np.float32))


def test_backward_empty_reductions(sbl, bwd):
    from sparse_linear_layers_b200.api import PreparedWeights
    K, O, T = 64, 40, 5
    w, xq_d, s_d, *_ = _layer(sbl, O, K, T, 2, 4, seed=1)
    # T == 0: dW is a sum over no tokens
    dW = torch.full((O, K), float("nan"), device="cuda")
    _, dW = bwd(torch.empty((0, O), device="cuda"), xq_d[:0], s_d[:0], w, need_dx=False, dW=dW)
    assert torch.count_nonzero(dW).item() == 0
    # O == 0: dX is a sum over no output rows
    w0 = PreparedWeights(torch.empty((0, K // 4), dtype=torch.uint8, device="cuda"),
                         torch.empty((0,), device="cuda"), 2, 4, K)
    dX = torch.full((T, K), float("nan"), device="cuda")
    dX, _ = bwd(torch.empty((T, 0), device="cuda"), xq_d, s_d, w0, need_dw=False, dX=dX)
    assert torch.count_nonzero(dX).item() == 0
    assert sbl.sbl_device_status() == 0
