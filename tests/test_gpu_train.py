"""The autograd layer (sparse_linear_layers_b200.train) on the GPU against the
CPU oracle: its forward equals the oracle's on the weights it prepares, its
gradients are the oracle's straight-through gradients within the fp32 bound
(plus the bf16 rounding of the activation gradient), and a training step that
moves the latent weights moves the mask the next forward uses."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_fp32_close, to_dev
from sparse_linear_layers_b200 import synthetic

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


@pytest.fixture(scope="module")
def train():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_linear_layers_b200 import train as m
    return m


def _layer(train, K, O, n, m, tern, seed):
    layer = train.SparseBitLinear(K, O, n, m, dw_ternary=tern, device="cuda")
    W = synthetic.latent_weights(O, K, seed=seed)
    with torch.no_grad():
        layer.weight.copy_(to_dev(W))
    return layer, W


# T = 150 takes a tensor-core prefill path, T = 1 the decode path
@pytest.mark.parametrize("B,S", [(3, 50), (1, 1)])
@pytest.mark.parametrize("n,m,tern", [(2, 4, False), (3, 4, True)])
def test_layer_forward_and_gradients(train, B, S, n, m, tern):
    K, O = 256, 384
    T = B * S
    layer, W = _layer(train, K, O, n, m, tern, seed=T + n)
    _, xv = synthetic.activations(T, K, seed=T)          # bf16 values: the cast to bf16 is exact
    x = to_dev(xv.reshape(B, S, K)).requires_grad_(True)
    dY = synthetic.output_grads(T, O, seed=T + 1)
    y = layer(x)
    (y * to_dev(dY.reshape(B, S, O))).sum().backward()

    _, scale, _, Wt = oracle.prepare_weights(W, n, m)
    y_ref, _, xq, s = oracle.linear(xv, Wt, scale)
    assert_fp32_close(y.detach().cpu().numpy().reshape(T, O), y_ref)
    dX_ref, dW_ref = oracle.ste_backward(dY, xq, s, Wt, scale, dw_ternary=tern)
    a = np.abs(dY).astype(np.float64)
    absx = (a * scale.astype(np.float64)[None, :]) @ np.abs(Wt).astype(np.float64)
    absw = a.T @ (np.abs(xq).astype(np.float64) / s.astype(np.float64)[:, None])
    if tern:
        absw = absw * scale.astype(np.float64)[:, None]
    gw = layer.weight.grad.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(gw - dW_ref) <= (T + 4) * U * absw + 1e-37)
    gx = x.grad.cpu().numpy().reshape(T, K).astype(np.float64)   # dX rounded to bf16, widened
    assert np.all(np.abs(gx - dX_ref) <= (O + 3) * U * absx + 2.0 ** -8 * np.abs(dX_ref) + 1e-37)


def test_training_step_moves_the_mask(train):
    """One SGD step on the latent weights; the next forward prepares the new
    weights (checked against the oracle) and their mask differs from the old."""
    import sparse_linear_layers_b200 as sbl
    K, O, T, n, m = 256, 384, 64, 2, 4
    layer, W = _layer(train, K, O, n, m, False, seed=2)
    _, xv = synthetic.activations(T, K, seed=3)
    x = to_dev(xv)
    opt = torch.optim.SGD(layer.parameters(), lr=1e-3)
    (layer(x) * to_dev(synthetic.output_grads(T, O, seed=4))).sum().backward()
    old = sbl.sbl_prepare_weights(layer.weight.detach(), n, m, with_mask=True).mask_bits
    opt.step()
    W2 = layer.weight.detach().cpu().numpy()
    new = sbl.sbl_prepare_weights(layer.weight.detach(), n, m, with_mask=True).mask_bits
    ch, bad, _ = oracle.mask_monitor(old.cpu().numpy(), new.cpu().numpy(), K, n, m)
    assert ch > 0 and bad == 0
    totals, _ = sbl.sbl_mask_monitor(old, new, K, n, m)
    assert totals.cpu().tolist() == [ch, 0]
    with torch.no_grad():
        y = layer(x)
    _, scale, _, Wt = oracle.prepare_weights(W2, n, m)
    assert_fp32_close(y.cpu().numpy(), oracle.linear(xv, Wt, scale)[0])


def test_forward_stops_on_nonfinite_input(train):
    """The kernels flag NaN and Inf instead of propagating them, so the layer
    reads the status word: a NaN activation or latent weight raises
    FloatingPointError; with check_finite=False the forward runs on."""
    K, O = 256, 128
    layer, W = _layer(train, K, O, 2, 4, False, seed=5)
    x = torch.randn((4, K), device="cuda")
    layer(x)  # finite: no error
    bad = x.clone()
    bad[2, 7] = float("nan")
    with pytest.raises(FloatingPointError):
        layer(bad)
    with torch.no_grad():
        layer.weight[3, 5] = float("inf")
    with pytest.raises(FloatingPointError):
        layer(x)
    layer.check_finite = False
    layer(x)
    torch.cuda.synchronize()
    from sparse_linear_layers_b200 import api
    assert api.sbl_device_status() == 3  # flagged, not raised
    assert api.sbl_device_status() == 0
