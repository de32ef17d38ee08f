"""sbl_linear_q: the contraction on activations quantised already, against the
oracle (Sparse-BitNet Guide, "Mathematical Formulation of Sparse-BitLinear":
y = (x_q . W_t^T) * scale_o / s_t with the activation step done by the caller).

The quantised activations come from the oracle (oracle.quant_act) or are any
int8 values with any positive scales, -128 included, which the activation
equation itself never yields; the expected accumulators and y are the
oracle's integer product and rescale of exactly those inputs."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_layer_outputs, layer_inputs, to_dev, x_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sbl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_linear_layers_b200 as m
    return m


def _run(sbl, W, n, m, xq, s, out):
    w = sbl.sbl_prepare_weights(torch.from_numpy(W).cuda(), n, m)
    T, O = xq.shape[0], W.shape[0]
    acc = torch.empty((T, O), dtype=torch.int32, device="cuda")
    y = sbl.sbl_linear_q(to_dev(xq), to_dev(s), w, out_dtype=out, acc_out=acc)
    torch.cuda.synchronize()
    assert sbl.sbl_device_status() == 0
    _, scale, _, Wt = oracle.prepare_weights(W, n, m)
    yn = y.cpu()
    assert_layer_outputs(acc.cpu().numpy(), yn.numpy() if out == torch.float32 else None,
                         yn.view(torch.int16).numpy().view(np.uint16) if out == torch.bfloat16 else None,
                         xq, s, Wt, scale, what=f"linear_q {O}x{W.shape[1]} T={T}")
    return w, y


# (O, K, T, n, m, output dtype, the path the sizes take)
CASES = [
    (512, 256, 1, 2, 4, torch.float32, "decode"),
    (896, 896, 16, 3, 4, torch.float32, "decode"),
    (200, 128, 7, 6, 8, torch.bfloat16, "decode"),          # O not a multiple of the row tile
    (896, 896, 300, 3, 4, torch.float32, "prefill_1cta"),  # a ragged token tile
    (4864, 896, 2048, 3, 4, torch.bfloat16, "prefill_pair"),
    (896, 4864, 2048, 4, 8, torch.float32, "prefill_1cta"),
    (384, 2048, 16384, 2, 4, torch.bfloat16, "prefill_sparse"),
]


@pytest.mark.parametrize("O,K,T,n,m,out,path", CASES)
def test_linear_q_matches_oracle(sbl, O, K, T, n, m, out, path):
    assert sbl.sbl_linear_plan(T, K, O, n, m) == path
    W, _, xval = layer_inputs(O, K, T, seed=11, tag="linq")
    xq, s = oracle.quant_act(xval)
    _run(sbl, W, n, m, xq, s, out)


@pytest.mark.parametrize("O,K,T,n,m", [(896, 896, 5, 3, 4), (1024, 896, 640, 2, 4)])
def test_linear_q_any_int8(sbl, O, K, T, n, m):
    """Full-range int8 activations (-128 included) and arbitrary positive scales."""
    rng = np.random.default_rng(7)
    W, _, _ = layer_inputs(O, K, T, seed=12, tag="linq8")
    xq = rng.integers(-128, 128, size=(T, K), dtype=np.int16).astype(np.int8)
    xq[:, 0] = -128
    s = (2.0 ** rng.uniform(-8, 8, size=T)).astype(np.float32)
    _run(sbl, W, n, m, xq, s, torch.float32)


@pytest.mark.parametrize("O,K,T,n,m", [(896, 896, 1, 3, 4), (896, 896, 12, 3, 4), (4864, 896, 2048, 3, 4)])
def test_linear_q_equals_linear(sbl, O, K, T, n, m):
    """On the quantisation sbl_quant_act gives, the same bits as sbl_linear."""
    W, xbits, _ = layer_inputs(O, K, T, seed=13, tag="linqeq")
    w = sbl.sbl_prepare_weights(torch.from_numpy(W).cuda(), n, m)
    x = x_dev(xbits)
    xq, s = sbl.sbl_quant_act(x)
    y_q = sbl.sbl_linear_q(xq, s, w)
    y = sbl.sbl_linear(x, w)
    torch.cuda.synchronize()
    assert torch.equal(y_q.view(torch.int32), y.view(torch.int32))


def test_linear_q_edges(sbl):
    W, _, _ = layer_inputs(128, 96, 4, seed=14, tag="linqedge")
    w96 = sbl.sbl_prepare_weights(torch.from_numpy(W).cuda(), 2, 4)
    xq = torch.zeros((4, 96), dtype=torch.int8, device="cuda")
    s = torch.ones(4, dtype=torch.float32, device="cuda")
    with pytest.raises(sbl.SblError):
        sbl.sbl_linear_q(xq, s, w96)  # K % 64 != 0
    W, _, _ = layer_inputs(256, 128, 1, seed=15, tag="linqedge")
    w = sbl.sbl_prepare_weights(torch.from_numpy(W).cuda(), 2, 4)
    y = sbl.sbl_linear_q(torch.zeros((0, 128), dtype=torch.int8, device="cuda"),
                         torch.zeros(0, dtype=torch.float32, device="cuda"), w)
    assert y.shape == (0, 256)
    # zero activations give zero outputs
    y = sbl.sbl_linear_q(torch.zeros((3, 128), dtype=torch.int8, device="cuda"),
                         torch.ones(3, dtype=torch.float32, device="cuda"), w)
    torch.cuda.synchronize()
    assert not y.any()
    with pytest.raises(ValueError):
        sbl.sbl_linear_q(torch.zeros((3, 128), dtype=torch.int8, device="cuda"),
                         torch.ones(2, dtype=torch.float32, device="cuda"), w)  # s_tok of the wrong length
