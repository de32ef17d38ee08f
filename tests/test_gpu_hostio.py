"""Host-buffer entry points: sbl_linear_hostio (x in and y out of host memory
around sbl_linear) and the copies sbl_copy_to_device / sbl_copy_to_host,
against the oracle (the Sparse-BitNet Guide, "Mathematical Formulation of
Sparse-BitLinear")."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_bf16_close, assert_fp32_close, layer_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sbl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_linear_layers_b200 as m
    return m


@pytest.mark.parametrize("O,K,T,n,m,out", [
    (512, 256, 16, 2, 4, torch.float32),    # the decode path
    (896, 896, 1, 3, 4, torch.float32),
    (896, 896, 300, 3, 4, torch.float32),   # the tensor-core path, a ragged token tile
    (4864, 896, 2048, 3, 4, torch.bfloat16),
    (200, 128, 7, 6, 8, torch.bfloat16),    # O not a multiple of the output tile
])
def test_linear_hostio_matches_oracle(sbl, O, K, T, n, m, out):
    W, xbits, xval = layer_inputs(O, K, T, seed=5, tag="hostio")
    w = sbl.sbl_prepare_weights(torch.from_numpy(W).cuda(), n, m)
    x_host = torch.from_numpy(np.ascontiguousarray(xbits).view(np.int16)).view(torch.bfloat16).pin_memory()
    s = torch.cuda.Stream()
    y_host = sbl.sbl_linear_hostio(x_host, w, out_dtype=out, stream=s)
    s.synchronize()
    assert not y_host.is_cuda and y_host.shape == (T, O) and y_host.dtype == out
    assert sbl.sbl_device_status() == 0
    _, o_scale, _, Wt = oracle.prepare_weights(W, n, m)
    y_o, _, _, _ = oracle.linear(xval, Wt, o_scale)
    if out == torch.float32:
        assert_fp32_close(y_host.numpy(), y_o)
    else:
        assert_bf16_close(y_host.view(torch.int16).numpy().view(np.uint16), y_o)
    # the same kernels as sbl_linear on device buffers: the same bits
    y_dev = sbl.sbl_linear(x_host.cuda(), w, out_dtype=out)
    assert torch.equal(y_dev.cpu().view(torch.int16), y_host.view(torch.int16))


def test_host_copies_round_trip(sbl):
    g = torch.Generator().manual_seed(3)
    a = torch.randint(0, 256, (1 << 20,), dtype=torch.uint8, generator=g).pin_memory()
    d = torch.empty_like(a, device="cuda")
    b = torch.empty_like(a).pin_memory()
    s = torch.cuda.Stream()
    sbl.copy_to_device(d, a, stream=s)
    sbl.copy_to_host(b, d, stream=s)
    s.synchronize()
    assert torch.equal(a, b)
    with pytest.raises(ValueError):
        sbl.copy_to_device(d, a[:16], stream=s)  # sizes differ
    with pytest.raises(ValueError):
        sbl.copy_to_host(d, d, stream=s)          # the destination is not host memory
