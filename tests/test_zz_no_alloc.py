"""sbl_linear_noalloc against the CPU oracle and against sbl_linear, through
the C ABI.

sbl_linear_noalloc is for callers that cannot allocate device memory (for
example a plugin whose host application owns the device-memory budget): it
keeps its scratch in a fixed array of static device memory inside the library
instead of a caller-provided workspace.  This file is collected last so that a
run stopping at the first failure has already run every other test; it passes
on its own in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from parity_util import FP32_RTOL, assert_fp32_close, layer_inputs, to_dev, x_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def abi():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_linear_layers_b200 import _lib
    return _lib


def _prepare(abi, W, n, m):
    O, K = W.shape
    Wd = to_dev(W)
    packed = torch.empty((O, K // 4), dtype=torch.uint8, device="cuda")
    scale = torch.empty((O,), dtype=torch.float32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert abi.lib.sbl_prepare_weights(Wd.data_ptr(), O, K, n, m, packed.data_ptr(), scale.data_ptr(), None, s) == 0
    return packed, scale


def _run_both(abi, O, K, T, n, m, seed):
    W, xbits, xval = layer_inputs(O, K, T, seed=seed, tag="noalloc", outlier_p=0.01)
    packed, scale = _prepare(abi, W, n, m)
    x = x_dev(xbits)
    s = torch.cuda.current_stream().cuda_stream
    # existing entry point, caller-provided workspace
    ws_bytes = abi.lib.sbl_linear_workspace_bytes(T, K, O, n, m)
    ws = torch.empty((ws_bytes,), dtype=torch.uint8, device="cuda")
    y_ref = torch.empty((T, O), dtype=torch.float32, device="cuda")
    acc_ref = torch.empty((T, O), dtype=torch.int32, device="cuda")
    assert abi.lib.sbl_linear(x.data_ptr(), T, K, packed.data_ptr(), scale.data_ptr(), O, n, m, y_ref.data_ptr(),
                              abi.SBL_F32, acc_ref.data_ptr(), ws.data_ptr(), ws_bytes, s) == 0
    # the allocation-free entry point
    y = torch.empty((T, O), dtype=torch.float32, device="cuda")
    acc = torch.empty((T, O), dtype=torch.int32, device="cuda")
    assert abi.lib.sbl_linear_noalloc(x.data_ptr(), T, K, packed.data_ptr(), scale.data_ptr(), O, n, m,
                                      y.data_ptr(), abi.SBL_F32, acc.data_ptr(), s) == 0
    assert abi.lib.sbl_device_status(s) == 0
    # against the oracle: accumulators bit-exact, y within 1e-5 relative
    _, o_scale, _, Wt = oracle.prepare_weights(W, n, m)
    assert np.array_equal(scale.cpu().numpy().view(np.uint32), o_scale.view(np.uint32))
    y_o, acc_o, _, _ = oracle.linear(xval, Wt, o_scale)
    assert np.array_equal(acc.cpu().numpy(), acc_o)
    assert_fp32_close(y.cpu().numpy(), y_o)
    # and against the entry point with a caller-provided workspace
    assert torch.equal(acc, acc_ref)
    yr = y_ref.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(y.cpu().numpy() - yr) <= FP32_RTOL * np.abs(yr))


def test_noalloc_matches_linear_on_two_calls_in_a_row(abi):
    # two different calls back to back: the second finds the first call's
    # contents in the shared scratch array and must not depend on them
    _run_both(abi, O=768, K=896, T=1000, n=3, m=4, seed=0)
    _run_both(abi, O=512, K=2048, T=384, n=2, m=4, seed=1)
    # long K, few tiles: both entry points split the one-CTA prefill along k;
    # the accumulators in the shared scratch hold the previous call's sums
    _run_both(abi, O=2048, K=7168, T=64, n=2, m=4, seed=2)
    _run_both(abi, O=2048, K=7168, T=64, n=2, m=4, seed=3)


def test_noalloc_rejects_calls_beyond_its_scratch(abi):
    limit = 8 << 20
    T, K = 1024, 8192  # needs 8 MiB + 4 KiB of scratch
    assert abi.lib.sbl_linear_workspace_bytes(T, K, 256, 2, 4) > limit
    p = 4096  # never dereferenced: the size check comes first
    assert abi.lib.sbl_linear_noalloc(p, T, K, p, p, 256, 2, 4, p, abi.SBL_F32, None, None) == abi.SBL_ERR_WORKSPACE
