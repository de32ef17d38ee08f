"""sbl_linear_grouped (layers that share x: q/k/v, gate/up) against the CPU
oracle, layer by layer: accumulators bit for bit, fp32 y within 1e-5
relative, bf16 y within 2 ulps, and the same bits as separate sbl_linear
calls.  Token counts reach every branch: one launch over the stacked rows
(T <= 2, with wide load batches for large groups), the warp-level MMA per
layer (3 <= T <= 16) and, for prefill, one quantisation and one launch of the
tensor-core GEMM (one CTA or CTA pairs) over up to four layers' output tiles
(more layers: several launches); ragged, unaligned and empty layers, rows of one warp straddling
two layers, and K not a multiple of 64."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_bf16_close, assert_fp32_close, layer_inputs, to_dev, x_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sbl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_linear_layers_b200 as m
    return m


def _layers(sbl, K, Os, n, m, seed):
    out = []
    for i, O in enumerate(Os):
        W, _, _ = layer_inputs(O, K, 1, seed=seed + i, tag=f"grp{i}")
        _, scale, _, Wt = oracle.prepare_weights(W, n, m)
        w = sbl.sbl_prepare_weights(to_dev(W), n, m)
        out.append((w, scale, Wt))
    return out


CASES = [
    # (K, Os, n, m, Ts)
    (896, (896, 128, 128), 3, 4, (1, 2, 5, 16, 300, 2048)),   # q, k, v of the 0.5B layer
    (896, (4864, 4864), 3, 4, (1, 2, 40, 2048)),               # gate, up (T = 2048: one CTA-pair launch)
    (896, (4864, 130), 3, 4, (1000,)),                         # CTA pairs with a ragged, unaligned layer
    (256, (1, 31, 0, 130, 7, 64, 128, 3), 2, 4, (1, 2, 3, 40, 300)),  # eight ragged layers, one empty
    (48, (40, 24, 8), 6, 8, (1, 2, 7)),                        # K % 64 != 0: the dp4a decode only
    (2048, (2048, 7168), 2, 4, (1, 129)),
    (2048, (7168, 7168, 7168, 7168), 2, 4, (1, 2)),           # too large for one batch per lane: wide batches
]


@pytest.mark.parametrize("K,Os,n,m,Ts", CASES)
def test_grouped_matches_oracle_and_separate_calls(sbl, K, Os, n, m, Ts):
    layers = _layers(sbl, K, Os, n, m, seed=K)
    ws = [w for w, _, _ in layers]
    for T in Ts:
        _, xbits, xval = layer_inputs(8, K, T, seed=T, tag="grp-x")
        x = x_dev(xbits)
        accs = [torch.empty((T, O), dtype=torch.int32, device="cuda") for O in Os]
        ys = sbl.sbl_linear_grouped(x, ws, acc_outs=accs)
        ybs = sbl.sbl_linear_grouped(x, ws, out_dtype=torch.bfloat16)
        assert sbl.sbl_device_status() == 0
        for (w, scale, Wt), y, yb, acc in zip(layers, ys, ybs, accs):
            y_ref, acc_ref, _, _ = oracle.linear(xval, Wt, scale)
            assert np.array_equal(acc.cpu().numpy(), acc_ref), (T, w.O)
            assert_fp32_close(y.cpu().numpy(), y_ref, f"T={T} O={w.O}")
            assert_bf16_close(yb.cpu().view(torch.int16).numpy(), y_ref, f"T={T} O={w.O}")
            if w.O:
                assert torch.equal(y, sbl.sbl_linear(x, w)), (T, w.O)


def test_grouped_rejects_mixed_layers(sbl):
    a, b = _layers(sbl, 256, (64, 64), 2, 4, seed=1)
    c = _layers(sbl, 512, (64,), 2, 4, seed=2)[0]
    x = x_dev(layer_inputs(8, 256, 2, seed=0)[1])
    with pytest.raises(ValueError):
        sbl.sbl_linear_grouped(x, [a[0], c[0]])
    with pytest.raises(ValueError):
        sbl.sbl_linear_grouped(x, [a[0]] * 9)


@pytest.mark.parametrize("T", [1, 2])
@pytest.mark.parametrize("K,O", [(2048, 28672), (4864, 8192)])
def test_single_large_layer_decode(sbl, T, K, O):
    """One layer too large for a single batch of loads per lane: the decode takes
    the wide batches (K = 4864 also quantises x with the strided loop);
    bit-exact against the oracle."""
    (w, scale, Wt), = _layers(sbl, K, (O,), 2, 4, seed=77)
    _, xbits, xval = layer_inputs(8, K, T, seed=5, tag="big-x")
    acc = torch.empty((T, O), dtype=torch.int32, device="cuda")
    y = sbl.sbl_linear(x_dev(xbits), w, acc_out=acc)
    assert sbl.sbl_device_status() == 0
    y_ref, acc_ref, _, _ = oracle.linear(xval, Wt, scale)
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_fp32_close(y.cpu().numpy(), y_ref)


@pytest.mark.parametrize("K,Os,n,m", [
    (896, (896, 128, 128, 896, 4864, 4864), 3, 4),   # the 0.5B layer's K = 896 projections
    (64, (1, 0, 33, 130, 7), 2, 4),                  # ragged and empty matrices
    (2048, (700, 2048), 6, 8),
    (9216, (40, 9), 4, 8),                            # rows longer than the register-resident kernel
])
def test_prepare_grouped_matches_oracle(sbl, K, Os, n, m):
    """sbl_prepare_weights_grouped: packed codes, row scales and mask bits of
    every matrix bit for bit against the oracle (and so against separate
    sbl_prepare_weights calls)."""
    Ws = [layer_inputs(O, K, 1, seed=O + i, tag=f"gprep{i}")[0] for i, O in enumerate(Os)]
    outs = sbl.sbl_prepare_weights_grouped([to_dev(W) for W in Ws], n, m, with_mask=True)
    assert sbl.sbl_device_status() == 0
    for W, o in zip(Ws, outs):
        packed, scale, mbits, _ = oracle.prepare_weights(W, n, m)
        assert np.array_equal(o.packed.cpu().numpy(), packed)
        assert np.array_equal(o.row_scale.cpu().numpy().view(np.uint32), scale.view(np.uint32))
        assert np.array_equal(o.mask_bits.cpu().numpy(), mbits)
