"""CUDA path against the CPU oracle, element by element, through the C ABI.

Bit-exact: packed codes, mask bits, row scales (as fp32 bit patterns), x_q,
s_tok and the int32 accumulators.  fp32 outputs within 1e-5 relative, bf16
outputs within 2 ulp of the rounded oracle value.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import (assert_bf16_close, assert_fp32_close, assert_layer_outputs, layer_inputs, oracle_layer, to_dev,
                         x_dev)

pytestmark = pytest.mark.gpu

PATTERNS = [(2, 4), (3, 4), (6, 8), (4, 8)]


@pytest.fixture(scope="module")
def sbl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_linear_layers_b200 as m
    return m


def _prep(sbl, W, n, m):
    w = sbl.sbl_prepare_weights(to_dev(W), n, m, with_mask=True)
    torch.cuda.synchronize()
    return w


# ------------------------------------------------------------------ weight prep

@pytest.mark.parametrize("n,m", PATTERNS)
@pytest.mark.parametrize("O,K", [(512, 256), (37, 48), (130, 320), (9, 16 * 8)])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_prepare_bit_exact(sbl, n, m, O, K, seed):
    if K % m:
        pytest.skip("K not a multiple of M")
    W, _, _ = layer_inputs(O, K, 1, seed=seed)
    # plant ties, zero groups and a zero row
    W[0, :m] = np.float32(0.03125)
    W[1, : 2 * m] = 0.0
    W[-1, :] = 0.0
    w = _prep(sbl, W, n, m)
    packed, scale, mbits, _ = oracle.prepare_weights(W, n, m)
    assert np.array_equal(w.packed.cpu().numpy(), packed)
    assert np.array_equal(w.row_scale.cpu().numpy().view(np.uint32), scale.view(np.uint32))
    assert np.array_equal(w.mask_bits.cpu().numpy(), mbits)


@pytest.mark.parametrize("n,m,O,K", [(3, 4, 4864, 896), (3, 4, 896, 4864), (2, 4, 7168, 2048),
                                     (6, 8, 2048, 7168), (4, 8, 7168, 2048), (4, 8, 2048, 16384)])
def test_prepare_bit_exact_full_layers(sbl, n, m, O, K):
    W, _, _ = layer_inputs(O, K, 1, seed=0)
    w = _prep(sbl, W, n, m)
    packed, scale, mbits, _ = oracle.prepare_weights(W, n, m)
    assert np.array_equal(w.row_scale.cpu().numpy().view(np.uint32), scale.view(np.uint32))
    assert np.array_equal(w.packed.cpu().numpy(), packed)
    assert np.array_equal(w.mask_bits.cpu().numpy(), mbits)


def test_prepare_extreme_magnitudes(sbl):
    # denormals, huge values and mixed exponents stress the exact row sum
    rng = np.random.default_rng(7)
    O, K = 64, 256
    e = rng.integers(-149, 120, size=(O, K)).astype(np.float64)
    W = (rng.choice([-1.0, 1.0], size=(O, K)) * rng.random((O, K)) * np.exp2(e)).astype(np.float32)
    W[3] = np.float32(1e-45)
    W[4] = np.float32(3.0e38)
    for n, m in PATTERNS:
        w = _prep(sbl, W, n, m)
        packed, scale, mbits, _ = oracle.prepare_weights(W, n, m)
        assert np.array_equal(w.row_scale.cpu().numpy().view(np.uint32), scale.view(np.uint32))
        assert np.array_equal(w.packed.cpu().numpy(), packed)


def test_prepare_window_boundaries(sbl):
    # Kept magnitudes placed at chosen binade distances d below each row's
    # largest one (d = 0 ... 200, both sides of 35/36 and 71/72, subnormals),
    # and a row whose exact sum is a double rounding tie broken only by a value
    # 100 binades down: the row scale must still be the exactly rounded mean.
    rng = np.random.default_rng(11)
    O, K = 96, 64
    dists = [0, 1, 23, 24, 34, 35, 36, 37, 47, 48, 70, 71, 72, 73, 100, 200]
    W = np.zeros((O, K), dtype=np.float32)
    for r in range(O - 1):
        p_max = int(rng.integers(0, 254))
        W[r, 0] = np.float32(np.ldexp(float(rng.integers(1 << 23, 1 << 24)), p_max - 149))
        for g in range(1, K // 4):
            p = p_max - int(rng.choice(dists))
            if p >= 0:
                mant = int(rng.integers(1 << 23, 1 << 24)) if p > 0 else int(rng.integers(1, 1 << 23))
                W[r, 4 * g] = np.float32(np.ldexp(float(mant), p - 149)) * np.float32(rng.choice([-1, 1]))
    W[O - 1, 0], W[O - 1, 4], W[O - 1, 8] = 1.0, np.float32(2.0 ** -53), np.float32(2.0 ** -100)
    for n, m in PATTERNS:
        w = _prep(sbl, W, n, m)
        packed, scale, mbits, _ = oracle.prepare_weights(W, n, m)
        assert np.array_equal(w.row_scale.cpu().numpy().view(np.uint32), scale.view(np.uint32))
        assert np.array_equal(w.packed.cpu().numpy(), packed)
        assert np.array_equal(w.mask_bits.cpu().numpy(), mbits)


# ------------------------------------------------------------------ activation quant

@pytest.mark.parametrize("T,K,p", [(16, 256, 0.0), (3, 48, 0.0), (257, 896, 0.01), (64, 4864, 0.01)])
def test_quant_bit_exact(sbl, T, K, p):
    _, xbits, xval = layer_inputs(8, K, T, seed=1, outlier_p=p)
    xbits[0] = 0  # zero token
    xval[0] = 0.0
    xq, s = sbl.sbl_quant_act(x_dev(xbits))
    rq, rs = oracle.quant_act(xval)
    assert np.array_equal(xq.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))


# ------------------------------------------------------------------ linear

def _run_linear(sbl, w, xbits, T, O, path, out_dtype=torch.float32):
    acc = torch.empty((T, O), dtype=torch.int32, device="cuda")
    y = sbl.sbl_linear(x_dev(xbits), w, out_dtype=out_dtype, acc_out=acc, path=path)
    assert sbl.sbl_device_status() == 0
    return y, acc


LINEAR_CASES = [
    # (O, K, T, n, m): config-1 shape, ragged tiles and tails, K % 128 == 64, narrow/wide N tiles
    (512, 256, 16, 2, 4),
    (40, 64, 3, 3, 4),
    (300, 320, 130, 6, 8),
    (130, 192, 17, 2, 4),
    (384, 896, 257, 3, 4),
    (896, 128, 1, 3, 4),
    (256, 512, 33, 4, 8),
    (640, 1024, 5, 4, 8),
]


@pytest.mark.parametrize("path", ["decode", "prefill", "prefill_1cta", "prefill_pair"])
@pytest.mark.parametrize("O,K,T,n,m", LINEAR_CASES)
def test_linear_parity(sbl, path, O, K, T, n, m):
    W, xbits, xval = layer_inputs(O, K, T, seed=2, outlier_p=0.01)
    ref = oracle_layer(W, n, m, xval)
    w = _prep(sbl, W, n, m)
    y, acc = _run_linear(sbl, w, xbits, T, O, path)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert_fp32_close(y.cpu().numpy(), ref["y"])
    yb, _ = _run_linear(sbl, w, xbits, T, O, path, torch.bfloat16)
    assert_bf16_close(yb.cpu().view(torch.int16).numpy(), ref["y"])


@pytest.mark.parametrize("T", [1, 2, 5, 8, 9, 16])
def test_decode_token_counts(sbl, T):
    O, K, n, m = 200, 448, 3, 4
    W, xbits, xval = layer_inputs(O, K, T, seed=0)
    ref = oracle_layer(W, n, m, xval)
    w = _prep(sbl, W, n, m)
    y, acc = _run_linear(sbl, w, xbits, T, O, "decode")
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert_fp32_close(y.cpu().numpy(), ref["y"])


@pytest.mark.parametrize("O,K,T", [(7168, 2048, 8), (896, 4864, 16), (4864, 896, 3), (48, 24576, 16),
                                   (136, 2048, 12), (24, 320, 7)])
def test_decode_mma_shapes(sbl, O, K, T):
    """Warp-MMA decode: every code-word width (K % 256, % 128, % 64), split-K
    row tiles, one and two n8 token tiles, passes limited by shared memory,
    activations re-read past four blocks per thread, ragged row tiles."""
    n, m = 2, 4
    W, xbits, xval = layer_inputs(O, K, T, seed=5, outlier_p=0.01)
    ref = oracle_layer(W, n, m, xval)
    w = _prep(sbl, W, n, m)
    y, acc = _run_linear(sbl, w, xbits, T, O, "decode")
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert_fp32_close(y.cpu().numpy(), ref["y"])
    yb, _ = _run_linear(sbl, w, xbits, T, O, "decode", torch.bfloat16)
    assert_bf16_close(yb.cpu().view(torch.int16).numpy(), ref["y"])


@pytest.mark.parametrize("O,K,T,n,m", [(2048, 7168, 64, 2, 4), (896, 4864, 64, 3, 4), (300, 4096, 40, 6, 8),
                                       (512, 2048, 200, 2, 4)])
def test_prefill_split_k(sbl, O, K, T, n, m):
    """One-CTA prefill split along k (few tiles, long K): the automatic path
    takes it, a second call on the same workspace agrees (the accumulators
    are zeroed every call), and ragged token and row counts are covered."""
    assert sbl.sbl_linear_plan(T, K, O, n, m) == "prefill_1cta"
    W, xbits, xval = layer_inputs(O, K, T, seed=6, outlier_p=0.01)
    ref = oracle_layer(W, n, m, xval)
    w = _prep(sbl, W, n, m)
    ws = sbl.workspace_for(T, K, O, n, m, "cuda")
    assert ws.numel() > T * K + 4 * T + 512  # the split area is part of the default workspace
    for out_dtype in (torch.float32, torch.bfloat16, torch.float32):
        acc = torch.empty((T, O), dtype=torch.int32, device="cuda")
        y = sbl.sbl_linear(x_dev(xbits), w, out_dtype=out_dtype, acc_out=acc, workspace=ws)
        assert sbl.sbl_device_status() == 0
        assert np.array_equal(acc.cpu().numpy(), ref["acc"])
        if out_dtype == torch.float32:
            assert_fp32_close(y.cpu().numpy(), ref["y"])
        else:
            assert_bf16_close(y.cpu().view(torch.int16).numpy(), ref["y"])


def test_decode_k_not_multiple_of_64(sbl):
    O, K, T, n, m = 77, 48, 4, 2, 4
    W, xbits, xval = layer_inputs(O, K, T, seed=3)
    ref = oracle_layer(W, n, m, xval)
    w = _prep(sbl, W, n, m)
    y, acc = _run_linear(sbl, w, xbits, T, O, "auto")
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert_fp32_close(y.cpu().numpy(), ref["y"])


def test_zero_rows_and_tokens(sbl):
    O, K, T, n, m = 256, 256, 40, 2, 4
    W, xbits, xval = layer_inputs(O, K, T, seed=4)
    W[5] = 0.0
    xbits[7] = 0
    xval[7] = 0.0
    ref = oracle_layer(W, n, m, xval)
    w = _prep(sbl, W, n, m)
    for path in ("decode", "prefill_1cta", "prefill_pair"):
        y, acc = _run_linear(sbl, w, xbits, T, O, path)
        yn = y.cpu().numpy()
        assert np.array_equal(acc.cpu().numpy(), ref["acc"])
        assert not yn[7].any() and not yn[:, 5].any()


PAIR_CASES = [
    # (O, K, T, n, m): full 256 x 256 pair tiles, a ragged half tile of outputs
    # (896 = 3.5 x 256) and of tokens, an odd CTA with no tokens at all, N:M patterns
    (4864, 896, 2048, 3, 4),
    (896, 4864, 300, 2, 4),
    (1000, 640, 513, 6, 8),
    (256, 128, 128, 2, 4),
]


@pytest.mark.parametrize("O,K,T,n,m", PAIR_CASES)
def test_pair_prefill_full(sbl, O, K, T, n, m):
    """The CTA-pair tensor-core kernel, fully compared (fp32 and bf16 outputs)."""
    W, xbits, xval = layer_inputs(O, K, T, seed=6, outlier_p=0.01)
    ref = oracle_layer(W, n, m, xval)
    w = _prep(sbl, W, n, m)
    y, acc = _run_linear(sbl, w, xbits, T, O, "prefill_pair")
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert_fp32_close(y.cpu().numpy(), ref["y"])
    yb, _ = _run_linear(sbl, w, xbits, T, O, "prefill_pair", torch.bfloat16)
    assert_bf16_close(yb.cpu().view(torch.int16).numpy(), ref["y"])


SPARSE_CASES = [
    # (O, K, T): 2:4 weights on the structured-sparse MMA.  A full 128 x 160 tile
    # and K multiple of 256; ragged output rows and token tiles; K % 256 = 64,
    # 128, 192 (a partial last k-block); the FFN gate and down shapes.
    (256, 256, 160),
    (300, 320, 130),
    (1000, 640, 513),
    (130, 448, 17),
    (4864, 896, 2048),
    (896, 4864, 300),
]


@pytest.mark.parametrize("O,K,T", SPARSE_CASES)
def test_sparse_prefill_full(sbl, O, K, T):
    """2:4 weights through the sparse tensor cores, fully compared (fp32 and bf16 outputs)."""
    W, xbits, xval = layer_inputs(O, K, T, seed=8, outlier_p=0.01)
    W[0, :8] = 0.0        # all-zero groups
    W[1, 1::4] = 0.0      # groups with a single kept nonzero at every position
    W[1, 2::4] = 0.0
    W[2, ::4] = 0.0
    W[2, 1::4] = 0.0
    ref = oracle_layer(W, 2, 4, xval)
    w = _prep(sbl, W, 2, 4)
    y, acc = _run_linear(sbl, w, xbits, T, O, "prefill_sparse")
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert_fp32_close(y.cpu().numpy(), ref["y"])
    yb, _ = _run_linear(sbl, w, xbits, T, O, "prefill_sparse", torch.bfloat16)
    assert_bf16_close(yb.cpu().view(torch.int16).numpy(), ref["y"])


def test_sparse_prefill_rejections(sbl):
    from sparse_linear_layers_b200._lib import SBL_ERR_UNSUPPORTED, SBL_ERR_WORKSPACE, SblError
    O, K, T = 128, 256, 64
    W, xbits, _ = layer_inputs(O, K, T, seed=9)
    w34 = _prep(sbl, W, 3, 4)
    with pytest.raises(SblError) as e:
        sbl.sbl_linear(x_dev(xbits), w34, path="prefill_sparse")
    assert e.value.code == SBL_ERR_UNSUPPORTED
    w24 = _prep(sbl, W, 2, 4)
    small = torch.empty((T * K + 4 * T + 512,), dtype=torch.uint8, device="cuda")  # no room for compressed weights
    with pytest.raises(SblError) as e:
        sbl.sbl_linear(x_dev(xbits), w24, workspace=small, path="prefill_sparse")
    assert e.value.code == SBL_ERR_WORKSPACE
    # the automatic choice falls back to a dense path in that workspace
    y = sbl.sbl_linear(x_dev(xbits), w24, workspace=small)
    assert sbl.sbl_device_status() == 0
    assert torch.isfinite(y).all()


def test_sparse_prefill_flags_non_24_codes(sbl):
    from sparse_linear_layers_b200._lib import SBL_ERR_INVALID_ARG
    O, K, T = 128, 256, 64
    W, xbits, _ = layer_inputs(O, K, T, seed=10)
    w = _prep(sbl, W, 2, 4)
    packed = w.packed.clone()
    packed[5, 3] = 0b01010101  # four +1 codes in one group of four
    bad = sbl.PreparedWeights(packed, w.row_scale, 2, 4, K)
    sbl.sbl_linear(x_dev(xbits), bad, path="prefill_sparse")
    assert sbl.sbl_device_status() == SBL_ERR_INVALID_ARG


# ------------------------------------------------------------------ full-size layers

@pytest.mark.parametrize("T", [1, 2048])
def test_qwen_layer_full(sbl, T):
    """Qwen2.5-0.5B-shaped projections at 3:4, fully compared."""
    from sparse_linear_layers_b200.synthetic import QWEN05_LAYER
    for name, K, O in QWEN05_LAYER:
        W, xbits, xval = layer_inputs(O, K, T, seed=0, tag=name)
        ref = oracle_layer(W, 3, 4, xval)
        w = _prep(sbl, W, 3, 4)
        y, acc = _run_linear(sbl, w, xbits, T, O, "auto")
        assert np.array_equal(acc.cpu().numpy(), ref["acc"]), name
        assert_fp32_close(y.cpu().numpy(), ref["y"], name)


@pytest.mark.parametrize("n,m", [(3, 4), (2, 4)])
def test_ffn_prefill_32k_full(sbl, n, m):
    """0.5B FFN shapes (gate, up, down) at T = 32768 with 1% outliers x20, 3:4
    and 2:4: every accumulator bit for bit, every fp32 and bf16 output within
    tolerance (the oracle's exact float64 product, token chunk by chunk)."""
    from sparse_linear_layers_b200.synthetic import QWEN05_FFN
    T = 32768
    for name, K, O in QWEN05_FFN:
        W, xbits, xval = layer_inputs(O, K, T, seed=0, outlier_p=0.01, tag=name)
        packed, scale, _, Wt = oracle.prepare_weights(W, n, m)
        xq, s = oracle.quant_act(xval)
        del xval
        w = _prep(sbl, W, n, m)
        assert np.array_equal(w.packed.cpu().numpy(), packed)
        x = x_dev(xbits)
        acc = torch.empty((T, O), dtype=torch.int32, device="cuda")
        y = sbl.sbl_linear(x, w, acc_out=acc)
        yb = sbl.sbl_linear(x, w, out_dtype=torch.bfloat16)
        assert sbl.sbl_device_status() == 0
        assert np.array_equal(s, sbl.sbl_quant_act(x)[1].cpu().numpy())
        assert_layer_outputs(acc.cpu().numpy(), y.cpu().numpy(), yb.cpu().view(torch.int16).numpy(), xq, s, Wt, scale,
                             what=f"{name} {n}:{m}")
        del acc, y, yb, x


# ------------------------------------------------------------------ device status paths

def test_nonfinite_inputs_raise_status(sbl):
    W, xbits, _ = layer_inputs(64, 128, 4, seed=5)
    W[3, 7] = np.nan
    sbl.sbl_prepare_weights(to_dev(W), 2, 4)
    assert sbl.sbl_device_status() == 3
    xbits[1, 2] = 0x7F80  # +inf
    sbl.sbl_quant_act(x_dev(xbits))
    assert sbl.sbl_device_status() == 3
    assert sbl.sbl_device_status() == 0  # cleared


def test_bounded_wait_times_out_cleanly(sbl):
    assert sbl.sbl_selftest_bounded_wait(200) == 5
    # the context stays usable
    W, xbits, xval = layer_inputs(64, 128, 4, seed=6)
    ref = oracle_layer(W, 2, 4, xval)
    w = _prep(sbl, W, 2, 4)
    _, acc = _run_linear(sbl, w, xbits, 4, 64, "prefill")
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])


# ------------------------------------------------------------------ streams and graphs

def test_concurrent_streams_in_a_graph(sbl):
    """Independent projections on separate streams, each with its own workspace,
    captured into one CUDA graph and replayed twice: every output matches the oracle."""
    shapes = [(512, 256, 300, 3, 4), (128, 256, 300, 3, 4), (640, 256, 1, 2, 4), (1024, 256, 40, 6, 8)]
    cases = []
    for i, (O, K, T, n, m) in enumerate(shapes):
        W, xbits, xval = layer_inputs(O, K, T, seed=20 + i)
        ref = oracle_layer(W, n, m, xval)
        w = _prep(sbl, W, n, m)
        x = x_dev(xbits)
        y = torch.empty((T, O), dtype=torch.float32, device="cuda")
        acc = torch.empty((T, O), dtype=torch.int32, device="cuda")
        ws = sbl.workspace_for(T, K, O, n, m, torch.device("cuda"))
        cases.append((w, x, y, acc, ws, ref))
    main = torch.cuda.Stream()
    side = [torch.cuda.Stream() for _ in cases]

    def launch():
        fork = torch.cuda.Event()
        fork.record(main)
        joins = []
        for (w, x, y, acc, ws, _), st in zip(cases, side):
            st.wait_event(fork)
            with torch.cuda.stream(st):
                sbl.sbl_linear(x, w, y=y, acc_out=acc, workspace=ws)
            ev = torch.cuda.Event()
            ev.record(st)
            joins.append(ev)
        for ev in joins:
            main.wait_event(ev)

    with torch.cuda.stream(main):
        launch()  # eager pass before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=main):
        launch()
    for _ in range(2):
        for _, _, y, acc, _, _ in cases:
            y.zero_()
            acc.zero_()
        torch.cuda.synchronize()
        with torch.cuda.stream(main):
            g.replay()
        torch.cuda.synchronize()
        assert sbl.sbl_device_status() == 0
        for _, _, y, acc, _, ref in cases:
            assert np.array_equal(acc.cpu().numpy(), ref["acc"])
            assert_fp32_close(y.cpu().numpy(), ref["y"])


def test_linear_plan(sbl):
    from sparse_linear_layers_b200._lib import SBL_ERR_UNSUPPORTED, SblError
    assert sbl.sbl_linear_plan(1, 2048, 7168, 2, 4) == "decode"
    assert sbl.sbl_linear_plan(16, 896, 896, 3, 4) == "decode"
    assert sbl.sbl_linear_plan(2048, 896, 896, 3, 4) == "prefill_1cta"
    assert sbl.sbl_linear_plan(32768, 896, 4864, 3, 4) == "prefill_pair"
    assert sbl.sbl_linear_plan(32768, 2048, 7168, 2, 4) == "prefill_sparse"
    # 2:4 without room for the compressed weights stays dense
    base = 32768 * 2048 + 32768 * 4 + 1024
    assert sbl.sbl_linear_plan(32768, 2048, 7168, 2, 4, workspace_bytes=base) == "prefill_pair"
    with pytest.raises(SblError) as e:
        sbl.sbl_linear_plan(64, 256, 128, 1, 4)
    assert e.value.code == SBL_ERR_UNSUPPORTED


@pytest.mark.parametrize("n,m", PATTERNS)
@pytest.mark.parametrize("O,K", [(300, 896), (64, 16384)])
def test_prepare_scale_bf16(sbl, n, m, O, K):
    """bf16 scale storage: the rounded scale ternarises the row; both prep
    kernels (rows held in registers, and the long-row kernel) bit-exact."""
    W, xbits, xval = layer_inputs(O, K, 5, seed=7)
    packed, scale, mbits, Wt = oracle.prepare_weights(W, n, m, scale_bf16=True)
    w = sbl.sbl_prepare_weights(to_dev(W), n, m, with_mask=True, scale_bf16=True)
    assert sbl.sbl_device_status() == 0
    assert np.array_equal(w.packed.cpu().numpy(), packed)
    assert np.array_equal(w.row_scale.cpu().numpy().view(np.uint32), scale.view(np.uint32))
    assert np.array_equal(w.mask_bits.cpu().numpy(), mbits)
    y_ref, acc_ref, _, _ = oracle.linear(xval, Wt, scale)
    y, acc = _run_linear(sbl, w, xbits, 5, O, "auto")
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_fp32_close(y.cpu().numpy(), y_ref)


@pytest.mark.parametrize("n,m", PATTERNS)
@pytest.mark.parametrize("O,K", [(300, 896), (64, 16384)])
@pytest.mark.parametrize("bf16", [False, True])
def test_prepare_scale_global(sbl, n, m, O, K, bf16):
    """The guide listing's single scale: the exact mean of |W| over the matrix
    (a huge and a tiny weight included), bit-exact, in both prep kernels."""
    W, xbits, xval = layer_inputs(O, K, 3, seed=9)
    W = W.copy()
    W[0, 5] = np.float32(2.5e6)
    W[O - 1, K - 1] = np.float32(3.0e-33)
    packed, scale, mbits, Wt = oracle.prepare_weights(W, n, m, scale_bf16=bf16, scale_global=True)
    w = sbl.sbl_prepare_weights(to_dev(W), n, m, with_mask=True, scale_bf16=bf16, scale_global=True)
    assert sbl.sbl_device_status() == 0
    assert np.array_equal(w.row_scale.cpu().numpy().view(np.uint32), scale.view(np.uint32))
    assert np.array_equal(w.packed.cpu().numpy(), packed)
    assert np.array_equal(w.mask_bits.cpu().numpy(), mbits)
    y_ref, acc_ref, _, _ = oracle.linear(xval, Wt, scale)
    y, acc = _run_linear(sbl, w, xbits, 3, O, "auto")
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_fp32_close(y.cpu().numpy(), y_ref)


@pytest.mark.parametrize("path", ["prefill", "prefill_1cta", "prefill_pair"])
def test_prefill_large_t_full(sbl, path):
    """T = 16500 on the dense paths (ragged last token tile), every output
    element compared, and a second call reusing the workspace."""
    O, K, T, n, m = 256, 256, 16500, 3, 4
    W, xbits, xval = layer_inputs(O, K, T, seed=10, outlier_p=0.01)
    ref = oracle_layer(W, n, m, xval)
    w = _prep(sbl, W, n, m)
    ws = sbl.workspace_for(T, K, O, n, m, "cuda")
    for _ in range(2):
        acc = torch.empty((T, O), dtype=torch.int32, device="cuda")
        y = sbl.sbl_linear(x_dev(xbits), w, acc_out=acc, workspace=ws, path=path)
        assert sbl.sbl_device_status() == 0
        assert np.array_equal(acc.cpu().numpy(), ref["acc"])
        assert_fp32_close(y.cpu().numpy(), ref["y"])


def test_graph_replay_of_split_rmsnorm_and_monitor(sbl):
    """A CUDA graph holding a split-K prefill (its accumulators zeroed inside
    the graph by the quantisation kernel), an RMSNorm-fronted decode and a mask
    monitor (a memset node), replayed three times: every replay matches."""
    O, K, T, n, m = 512, 4096, 40, 2, 4
    W, xbits, xval = layer_inputs(O, K, T, seed=12)
    W2 = W + np.float32(0.003)
    ref = oracle_layer(W, n, m, xval)
    g = np.random.default_rng(4).uniform(0.5, 1.5, K).astype(np.float32)
    _, scale, mb1, Wt = oracle.prepare_weights(W, n, m)
    _, _, mb2, _ = oracle.prepare_weights(W2, n, m)
    y_rms, acc_rms, _, _ = oracle.linear(xval[:8], Wt, scale, g=g, eps=2.0 ** -23)
    changed, bad, _ = oracle.mask_monitor(mb1, mb2, K, n, m)
    w = sbl.sbl_prepare_weights(to_dev(W), n, m, with_mask=True)
    w2 = sbl.sbl_prepare_weights(to_dev(W2), n, m, with_mask=True)
    assert sbl.sbl_linear_plan(T, K, O, n, m) == "prefill_1cta"
    x, x8, gd = x_dev(xbits), x_dev(xbits[:8]), to_dev(g)
    ws = sbl.workspace_for(T, K, O, n, m, "cuda")
    ws8 = sbl.workspace_for(8, K, O, n, m, "cuda")
    acc = torch.empty((T, O), dtype=torch.int32, device="cuda")
    y = torch.empty((T, O), dtype=torch.float32, device="cuda")
    acc8 = torch.empty((8, O), dtype=torch.int32, device="cuda")
    y8 = torch.empty((8, O), dtype=torch.float32, device="cuda")
    out = {}
    s = torch.cuda.Stream()

    def step():
        sbl.sbl_linear(x, w, y=y, acc_out=acc, workspace=ws)
        sbl.sbl_linear_rmsnorm(x8, w, gd, y=y8, acc_out=acc8, workspace=ws8)
        out["tot"], _ = sbl.sbl_mask_monitor(w.mask_bits, w2.mask_bits, K, n, m)

    with torch.cuda.stream(s):
        step()
    s.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        step()
    for _ in range(3):
        acc.zero_(), acc8.zero_(), y.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert sbl.sbl_device_status() == 0
        assert np.array_equal(acc.cpu().numpy(), ref["acc"])
        assert_fp32_close(y.cpu().numpy(), ref["y"])
        assert np.array_equal(acc8.cpu().numpy(), acc_rms)
        assert_fp32_close(y8.cpu().numpy(), y_rms)
        assert out["tot"].cpu().tolist() == [changed, bad]
