"""The C ABI library loads, exports every entry point include/sbl.h declares, and
rejects bad arguments on the host before touching a device (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sbl.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sbl_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("sbl_prepare_weights", "sbl_quant_act", "sbl_linear", "sbl_linear_workspace_bytes"):
        assert must in names


def test_library_exports_every_declared_symbol():
    from sparse_linear_layers_b200 import _lib
    raw = ctypes.CDLL(_lib.LIB_PATH)
    for name in _declared():
        assert hasattr(raw, name), name
    assert set(_declared()) == set(_lib.SIGNATURES), "binding signatures out of sync with sbl.h"


def test_version_and_status_strings():
    from sparse_linear_layers_b200._lib import lib, status_string
    assert b"sm_100a" in lib.sbl_version()
    for code in range(7):
        assert status_string(code)
    assert status_string(99) == "unknown status"


def test_workspace_bytes():
    from sparse_linear_layers_b200._lib import lib
    assert lib.sbl_linear_workspace_bytes(0, 896, 896, 3, 4) == 0
    # x_q (T*K rounded to 256) + s_tok (T*4 rounded to 256)
    assert lib.sbl_linear_workspace_bytes(2048, 896, 896, 3, 4) == 2048 * 896 + 8192
    assert lib.sbl_linear_workspace_bytes(3, 48, 16, 2, 4) == 256 + 256


@pytest.mark.parametrize("args,code", [
    # (O, K, n, m)
    ((-1, 64, 2, 4), 1),     # negative O
    ((8, 0, 2, 4), 1),       # K == 0
    ((8, 40, 2, 4), 1),      # K % 16 != 0
    ((8, 64, 1, 4), 2),      # unsupported N:M
    ((8, 64, 5, 8), 2),
    ((8, 1 << 25, 2, 4), 2), # K beyond the int32-accumulator bound
])
def test_prepare_rejects_on_host(args, code):
    from sparse_linear_layers_b200._lib import lib
    O, K, n, m = args
    assert lib.sbl_prepare_weights(None, O, K, n, m, None, None, None, None) == code


def test_prepare_ex_rejects_unknown_flags():
    from sparse_linear_layers_b200._lib import lib
    p = 4096
    assert lib.sbl_prepare_weights_ex(p, 8, 64, 2, 4, p, p, None, 4, None) == 1
    assert lib.sbl_prepare_weights_ex(p, 8, 64, 2, 4, p, p, None, -1, None) == 1
    assert lib.sbl_prepare_weights_ex(p, 1 << 20, 4096, 2, 4, p, p, None, 2, None) == 2  # global scale: O*K >= 2^32


def test_zero_sizes_are_noops_without_a_device():
    from sparse_linear_layers_b200._lib import lib
    assert lib.sbl_prepare_weights(None, 0, 64, 2, 4, None, None, None, None) == 0
    assert lib.sbl_quant_act(None, 0, 64, None, None, None) == 0
    assert lib.sbl_linear(None, 0, 64, None, None, 16, 2, 4, None, 0, None, None, 0, None) == 0
    assert lib.sbl_linear(None, 4, 64, None, None, 0, 2, 4, None, 0, None, None, 0, None) == 0


def test_linear_rejects_on_host():
    from sparse_linear_layers_b200._lib import lib
    L = lib.sbl_linear_path
    p = 4096  # a fake, 16-byte aligned address: never dereferenced, validation fails first
    # bad output dtype
    assert L(p, 4, 64, p, p, 16, 2, 4, p, 7, None, p, 1 << 20, 0, None) == 1
    # bad path
    assert L(p, 4, 64, p, p, 16, 2, 4, p, 0, None, p, 1 << 20, 9, None) == 1
    # prefill needs K % 64 == 0
    assert L(p, 4, 48, p, p, 16, 2, 4, p, 0, None, p, 1 << 20, 2, None) == 2
    # unaligned y
    assert L(p, 4, 64, p, p, 16, 2, 4, p + 4, 0, None, p, 1 << 20, 0, None) == 1
    # workspace too small / unaligned
    assert L(p, 4, 64, p, p, 16, 2, 4, p, 0, None, p, 16, 0, None) == 6
    assert L(p, 4, 64, p, p, 16, 2, 4, p, 0, None, p + 16, 1 << 20, 0, None) == 6
    assert L(p, 4, 64, p, p, 16, 2, 4, p, 0, None, None, 1 << 20, 0, None) == 6


def test_rmsnorm_rejects_on_host():
    from sparse_linear_layers_b200._lib import lib
    p = 4096
    R = lib.sbl_rmsnorm_quant_act
    assert R(None, None, 1e-6, 0, 64, None, None, None) == 0          # T == 0: nothing to do
    assert R(p, p, 1e-6, 4, 40, p, p, None) == 1                       # K % 16 != 0
    assert R(p, p, -1.0, 4, 64, p, p, None) == 1                       # negative eps
    assert R(p, p, float("nan"), 4, 64, p, p, None) == 1               # NaN eps
    assert R(p, p + 4, 1e-6, 4, 64, p, p, None) == 1                   # unaligned g
    L = lib.sbl_linear_rmsnorm
    assert L(p, None, 1e-6, 4, 64, p, p, 16, 2, 4, p, 0, None, p, 1 << 20, 0, None) == 1   # g is required
    assert L(p, p, -1.0, 4, 64, p, p, 16, 2, 4, p, 0, None, p, 1 << 20, 0, None) == 1     # negative eps
    assert L(p, p, 1e-6, 4, 40, p, p, 16, 2, 4, p, 0, None, p, 1 << 20, 0, None) == 1     # K % 16 != 0
    assert L(p, p, 1e-6, 4, 48, p, p, 16, 2, 4, p, 0, None, p, 1 << 20, 1, None) == 2     # decode needs K % 64
    assert L(p, p, 1e-6, 4, 64, p, p, 16, 2, 4, p, 0, None, p, 16, 0, None) == 6          # workspace too small


def test_mask_monitor_rejects_on_host():
    from sparse_linear_layers_b200._lib import lib
    p = 4096
    M = lib.sbl_mask_monitor
    assert M(p, p, 8, 40, 2, 4, p, None, None) == 1          # K % 16 != 0
    assert M(p, p, 8, 64, 5, 8, p, None, None) == 2          # unsupported pattern
    assert M(p, p, 8, 64, 2, 4, None, None, None) == 1       # totals required
    assert M(p + 8, p, 8, 64, 2, 4, p, None, None) == 1      # unaligned bitmap
    assert M(p, p, 8, 64, 2, 4, p, p + 2, None) == 1         # unaligned row counts
    assert M(p, p, -1, 64, 2, 4, p, None, None) == 1         # negative O


def _has_device():
    import torch
    return torch.cuda.is_available()


def test_backward_rejects_on_host():
    from sparse_linear_layers_b200._lib import lib
    p = 4096
    B = lib.sbl_linear_backward
    # (dY, T, O, x_q, s_tok, K, packed, row_scale, dX, dW, flags, stream)
    assert B(p, 4, 8, p, p, 40, p, p, p, p, 0, None) == 1          # K % 16 != 0
    assert B(p, -1, 8, p, p, 64, p, p, p, p, 0, None) == 1         # negative T
    assert B(p, 4, -1, p, p, 64, p, p, p, p, 0, None) == 1         # negative O
    assert B(p, 4, 8, p, p, 64, p, p, None, None, 0, None) == 1    # no output asked for
    assert B(p, 4, 8, p, p, 64, p, p, p, p, 2, None) == 1          # unknown flag
    assert B(p, 4, 8, p, p, 64, None, p, p, None, 0, None) == 1    # dX needs the packed weights
    assert B(p, 4, 8, None, p, 64, p, p, None, p, 0, None) == 1    # dW needs x_q
    assert B(p, 4, 8, p, None, 64, p, p, None, p, 0, None) == 1    # dW needs s_tok
    assert B(p, 4, 8, p, p, 64, p, None, None, p, 1, None) == 1    # the ternary form needs row_scale
    assert B(p + 4, 4, 8, p, p, 64, p, p, p, None, 0, None) == 1   # unaligned dY
    assert B(p, 4, 8, p, p, 64, p, p, p + 8, None, 0, None) == 1   # unaligned dX
    assert B(p, 4, 8, p, p, 1 << 25, p, p, p, None, 0, None) == 2  # K above the library's limit
    # both outputs and the ternary flag: every host check passes and the missing
    # device is reported (only without a device: these pointers are not real)
    if not _has_device():
        assert B(p, 4, 8, p, p, 64, p, p, p, p, 1, None) == 4
        assert B(p, 4, 8, p, p, 64, p, p, p + 16, p + 32, 0, None) == 4
    # nothing to write: accepted before any device work
    assert B(None, 0, 8, None, None, 64, None, None, p, None, 0, None) == 0
    assert B(None, 4, 0, None, None, 64, None, None, None, p, 0, None) == 0


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    import importlib
    from sparse_linear_layers_b200 import _lib
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(ImportError):
        _lib._load()
    importlib.reload(_lib)  # restore the real module state


def test_training_layer_has_no_cpu_fallback():
    """The autograd layer reaches the library for every step; CPU tensors are refused."""
    import torch
    import sparse_linear_layers_b200 as sbl
    layer = sbl.SparseBitLinear(64, 128, 2, 4)
    assert tuple(layer.weight.shape) == (128, 64) and layer.weight.dtype == torch.float32
    with pytest.raises(ValueError, match="CUDA"):
        layer(torch.zeros(3, 64))


def test_grouped_rejects_on_host():
    import ctypes as C
    from sparse_linear_layers_b200 import _lib
    lib = _lib.lib
    src = open(HEADER).read()
    assert int(re.search(r"#define SBL_MAX_GROUP (\d+)", src).group(1)) == _lib.SBL_MAX_GROUP
    G = 3
    p = 4096  # never dereferenced: host checks come first
    ptrs = (C.c_void_p * G)(p, p, p)
    rows = (C.c_int64 * G)(896, 128, 128)
    args = lambda T, K, g, n=3, m=4, rows=rows, ws=None, wsb=0: lib.sbl_linear_grouped(
        p, T, K, g, ptrs, ptrs, rows, n, m, ptrs, 0, None, ws, wsb, None)
    assert args(2048, 896, 0) == 1                       # no layers
    assert args(2048, 896, _lib.SBL_MAX_GROUP + 1) == 1  # too many
    assert args(2048, 40, G) == 1                        # K % 16
    assert args(2048, 896, G, n=1) == 2                  # pattern
    assert args(0, 896, G) == 0                          # no tokens: nothing to do
    assert args(2048, 896, G) == 6                       # prefill sizes need the workspace
    assert args(2048, 896, G, ws=p, wsb=16) == 6
    assert args(2048, 896, G, rows=(C.c_int64 * G)(0, 0, 0)) == 0
    assert args(2048, 896, G, rows=(C.c_int64 * G)(-1, 0, 0)) == 1
    assert lib.sbl_linear_grouped_workspace_bytes(2048, 896) == lib.sbl_linear_workspace_bytes(2048, 896, 896, 3, 4)


def test_backward_ws_rejects_on_host():
    from sparse_linear_layers_b200._lib import lib
    p = 4096
    B = lib.sbl_linear_backward_ws
    assert B(p, 8, 16, p, p, 64, p, p, p, p, 4, p, 1 << 20, None) == 1      # unknown flag
    assert B(p, 8, 16, p, p, 40, p, p, p, p, 0, p, 1 << 20, None) == 1      # K % 16
    assert B(p, 8, 16, p, p, 64, p, p, None, None, 0, p, 1 << 20, None) == 1  # no output asked for
    assert B(p, 8, 16, p, p, 64, p, p, p, p, 0, None, 0, None) == 6          # no workspace
    assert B(p, 8, 16, p, p, 64, p, p, p, p, 0, p + 16, 1 << 20, None) == 6  # unaligned workspace
    need = lib.sbl_linear_backward_workspace_bytes(8, 16, 64, 1, 1)
    assert need > 0 and B(p, 8, 16, p, p, 64, p, p, p, p, 0, p, need - 1, None) == 6
    assert B(p, 1 << 22, 16, p, p, 64, p, p, p, p, 0, p, 1 << 40, None) == 2  # T beyond the tensor-core path
    # workspace: A' [M, 3 * 64] and B [64, 64] bf16 per gradient, the larger of the two
    assert lib.sbl_linear_backward_workspace_bytes(8, 16, 64, 1, 0) == 3 * 8 * 64 * 2 + 64 * 64 * 2
    assert lib.sbl_linear_backward_workspace_bytes(0, 16, 64, 1, 1) == 0


def test_prepare_grouped_rejects_on_host():
    import ctypes as C
    from sparse_linear_layers_b200 import _lib
    lib = _lib.lib
    p = 4096
    G = 2
    ptrs = (C.c_void_p * G)(p, p)
    P = lambda g, rows, K=64, n=2, m=4: lib.sbl_prepare_weights_grouped(g, ptrs, rows, K, n, m, ptrs, ptrs, None, None)
    ok_rows = (C.c_int64 * G)(8, 8)
    assert P(0, ok_rows) == 1                                  # no matrices
    assert P(_lib.SBL_MAX_GROUP + 1, ok_rows) == 1
    assert P(G, ok_rows, K=40) == 1                            # K % 16
    assert P(G, ok_rows, n=5, m=8) == 2                        # pattern
    assert P(G, (C.c_int64 * G)(-1, 8)) == 1                   # negative rows
    assert P(G, (C.c_int64 * G)(0, 0)) == 0                    # nothing to do
    bad = (C.c_void_p * G)(p + 4, p)                           # unaligned latent weights
    assert lib.sbl_prepare_weights_grouped(G, bad, ok_rows, 64, 2, 4, ptrs, ptrs, None, None) == 1


def test_host_copies_reject_on_host():
    from sparse_linear_layers_b200._lib import lib
    p = 4096  # a fake address: validation fails (or the size is 0) before it could be read
    assert lib.sbl_copy_to_device(None, None, 0, None) == 0
    assert lib.sbl_copy_to_host(None, None, 0, None) == 0
    assert lib.sbl_copy_to_device(None, p, 16, None) == 1
    assert lib.sbl_copy_to_device(p, None, 16, None) == 1
    assert lib.sbl_copy_to_host(None, p, 16, None) == 1
    assert lib.sbl_copy_to_host(p, None, 16, None) == 1


def test_linear_hostio_rejects_on_host():
    from sparse_linear_layers_b200._lib import lib
    H = lib.sbl_linear_hostio
    p = 4096
    # empty problems enqueue nothing
    assert H(None, 0, 64, None, None, None, 16, 2, 4, None, None, 0, None, 0, None) == 0
    assert H(None, 4, 64, None, None, None, 0, 2, 4, None, None, 0, None, 0, None) == 0
    # sbl_linear's checks run first: output dtype, alignment, workspace
    assert H(p, 4, 64, p, p, p, 16, 2, 4, p, p, 7, p, 1 << 20, None) == 1
    assert H(p, 4, 64, p + 4, p, p, 16, 2, 4, p, p, 0, p, 1 << 20, None) == 1
    assert H(p, 4, 64, p, p, p, 16, 2, 4, p, p, 0, p, 16, None) == 6
    # then the host buffers
    assert H(None, 4, 64, p, p, p, 16, 2, 4, p, p, 0, p, 1 << 20, None) == 1
    assert H(p, 4, 64, p, p, p, 16, 2, 4, p, None, 0, p, 1 << 20, None) == 1


def test_linear_q_rejects_on_host():
    from sparse_linear_layers_b200._lib import lib
    Q = lib.sbl_linear_q
    p = 4096
    # empty problems enqueue nothing
    assert Q(None, None, 0, 64, None, None, 16, 2, 4, None, 0, None, None, 0, None) == 0
    assert Q(None, None, 4, 64, None, None, 0, 2, 4, None, 0, None, None, 0, None) == 0
    # K % 64 != 0, an unsupported pattern, a bad output dtype
    assert Q(p, p, 4, 48, p, p, 16, 2, 4, p, 0, None, p, 1 << 20, None) == 2
    assert Q(p, p, 4, 64, p, p, 16, 1, 4, p, 0, None, p, 1 << 20, None) == 2
    assert Q(p, p, 4, 64, p, p, 16, 2, 4, p, 7, None, p, 1 << 20, None) == 1
    # missing or unaligned activations and scales
    assert Q(None, p, 4, 64, p, p, 16, 2, 4, p, 0, None, p, 1 << 20, None) == 1
    assert Q(p, None, 4, 64, p, p, 16, 2, 4, p, 0, None, p, 1 << 20, None) == 1
    assert Q(p + 8, p, 4, 64, p, p, 16, 2, 4, p, 0, None, p, 1 << 20, None) == 1
    assert Q(p, p + 4, 4, 64, p, p, 16, 2, 4, p, 0, None, p, 1 << 20, None) == 1
    assert Q(p, p, 4, 64, p, p, 16, 2, 4, p, 0, p + 4, p, 1 << 20, None) == 1
    # workspace missing, too small or unaligned
    assert Q(p, p, 4, 64, p, p, 16, 2, 4, p, 0, None, None, 1 << 20, None) == 6
    assert Q(p, p, 4, 64, p, p, 16, 2, 4, p, 0, None, p, 16, None) == 6
    assert Q(p, p, 4, 64, p, p, 16, 2, 4, p, 0, None, p + 16, 1 << 20, None) == 6
    # negative sizes
    assert Q(p, p, -1, 64, p, p, 16, 2, 4, p, 0, None, p, 1 << 20, None) == 1
