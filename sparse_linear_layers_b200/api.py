"""PyTorch-facing calls of the Sparse-BitLinear library.

PyTorch provides device memory and streams; every call forwards raw pointers
to the C ABI (include/sbl.h) and the CUDA kernels do all the arithmetic.
The function names follow the C entry points.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

from . import _lib
from ._lib import check, lib

_PATHS = {"auto": _lib.SBL_PATH_AUTO, "decode": _lib.SBL_PATH_DECODE, "prefill": _lib.SBL_PATH_PREFILL,
          "prefill_1cta": _lib.SBL_PATH_PREFILL_1CTA, "prefill_pair": _lib.SBL_PATH_PREFILL_PAIR,
          "prefill_sparse": _lib.SBL_PATH_PREFILL_SPARSE}


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _need_cuda(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None, device=None) -> None:
    """Raise ValueError unless ``t`` is a contiguous CUDA tensor of ``dtype``
    (and, when given, exactly ``shape`` and on ``device``): the kernels write
    and read through raw pointers, so a tensor of the wrong size or on another
    GPU must never reach them."""
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the other operands on {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def _need_2d(t: torch.Tensor, name: str):
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D, got shape {tuple(t.shape)}")
    return t.shape


def _need_weights(w: "PreparedWeights", device) -> None:
    _need_cuda(w.packed, "packed", torch.uint8, (w.O, w.K // 4), device)
    _need_cuda(w.row_scale, "row_scale", torch.float32, (w.O,), device)


def _need_workspace(ws: torch.Tensor, device) -> None:
    if ws.dim() != 1:
        raise ValueError("workspace must be a 1-D uint8 tensor")
    _need_cuda(ws, "workspace", torch.uint8, None, device)


@dataclass
class PreparedWeights:
    """2-bit packed ternary weights of one layer plus its per-row scales."""
    packed: torch.Tensor      # uint8 [O, K/4]
    row_scale: torch.Tensor   # fp32 [O]
    n: int
    m: int
    K: int
    mask_bits: Optional[torch.Tensor] = None  # uint8 [O, K/8]

    @property
    def O(self) -> int:
        return self.packed.shape[0]


def sbl_prepare_weights(W: torch.Tensor, n: int, m: int, with_mask: bool = False,
                        out: Optional[PreparedWeights] = None, scale_bf16: bool = False,
                        scale_global: bool = False,
                        stream: Optional[torch.cuda.Stream] = None) -> PreparedWeights:
    """N:M mask, per-row absmean scale, ternarise and pack (one kernel).  With
    ``scale_bf16`` the scale is rounded to bf16 (the halo card's storage) first;
    with ``scale_global`` one scale, the mean of |W| over the whole matrix (the
    guide's module listing), serves every row."""
    O, K = _need_2d(W, "W")
    _need_cuda(W, "W", torch.float32)
    if out is None:
        packed = torch.empty((O, K // 4), dtype=torch.uint8, device=W.device)
        scale = torch.empty((O,), dtype=torch.float32, device=W.device)
        mask = torch.empty((O, K // 8), dtype=torch.uint8, device=W.device) if with_mask else None
        out = PreparedWeights(packed, scale, n, m, K, mask)
    if out.K != K or out.O != O:
        raise ValueError(f"out holds [{out.O}, {out.K}] weights, W is [{O}, {K}]")
    _need_weights(out, W.device)
    if out.mask_bits is not None:
        _need_cuda(out.mask_bits, "mask_bits", torch.uint8, (O, K // 8), W.device)
    mb = out.mask_bits.data_ptr() if out.mask_bits is not None else None
    check(lib.sbl_prepare_weights_ex(W.data_ptr(), O, K, n, m, out.packed.data_ptr(), out.row_scale.data_ptr(), mb,
                                     (_lib.SBL_PREP_SCALE_BF16 if scale_bf16 else 0) |
                                     (_lib.SBL_PREP_SCALE_GLOBAL if scale_global else 0), _stream(stream)),
          "sbl_prepare_weights")
    return out


def sbl_prepare_weights_grouped(Ws, n: int, m: int, outs=None, with_mask: bool = False,
                                stream: Optional[torch.cuda.Stream] = None):
    """sbl_prepare_weights for several latent matrices of the same K in one call
    (per-row scales); returns the list of PreparedWeights."""
    import ctypes
    G = len(Ws)
    if not 1 <= G <= _lib.SBL_MAX_GROUP:
        raise ValueError(f"between 1 and {_lib.SBL_MAX_GROUP} matrices, got {G}")
    K = _need_2d(Ws[0], "W[0]")[1]
    dev = Ws[0].device
    for g, W in enumerate(Ws):
        if _need_2d(W, f"W[{g}]")[1] != K:
            raise ValueError("every matrix must have the same K")
        _need_cuda(W, f"W[{g}]", torch.float32, None, dev)
    if outs is None:
        outs = [PreparedWeights(torch.empty((W.shape[0], K // 4), dtype=torch.uint8, device=dev),
                                torch.empty((W.shape[0],), dtype=torch.float32, device=dev), n, m, K,
                                torch.empty((W.shape[0], K // 8), dtype=torch.uint8, device=dev) if with_mask else None)
                for W in Ws]
    if len(outs) != G:
        raise ValueError("one output per matrix")
    for W, o in zip(Ws, outs):
        if o.K != K or o.O != W.shape[0]:
            raise ValueError("outputs must match the matrices' shapes")
        _need_weights(o, dev)
        if o.mask_bits is not None:
            _need_cuda(o.mask_bits, "mask_bits", torch.uint8, (o.O, K // 8), dev)
    ptrs = lambda ts: (ctypes.c_void_p * G)(*[t.data_ptr() if t is not None else None for t in ts])
    rows = (ctypes.c_int64 * G)(*[W.shape[0] for W in Ws])
    masks = ptrs([o.mask_bits for o in outs]) if any(o.mask_bits is not None for o in outs) else None
    check(lib.sbl_prepare_weights_grouped(G, ptrs(Ws), rows, K, n, m, ptrs([o.packed for o in outs]),
                                          ptrs([o.row_scale for o in outs]), masks, _stream(stream)),
          "sbl_prepare_weights_grouped")
    return outs


def sbl_quant_act(x: torch.Tensor, stream: Optional[torch.cuda.Stream] = None):
    """Per-token absmax int8 quantisation: returns (x_q int8 [T,K], s_tok fp32 [T])."""
    T, K = _need_2d(x, "x")
    _need_cuda(x, "x", torch.bfloat16)
    xq = torch.empty((T, K), dtype=torch.int8, device=x.device)
    s = torch.empty((T,), dtype=torch.float32, device=x.device)
    check(lib.sbl_quant_act(x.data_ptr(), T, K, xq.data_ptr(), s.data_ptr(), _stream(stream)), "sbl_quant_act")
    return xq, s


RMSNORM_EPS_F32 = 2.0 ** -23  # torch's default RMSNorm epsilon for float32 (machine epsilon)


def sbl_rmsnorm_quant_act(x: torch.Tensor, g: torch.Tensor, eps: float = RMSNORM_EPS_F32,
                          stream: Optional[torch.cuda.Stream] = None):
    """RMSNorm (weight g, fp32 [K]) then per-token absmax int8: (x_q int8 [T,K], s_tok fp32 [T])."""
    T, K = _need_2d(x, "x")
    _need_cuda(x, "x", torch.bfloat16)
    _need_cuda(g, "g", torch.float32, (K,), x.device)
    xq = torch.empty((T, K), dtype=torch.int8, device=x.device)
    s = torch.empty((T,), dtype=torch.float32, device=x.device)
    check(lib.sbl_rmsnorm_quant_act(x.data_ptr(), g.data_ptr(), float(eps), T, K, xq.data_ptr(), s.data_ptr(),
                                    _stream(stream)), "sbl_rmsnorm_quant_act")
    return xq, s


def sbl_linear_workspace_bytes(T: int, K: int, O: int, n: int, m: int) -> int:
    return int(lib.sbl_linear_workspace_bytes(T, K, O, n, m))


def workspace_for(T: int, K: int, O: int, n: int, m: int, device) -> torch.Tensor:
    """A workspace tensor of the size sbl_linear needs (256-byte aligned by the caching allocator)."""
    return torch.empty((max(1, sbl_linear_workspace_bytes(T, K, O, n, m)),), dtype=torch.uint8, device=device)


def sbl_linear(x: torch.Tensor, w: PreparedWeights, out_dtype: torch.dtype = torch.float32,
               y: Optional[torch.Tensor] = None, acc_out: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None, path: str = "auto",
               stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """y = dequant(int8(x) . W_t^T); ``acc_out`` (int32 [T,O]) receives the integer accumulators."""
    T, K = _need_2d(x, "x")
    _need_cuda(x, "x", torch.bfloat16)
    if K != w.K:
        raise ValueError(f"x has K={K}, weights were prepared with K={w.K}")
    _need_weights(w, x.device)
    O = w.O
    if y is None:
        y = torch.empty((T, O), dtype=out_dtype, device=x.device)
    if y.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("y must be float32 or bfloat16")
    _need_cuda(y, "y", y.dtype, (T, O), x.device)
    ydt = _lib.SBL_F32 if y.dtype == torch.float32 else _lib.SBL_BF16
    if acc_out is not None:
        _need_cuda(acc_out, "acc_out", torch.int32, (T, O), x.device)
    if workspace is None:
        workspace = workspace_for(T, K, O, w.n, w.m, x.device)
    _need_workspace(workspace, x.device)
    check(lib.sbl_linear_path(x.data_ptr(), T, K, w.packed.data_ptr(), w.row_scale.data_ptr(), O, w.n, w.m,
                              y.data_ptr(), ydt, acc_out.data_ptr() if acc_out is not None else None,
                              workspace.data_ptr(), workspace.numel(), _PATHS[path], _stream(stream)),
          "sbl_linear")
    return y


def sbl_linear_q(x_q: torch.Tensor, s_tok: torch.Tensor, w: PreparedWeights, out_dtype: torch.dtype = torch.float32,
                 y: Optional[torch.Tensor] = None, acc_out: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """sbl_linear on activations quantised already: x_q (int8 [T,K]) and s_tok
    (fp32 [T]) as sbl_quant_act returns them.  Needs K % 64 == 0."""
    T, K = _need_2d(x_q, "x_q")
    _need_cuda(x_q, "x_q", torch.int8)
    _need_cuda(s_tok, "s_tok", torch.float32, (T,), x_q.device)
    if K != w.K:
        raise ValueError(f"x_q has K={K}, weights were prepared with K={w.K}")
    _need_weights(w, x_q.device)
    O = w.O
    if y is None:
        y = torch.empty((T, O), dtype=out_dtype, device=x_q.device)
    if y.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("y must be float32 or bfloat16")
    _need_cuda(y, "y", y.dtype, (T, O), x_q.device)
    ydt = _lib.SBL_F32 if y.dtype == torch.float32 else _lib.SBL_BF16
    if acc_out is not None:
        _need_cuda(acc_out, "acc_out", torch.int32, (T, O), x_q.device)
    if workspace is None:
        workspace = workspace_for(T, K, O, w.n, w.m, x_q.device)
    _need_workspace(workspace, x_q.device)
    check(lib.sbl_linear_q(x_q.data_ptr(), s_tok.data_ptr(), T, K, w.packed.data_ptr(), w.row_scale.data_ptr(), O,
                           w.n, w.m, y.data_ptr(), ydt, acc_out.data_ptr() if acc_out is not None else None,
                           workspace.data_ptr(), workspace.numel(), _stream(stream)),
          "sbl_linear_q")
    return y


def _need_host_pair(host: torch.Tensor, dev: torch.Tensor, hname: str, dname: str) -> int:
    """Byte count of a host <-> device copy between two contiguous tensors of
    equal size in bytes, the host one in CPU memory, the other on a GPU."""
    if host.is_cuda or not dev.is_cuda:
        raise ValueError(f"{hname} must be a CPU tensor and {dname} a CUDA tensor")
    if not host.is_contiguous() or not dev.is_contiguous():
        raise ValueError(f"{hname} and {dname} must be contiguous")
    nb = host.numel() * host.element_size()
    if nb != dev.numel() * dev.element_size():
        raise ValueError(f"{hname} and {dname} differ in size ({nb} and {dev.numel() * dev.element_size()} bytes)")
    return nb


def copy_to_device(dst: torch.Tensor, src: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Asynchronous copy of the host tensor ``src`` (pinned for overlap) into
    the device tensor ``dst`` on the stream, through sbl_copy_to_device."""
    nb = _need_host_pair(src, dst, "src", "dst")
    check(lib.sbl_copy_to_device(dst.data_ptr(), src.data_ptr(), nb, _stream(stream)), "sbl_copy_to_device")
    return dst


def copy_to_host(dst: torch.Tensor, src: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Asynchronous copy of the device tensor ``src`` into the host tensor
    ``dst`` (pinned for overlap) on the stream, through sbl_copy_to_host;
    synchronise the stream before reading ``dst``."""
    nb = _need_host_pair(dst, src, "dst", "src")
    check(lib.sbl_copy_to_host(dst.data_ptr(), src.data_ptr(), nb, _stream(stream)), "sbl_copy_to_host")
    return dst


def sbl_linear_hostio(x_host: torch.Tensor, w: PreparedWeights, out_dtype: torch.dtype = torch.float32,
                      y_host: Optional[torch.Tensor] = None, x_dev: Optional[torch.Tensor] = None,
                      y_dev: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                      stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """sbl_linear with x and y in host memory (sbl_linear_hostio): copies
    ``x_host`` (bf16 [T, K], pinned for overlap) in, contracts, copies y out
    into ``y_host``, all enqueued on the stream; returns ``y_host``, valid once
    the stream has been synchronised.  ``x_dev``/``y_dev`` are the device
    staging buffers (allocated here when not given)."""
    T, K = _need_2d(x_host, "x_host")
    if x_host.dtype != torch.bfloat16 or x_host.is_cuda or not x_host.is_contiguous():
        raise ValueError("x_host must be a contiguous bf16 CPU tensor")
    if K != w.K:
        raise ValueError(f"x has K={K}, weights were prepared with K={w.K}")
    dev = w.packed.device
    _need_weights(w, dev)
    if out_dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("out_dtype must be float32 or bfloat16")
    if y_host is None:
        y_host = torch.empty((T, w.O), dtype=out_dtype, pin_memory=True)
    if x_dev is None:
        x_dev = torch.empty((T, K), dtype=torch.bfloat16, device=dev)
    if y_dev is None:
        y_dev = torch.empty((T, w.O), dtype=y_host.dtype, device=dev)
    if y_host.dtype != y_dev.dtype or y_host.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("y_host and y_dev must both be float32 or both bfloat16")
    _need_cuda(x_dev, "x_dev", torch.bfloat16, (T, K), dev)
    _need_cuda(y_dev, "y_dev", y_host.dtype, (T, w.O), dev)
    _need_host_pair(y_host, y_dev, "y_host", "y_dev")
    if workspace is None:
        workspace = workspace_for(T, K, w.O, w.n, w.m, dev)
    _need_workspace(workspace, dev)
    ydt = _lib.SBL_F32 if y_host.dtype == torch.float32 else _lib.SBL_BF16
    check(lib.sbl_linear_hostio(x_host.data_ptr(), T, K, x_dev.data_ptr(), w.packed.data_ptr(), w.row_scale.data_ptr(),
                                w.O, w.n, w.m, y_dev.data_ptr(), y_host.data_ptr(), ydt, workspace.data_ptr(),
                                workspace.numel(), _stream(stream)), "sbl_linear_hostio")
    return y_host


def sbl_linear_grouped(x: torch.Tensor, ws, out_dtype: torch.dtype = torch.float32, ys=None, acc_outs=None,
                       workspace: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None):
    """Several layers that read the same x (q/k/v, gate/up) in one call: x is
    quantised once; returns the list of y [T, O_g].  Each result is exactly
    sbl_linear's for that layer.  ``ws``: PreparedWeights with one N:M
    pattern and one K; ``acc_outs``: None or a list (entries may be None)."""
    import ctypes
    T, K = _need_2d(x, "x")
    _need_cuda(x, "x", torch.bfloat16)
    G = len(ws)
    if not 1 <= G <= _lib.SBL_MAX_GROUP:
        raise ValueError(f"between 1 and {_lib.SBL_MAX_GROUP} layers, got {G}")
    n, m = ws[0].n, ws[0].m
    for w in ws:
        if w.K != K or (w.n, w.m) != (n, m):
            raise ValueError("every layer must have the activations' K and one N:M pattern")
        _need_weights(w, x.device)
    if ys is None:
        ys = [torch.empty((T, w.O), dtype=out_dtype, device=x.device) for w in ws]
    if len(ys) != G or (acc_outs is not None and len(acc_outs) != G):
        raise ValueError("one output (and accumulator) per layer")
    for g, (w, yg) in enumerate(zip(ws, ys)):
        if yg.dtype not in (torch.float32, torch.bfloat16) or yg.dtype != ys[0].dtype:
            raise ValueError("outputs must all be float32 or all bfloat16")
        _need_cuda(yg, f"y[{g}]", yg.dtype, (T, w.O), x.device)
        if acc_outs is not None and acc_outs[g] is not None:
            _need_cuda(acc_outs[g], f"acc_out[{g}]", torch.int32, (T, w.O), x.device)
    if workspace is None:
        workspace = torch.empty((max(1, int(lib.sbl_linear_grouped_workspace_bytes(T, K))),), dtype=torch.uint8,
                                device=x.device)
    _need_workspace(workspace, x.device)
    ptrs = lambda ts: (ctypes.c_void_p * G)(*[t.data_ptr() if t is not None else None for t in ts])
    rows = (ctypes.c_int64 * G)(*[w.O for w in ws])
    accs = ptrs(acc_outs) if acc_outs is not None else None
    ydt = _lib.SBL_F32 if ys[0].dtype == torch.float32 else _lib.SBL_BF16
    check(lib.sbl_linear_grouped(x.data_ptr(), T, K, G, ptrs([w.packed for w in ws]), ptrs([w.row_scale for w in ws]),
                                 rows, n, m, ptrs(ys), ydt, accs, workspace.data_ptr(), workspace.numel(),
                                 _stream(stream)), "sbl_linear_grouped")
    return ys


def sbl_linear_rmsnorm(x: torch.Tensor, w: PreparedWeights, g: torch.Tensor, eps: float = RMSNORM_EPS_F32,
                       out_dtype: torch.dtype = torch.float32, y: Optional[torch.Tensor] = None,
                       acc_out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                       path: str = "auto", stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """The guide module's forward: y = dequant(int8(RMSNorm(x; g, eps)) . W_t^T)."""
    T, K = _need_2d(x, "x")
    _need_cuda(x, "x", torch.bfloat16)
    if K != w.K or g.numel() != K:
        raise ValueError(f"x has K={K}; weights were prepared with K={w.K}; g has {g.numel()} entries")
    _need_cuda(g, "g", torch.float32, (K,), x.device)
    _need_weights(w, x.device)
    O = w.O
    if y is None:
        y = torch.empty((T, O), dtype=out_dtype, device=x.device)
    if y.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("y must be float32 or bfloat16")
    _need_cuda(y, "y", y.dtype, (T, O), x.device)
    ydt = _lib.SBL_F32 if y.dtype == torch.float32 else _lib.SBL_BF16
    if acc_out is not None:
        _need_cuda(acc_out, "acc_out", torch.int32, (T, O), x.device)
    if workspace is None:
        workspace = workspace_for(T, K, O, w.n, w.m, x.device)
    _need_workspace(workspace, x.device)
    check(lib.sbl_linear_rmsnorm(x.data_ptr(), g.data_ptr(), float(eps), T, K, w.packed.data_ptr(),
                                 w.row_scale.data_ptr(), O, w.n, w.m, y.data_ptr(), ydt,
                                 acc_out.data_ptr() if acc_out is not None else None, workspace.data_ptr(),
                                 workspace.numel(), _PATHS[path], _stream(stream)), "sbl_linear_rmsnorm")
    return y


def sbl_mask_monitor(old_bits: torch.Tensor, new_bits: torch.Tensor, K: int, n: int, m: int, per_row: bool = False,
                     stream: Optional[torch.cuda.Stream] = None):
    """Mask change and verification on the device: (totals int64 [2] = [changed
    positions, groups not keeping exactly N], row_changed int32 [O] or None).
    Nothing is copied to the host."""
    O = _need_2d(old_bits, "old_bits")[0]
    _need_cuda(old_bits, "old_bits", torch.uint8, (O, K // 8))
    _need_cuda(new_bits, "new_bits", torch.uint8, (O, K // 8), old_bits.device)
    totals = torch.empty(2, dtype=torch.int64, device=old_bits.device)
    rows = torch.empty(O, dtype=torch.int32, device=old_bits.device) if per_row else None
    check(lib.sbl_mask_monitor(old_bits.data_ptr(), new_bits.data_ptr(), O, K, n, m, totals.data_ptr(),
                               rows.data_ptr() if rows is not None else None, _stream(stream)), "sbl_mask_monitor")
    return totals, rows


def sbl_linear_backward_workspace_bytes(T: int, O: int, K: int, need_dx: bool = True, need_dw: bool = True) -> int:
    return int(lib.sbl_linear_backward_workspace_bytes(T, O, K, int(need_dx), int(need_dw)))


def sbl_linear_backward(dY: torch.Tensor, x_q: torch.Tensor, s_tok: torch.Tensor, w: PreparedWeights,
                        need_dx: bool = True, need_dw: bool = True, dw_ternary: bool = False,
                        dX: Optional[torch.Tensor] = None, dW: Optional[torch.Tensor] = None,
                        tensor_cores: bool = True, workspace: Optional[torch.Tensor] = None,
                        stream: Optional[torch.cuda.Stream] = None):
    """Straight-through gradients of sbl_linear: (dX fp32 [T,K] or None, dW fp32 [O,K] or None).

    dX = dY . (scale * W_t) and dW = dY^T . (x_q / s_t) over every weight position
    (``dw_ternary``: dW rows scaled by scale_o once more, the guide module's form).
    ``x_q``/``s_tok`` are the forward's quantised activations in natural order
    (sbl_quant_act or sbl_rmsnorm_quant_act).  ``tensor_cores`` (default) runs
    the tcgen05 path (sbl_linear_backward_ws; a workspace of
    sbl_linear_backward_workspace_bytes() is allocated unless given), else the
    CUDA-core kernels (sbl_linear_backward)."""
    T, O = _need_2d(dY, "dY")
    K = w.K
    if O != w.O or x_q.shape != (T, K) or s_tok.shape != (T,):
        raise ValueError(f"dY {tuple(dY.shape)}, x_q {tuple(x_q.shape)} and s_tok {tuple(s_tok.shape)} do not match "
                         f"weights with O={w.O}, K={K}")
    _need_cuda(dY, "dY", torch.float32)
    dev = dY.device
    _need_cuda(x_q, "x_q", torch.int8, (T, K), dev)
    _need_cuda(s_tok, "s_tok", torch.float32, (T,), dev)
    _need_weights(w, dev)
    if not (need_dx or need_dw):
        raise ValueError("ask for dX, dW or both")
    if need_dx:
        dX = torch.empty((T, K), dtype=torch.float32, device=dev) if dX is None else dX
        _need_cuda(dX, "dX", torch.float32, (T, K), dev)
    if need_dw:
        dW = torch.empty((O, K), dtype=torch.float32, device=dev) if dW is None else dW
        _need_cuda(dW, "dW", torch.float32, (O, K), dev)
    flags = _lib.SBL_BWD_DW_TERNARY if dw_ternary else 0
    if tensor_cores:
        if workspace is None:
            workspace = torch.empty((max(1, sbl_linear_backward_workspace_bytes(T, O, K, need_dx, need_dw)),),
                                    dtype=torch.uint8, device=dev)
        _need_workspace(workspace, dev)
        check(lib.sbl_linear_backward_ws(dY.data_ptr(), T, O, x_q.data_ptr(), s_tok.data_ptr(), K,
                                         w.packed.data_ptr(), w.row_scale.data_ptr(), dX.data_ptr() if need_dx else None,
                                         dW.data_ptr() if need_dw else None, flags, workspace.data_ptr(),
                                         workspace.numel(), _stream(stream)), "sbl_linear_backward_ws")
    else:
        check(lib.sbl_linear_backward(dY.data_ptr(), T, O, x_q.data_ptr(), s_tok.data_ptr(), K, w.packed.data_ptr(),
                                      w.row_scale.data_ptr(), dX.data_ptr() if need_dx else None,
                                      dW.data_ptr() if need_dw else None, flags, _stream(stream)),
              "sbl_linear_backward")
    return (dX if need_dx else None), (dW if need_dw else None)


_PATH_NAMES = {v: k for k, v in _PATHS.items()}


def sbl_linear_plan(T: int, K: int, O: int, n: int, m: int, workspace_bytes: Optional[int] = None) -> str:
    """Name of the path sbl_linear takes for these sizes ("decode", "prefill_1cta",
    "prefill_pair" or "prefill_sparse"); the default workspace is workspace_for's."""
    if workspace_bytes is None:
        workspace_bytes = max(1, sbl_linear_workspace_bytes(T, K, O, n, m))
    r = int(lib.sbl_linear_plan(T, K, O, n, m, workspace_bytes))
    if r < 0:
        raise _lib.SblError(-r, "sbl_linear_plan")
    return _PATH_NAMES[r]


def sbl_decode_max_tokens() -> int:
    return int(lib.sbl_decode_max_tokens())


def sbl_device_status(stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronise and return (and clear) the device status code (0 = ok)."""
    return int(lib.sbl_device_status(_stream(stream)))


def sbl_selftest_bounded_wait(max_polls: int = 1000, stream: Optional[torch.cuda.Stream] = None) -> int:
    return int(lib.sbl_selftest_bounded_wait(max_polls, _stream(stream)))
