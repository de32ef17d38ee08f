"""Sparse-BitLinear forward for NVIDIA B200 (sm_100a).

y = dequant(int8(x) . ternary_NM(W)^T) behind a C ABI (include/sbl.h) with
hand-written CUDA kernels: fused weight preparation, per-token activation
quantisation (optionally after RMSNorm, as the guide's module does), decode
paths on CUDA cores and the warp-level MMA, tcgen05 tensor-core prefill, a
mask monitor and the straight-through backward of the training path.

The library entry points (sbl_prepare_weights, sbl_quant_act, sbl_linear, ...)
load libsbl.so on first use and raise ImportError if it has not been built;
there is no CPU fallback.  ``synthetic`` (seeded input generators) needs no
GPU library.
"""
__version__ = "0.1.0"

_API = ("PreparedWeights", "copy_to_device", "copy_to_host", "sbl_decode_max_tokens", "sbl_device_status", "sbl_linear", "sbl_linear_backward", "sbl_linear_backward_workspace_bytes", "sbl_linear_grouped", "sbl_linear_hostio", "sbl_linear_plan", "sbl_linear_q",
        "sbl_linear_rmsnorm", "sbl_linear_workspace_bytes", "sbl_mask_monitor", "sbl_prepare_weights", "sbl_prepare_weights_grouped", "sbl_quant_act",
        "sbl_rmsnorm_quant_act", "sbl_selftest_bounded_wait", "workspace_for", "RMSNORM_EPS_F32", "SblError")


_TRAIN = ("SparseBitLinear", "SparseBitLinearFunction")


def __getattr__(name):
    if name in _TRAIN:
        from . import train
        return getattr(train, name)
    if name in _API:
        from . import api
        from ._lib import SblError
        return SblError if name == "SblError" else getattr(api, name)
    raise AttributeError(name)


__all__ = list(_API) + list(_TRAIN)
