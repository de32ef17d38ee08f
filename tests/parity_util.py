"""Helpers shared by the GPU parity tests: seeded inputs, oracle results and the
comparison rules (bit-exact integers, 1e-5 relative fp32, 2 ulp bf16)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_linear_layers_b200 import synthetic

FP32_RTOL = 1e-5
BF16_ULPS = 2


def to_dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def x_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def assert_fp32_close(y_gpu: np.ndarray, y_ref: np.ndarray, what: str = "y"):
    y_gpu = np.asarray(y_gpu, np.float64)
    err = np.abs(y_gpu - y_ref)
    bad = err > FP32_RTOL * np.abs(y_ref)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} elements beyond 1e-5 relative; first at {tuple(i)}: "
                             f"gpu {y_gpu[tuple(i)]!r} ref {y_ref[tuple(i)]!r}")


def _bf16_ordered(bits: np.ndarray) -> np.ndarray:
    b = bits.astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def assert_bf16_close(y_gpu_bits: np.ndarray, y_ref: np.ndarray, what: str = "y"):
    ref_bits = synthetic.f32_to_bf16_bits(y_ref.astype(np.float32))
    d = np.abs(_bf16_ordered(y_gpu_bits.view(np.uint16)) - _bf16_ordered(ref_bits))
    if (d > BF16_ULPS).any():
        i = np.argwhere(d > BF16_ULPS)[0]
        raise AssertionError(f"{what}: {(d > BF16_ULPS).sum()} bf16 elements beyond {BF16_ULPS} ulp; first at "
                             f"{tuple(i)}")


def layer_inputs(O, K, T, seed=0, outlier_p=0.0, tag=""):
    W = synthetic.latent_weights(O, K, seed=seed, tag=f"W{tag}{O}x{K}")
    xbits, xval = synthetic.activations(T, K, seed=seed, tag=f"x{tag}{T}x{K}", outlier_p=outlier_p)
    return W, xbits, xval


def oracle_layer(W, n, m, xval):
    packed, scale, mbits, Wt = oracle.prepare_weights(W, n, m)
    y, acc, xq, s = oracle.linear(xval, Wt, scale)
    return dict(packed=packed, scale=scale, mbits=mbits, Wt=Wt, y=y, acc=acc, xq=xq, s=s)


def oracle_acc(xq, Wt, chunk=4096):
    """The oracle's int32 accumulators x_q . W_t^T, taken in token chunks so the
    float64 operands of its (exact) matrix product stay a few hundred MB."""
    T = xq.shape[0]
    out = np.empty((T, Wt.shape[0]), np.int32)
    for t0 in range(0, T, chunk):
        out[t0:t0 + chunk] = oracle.int_contract(xq[t0:t0 + chunk], Wt)
    return out


def assert_layer_outputs(acc_gpu, y_gpu, yb_gpu_bits, xq, s, Wt, scale, what="", chunk=4096):
    """Every accumulator bit-exact, every fp32 y within 1e-5 relative and every
    bf16 y within 2 ulps of the oracle, chunk by chunk of tokens."""
    T = xq.shape[0]
    for t0 in range(0, T, chunk):
        sl = slice(t0, t0 + chunk)
        ref = oracle.int_contract(xq[sl], Wt)
        got = acc_gpu[sl]
        if not np.array_equal(got, ref):
            bad = np.argwhere(got != ref)[0]
            raise AssertionError(f"{what}: acc differs at token {t0 + bad[0]}, output {bad[1]}")
        y_ref = oracle.dequant(ref, scale, s[sl])
        if y_gpu is not None:
            assert_fp32_close(y_gpu[sl], y_ref, f"{what} y (tokens {t0}..)")
        if yb_gpu_bits is not None:
            assert_bf16_close(yb_gpu_bits[sl], y_ref, f"{what} bf16 y (tokens {t0}..)")
