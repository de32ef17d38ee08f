"""CPU oracle for the Sparse-BitLinear forward — TEST INFRASTRUCTURE ONLY.

Only the test-suite, the package smoke check and the benchmark's CPU-baseline
leg may import this module.  The library never does: it shares no code,
table or helper with the CUDA path and must not be used as a fallback.

What it computes (the Sparse-BitLinear operator of "Sparse-BitNet Guide: 1.58-Bit
LLMs Meet 2:4 Sparsity", section "Mathematical Formulation of Sparse-BitLinear",
with the per-row scale of the halo-sparse-bitnet-3:4-500m card's "Recipe" and
the 2-bit code table of its "What ships with this repo / Packed vs raw"):

    mask      keep the N largest |W| of every M contiguous input-dim weights
    scale_i   absmean of the kept |W| of row i
    W_t       clip(round(W / scale), -1, 1) on kept positions, 0 elsewhere
    packed    2 bits per weight, 00 = 0, 01 = +1, 10 = -1, 4 codes per byte
    x_q       clip(round(x * 127 / max|x|), -128, 127) per token
    (RMSNorm) x <- x / sqrt(mean(x^2) + eps) * g before x_q, as the guide's
              module does (optional, the fused RMSNorm entry points)
    acc       x_q . W_t^T in integers
    y         acc * scale_i / s_t,  s_t = 127 / max|x_t|
    (backward) straight-through gradients dX = dY . (scale * W_t),
              dW = dY^T . (x_q / s_t) (the training path)

Readings taken where the pages are silent or disagree (each one is listed
with its reason in the design notes):

* ties in the Top-N go to the lower index; -0 and +0 tie;
* scale: per row over the kept weights; sum of |w| formed exactly and
  rounded once to double (``math.fsum``), divided by the kept count in double,
  rounded to float, then clamped below at 1e-5 (the epsilon of the guide's
  module listing);
* round() is round-half-to-even (``torch.round`` semantics in the guide's
  listing); W / scale is evaluated in double, which decides |W|/scale against
  the 0.5 threshold exactly for float inputs;
* the activation scale and x * s are float32 operations (the guide's module
  computes in the activation's float type); x is bf16 widened exactly;
* 2-bit codes are stored LSB-first: weight k sits in byte k // 4 at bits
  2 (k % 4) .. 2 (k % 4) + 1; mask bits: bit k % 8 of byte k // 8;
* dequantisation in double: y = acc * scale / s_t;
* RMSNorm (the guide's module normalises x with torch's RMSNorm before the
  absmax; the pages give no arithmetic order): the sum of squares is the
  exact sum rounded once to float32, which no summation order changes; then
  float32 steps, each an IEEE-rounded operation: mean = sum / K;
  inv = 1 / sqrt(mean + eps); x_norm = (x * inv) * g.
* training (straight-through) backward: every quantiser acts as the identity,
  so dX = dY . (scale * W_t) and dW = dY^T . (x_q / s_t) over all positions,
  masked ones included; optionally (the guide's module) dW taken at the
  ternary matrix, i.e. scaled once more by scale_o.

Every function here is pinned by tests that do not call it to build their
expected values (worked examples from the pages, closed forms, brute force).
Parity pinned for all functions; none is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

EPS_SCALE = np.float32(1e-5)   # clamp of the weight absmean (guide's module listing)
EPS_ACT = np.float32(1e-5)     # clamp of the activation absmax (guide's module listing)
SUPPORTED_NM = ((2, 4), (3, 4), (6, 8), (4, 8))


def _check_nm(K: int, n: int, m: int) -> None:
    if (n, m) not in SUPPORTED_NM:
        raise ValueError(f"unsupported N:M pattern {n}:{m}")
    if K % m or K % 4:
        raise ValueError("K must be a multiple of M and of 4")


def nm_mask(W: np.ndarray, n: int, m: int) -> np.ndarray:
    """Boolean keep-mask [O, K]: Top-N |W| in each group of M input-dim weights.

    Sparse-BitNet Guide, "Mathematical Formulation of Sparse-BitLinear", the
    mask equation (Top-N indices of |W[i, Mk : Mk+M]|); Sparse-BitNet README,
    "How It Works / N:M Structured Sparsity".  Equal magnitudes: the lower
    index is kept first (a stable sort on -|w|).
    """
    W = np.asarray(W, dtype=np.float32)
    O, K = W.shape
    _check_nm(K, n, m)
    if not np.all(np.isfinite(W)):
        raise ValueError("non-finite weight")
    a = np.abs(W.astype(np.float64)).reshape(O, K // m, m)
    order = np.argsort(-a, axis=-1, kind="stable")
    keep = np.zeros(a.shape, dtype=bool)
    np.put_along_axis(keep, order[..., :n], True, axis=-1)
    return keep.reshape(O, K)


def row_scale(W: np.ndarray, mask: np.ndarray) -> np.ndarray:
    """fp32 [O]: per-row absmean of the kept weights, clamped at 1e-5.

    halo-sparse-bitnet-3:4-500m card, "Recipe" (per-row absmean scale); the
    guide's gamma equation gives the absmean form.  The sum is exact up to one
    final rounding to double (``math.fsum``).
    """
    W = np.asarray(W, dtype=np.float32)
    O = W.shape[0]
    out = np.empty(O, dtype=np.float32)
    for i in range(O):
        kept = np.abs(W[i][mask[i]]).astype(np.float64)
        mean = math.fsum(kept.tolist()) / float(kept.size)
        out[i] = max(np.float32(mean), EPS_SCALE)
    return out


def ternarise(W: np.ndarray, scale: np.ndarray, mask: np.ndarray) -> np.ndarray:
    """int8 [O, K] in {-1, 0, +1}: mask * clip(round(W / scale), -1, 1).

    Sparse-BitNet Guide, "Mathematical Formulation of Sparse-BitLinear", the
    joint sparse-ternary equation; the README's "Sparse-BitNet" section
    (mask first, then quantise what remains).
    """
    q = np.rint(np.asarray(W, np.float64) / np.asarray(scale, np.float64)[:, None])
    q = np.clip(q, -1.0, 1.0) * mask
    return q.astype(np.int8)


def pack_codes(Wt: np.ndarray) -> np.ndarray:
    """uint8 [O, K/4]: 2-bit codes 00 = 0, 01 = +1, 10 = -1, LSB-first.

    halo-sparse-bitnet-3:4-500m card, "What ships with this repo" /
    "Packed vs raw" (NAME.packed, 4 codes per byte).
    """
    Wt = np.asarray(Wt)
    O, K = Wt.shape
    code = np.zeros(Wt.shape, dtype=np.uint8)
    code[Wt == 1] = 1
    code[Wt == -1] = 2
    c = code.reshape(O, K // 4, 4)
    return (c[..., 0] | (c[..., 1] << 2) | (c[..., 2] << 4) | (c[..., 3] << 6)).astype(np.uint8)


def pack_mask_bits(mask: np.ndarray) -> np.ndarray:
    """uint8 [O, K/8]: bit k % 8 of byte k // 8 is set when weight k is kept."""
    O, K = mask.shape
    b = mask.reshape(O, K // 8, 8).astype(np.uint8)
    out = np.zeros((O, K // 8), dtype=np.uint8)
    for j in range(8):
        out |= (b[..., j] << j).astype(np.uint8)
    return out


def round_to_bf16(v: np.ndarray) -> np.ndarray:
    """float32 values rounded to the nearest bf16 (ties to even), as float32.

    The halo-sparse-bitnet-3:4-500m card, "What ships with this repo / Packed vs
    raw": row_scale is stored as bf16.  bf16 keeps the top 16 bits of a float32;
    round to nearest even on the dropped 16 (finite inputs)."""
    b = np.asarray(v, np.float32).view(np.uint32).astype(np.uint64)
    r = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return r.astype(np.uint32).view(np.float32)


def global_scale(W: np.ndarray) -> np.float32:
    """One scale for the whole matrix: mean of |W| over all O*K weights, masked
    ones included, clamped below at 1e-5 — the gamma of the Sparse-BitNet
    Guide's module listing (``torch.mean(torch.abs(weight)).clamp(min=1e-5)``).
    The sum is exact up to one final rounding to double (``math.fsum``)."""
    a = np.abs(np.asarray(W, dtype=np.float32)).astype(np.float64).ravel()
    mean = math.fsum(a.tolist()) / float(a.size)
    return max(np.float32(mean), EPS_SCALE)


def prepare_weights(W: np.ndarray, n: int, m: int, scale_bf16: bool = False, scale_global: bool = False):
    """Latent fp32 weights -> (packed uint8 [O,K/4], scale fp32 [O], mask bits uint8 [O,K/8], W_t int8 [O,K]).

    With ``scale_bf16`` the row scale is rounded to bf16 (:func:`round_to_bf16`)
    before it ternarises the row; the returned scale is that bf16 value.  With
    ``scale_global`` every row takes :func:`global_scale` instead."""
    mask = nm_mask(W, n, m)
    if scale_global:
        scale = np.full(np.asarray(W).shape[0], global_scale(W), dtype=np.float32)
    else:
        scale = row_scale(W, mask)
    if scale_bf16:
        scale = round_to_bf16(scale)
    Wt = ternarise(W, scale, mask)
    return pack_codes(Wt), scale, pack_mask_bits(mask), Wt


def quant_act(x: np.ndarray):
    """Per-token absmax int8: (x_q int8 [T,K], s_tok fp32 [T]), s_t = 127 / max(max|x_t|, 1e-5).

    Sparse-BitNet Guide, "Mathematical Formulation of Sparse-BitLinear", the
    activation equation (per-token beta = max |x_j|, clip to [-128, 127]);
    BitNet-TinyDialogues card (W1.58A8, 8-bit per-token activations).
    ``x`` holds bf16 values widened to fp32.
    """
    x = np.asarray(x, dtype=np.float32)
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite activation")
    amax = np.max(np.abs(x), axis=1) if x.shape[1] else np.zeros(x.shape[0], np.float32)
    s = (np.float32(127.0) / np.maximum(amax, EPS_ACT)).astype(np.float32)
    q = np.rint((x * s[:, None]).astype(np.float32))
    return np.clip(q, -128, 127).astype(np.int8), s


def round_exact_to_f32(num: int, exp2: int) -> np.float32:
    """The float32 nearest to the exact value num * 2**exp2 (num >= 0 an
    integer), ties to the even significand; values at or past the float32
    overflow threshold give +inf.  A float32 keeps 24 significant bits down to
    2**-126 and a fixed spacing of 2**-149 below it."""
    if num < 0:
        raise ValueError("num must be >= 0")
    if num == 0:
        return np.float32(0.0)
    e = num.bit_length() - 1 + exp2           # the value lies in [2**e, 2**(e + 1))
    q = max(e - 23, -149)                      # weight of the last bit float32 keeps there
    drop = q - exp2
    if drop <= 0:
        m = num << -drop
    else:
        m = num >> drop
        rest = num - (m << drop)
        half = 1 << (drop - 1)
        if rest > half or (rest == half and m & 1):
            m += 1
    if m.bit_length() - 1 + q >= 128:
        return np.float32(np.inf)
    return np.float32(math.ldexp(m, q))


def rms_sumsq(x: np.ndarray) -> np.ndarray:
    """float32 [T]: sum_k x_k^2 of every token, formed exactly and rounded once
    to float32 (nearest, ties to even; +inf past the float32 range).

    The sum of squares of torch's RMSNorm (the guide's SparseBitLinear module
    listing), whose order the pages leave open; the exact sum is independent of
    it.  ``x`` holds bf16 values (widened to float32): each is
    x = M * 2**(E - 134), M its 8-bit significand (implicit bit included) and
    E = max(biased exponent, 1), so x**2 = M**2 * 2**(2E - 268) is an integer
    multiple of 2**-266 and the sum is an exact integer in that unit: the
    squares are gathered per exponent (sums of M**2, exact) and the
    per-exponent totals added as Python integers.
    """
    x = np.asarray(x, dtype=np.float32)
    T, K = x.shape
    u = x.view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("x must hold bf16 values")
    mag = (u >> 16) & 0x7FFF
    if np.any(mag >= 0x7F80):
        raise ValueError("non-finite input")
    bexp = mag >> 7
    M = np.where(bexp > 0, (mag & 0x7F) | 0x80, mag & 0x7F).astype(np.int64)
    E = np.maximum(bexp, 1).astype(np.int64)            # 1 .. 254
    # per-exponent sums of M**2: each below 2**16 * K < 2**53, so the float64
    # accumulation of bincount is exact
    idx = (np.arange(T, dtype=np.int64)[:, None] * 255 + E).ravel()
    per_exp = np.bincount(idx, weights=(M * M).ravel().astype(np.float64), minlength=T * 255)
    per_exp = per_exp.reshape(T, 255).astype(np.int64)
    out = np.empty(T, np.float32)
    for t in range(T):
        nz = np.nonzero(per_exp[t])[0]
        total = sum(int(per_exp[t, e]) << (2 * int(e) - 2) for e in nz)   # units of 2**-266
        out[t] = round_exact_to_f32(total, -266)
    return out


def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """float32 [T, K]: x * (1 / sqrt(sum_k x_k^2 / K + eps)) * g.

    Sparse-BitNet Guide, "Mathematical Formulation of Sparse-BitLinear" (x is
    normalised by RMSNorm before the absmax) and its SparseBitLinear module
    listing (torch RMSNorm over the input features, elementwise weight g,
    default eps = float32 machine epsilon).  Every step is one IEEE float32
    operation after the exact sum of squares of :func:`rms_sumsq`: a division
    by K, an addition of eps, a square root, a division of 1 by it, and two
    products.  A sum of squares past the float32 range is +inf, which makes
    every normalised value 0 (the library flags such a token).
    """
    x = np.asarray(x, dtype=np.float32)
    g = np.asarray(g, dtype=np.float32)
    if not (np.all(np.isfinite(x)) and np.all(np.isfinite(g))):
        raise ValueError("non-finite input")
    T, K = x.shape
    if g.shape != (K,):
        raise ValueError("g must have K entries")
    ms = (rms_sumsq(x) / np.float32(K)).astype(np.float32)
    den = np.sqrt((ms + np.float32(eps)).astype(np.float32)).astype(np.float32)
    inv = (np.float32(1.0) / den).astype(np.float32)
    return ((x * inv[:, None]).astype(np.float32) * g[None, :]).astype(np.float32)


def rmsnorm_quant_act(x: np.ndarray, g: np.ndarray, eps: float):
    """(x_q int8 [T,K], s_tok fp32 [T]) of the RMS-normalised activations: the
    guide module's normalise-then-absmax-quantise front end."""
    return quant_act(rmsnorm(x, g, eps))


def mask_monitor(old_bits: np.ndarray, new_bits: np.ndarray, K: int, n: int, m: int):
    """Mask change rate and verification between two mask bitmaps uint8 [O, K/8]
    (bit k % 8 of byte k // 8 set when weight k is kept).

    Returns (changed, bad_groups, row_changed): the number of positions whose
    kept state differs, the number of M-groups of ``new_bits`` that do not keep
    exactly N weights, and the changed count per row (int64 [O]).
    The Sparse-BitNet README ("Features": dynamic mask monitoring; the CLI's
    mask-monitor interval: the mask change rate every N steps) and the
    halo-sparse-bitnet-3:4-500m card ("Recipe": mask-verify every 500 steps);
    the rate is changed / (O * K).
    """
    _check_nm(K, n, m)
    old = np.unpackbits(np.asarray(old_bits, np.uint8), axis=1, bitorder="little")[:, :K].astype(bool)
    new = np.unpackbits(np.asarray(new_bits, np.uint8), axis=1, bitorder="little")[:, :K].astype(bool)
    row_changed = np.count_nonzero(old != new, axis=1).astype(np.int64)
    kept = new.reshape(new.shape[0], K // m, m).sum(axis=2)
    return int(row_changed.sum()), int(np.count_nonzero(kept != n)), row_changed


def int_contract(xq: np.ndarray, Wt: np.ndarray) -> np.ndarray:
    """int32 [T, O] = x_q . W_t^T (the guide's integer product before rescaling).

    Evaluated as a float64 matrix product: every product and partial sum is an
    integer of magnitude <= 128 * K < 2**53, so each is exact whatever the
    summation order; the result is checked to be integral and to fit int32.
    """
    acc = np.asarray(xq, np.float64) @ np.asarray(Wt, np.float64).T
    r = np.rint(acc)
    if not np.array_equal(r, acc):
        raise ArithmeticError("non-integral contraction")
    if r.size and np.max(np.abs(r)) >= 2**31:
        raise OverflowError("accumulator exceeds int32")
    return r.astype(np.int32)


def dequant(acc: np.ndarray, scale: np.ndarray, s_tok: np.ndarray) -> np.ndarray:
    """float64 [T, O] = acc * scale_o / s_t (the guide's beta * gamma / 127 rescale)."""
    return (np.asarray(acc, np.float64) * np.asarray(scale, np.float64)[None, :]
            / np.asarray(s_tok, np.float64)[:, None])


def linear(x: np.ndarray, Wt: np.ndarray, scale: np.ndarray, g=None, eps=None):
    """Full forward on prepared weights: (y float64 [T,O], acc int32 [T,O], x_q, s_tok).

    With ``g`` (and ``eps``) the activations are RMS-normalised first."""
    xq, s = quant_act(x) if g is None else rmsnorm_quant_act(x, g, eps)
    acc = int_contract(xq, Wt)
    return dequant(acc, scale, s), acc, xq, s


def unpack_codes(packed: np.ndarray, K: int) -> np.ndarray:
    """Inverse of :func:`pack_codes` (code 11 is invalid and raises)."""
    p = np.asarray(packed, dtype=np.uint8)
    O = p.shape[0]
    c = np.stack([(p >> (2 * j)) & 3 for j in range(4)], axis=-1).reshape(O, K)
    if np.any(c == 3):
        raise ValueError("invalid 2-bit code 11")
    return np.where(c == 1, 1, np.where(c == 2, -1, 0)).astype(np.int8)


def acc_entries(xq: np.ndarray, Wt: np.ndarray, idx_t, idx_o) -> np.ndarray:
    """int64 acc[t, o] for the listed (t, o) pairs, one dot product each (sampled checks)."""
    xq = np.asarray(xq, np.int64)
    Wt = np.asarray(Wt, np.int64)
    return np.array([int(np.dot(xq[t], Wt[o])) for t, o in zip(idx_t, idx_o)], dtype=np.int64)


def ste_backward(dY: np.ndarray, xq: np.ndarray, s_tok: np.ndarray, Wt: np.ndarray, scale: np.ndarray,
                 dw_ternary: bool = False):
    """Straight-through gradients of the forward y = (x_q . W_t^T) * scale_o / s_t:
    (dX float64 [T, K], dW float64 [O, K]) for the loss gradient dY [T, O].

    Reading (the guide's "Training Stability & The Straight-Through Estimator":
    the backward bypasses the N:M mask and the ternary rounding and reaches the
    latent weights; the Sparse-BitNet README, "How It Works / BitLinear": the
    gradient passes the quantiser by straight-through estimation): in the
    backward every quantiser is the identity, so the forward reads as
    y = x_hat . W_hat^T with x_hat[t,k] = x_q[t,k] / s_t (the activations the
    forward used) and W_hat[o,k] = scale_o * W_t[o,k] (the weights it used):

        dX[t,k] = sum_o dY[t,o] * scale_o * W_t[o,k]
        dW[o,k] = sum_t dY[t,o] * x_q[t,k] / s_t     (every position, masked ones too)

    dX is the gradient at the quantiser's input (after the RMSNorm, when the
    fused front end ran).  With ``dw_ternary`` the weight gradient is the one the
    guide's module returns: taken at the ternary matrix of its equation
    y = (x~ . W~^T) * beta * gamma / 127, i.e. dW[o,k] scaled once more by scale_o.
    Products and sums in float64 (numpy matrix products).
    """
    dY = np.asarray(dY, np.float64)
    xhat = np.asarray(xq, np.float64) / np.asarray(s_tok, np.float64)[:, None]
    sc = np.asarray(scale, np.float64)
    Wt = np.asarray(Wt, np.float64)
    dX = (dY * sc[None, :]) @ Wt
    dW = dY.T @ xhat
    if dw_ternary:
        dW = dW * sc[:, None]
    return dX, dW
