"""Pins of the CPU oracle to facts that do not come from the oracle itself.

* worked examples: the 4-element block the Sparse-BitNet Guide prints in
  "The Hardware Mechanics of 2:4 Sparsity", plus hand-derived tie, rounding and
  degenerate cases (tests/golden/worked_examples.json, each with its source);
* brute force on tiny shapes: the Top-N set found by enumerating every subset,
  exact rational means (fractions.Fraction), the |w| > scale/2 threshold form
  of clip(round(w/scale)), bit-string packing, explicit integer loops;
* invariants that hold at any size (codes in {-1,0,1}, at most N nonzeros per
  group, sign agreement, packed size O*K/4, argmax token element -> +-127);
* the guide's own rescale form y = acc * beta * gamma / 127;
* RMSNorm front end: torch's rms_norm in float64 (the library routine the
  guide's module calls); the sum of squares against exact rational sums
  (fractions.Fraction) rounded by a nearest-float search, hand-derived sums at
  float32 rounding boundaries (ties, a double-rounding trap, subnormal and
  overflowing squares) and invariance under any reordering; constant rows,
  and invariance under x -> 4x.

Each plausible mistake (a reversed input index, scale over all weights, half away
from zero, ties to the higher index, MSB-first packing, a dropped clamp, a sign
flip) is planted in a copy of the oracle at the end of this file, and some pin
below must reject it.
"""
import itertools
import math
import json
import os
import types
from fractions import Fraction

import numpy as np
import pytest

import oracle
from sparse_linear_layers_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")
PATTERNS = [(2, 4), (3, 4), (6, 8), (4, 8)]


def _cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


# --------------------------------------------------------------------------
# pins written as functions of an oracle-like namespace, so the planted
# mistakes at the bottom can be run through the very same checks
# --------------------------------------------------------------------------

def pin_golden(o):
    for c in _cases():
        if "w" in c and "w_t" in c:
            W = np.array([c["w"]], dtype=np.float32)
            n, m = c["n"], c["m"]
            mask = o.nm_mask(W, n, m)
            assert sorted(np.nonzero(mask[0])[0].tolist()) == c["kept_indices"], c["name"]
            scale = o.row_scale(W, mask)
            assert abs(float(scale[0]) - c["scale"]) <= 1e-6 * c["scale"], c["name"]
            Wt = o.ternarise(W, scale, mask)
            assert Wt[0].tolist() == c["w_t"], c["name"]
            assert o.pack_codes(Wt)[0].tolist() == c["packed"], c["name"]
            # mask bits need K % 8 == 0: pad with a second group of zeros
            W8 = np.concatenate([W, np.zeros((1, 4), np.float32)], axis=1)
            mb = o.pack_mask_bits(o.nm_mask(W8, n, m))
            assert int(mb[0, 0]) & 0xF == c["mask_byte_low_nibble"], c["name"]
        if "x" in c and "x_q" in c:
            x = np.array([c["x"]], dtype=np.float32)
            xq, s = o.quant_act(x)
            assert xq[0].tolist() == c["x_q"], c["name"]
            if "s_tok" in c:
                assert float(s[0]) == c["s_tok"], c["name"]
        if "acc" in c:
            W = np.array([c["w"]], dtype=np.float32)
            mask = o.nm_mask(W, c["n"], c["m"])
            scale = o.row_scale(W, mask)
            Wt = o.ternarise(W, scale, mask)
            y, acc, _, _ = o.linear(np.array([c["x"]], np.float32), Wt, scale)
            assert int(acc[0, 0]) == c["acc"], c["name"]
            if c["y"] == 0.0:
                assert y[0, 0] == 0.0
            else:
                assert abs(y[0, 0] - c["y"]) <= 1e-6 * abs(c["y"]), c["name"]


def _brute_mask_group(a, n):
    """The unique N-subset S with |a_i| > |a_j| or (equal and i < j) for all i in S, j not in S."""
    m = len(a)
    found = []
    for S in itertools.combinations(range(m), n):
        ok = all((abs(a[i]) > abs(a[j])) or (abs(a[i]) == abs(a[j]) and i < j)
                 for i in S for j in range(m) if j not in S)
        if ok:
            found.append(S)
    assert len(found) == 1
    return found[0]


def _exact_scale(row, kept):
    tot = sum((Fraction(float(abs(row[k]))) for k in kept), Fraction(0))
    mean = float(tot) / float(len(kept))       # float(Fraction) rounds correctly to double
    return max(np.float32(mean), np.float32(1e-5))


def _brute_prepare(W, n, m):
    O, K = W.shape
    mask = np.zeros((O, K), bool)
    for i in range(O):
        for g in range(K // m):
            for j in _brute_mask_group([float(v) for v in W[i, g * m:(g + 1) * m]], n):
                mask[i, g * m + j] = True
    scale = np.array([_exact_scale(W[i], np.nonzero(mask[i])[0]) for i in range(O)], np.float32)
    Wt = np.zeros((O, K), np.int8)
    for i in range(O):
        half = np.float32(0.5) * scale[i]          # exact in float32
        for k in range(K):
            if mask[i, k] and abs(W[i, k]) > half:  # round(w/s) != 0  <=>  |w|/s > 1/2
                Wt[i, k] = 1 if W[i, k] > 0 else -1
    return mask, scale, Wt


def _bitstring_pack(Wt):
    O, K = Wt.shape
    out = np.zeros((O, K // 4), np.uint8)
    for i in range(O):
        for b in range(K // 4):
            bits = ""
            for j in reversed(range(4)):           # most significant code first in the string
                v = int(Wt[i, 4 * b + j])
                bits += {0: "00", 1: "01", -1: "10"}[v]
            out[i, b] = int(bits, 2)
    return out


def _loop_contract(xq, Wt):
    T, K = xq.shape
    O = Wt.shape[0]
    acc = np.zeros((T, O), np.int64)
    for t in range(T):
        for o in range(O):
            s = 0
            for k in range(K):
                s += int(xq[t, k]) * int(Wt[o, k])
            acc[t, o] = s
    return acc


def pin_brute_force(o, shapes=((8, 16), (5, 24), (3, 64)), T=3, seeds=(0, 1, 2)):
    for seed in seeds:
        for (O, K) in shapes:
            for (n, m) in PATTERNS:
                if K % m:
                    continue
                W = synthetic.latent_weights(O, K, seed=seed, tag=f"bf{O}x{K}")
                # plant exact ties and zeros so the tie rule is exercised
                W[0, :m] = np.float32(0.25)
                W[-1, m:2 * m] = 0.0
                W[1 % O, :4] = [np.float32(0.5), np.float32(-0.5), np.float32(0.5), np.float32(0.125)]
                mask_b, scale_b, Wt_b = _brute_prepare(W, n, m)
                packed, scale, mbits, Wt = o.prepare_weights(W, n, m)
                assert np.array_equal(o.nm_mask(W, n, m), mask_b)
                assert np.array_equal(scale.view(np.uint32), scale_b.view(np.uint32))
                assert np.array_equal(Wt, Wt_b)
                assert np.array_equal(packed, _bitstring_pack(Wt_b))
                _, xv = synthetic.activations(T, K, seed=seed, tag=f"bfx{K}")
                xq, s = o.quant_act(xv)
                acc_b = _loop_contract(xq, Wt_b)
                y, acc, _, _ = o.linear(xv, Wt, scale)
                assert np.array_equal(acc.astype(np.int64), acc_b)
                # the guide's rescale: y = acc * beta * gamma / 127, beta = max|x_t|
                beta = np.maximum(np.max(np.abs(xv.astype(np.float64)), axis=1), 1e-5)
                y_page = acc_b * beta[:, None] * scale.astype(np.float64)[None, :] / 127.0
                assert np.allclose(y, y_page, rtol=1e-6, atol=0.0)


def pin_invariants(o, O=64, K=512, T=16):
    for (n, m) in PATTERNS:
        for seed in (0, 1):
            W = synthetic.latent_weights(O, K, seed=seed, tag="inv")
            packed, scale, mbits, Wt = o.prepare_weights(W, n, m)
            assert packed.shape == (O, K // 4) and packed.dtype == np.uint8   # 2 bits per weight
            assert set(np.unique(Wt).tolist()) <= {-1, 0, 1}
            codes = np.stack([(packed >> (2 * j)) & 3 for j in range(4)], -1)
            assert not np.any(codes == 3)
            mask = np.unpackbits(mbits, axis=1, bitorder="little").astype(bool)
            assert np.all(mask.reshape(O, K // m, m).sum(-1) == n)
            assert np.all((Wt != 0).reshape(O, K // m, m).sum(-1) <= n)
            assert np.all(mask[Wt != 0])
            nz = Wt != 0
            assert np.all(np.sign(W[nz]) == Wt[nz])
            # kept weights dominate dropped ones inside every group
            a = np.abs(W).reshape(O, K // m, m)
            mk = mask.reshape(O, K // m, m)
            kept_min = np.where(mk, a, np.inf).min(-1)
            drop_max = np.where(~mk, a, -np.inf).max(-1)
            assert np.all(kept_min >= drop_max)
            # scale is the mean of the kept magnitudes (loose check against float64 mean)
            mean = np.where(mask, np.abs(W.astype(np.float64)), 0).sum(1) / (K * n // m)
            assert np.allclose(scale, mean, rtol=1e-6)
            # round(w/s) != 0 exactly when |w| > s/2
            assert np.array_equal(nz, mask & (np.abs(W) > np.float32(0.5) * scale[:, None]))
    _, x = synthetic.activations(T, K, seed=3, tag="invx", outlier_p=0.01)
    xq, s = o.quant_act(x)
    assert xq.min() >= -127 and xq.max() <= 127
    arg = np.argmax(np.abs(x), axis=1)
    assert np.all(np.abs(xq[np.arange(T), arg]) == 127)
    exact = x.astype(np.float64) * s.astype(np.float64)[:, None]
    assert np.all(np.abs(xq - exact) <= 0.5 + 1e-6)
    # monotone in x within each token
    for t in range(T):
        order = np.argsort(x[t], kind="stable")
        assert np.all(np.diff(xq[t][order].astype(np.int32)) >= 0)


def pin_closed_forms(o):
    # every kept magnitude equal to c: scale == c exactly, W_t == sign(W) on kept positions
    c = np.float32(0.0375)
    K = 64
    for (n, m) in PATTERNS:
        W = np.full((2, K), c, np.float32)
        W[1, ::2] = -c
        mask = o.nm_mask(W, n, m)
        scale = o.row_scale(W, mask)
        assert np.all(scale == c)
        Wt = o.ternarise(W, scale, mask)
        assert np.array_equal(Wt, (np.sign(W) * mask).astype(np.int8))
        # first N of each group kept (all tie)
        assert np.array_equal(mask.reshape(2, K // m, m)[..., :n], np.ones((2, K // m, n), bool))
    # zero token -> zero codes, zero output
    x = np.zeros((1, K), np.float32)
    xq, s = o.quant_act(x)
    assert not xq.any() and s[0] == np.float32(127.0) / np.float32(1e-5)


# --------------------------------------------------------------------------

def test_golden_worked_examples():
    pin_golden(oracle)


def test_brute_force_tiny_shapes():
    pin_brute_force(oracle)


def test_invariants():
    pin_invariants(oracle)


def test_closed_forms():
    pin_closed_forms(oracle)


def test_unpack_roundtrip_and_bad_code():
    W = synthetic.latent_weights(16, 128, seed=5)
    packed, _, _, Wt = oracle.prepare_weights(W, 3, 4)
    assert np.array_equal(oracle.unpack_codes(packed, 128), Wt)
    bad = packed.copy()
    bad[0, 0] = 0xFF
    with pytest.raises(ValueError):
        oracle.unpack_codes(bad, 128)


def test_rejects_bad_input():
    with pytest.raises(ValueError):
        oracle.nm_mask(np.ones((2, 8), np.float32), 1, 4)
    W = np.ones((2, 8), np.float32)
    W[0, 3] = np.nan
    with pytest.raises(ValueError):
        oracle.nm_mask(W, 2, 4)
    x = np.ones((1, 8), np.float32)
    x[0, 0] = np.inf
    with pytest.raises(ValueError):
        oracle.quant_act(x)


def test_acc_entries_matches_contract():
    W = synthetic.latent_weights(32, 256, seed=1)
    _, scale, _, Wt = oracle.prepare_weights(W, 2, 4)
    _, x = synthetic.activations(4, 256, seed=1)
    xq, _ = oracle.quant_act(x)
    full = oracle.int_contract(xq, Wt)
    t = np.array([0, 1, 3, 2])
    o_ = np.array([0, 31, 7, 19])
    assert np.array_equal(oracle.acc_entries(xq, Wt, t, o_), full[t, o_])


# --------------------------------------------------------------------------
# planted mistakes: each mutant must fail at least one pin
# --------------------------------------------------------------------------

def _mutant(**over):
    ns = types.SimpleNamespace(**{k: getattr(oracle, k) for k in (
        "nm_mask", "row_scale", "ternarise", "pack_codes", "pack_mask_bits", "quant_act",
        "int_contract", "dequant")})
    ns.__dict__.update(over)

    def prepare_weights(W, n, m):
        mask = ns.nm_mask(W, n, m)
        scale = ns.row_scale(W, mask)
        Wt = ns.ternarise(W, scale, mask)
        return ns.pack_codes(Wt), scale, ns.pack_mask_bits(mask), Wt

    def linear(x, Wt, scale):
        xq, s = ns.quant_act(x)
        acc = ns.int_contract(xq, Wt)
        return ns.dequant(acc, scale, s), acc, xq, s

    ns.prepare_weights = prepare_weights
    ns.linear = linear
    return ns


def _ties_high(W, n, m):
    O, K = W.shape
    a = np.abs(W.astype(np.float64)).reshape(O, K // m, m)[..., ::-1]
    order = np.argsort(-a, axis=-1, kind="stable")
    keep = np.zeros(a.shape, bool)
    np.put_along_axis(keep, order[..., :n], True, axis=-1)
    return keep[..., ::-1].reshape(O, K)


def _scale_all(W, mask):
    return np.maximum(np.mean(np.abs(W.astype(np.float64)), axis=1).astype(np.float32), np.float32(1e-5))


def _half_away(W, scale, mask):
    r = np.asarray(W, np.float64) / np.asarray(scale, np.float64)[:, None]
    q = np.sign(r) * np.floor(np.abs(r) + 0.5)
    return (np.clip(q, -1, 1) * mask).astype(np.int8)


def _msb_first(Wt):
    O, K = Wt.shape
    code = np.where(Wt == 1, 1, np.where(Wt == -1, 2, 0)).astype(np.uint8).reshape(O, K // 4, 4)
    return (code[..., 3] | (code[..., 2] << 2) | (code[..., 1] << 4) | (code[..., 0] << 6)).astype(np.uint8)


def _swapped_codes(Wt):
    return oracle.pack_codes(-np.asarray(Wt))


def _no_mask(W, scale, mask):
    return oracle.ternarise(W, scale, np.ones_like(mask))


def _k_reversed(xq, Wt):
    return oracle.int_contract(xq, np.asarray(Wt)[:, ::-1])


def _quant_no_round(x):
    xq, s = oracle.quant_act(x)
    x = np.asarray(x, np.float32)
    q = np.trunc(x * s[:, None])
    return np.clip(q, -128, 127).astype(np.int8), s


def _dequant_inverted(acc, scale, s_tok):
    return np.asarray(acc, np.float64) * np.asarray(scale, np.float64)[None, :] * np.asarray(s_tok, np.float64)[:, None] / 127.0 ** 2


MUTANTS = {
    "ties_to_higher_index": dict(nm_mask=_ties_high),
    "scale_over_all_weights": dict(row_scale=_scale_all),
    "round_half_away": dict(ternarise=_half_away),
    "msb_first_packing": dict(pack_codes=_msb_first),
    "swapped_code_table": dict(pack_codes=_swapped_codes),
    "mask_not_applied": dict(ternarise=_no_mask),
    "input_dim_reversed": dict(int_contract=_k_reversed),
    "activation_truncated": dict(quant_act=_quant_no_round),
    "rescale_inverted": dict(dequant=_dequant_inverted),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    o = _mutant(**MUTANTS[name])
    caught = []
    for pin in (pin_golden, pin_closed_forms, pin_brute_force, pin_invariants):
        try:
            if pin is pin_brute_force:
                pin(o, shapes=((8, 16), (4, 32)), T=2, seeds=(0,))
            else:
                pin(o)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"


# --------------------------------------------------------------------------
# RMSNorm front end (the guide's module normalises x before the absmax)
# --------------------------------------------------------------------------

def pin_rms_library(o):
    """torch's own rms_norm in float64 (the guide's module uses torch RMSNorm):
    the float32 oracle agrees within a few float32 roundings; eps = 0.5 and a
    random weight make the placement of eps and of g visible."""
    import torch
    rng = np.random.default_rng(7)
    for K in (64, 256):
        x = synthetic.activations(5, K, seed=3)[1]
        g = rng.uniform(0.5, 1.5, K).astype(np.float32)
        for eps in (0.5, 2.0 ** -23):
            ref = torch.nn.functional.rms_norm(torch.from_numpy(x.astype(np.float64)), (K,),
                                               weight=torch.from_numpy(g.astype(np.float64)), eps=eps).numpy()
            got = o.rmsnorm(x, g, eps).astype(np.float64)
            assert np.all(np.abs(got - ref) <= 2e-5 * np.abs(ref) + 1e-30)


def _bf16_row(vals, K=None):
    x = np.zeros((1, K or len(vals)), np.float32)
    x[0, :len(vals)] = np.asarray(vals, np.float64).astype(np.float32)
    assert not np.any(x.view(np.uint32) & 0xFFFF), "test values must be bf16"
    return x


def _nearest_f32(q: Fraction) -> np.float32:
    """The float32 nearest to the rational q >= 0 (ties to the even bit
    pattern; +inf from the overflow threshold (2 - 2^-24) * 2^127 on), by
    comparing the distances of the candidates around the double nearest to q."""
    if q >= Fraction(2 ** 128 - 2 ** 103):
        return np.float32(np.inf)
    c0 = np.float32(float(q))
    cands = {c0, np.nextafter(c0, np.float32(0)), np.nextafter(c0, np.float32(np.inf))}
    cands = [c for c in cands if np.isfinite(c)]
    return min(cands, key=lambda c: (abs(Fraction(float(c)) - q), int(np.asarray(c).view(np.uint32)) & 1))


def pin_rms_exact(o):
    """The sum of squares is the exact sum rounded once to float32.

    Hand-derived (float32 spacing is 2 between 2^24 and 2^25):
      [4096, 1]: 2^24 + 1 is a tie between 2^24 and 2^24 + 2 -> even 2^24
        (half away from zero would give 2^24 + 2);
      [4096, 1 x 15]: 16777231, a tie -> even 16777232 (a float32 running
        sum stays at 2^24: every + 1 ties back down);
      K = 512, x_0 = 4096, the first element of blocks 1..31 = 1: 16777247,
        a tie -> 16777248 (32 float32 lane sums combined by a butterfly give
        16777246);
      [4096, 1, 2^-30]: 2^24 + 1 + 2^-60 lies above the tie -> 16777218;
        the exact sum rounded to double first is the tie itself, which then
        rounds to 2^24 (double rounding);
      [2^-75]: 2^-150 is half the smallest float32 -> ties to 0;
        [2^-75, 2^-75]: 2^-149 exactly;
      [2^64]: 2^128 overflows -> +inf; [1.5 * 2^63]: 1.125 * 2^127 exactly.
    Brute force: random rows mixing bf16 subnormals, tiny, ordinary and large
    magnitudes, against sum(Fraction(x)^2) rounded by a nearest-float search.
    Any reordering of a row gives the same float."""
    cases = [
        ([4096.0, 1.0], 16777216.0),
        ([4096.0] + [1.0] * 15, 16777232.0),
        ([4096.0, 1.0, 2.0 ** -30], 16777218.0),
        ([2.0 ** -75], 0.0),
        ([2.0 ** -75, 2.0 ** -75], 2.0 ** -149),
        ([2.0 ** 64], math.inf),
        ([1.5 * 2.0 ** 63], 1.125 * 2.0 ** 127),
    ]
    for vals, want in cases:
        assert float(o.rms_sumsq(_bf16_row(vals, K=16 * ((len(vals) + 15) // 16)))[0]) == want, vals
    x = np.zeros((1, 512), np.float32)
    x[0, 0] = 4096.0
    x[0, 16::16] = 1.0
    assert float(o.rms_sumsq(x)[0]) == 16777248.0
    rng = np.random.default_rng(11)
    pool = [0.0, 2.0 ** -133, 3 * 2.0 ** -133, 2.0 ** -126, 1e-30, 1e-12, 1e-4, 0.5, 1.0, 3.0, 1e4, 1e15, 3e18]
    rows = []
    for _ in range(40):
        K = int(rng.choice([16, 32, 48]))
        v = rng.choice(pool, K) * rng.choice([-1.0, 1.0], K) * (1 + rng.integers(0, 128, K) / 128.0)
        v = synthetic.bf16_bits_to_f32(synthetic.f32_to_bf16_bits(v.astype(np.float32)))
        rows.append(v)
    for v in rows:
        want = _nearest_f32(sum(Fraction(float(e)) ** 2 for e in v))
        got = o.rms_sumsq(v[None, :])[0]
        assert got.view(np.uint32) == want.view(np.uint32), (v, got, want)
        perm = rng.permutation(v.size)
        assert o.rms_sumsq(v[None, perm])[0].view(np.uint32) == got.view(np.uint32)


def pin_rms_closed_forms(o):
    """Constant rows normalise to +-1 (fl(1/3) * 3 rounds to 1 in float32), so
    every code is +-127 with s = 127; with eps = 0 the front end is invariant
    under x -> 4x (powers of two scale every step exactly); the largest |x g|
    of a token maps to +-127."""
    K = 32
    x = np.full((2, K), 3.0, np.float32)
    x[1, 1::2] = -3.0
    xq, s = o.rmsnorm_quant_act(x, np.ones(K, np.float32), 0.0)
    assert xq[0].tolist() == [127] * K and s[0] == np.float32(127.0)
    assert xq[1].tolist() == [127, -127] * (K // 2)
    xb, xv = synthetic.activations(6, 128, seed=4)
    g = np.random.default_rng(2).uniform(0.25, 2.0, 128).astype(np.float32)
    q1, s1 = o.rmsnorm_quant_act(xv, g, 0.0)
    q4, s4 = o.rmsnorm_quant_act(xv * np.float32(4.0), g, 0.0)
    assert np.array_equal(q1, q4) and np.array_equal(s1, s4)
    q, _ = o.rmsnorm_quant_act(xv, g, 2.0 ** -23)
    am = np.argmax(np.abs(xv.astype(np.float64) * g), axis=1)
    assert np.all(np.abs(q[np.arange(6), am]) == 127)


def test_rms_pins():
    for pin in (pin_rms_library, pin_rms_exact, pin_rms_closed_forms):
        pin(oracle)


def _rms_ns(**over):
    ns = types.SimpleNamespace(rms_sumsq=oracle.rms_sumsq, quant_act=oracle.quant_act)
    ns.__dict__.update(over)

    def rmsnorm(x, g, eps):
        x = np.asarray(x, np.float32)
        K = x.shape[1]
        ms = (ns.rms_sumsq(x) / np.float32(K)).astype(np.float32)
        inv = (np.float32(1.0) / np.sqrt((ms + np.float32(eps)).astype(np.float32))).astype(np.float32)
        return ((x * inv[:, None]).astype(np.float32) * np.asarray(g, np.float32)[None, :]).astype(np.float32)

    if "rmsnorm" not in over:
        ns.rmsnorm = rmsnorm
    ns.rmsnorm_quant_act = lambda x, g, eps: ns.quant_act(ns.rmsnorm(x, g, eps))
    return ns


def _rms_seq(x):
    x = np.asarray(x, np.float32)
    acc = np.zeros(x.shape[0], np.float32)
    for k in range(x.shape[1]):
        acc = (acc + (x[:, k] * x[:, k]).astype(np.float32)).astype(np.float32)
    return acc


def _rms_lane_butterfly(x):
    """32 float32 lane sums of 16-element blocks, combined by an xor butterfly
    (an order-dependent float32 sum)."""
    x = np.asarray(x, np.float32)
    part = np.zeros((x.shape[0], 32), np.float32)
    for k in range(x.shape[1]):
        lane = (k // 16) % 32
        part[:, lane] = (part[:, lane] + (x[:, k] * x[:, k]).astype(np.float32)).astype(np.float32)
    idx = np.arange(32)
    for off in (16, 8, 4, 2, 1):
        part = (part + part[:, idx ^ off]).astype(np.float32)
    return part[:, 0].copy()


def _rms_fsum_then_f32(x):
    """The exact sum rounded to double (fsum), then to float32: double rounding."""
    x = np.asarray(x, np.float64)
    return np.array([np.float32(math.fsum((r * r).tolist())) for r in x], np.float32)


def _rms_ties_away(x):
    """Exact sum, but ties rounded away from zero."""
    x = np.asarray(x, np.float32)
    out = np.empty(x.shape[0], np.float32)
    for t, r in enumerate(x):
        q = sum(Fraction(float(e)) ** 2 for e in r)
        c = np.float32(float(q))
        lo = c if Fraction(float(c)) <= q else np.nextafter(c, np.float32(0))
        hi = np.nextafter(lo, np.float32(np.inf))
        dlo, dhi = q - Fraction(float(lo)), Fraction(float(hi)) - q
        out[t] = hi if dhi <= dlo else lo
    return out


def _rms_flush_subnormal_squares(x):
    """Exact sum of the squares, but squares below 2^-126 dropped."""
    x = np.asarray(x, np.float32)
    sq = np.where(np.abs(x.astype(np.float64)) ** 2 < 2.0 ** -126, np.float32(0), x)
    return oracle.rms_sumsq(sq.astype(np.float32))


def _rms_saturate(x):
    """Exact sum, but an overflowing sum saturated at the largest float32."""
    s = oracle.rms_sumsq(x)
    return np.where(np.isinf(s), np.finfo(np.float32).max, s).astype(np.float32)


def _rms_no_sqrt(x, g, eps):
    x = np.asarray(x, np.float32)
    ms = (oracle.rms_sumsq(x) / np.float32(x.shape[1])).astype(np.float32)
    return (x / (ms + np.float32(eps))[:, None] * np.asarray(g, np.float32)[None, :]).astype(np.float32)


def _rms_eps_outside(x, g, eps):
    x = np.asarray(x, np.float32)
    ms = (oracle.rms_sumsq(x) / np.float32(x.shape[1])).astype(np.float32)
    return (x / (np.sqrt(ms) + np.float32(eps))[:, None] * np.asarray(g, np.float32)[None, :]).astype(np.float32)


def _rms_no_weight(x, g, eps):
    return oracle.rmsnorm(x, np.ones_like(np.asarray(g, np.float32)), eps)


def _rms_mean_k_minus_1(x, g, eps):
    x = np.asarray(x, np.float32)
    ms = (oracle.rms_sumsq(x) / np.float32(x.shape[1] - 1)).astype(np.float32)
    inv = (np.float32(1.0) / np.sqrt((ms + np.float32(eps)).astype(np.float32))).astype(np.float32)
    return ((x * inv[:, None]).astype(np.float32) * np.asarray(g, np.float32)[None, :]).astype(np.float32)


RMS_MUTANTS = {
    "rms_sequential_sum": dict(rms_sumsq=_rms_seq),
    "rms_lane_butterfly": dict(rms_sumsq=_rms_lane_butterfly),
    "rms_fsum_then_float32": dict(rms_sumsq=_rms_fsum_then_f32),
    "rms_ties_away": dict(rms_sumsq=_rms_ties_away),
    "rms_flush_subnormal_squares": dict(rms_sumsq=_rms_flush_subnormal_squares),
    "rms_saturate_overflow": dict(rms_sumsq=_rms_saturate),
    "rms_no_sqrt": dict(rmsnorm=_rms_no_sqrt),
    "rms_eps_outside_sqrt": dict(rmsnorm=_rms_eps_outside),
    "rms_weight_dropped": dict(rmsnorm=_rms_no_weight),
    "rms_mean_over_k_minus_1": dict(rmsnorm=_rms_mean_k_minus_1),
}


@pytest.mark.parametrize("name", sorted(RMS_MUTANTS))
def test_planted_rms_mistake_is_caught(name):
    o = _rms_ns(**RMS_MUTANTS[name])
    caught = []
    for pin in (pin_rms_library, pin_rms_exact, pin_rms_closed_forms):
        try:
            pin(o)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"


# --------------------------------------------------------------------------
# mask monitor (change rate between two masks, mask verification)
# --------------------------------------------------------------------------

def _brute_monitor(old_bits, new_bits, K, n, m):
    """Bit by bit with Python integers: byte k // 8, bit k % 8."""
    O = old_bits.shape[0]
    changed, bad, rows = 0, 0, []
    for i in range(O):
        r = 0
        for k in range(K):
            a = (int(old_bits[i, k // 8]) >> (k % 8)) & 1
            b = (int(new_bits[i, k // 8]) >> (k % 8)) & 1
            r += a != b
        rows.append(r)
        changed += r
        for grp in range(K // m):
            kept = sum((int(new_bits[i, k // 8]) >> (k % 8)) & 1 for k in range(grp * m, grp * m + m))
            bad += kept != n
    return changed, bad, rows


def pin_mask_monitor(o):
    rng = np.random.default_rng(11)
    for (O, K, n, m) in ((3, 16, 2, 4), (5, 64, 3, 4), (2, 48, 6, 8), (4, 32, 2, 4)):
        a = rng.integers(0, 256, (O, K // 8), dtype=np.uint8)
        b = rng.integers(0, 256, (O, K // 8), dtype=np.uint8)
        ch, bad, rows = o.mask_monitor(a, b, K, n, m)
        bch, bbad, brows = _brute_monitor(a, b, K, n, m)
        assert (ch, bad, list(rows)) == (bch, bbad, brows)
        assert o.mask_monitor(a, a, K, n, m)[0] == 0
        assert o.mask_monitor(a, ~a, K, n, m)[0] == O * K
        assert o.mask_monitor(b, a, K, n, m)[0] == ch
    # masks made by the weight preparation keep exactly N per group; one flipped
    # bit is one changed position and one bad group
    for n, m in PATTERNS:
        W = synthetic.latent_weights(6, 64, seed=5)
        _, _, mb, _ = oracle.prepare_weights(W, n, m)
        assert o.mask_monitor(mb, mb, 64, n, m)[:2] == (0, 0)
        mb2 = mb.copy()
        mb2[2, 3] ^= 0x10  # weight 28 of row 2
        ch, bad, rows = o.mask_monitor(mb, mb2, 64, n, m)
        assert (ch, bad) == (1, 1) and rows.tolist() == [0, 0, 1, 0, 0, 0]


def test_mask_monitor_pins():
    pin_mask_monitor(oracle)


def _mm_changed_bytes(old_bits, new_bits, K, n, m):
    _, bad, _ = oracle.mask_monitor(old_bits, new_bits, K, n, m)
    rows = np.count_nonzero(np.asarray(old_bits) != np.asarray(new_bits), axis=1).astype(np.int64)
    return int(rows.sum()), bad, rows


def _mm_verify_old(old_bits, new_bits, K, n, m):
    return oracle.mask_monitor(new_bits, old_bits, K, n, m)[0], oracle.mask_monitor(new_bits, old_bits, K, n, m)[1], \
        oracle.mask_monitor(old_bits, new_bits, K, n, m)[2]


def _mm_kept_at_most(old_bits, new_bits, K, n, m):
    ch, _, rows = oracle.mask_monitor(old_bits, new_bits, K, n, m)
    new = np.unpackbits(np.asarray(new_bits, np.uint8), axis=1, bitorder="little")[:, :K].astype(bool)
    kept = new.reshape(new.shape[0], K // m, m).sum(axis=2)
    return ch, int(np.count_nonzero(kept > n)), rows


@pytest.mark.parametrize("name,fn", [("changed_bytes_not_bits", _mm_changed_bytes), ("verifies_old_mask", _mm_verify_old),
                                     ("counts_only_excess", _mm_kept_at_most)])
def test_planted_mask_monitor_mistake_is_caught(name, fn):
    o = types.SimpleNamespace(mask_monitor=fn)
    with pytest.raises(AssertionError):
        pin_mask_monitor(o)


# --------------------------------------------------------------------------
# bf16 scale storage (the halo card keeps one bf16 row_scale per row)
# --------------------------------------------------------------------------

def pin_scale_bf16(o):
    """The rounding agrees with torch's float32 -> bfloat16 conversion (a library
    routine, round to nearest even) on random values and on exact ties; the
    weights are ternarised with the rounded scale (|w| > s/2 on kept weights)."""
    import torch
    v = np.random.default_rng(12).uniform(1e-6, 1.0, 4096).astype(np.float32)
    ties = (np.array([0x3F808000, 0x3F818000, 0x3F80FFFF, 0x3F807FFF], np.uint32)).view(np.float32)
    for a in (v, ties):
        ref = torch.from_numpy(a).to(torch.bfloat16).float().numpy()
        assert np.array_equal(o.round_to_bf16(a).view(np.uint32), ref.view(np.uint32))
    for n, m in PATTERNS:
        W = synthetic.latent_weights(16, 64, seed=9)
        _, s32, _, _ = o.prepare_weights(W, n, m)
        _, s16, mb, Wt = o.prepare_weights(W, n, m, scale_bf16=True)
        assert np.array_equal(s16.view(np.uint32), torch.from_numpy(s32).to(torch.bfloat16).float().numpy().view(np.uint32))
        keep = np.unpackbits(mb, axis=1, bitorder="little")[:, :64].astype(bool)
        expect = np.where(keep & (np.abs(W) > np.float32(0.5) * s16[:, None]), np.sign(W), 0).astype(np.int8)
        assert np.array_equal(Wt, expect)


def test_scale_bf16_pins():
    pin_scale_bf16(oracle)


def test_planted_scale_bf16_truncation_is_caught():
    def trunc(v):
        return (np.asarray(v, np.float32).view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
    o = types.SimpleNamespace(round_to_bf16=trunc, prepare_weights=oracle.prepare_weights)
    with pytest.raises(AssertionError):
        pin_scale_bf16(o)


# --------------------------------------------------------------------------
# global scale (the guide's module listing: one mean |W| over the whole matrix)
# --------------------------------------------------------------------------

def pin_global_scale(o):
    """Exact rational mean (fractions) on small matrices, including values whose
    float sum would lose low bits; torch's float64 mean of |W| agrees within
    rounding; the weights are ternarised with that single scale."""
    import torch
    rng = np.random.default_rng(21)
    for O, K in ((3, 16), (8, 64), (5, 48)):
        W = (rng.standard_normal((O, K)) * 0.02).astype(np.float32)
        W[0, 0] = np.float32(3.0e7)       # a huge and a tiny weight in one sum
        W[1, 3] = np.float32(1.0e-30)
        exact = sum((Fraction(float(abs(v))) for v in W.ravel()), Fraction(0))
        want = max(np.float32(float(exact) / float(O * K)), np.float32(1e-5))
        assert o.global_scale(W) == want
        ref = float(torch.from_numpy(np.abs(W).astype(np.float64)).mean())
        assert abs(float(o.global_scale(W)) - ref) <= 1e-6 * ref
        for n, m in PATTERNS:
            _, s, mb, Wt = o.prepare_weights(W, n, m, scale_global=True)
            assert np.all(s == want)
            keep = np.unpackbits(mb, axis=1, bitorder="little")[:, :K].astype(bool)
            expect = np.where(keep & (np.abs(W) > np.float32(0.5) * want), np.sign(W), 0).astype(np.int8)
            assert np.array_equal(Wt, expect)
    tiny = np.full((2, 16), 1e-9, np.float32)
    assert o.global_scale(tiny) == np.float32(1e-5)  # the clamp


def test_global_scale_pins():
    pin_global_scale(oracle)


@pytest.mark.parametrize("name", ["kept_only", "divided_by_kept_count", "float32_sum"])
def test_planted_global_scale_mistake_is_caught(name):
    def kept_only(W):
        mask = oracle.nm_mask(W, 2, 4)
        a = np.abs(W[mask]).astype(np.float64)
        return max(np.float32(math.fsum(a.tolist()) / a.size), np.float32(1e-5))

    def divided_by_kept_count(W):
        tot = math.fsum(np.abs(W).astype(np.float64).ravel().tolist())
        return max(np.float32(tot / (W.size // 2)), np.float32(1e-5))

    def float32_sum(W):
        return max(np.float32(np.sum(np.abs(W), dtype=np.float32) / np.float32(W.size)), np.float32(1e-5))

    fn = {"kept_only": kept_only, "divided_by_kept_count": divided_by_kept_count, "float32_sum": float32_sum}[name]

    def prep(W, n, m, scale_global=False):
        mask = oracle.nm_mask(W, n, m)
        scale = np.full(W.shape[0], fn(W), np.float32)
        Wt = oracle.ternarise(W, scale, mask)
        return oracle.pack_codes(Wt), scale, oracle.pack_mask_bits(mask), Wt

    o = types.SimpleNamespace(global_scale=fn, prepare_weights=prep)
    with pytest.raises(AssertionError):
        pin_global_scale(o)


# --------------------------------------------------------------------------
# training path: straight-through backward
# --------------------------------------------------------------------------

def _ste_inputs(O, K, T, n, m, seed):
    W = synthetic.latent_weights(O, K, seed=seed)
    _, x = synthetic.activations(T, K, seed=seed)
    dY = synthetic.output_grads(T, O, seed=seed)
    _, scale, mb, Wt = oracle.prepare_weights(W, n, m)
    xq, s = oracle.quant_act(x)
    keep = np.unpackbits(mb, axis=1, bitorder="little")[:, :K].astype(bool)
    return W, x, dY, Wt, scale, xq, s, keep


def pin_ste_backward(o):
    """torch autograd (float64) through the straight-through surrogate of the
    forward — x_hat = x + (x_q/s - x).detach(), W_hat = W + (scale*W_t - W).detach(),
    and for the guide's module form W~ = W + (W_t - W).detach() with the scale
    applied after the product — whose value is checked to equal the forward's y;
    one-hot loss gradients place single rows; the gradient reaches masked weights."""
    import torch
    f64 = torch.float64
    for (O, K, T, n, m, seed) in ((8, 32, 5, 2, 4, 0), (16, 64, 3, 3, 4, 1), (12, 48, 7, 6, 8, 2),
                                  (32, 32, 4, 4, 8, 3)):
        W, x, dY, Wt, scale, xq, s, keep = _ste_inputs(O, K, T, n, m, seed)
        y_fwd = oracle.linear(x, Wt, scale)[0]
        xl = torch.tensor(x, dtype=f64, requires_grad=True)
        Wl = torch.tensor(W, dtype=f64, requires_grad=True)
        x_hat = xl + (torch.tensor(xq, dtype=f64) / torch.tensor(s, dtype=f64)[:, None] - xl).detach()
        W_hat = Wl + (torch.tensor(Wt, dtype=f64) * torch.tensor(scale, dtype=f64)[:, None] - Wl).detach()
        y = x_hat @ W_hat.T
        np.testing.assert_allclose(y.detach().numpy(), y_fwd, rtol=1e-12, atol=1e-15)
        (y * torch.tensor(dY, dtype=f64)).sum().backward()
        dX, dW = o.ste_backward(dY, xq, s, Wt, scale)
        assert dX.shape == (T, K) and dW.shape == (O, K)
        np.testing.assert_allclose(dX, xl.grad.numpy(), rtol=1e-12, atol=1e-12 * np.abs(dX).max())
        np.testing.assert_allclose(dW, Wl.grad.numpy(), rtol=1e-12, atol=1e-12 * np.abs(dW).max())
        assert np.count_nonzero(dW[~keep]) == np.count_nonzero(~keep)  # masked weights get gradient

        W2 = torch.tensor(W, dtype=f64, requires_grad=True)
        W_tern = W2 + (torch.tensor(Wt, dtype=f64) - W2).detach()
        y2 = (x_hat.detach() @ W_tern.T) * torch.tensor(scale, dtype=f64)[None, :]
        np.testing.assert_allclose(y2.detach().numpy(), y_fwd, rtol=1e-12, atol=1e-15)
        (y2 * torch.tensor(dY, dtype=f64)).sum().backward()
        dX2, dW2 = o.ste_backward(dY, xq, s, Wt, scale, dw_ternary=True)
        np.testing.assert_allclose(dW2, W2.grad.numpy(), rtol=1e-12, atol=1e-12 * np.abs(dW2).max())
        np.testing.assert_array_equal(dX2, dX)

        t, i = T // 2, O - 1                               # one-hot loss gradient
        e = np.zeros((T, O), np.float32)
        e[t, i] = 1.0
        dXe, dWe = o.ste_backward(e, xq, s, Wt, scale)
        assert np.array_equal(np.nonzero(np.any(dXe != 0, axis=1))[0], [t])
        np.testing.assert_array_equal(dXe[t], scale[i].astype(np.float64) * Wt[i])
        assert np.array_equal(np.nonzero(np.any(dWe != 0, axis=1))[0], [i])
        np.testing.assert_allclose(dWe[i], xq[t].astype(np.float64) / float(s[t]), rtol=1e-15, atol=0)
    dX, dW = o.ste_backward(np.zeros((0, 4), np.float32), np.zeros((0, 16), np.int8), np.zeros(0, np.float32),
                            np.ones((4, 16), np.int8), np.ones(4, np.float32))
    assert dX.shape == (0, 16) and dW.shape == (4, 16) and not np.any(dW)


def test_ste_backward_pins():
    pin_ste_backward(oracle)


@pytest.mark.parametrize("name", ["dw_masked", "dx_no_scale", "dw_no_token_scale", "dw_transposed",
                                  "ternary_flag_ignored", "dx_latent_weights"])
def test_planted_ste_backward_mistake_is_caught(name):
    def bwd(dY, xq, s_tok, Wt, scale, dw_ternary=False):
        dY = np.asarray(dY, np.float64)
        sc = np.asarray(scale, np.float64)
        xhat = np.asarray(xq, np.float64) / np.asarray(s_tok, np.float64)[:, None]
        if name == "dw_no_token_scale":
            xhat = np.asarray(xq, np.float64)
        dX = (dY * (1.0 if name == "dx_no_scale" else sc[None, :])) @ np.asarray(Wt, np.float64)
        if name == "dx_latent_weights":   # the dense latent-scale product, not the ternary one
            dX = dY @ (np.sign(np.asarray(Wt, np.float64)) * sc[:, None] + 1e-3)
        dW = dY.T @ xhat
        if name == "dw_masked":
            dW = dW * (np.asarray(Wt) != 0)
        if name == "dw_transposed":
            dW = (xhat.T @ dY) if dW.shape[0] == dW.shape[1] else dW.T
        if dw_ternary and name != "ternary_flag_ignored":
            dW = dW * sc[:, None]
        return dX, dW

    with pytest.raises(AssertionError):
        pin_ste_backward(types.SimpleNamespace(ste_backward=bwd))


def test_ste_backward_worked_block():
    """The guide's 4-element block carried through the backward by hand
    (tests/golden/ste_backward_worked.json)."""
    with open(os.path.join(os.path.dirname(__file__), "golden", "ste_backward_worked.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        W = np.array([c["w"]], np.float32)
        mask = oracle.nm_mask(W, c["n"], c["m"])
        scale = oracle.row_scale(W, mask)
        Wt = oracle.ternarise(W, scale, mask)
        xq, s = oracle.quant_act(np.array([c["x"]], np.float32))
        dY = np.array([[c["dY"]]], np.float32)
        dX, dW = oracle.ste_backward(dY, xq, s, Wt, scale)
        _, dWt = oracle.ste_backward(dY, xq, s, Wt, scale, dw_ternary=True)
        np.testing.assert_allclose(dX[0], c["dX"], rtol=1e-6, atol=0)
        np.testing.assert_allclose(dW[0], c["dW"], rtol=1e-6, atol=0)
        np.testing.assert_allclose(dWt[0], c["dW_ternary"], rtol=1e-6, atol=0)


# --------------------------------------------------------------------------
# property-based: adversarial weight values against the brute force
# --------------------------------------------------------------------------

from hypothesis import given, settings, strategies as st  # noqa: E402

# exact ties, both zeros, tiny and huge magnitudes, and values on the 0.5 * scale threshold
_POOL = (0.0, -0.0, 1e-30, -1e-30, 1e-7, 0.25, -0.25, 0.5, -0.5, 0.75, 1.0, -1.0, 1.5, 3.0e4, -3.0e4, 1e30)


@st.composite
def _weight_case(draw):
    n, m = draw(st.sampled_from(PATTERNS))
    O = draw(st.integers(1, 3))
    K = 8 * draw(st.integers(1, 3))
    elem = st.one_of(st.sampled_from(_POOL), st.floats(-2.0, 2.0, width=32, allow_subnormal=False))
    vals = draw(st.lists(elem, min_size=O * K, max_size=O * K))
    return np.array(vals, np.float32).reshape(O, K), n, m


@settings(max_examples=150, deadline=None)
@given(_weight_case())
def test_prepare_matches_brute_force_on_adversarial_values(case):
    W, n, m = case
    packed, scale, mbits, Wt = oracle.prepare_weights(W, n, m)
    mask_b, scale_b, Wt_b = _brute_prepare(W, n, m)
    assert np.array_equal(np.unpackbits(mbits, axis=1, bitorder="little").astype(bool), mask_b)
    assert np.array_equal(scale.view(np.uint32), scale_b.view(np.uint32))
    assert np.array_equal(Wt, Wt_b)
    assert np.array_equal(packed, _bitstring_pack(Wt_b))


@settings(max_examples=150, deadline=None)
@given(st.lists(st.one_of(st.sampled_from(_POOL), st.floats(-1e4, 1e4, width=32, allow_subnormal=False)),
                min_size=16, max_size=48).filter(lambda v: len(v) % 16 == 0))
def test_quant_invariants_on_adversarial_values(vals):
    x = np.array([vals], np.float32)
    xq, s = oracle.quant_act(x)
    amax = float(np.max(np.abs(x)))
    assert s[0] == np.float32(127.0) / max(np.float32(amax), np.float32(1e-5))
    exact = x.astype(np.float64) * float(s[0])
    assert np.all(np.abs(xq - exact) <= 0.5 + 2.0 ** -17 * np.abs(exact))
    assert xq.min() >= -127 and xq.max() <= 127
    if amax >= 1e-5:
        assert abs(int(xq[0, np.argmax(np.abs(x[0]))])) == 127


@settings(max_examples=60, deadline=None)
@given(st.sampled_from(PATTERNS), st.integers(1, 6), st.sampled_from([16, 32]), st.integers(0, 5),
       st.integers(0, 2 ** 16), st.booleans())
def test_ste_backward_matches_autograd_on_random_shapes(nm, O, K, T, seed, tern):
    """Any shape, the empty token set included: float64 autograd through the
    straight-through surrogate agrees with the oracle's gradients."""
    import torch
    n, m = nm
    f64 = torch.float64
    W = synthetic.latent_weights(O, K, seed=seed, tag="hyp")
    _, x = synthetic.activations(T, K, seed=seed, tag="hyp")
    dY = synthetic.output_grads(T, O, seed=seed, tag="hyp")
    _, scale, _, Wt = oracle.prepare_weights(W, n, m)
    xq, s = oracle.quant_act(x) if T else (np.zeros((0, K), np.int8), np.zeros(0, np.float32))
    xl = torch.tensor(x, dtype=f64, requires_grad=True)
    Wl = torch.tensor(W, dtype=f64, requires_grad=True)
    x_hat = xl + (torch.tensor(xq, dtype=f64) / torch.tensor(s, dtype=f64)[:, None] - xl).detach()
    wq = torch.tensor(Wt, dtype=f64)
    sc = torch.tensor(scale, dtype=f64)
    if tern:
        y = (x_hat @ (Wl + (wq - Wl).detach()).T) * sc[None, :]
    else:
        y = x_hat @ (Wl + (wq * sc[:, None] - Wl).detach()).T
    (y * torch.tensor(dY, dtype=f64)).sum().backward()
    dX, dW = oracle.ste_backward(dY, xq, s, Wt, scale, dw_ternary=tern)
    gx = xl.grad.numpy() if xl.grad is not None else np.zeros((T, K))
    np.testing.assert_allclose(dX, gx, rtol=1e-12, atol=1e-12 * (np.abs(gx).max(initial=0.0) + 1e-300))
    np.testing.assert_allclose(dW, Wl.grad.numpy(), rtol=1e-12, atol=1e-12 * (np.abs(dW).max(initial=0.0) + 1e-300))


def test_ternarise_threshold_equals_float32_division_reading():
    """round(W / scale) read as an IEEE float32 division then round-half-even
    (the other plausible reading of the guide's W~ equation) and the oracle's
    exact reading (nonzero iff |w| > scale / 2) give the same codes for every
    float w and normal scale: scale / 2 is a float, the next float above it,
    h + ulp(h), gives w / scale - 1/2 >= 2^-24 / m > 2^-25 (h = m * 2^e), half
    the float spacing just above 1/2, so the float32 quotient is already above
    1/2.  Checked on the floats around the threshold of 400k scales."""
    rng = np.random.default_rng(21)
    n = 400_000
    s = (rng.uniform(1, 2, n) * 2.0 ** rng.integers(-16, 16, n)).astype(np.float32)
    s = np.maximum(s, oracle.EPS_SCALE)
    h = (s / np.float32(2)).astype(np.float32)
    for k in range(-3, 4):
        w = h.copy()
        for _ in range(abs(k)):
            w = np.nextafter(w, np.float32(np.inf if k > 0 else -np.inf))
        w = w * np.where(rng.random(n) < 0.5, np.float32(-1), np.float32(1))
        fp32_reading = np.clip(np.rint((w / s).astype(np.float32)), -1, 1).astype(np.int8)
        exact = oracle.ternarise(w[:, None], s, np.ones((n, 1), bool))[:, 0]
        assert np.array_equal(fp32_reading, exact), k
