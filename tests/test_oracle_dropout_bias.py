"""Pins of the bias / dropout oracle (CPU only), and planted mistakes.

What pins it, besides itself: the published known-answer vectors of
Philox4x32-10 (tests/golden/philox4x32_10_kat.json); the Weyl constants'
closed forms; the keep
fraction and byte uniformity within binomial / chi-square bounds; p = 0
reducing to the plain oracle; a -inf bias above the diagonal reducing to the
causal oracle; a bias scale * Q' K'^T reducing to the plain attention of the
concatenated operands (a different code path: extra head dimensions); a
per-row constant bias (softmax shift invariance); the mean over seeds
approaching the undropped result; and the backward against central finite
differences of the forward at a fixed mask.
"""
import contextlib
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import dropout_bias as DB


def _rand(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


_KAT = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.json")


def pin_philox_known_answers():
    """Philox4x32-10 reproduces the generator authors' published
    known-answer vectors bit for bit (an independent reference: a wrong
    multiplier, round count, word order or key schedule changes every
    output word)."""
    with open(_KAT) as f:
        vectors = json.load(f)["vectors"]
    assert len(vectors) == 3
    for vec in vectors:
        c = [np.array([int(x, 16)], dtype=np.uint64) for x in vec["counter"]]
        k0, k1 = (int(x, 16) for x in vec["key"])
        got = [int(np.asarray(w).ravel()[0]) for w in DB.philox4x32_10(*c, k0, k1)]
        want = [int(x, 16) for x in vec["output"]]
        assert got == want, (vec["name"], [f"{x:08x}" for x in got])


def pin_weyl_constants():
    phi = (1 + math.sqrt(5)) / 2
    assert DB.PHILOX_W0 == int((phi - 1) * 2 ** 32)
    assert DB.PHILOX_W1 == int((math.sqrt(3) - 1) * 2 ** 32)
    assert DB.PHILOX_M0 & 1 and DB.PHILOX_M1 & 1  # odd multipliers


def pin_bytes_uniform_and_keep_fraction():
    keep, sc = DB.dropout_keep(2, 2, 256, seed=123456789, offset=7, p_drop=0.25)
    t = DB.keep_threshold(0.25)
    assert t == 192 and sc == 256 / 192
    n = keep.size
    frac = keep.mean()
    sd = math.sqrt(0.75 * 0.25 / n)
    assert abs(frac - 0.75) < 5 * sd
    # raw bytes: chi-square over 256 bins
    w = DB.philox4x32_10(np.arange(4096), 3, 5, 9, 0x12345678, 0x9ABCDEF0)
    by = np.concatenate([((x[:, None] >> (8 * np.arange(4, dtype=np.uint32))) & 0xFF).ravel()
                         for x in w])
    counts = np.bincount(by, minlength=256)
    exp = by.size / 256
    chi2 = float(np.sum((counts - exp) ** 2 / exp))
    assert chi2 < 255 + 6 * math.sqrt(2 * 255)
    # bits of word 0 vs word 1 are not correlated
    corr = np.corrcoef(w[0].astype(np.float64), w[1].astype(np.float64))[0, 1]
    assert abs(corr) < 0.05


def pin_mask_depends_on_seed_offset_head():
    a, _ = DB.dropout_keep(1, 2, 128, seed=1, offset=0, p_drop=0.5)
    b, _ = DB.dropout_keep(1, 2, 128, seed=2, offset=0, p_drop=0.5)
    c, _ = DB.dropout_keep(1, 2, 128, seed=1, offset=1, p_drop=0.5)
    d, _ = DB.dropout_keep(1, 2, 128, seed=1 << 32, offset=0, p_drop=0.5)
    for other in (b, c, d):
        assert 0.4 < np.mean(a != other) < 0.6
    assert 0.4 < np.mean(a[0, 0] != a[0, 1]) < 0.6
    again, _ = DB.dropout_keep(1, 2, 128, seed=1, offset=0, p_drop=0.5)
    assert np.array_equal(a, again)
    assert DB.dropout_keep(1, 1, 64, 5, 0, 0.0)[0].all()  # p = 0 keeps all


def pin_no_dropout_no_bias_is_plain():
    q, k, v = _rand(1, 2, 2, 70, 16), _rand(2, 2, 2, 70, 16), _rand(3, 2, 2, 70, 16)
    for causal in (False, True):
        o, l = DB.attention_fwd_ex(q, k, v, 0.25, causal)
        ro, rl = oracle.attention_fwd(q, k, v, 0.25, causal)
        np.testing.assert_allclose(o, ro, atol=1e-12)
        np.testing.assert_allclose(l, rl, atol=1e-12)
        keep, sc = DB.dropout_keep(2, 2, 70, 9, 0, 0.0)
        o2, _ = DB.attention_fwd_ex(q, k, v, 0.25, causal, keep=keep, keep_scale=sc)
        np.testing.assert_allclose(o2, ro, atol=1e-12)


def pin_bias_as_causal_mask():
    q, k, v = _rand(4, 1, 2, 50, 8), _rand(5, 1, 2, 50, 8), _rand(6, 1, 2, 50, 8)
    n = 50
    bias = np.where(np.arange(n)[None, :] <= np.arange(n)[:, None], 0.0, -np.inf)[None, None]
    o, l = DB.attention_fwd_ex(q, k, v, 0.3, False, bias=bias)
    ro, rl = oracle.attention_fwd(q, k, v, 0.3, True)
    np.testing.assert_allclose(o, ro, atol=1e-12)
    np.testing.assert_allclose(l, rl, atol=1e-12)


def pin_bias_as_extra_dimensions():
    """bias = scale Q' K'^T is the attention of [Q, Q'] and [K, K']; a
    transposed or mis-broadcast bias would not be."""
    B, H, N, d, e = 2, 3, 40, 8, 4
    q, k, v = _rand(7, B, H, N, d), _rand(8, B, H, N, d), _rand(9, B, H, N, d)
    qe, ke = _rand(10, B, H, N, e), _rand(11, B, H, N, e)
    scale = 0.35
    bias = scale * np.einsum("bhie,bhje->bhij", qe, ke)
    for causal in (False, True):
        o, l = DB.attention_fwd_ex(q, k, v, scale, causal, bias=bias)
        ro, rl = oracle.attention_fwd(np.concatenate([q, qe], -1), np.concatenate([k, ke], -1),
                                      v, scale, causal)
        np.testing.assert_allclose(o, ro, atol=1e-12)
        np.testing.assert_allclose(l, rl, atol=1e-12)
    # broadcasting over the batch: bias [1, H, N, N]
    bias1 = bias[:1]
    o, _ = DB.attention_fwd_ex(q, k, v, scale, False, bias=bias1)
    ro, _ = oracle.attention_fwd(np.concatenate([q, qe[:1].repeat(B, 0)], -1),
                                 np.concatenate([k, ke[:1].repeat(B, 0)], -1), v, scale, False)
    np.testing.assert_allclose(o, ro, atol=1e-12)


def pin_row_constant_bias():
    q, k, v = _rand(12, 1, 1, 30, 8), _rand(13, 1, 1, 30, 8), _rand(14, 1, 1, 30, 8)
    c = _rand(15, 30)
    o, l = DB.attention_fwd_ex(q, k, v, 0.5, False, bias=np.repeat(c[:, None], 30, 1)[None, None])
    ro, rl = oracle.attention_fwd(q, k, v, 0.5, False)
    np.testing.assert_allclose(o, ro, atol=1e-12)
    np.testing.assert_allclose(l, rl + c[None, None], atol=1e-12)


def pin_dropout_mean_over_seeds():
    """E[O] over masks is the undropped O (the 256/t rescale); 400 seeds."""
    q, k, v = _rand(16, 1, 1, 24, 8), _rand(17, 1, 1, 24, 8), _rand(18, 1, 1, 24, 8)
    ro, _ = oracle.attention_fwd(q, k, v, 0.5, False)
    acc = np.zeros_like(ro)
    n = 400
    for s in range(n):
        keep, sc = DB.dropout_keep(1, 1, 24, seed=1000 + s, offset=0, p_drop=0.3)
        acc += DB.attention_fwd_ex(q, k, v, 0.5, False, keep=keep, keep_scale=sc)[0]
    err = np.abs(acc / n - ro)
    assert err.max() < 0.12 and err.mean() < 0.03


def pin_backward_finite_differences():
    B, H, N, d = 1, 2, 20, 6
    q, k, v, do = (_rand(20 + i, B, H, N, d) for i in range(4))
    bias = _rand(30, 1, H, N, N)
    keep, sc = DB.dropout_keep(B, H, N, seed=77, offset=3, p_drop=0.2)
    scale = 0.4
    for causal in (False, True):
        dq, dk, dv = DB.attention_bwd_ex(q, k, v, do, scale, causal, bias, keep, sc)

        def f(q_, k_, v_):
            return float(np.sum(DB.attention_fwd_ex(q_, k_, v_, scale, causal, bias, keep, sc)[0] * do))

        h = 1e-6
        rng = np.random.default_rng(31)
        for g, idx in ((dq, 0), (dk, 1), (dv, 2)):
            for _ in range(6):
                pos = tuple(int(rng.integers(0, s)) for s in q.shape)
                args = [q.copy(), k.copy(), v.copy()]
                args[idx][pos] += h
                fp = f(*args)
                args[idx][pos] -= 2 * h
                fm = f(*args)
                num = (fp - fm) / (2 * h)
                assert abs(num - g[pos]) <= 1e-6 * max(1.0, abs(num)), (idx, pos, num, g[pos])


PINS = [
    pin_philox_known_answers,
    pin_weyl_constants,
    pin_bytes_uniform_and_keep_fraction,
    pin_mask_depends_on_seed_offset_head,
    pin_no_dropout_no_bias_is_plain,
    pin_bias_as_causal_mask,
    pin_bias_as_extra_dimensions,
    pin_row_constant_bias,
    pin_dropout_mean_over_seeds,
    pin_backward_finite_differences,
]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# ---------------------------------------------------------------------------
# planted mistakes
# ---------------------------------------------------------------------------

_orig = {n: getattr(DB, n) for n in ("philox4x32_10", "dropout_keep", "attention_fwd_ex",
                                     "attention_bwd_ex", "_scores_ex")}


def _mut_bias_transposed(q, k, scale, causal, bias):
    return _orig["_scores_ex"](q, k, scale, causal, None if bias is None else bias.T)


def _mut_bias_after_mask(q, k, scale, causal, bias):
    s = _orig["_scores_ex"](q, k, scale, causal, None)
    return s if bias is None else s + np.where(np.isfinite(bias), bias, 0.0)


def _mut_no_rescale(B, H, N, seed, offset, p_drop):
    keep, _ = _orig["dropout_keep"](B, H, N, seed, offset, p_drop)
    return keep, 1.0


def _mut_keep_inverted(B, H, N, seed, offset, p_drop):
    keep, sc = _orig["dropout_keep"](B, H, N, seed, offset, p_drop)
    return ~keep if p_drop > 0 else keep, sc


def _mut_bwd_dp_unmasked(q, k, v, do, scale, causal, bias=None, keep=None, keep_scale=1.0):
    """dV uses the dropped P, but dP is not masked."""
    q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
    dq, dk, dv = (np.empty_like(x) for x in (q, k, v))
    for b in range(q.shape[0]):
        for h in range(q.shape[1]):
            p, _ = oracle.softmax_rows(DB._scores_ex(q[b, h], k[b, h], scale, causal,
                                                     DB._head_bias(bias, b, h)))
            z = keep[b, h] * keep_scale if keep is not None else 1.0
            o = (p * z) @ v[b, h]
            dv[b, h] = (p * z).T @ do[b, h]
            ds = p * (do[b, h] @ v[b, h].T - np.sum(do[b, h] * o, axis=1)[:, None])
            dq[b, h], dk[b, h] = scale * (ds @ k[b, h]), scale * (ds.T @ q[b, h])
    return dq, dk, dv


def _philox_variant(rounds=10, swap_words=False, bump_first=False, swap_mult=False):
    """A Philox4x32 with one plausible slip, written out independently of
    the oracle's function so the slip is the only difference."""
    M32 = 0xFFFFFFFF
    m0, m1 = (DB.PHILOX_M1, DB.PHILOX_M0) if swap_mult else (DB.PHILOX_M0, DB.PHILOX_M1)

    def f(c0, c1, c2, c3, k0, k1):
        cs = np.broadcast_arrays(*[np.asarray(x, dtype=np.uint64) & np.uint64(M32)
                                   for x in (c0, c1, c2, c3)])
        a, b, c, d = (x.copy() for x in cs)
        ka, kb = np.uint64(k0 & M32), np.uint64(k1 & M32)
        for r in range(rounds):
            if bump_first:
                ka = (ka + np.uint64(DB.PHILOX_W0)) & np.uint64(M32)
                kb = (kb + np.uint64(DB.PHILOX_W1)) & np.uint64(M32)
            p0, p1 = np.uint64(m0) * a, np.uint64(m1) * c
            a, b, c, d = ((p1 >> np.uint64(32)) ^ b ^ ka, p1 & np.uint64(M32),
                          (p0 >> np.uint64(32)) ^ d ^ kb, p0 & np.uint64(M32))
            if not bump_first:
                ka = (ka + np.uint64(DB.PHILOX_W0)) & np.uint64(M32)
                kb = (kb + np.uint64(DB.PHILOX_W1)) & np.uint64(M32)
        out = [x.astype(np.uint32) for x in (a, b, c, d)]
        if swap_words:
            out = [out[1], out[0], out[3], out[2]]
        return tuple(out)

    return f


MUTANTS = {
    "philox_7_rounds": {"philox4x32_10": _philox_variant(rounds=7)},
    "philox_output_words_swapped": {"philox4x32_10": _philox_variant(swap_words=True)},
    "philox_key_bumped_before_round": {"philox4x32_10": _philox_variant(bump_first=True)},
    "philox_multipliers_swapped": {"philox4x32_10": _philox_variant(swap_mult=True)},
    "bias_transposed": {"_scores_ex": _mut_bias_transposed},
    "bias_added_after_mask": {"_scores_ex": _mut_bias_after_mask},
    "dropout_without_rescale": {"dropout_keep": _mut_no_rescale},
    "dropout_keep_inverted": {"dropout_keep": _mut_keep_inverted},
    "bwd_ignores_dropout": {"attention_bwd_ex": _mut_bwd_dp_unmasked},
}


@contextlib.contextmanager
def planted(patches):
    saved = []
    for name, fn in patches.items():
        for mod in (DB, oracle):
            if hasattr(mod, name):
                saved.append((mod, name, getattr(mod, name)))
                setattr(mod, name, fn)
    try:
        yield
    finally:
        for mod, name, fn in reversed(saved):
            setattr(mod, name, fn)


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_mutant_is_caught(mutant):
    caught = []
    with planted(MUTANTS[mutant]):
        for pin in PINS:
            try:
                pin()
            except Exception:
                caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {mutant}"
