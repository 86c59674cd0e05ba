"""Pins for the fp64 oracle: properties the pages and the mathematics fix.

Each ``pin_*`` function raises AssertionError when the oracle breaks the
property. The tests below call them on the real oracle, and
``test_oracle_mutants.py`` calls them on oracles with a planted mistake to
show that each plausible mistake is caught by at least one pin.

Sources of the properties (page title, section):
* "Bellek Duvarinin Fizigi", "Softmax'in Kalesi": softmax rows sum to one;
  subtracting (or adding) a constant in a row leaves softmax unchanged.
* same page, "Online Softmax": the one-pass recurrence reaches the two-pass
  result exactly up to floating-point ordering.
* same page, "Maskeleme ve Dropout": query 0 sees only key 0 under the
  causal mask.
* same page, "Geri Yayilim": the gradients of sum(O * dO), checked against
  central finite differences; D = rowsum(dO * O) = rowsum(P * dP).
* same page, "Decode Asamasi: Flash-Decoding": splitting the key/value axis
  into chunks and merging by log-sum-exp equals the unsplit result.
* same page, "Duvarin Otesi": a paged, grouped-query KV cache is only a
  different storage of the same keys and values: its decode equals the
  decode of the contiguous cache with each KV head repeated for its query
  heads, whatever the page size or page order.
* "FlashAttention'i Anlamak Bolum 1", 0.2 Notasyon: the function itself,
  compared with an independent library implementation (PyTorch's
  scaled_dot_product_attention in float64, and its autograd).
"""
import math

import numpy as np
import pytest

import oracle
from oracle import attention as A

RNG_SEED = 1234


def _rand(rng, *shape):
    return rng.standard_normal(shape)


# ---------------------------------------------------------------------------
# pins
# ---------------------------------------------------------------------------

def pin_rows_sum_to_one():
    rng = np.random.default_rng(RNG_SEED)
    for causal in (False, True):
        q, k = _rand(rng, 37, 8), _rand(rng, 37, 8)
        p, _ = A.softmax_rows(A.scores(q, k, 0.3, causal))
        assert np.allclose(p.sum(axis=1), 1.0, atol=1e-12, rtol=0)
        assert np.all(p >= 0)
        if causal:
            assert np.all(np.triu(p, 1) == 0)


def pin_row_shift_invariance():
    """Adding c_i to every score of row i: O unchanged, LSE_i + c_i.

    The shift enters through the inputs only: q gains a coordinate c_i/scale
    and every key gains a coordinate 1, so S'_ij = S_ij + c_i.
    """
    rng = np.random.default_rng(RNG_SEED + 1)
    n, d, scale = 29, 6, 0.41
    q, k, v = _rand(rng, n, d), _rand(rng, n, d), _rand(rng, n, 5)
    c = 3.0 * _rand(rng, n)
    q2 = np.concatenate([q, (c / scale)[:, None]], axis=1)
    k2 = np.concatenate([k, np.ones((n, 1))], axis=1)
    for causal in (False, True):
        o1, l1 = oracle.attention_fwd(q, k, v, scale, causal)
        o2, l2 = oracle.attention_fwd(q2, k2, v, scale, causal)
        assert np.allclose(o1, o2, atol=1e-12, rtol=1e-12)
        assert np.allclose(l2 - l1, c, atol=1e-12, rtol=1e-12)


def pin_single_key():
    """One key: O = v_0 for every query; LSE = scale * q . k_0."""
    rng = np.random.default_rng(RNG_SEED + 2)
    q, k, v = _rand(rng, 5, 7), _rand(rng, 1, 7), _rand(rng, 1, 3)
    o, lse = oracle.attention_fwd(q, k, v, 0.7, False)
    assert np.allclose(o, np.repeat(v, 5, axis=0), atol=1e-14)
    assert np.allclose(lse, 0.7 * (q @ k[0]), atol=1e-13)
    # N = 1 with the causal mask is the same problem
    o1, l1 = oracle.attention_fwd(q[:1], k, v, 0.7, True)
    assert np.allclose(o1[0], v[0], atol=1e-14)
    assert abs(l1[0] - 0.7 * float(q[0] @ k[0])) < 1e-13


def pin_identical_keys():
    """All keys equal: P uniform, O = mean(V), LSE = s_i + ln N."""
    rng = np.random.default_rng(RNG_SEED + 3)
    n, d = 23, 4
    q = _rand(rng, n, d)
    k = np.repeat(_rand(rng, 1, d), n, axis=0)
    v = _rand(rng, n, 6)
    o, lse = oracle.attention_fwd(q, k, v, 0.5, False)
    assert np.allclose(o, np.repeat(v.mean(axis=0)[None], n, axis=0),
                       atol=1e-13)
    assert np.allclose(lse, 0.5 * (q @ k[0]) + math.log(n), atol=1e-12)


def pin_causal_first_and_prefix_rows():
    """Causal row 0 sees only key 0; row i equals attention over keys 0..i."""
    rng = np.random.default_rng(RNG_SEED + 4)
    n, d = 19, 5
    q, k, v = _rand(rng, n, d), _rand(rng, n, d), _rand(rng, n, 4)
    o, lse = oracle.attention_fwd(q, k, v, 0.45, True)
    assert np.allclose(o[0], v[0], atol=1e-14)
    assert abs(lse[0] - 0.45 * float(q[0] @ k[0])) < 1e-13
    for i in (3, 11, n - 1):
        oi, li = oracle.attention_fwd(q[i:i + 1], k[:i + 1], v[:i + 1], 0.45,
                                      False)
        assert np.allclose(o[i], oi[0], atol=1e-13)
        assert abs(lse[i] - li[0]) < 1e-12


def pin_closed_form_two_by_two():
    """Hand-solvable case: Q = K = I_2, scale 1, so S = I_2.

    Row 0: P = [e, 1] / (e + 1); O_0 = (e v_0 + v_1) / (e + 1);
    LSE_0 = ln(e + 1). Causal: row 0 gives v_0 and LSE 1; row 1 gives
    P = [1, e] / (1 + e).
    """
    q = np.eye(2)
    k = np.eye(2)
    v = np.array([[1.0, 2.0, -1.0], [3.0, 4.0, 5.0]])
    e = math.e
    o, lse = oracle.attention_fwd(q, k, v, 1.0, False)
    assert np.allclose(o[0], (e * v[0] + v[1]) / (e + 1), atol=1e-15)
    assert np.allclose(o[1], (v[0] + e * v[1]) / (e + 1), atol=1e-15)
    assert np.allclose(lse, math.log(e + 1), atol=1e-15)
    oc, lc = oracle.attention_fwd(q, k, v, 1.0, True)
    assert np.allclose(oc[0], v[0], atol=1e-15) and abs(lc[0] - 1.0) < 1e-15
    assert np.allclose(oc[1], (v[0] + e * v[1]) / (1 + e), atol=1e-15)
    assert abs(lc[1] - math.log(1 + e)) < 1e-15


def pin_online_equals_two_pass():
    rng = np.random.default_rng(RNG_SEED + 5)
    for trial in range(6):
        n = int(rng.integers(1, 40))
        d = int(rng.integers(1, 9))
        q, k, v = _rand(rng, n, d) * 2, _rand(rng, n, d) * 2, _rand(rng, n, 3)
        widths = []
        left = n
        while left:
            w = int(rng.integers(1, left + 1))
            widths.append(w)
            left -= w
        for causal in (False, True):
            o1, l1 = oracle.attention_fwd(q, k, v, 0.6, causal)
            o2, l2 = oracle.online_attention_fwd(q, k, v, 0.6, causal, widths)
            assert np.allclose(o1, o2, atol=1e-12, rtol=1e-12), (trial, causal)
            assert np.allclose(l1, l2, atol=1e-12, rtol=1e-12), (trial, causal)


def _loss(q, k, v, do, scale, causal):
    o, _ = oracle.attention_fwd(q, k, v, scale, causal)
    return float(np.sum(o * do))


def pin_backward_finite_differences():
    rng = np.random.default_rng(RNG_SEED + 6)
    for causal in (False, True):
        n, d = 9, 4
        q, k, v, do = (_rand(rng, n, d) for _ in range(4))
        scale = 0.55
        dq, dk, dv = oracle.attention_bwd(q, k, v, do, scale, causal)
        h = 1e-6
        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            num = np.zeros_like(x)
            for idx in np.ndindex(*x.shape):
                xp = x.copy()
                xm = x.copy()
                xp[idx] += h
                xm[idx] -= h
                args_p = {"q": q, "k": k, "v": v}
                args_m = {"q": q, "k": k, "v": v}
                args_p[name] = xp
                args_m[name] = xm
                num[idx] = (_loss(args_p["q"], args_p["k"], args_p["v"], do,
                                  scale, causal)
                            - _loss(args_m["q"], args_m["k"], args_m["v"], do,
                                    scale, causal)) / (2 * h)
            rel = np.linalg.norm(num - g) / max(np.linalg.norm(num), 1e-30)
            assert rel < 1e-6, (name, causal, rel)


def pin_d_identity():
    """rowsum(P * dP) = rowsum(dO * O) (the D vector of the backward)."""
    rng = np.random.default_rng(RNG_SEED + 7)
    n, d = 21, 6
    q, k, v, do = (_rand(rng, n, d) for _ in range(4))
    for causal in (False, True):
        p, _ = A.softmax_rows(A.scores(q, k, 0.4, causal))
        o, _ = oracle.attention_fwd(q, k, v, 0.4, causal)
        dp = do @ v.T
        assert np.allclose(np.sum(p * dp, axis=1), np.sum(do * o, axis=1),
                           atol=1e-12)


def pin_decode_split_merge():
    rng = np.random.default_rng(RNG_SEED + 8)
    B, H, L, d = 3, 2, 50, 8
    q = _rand(rng, B, H, d)
    kc, vc = _rand(rng, B, H, L, d), _rand(rng, B, H, L, d)
    lens = np.array([50, 1, 17])
    o, lse = oracle.decode(q, kc, vc, lens, 0.35)
    for chunks in (1, 2, 3, 7, 64):
        o2, l2 = oracle.decode_split(q, kc, vc, lens, 0.35, chunks)
        assert np.allclose(o, o2, atol=1e-12), chunks
        assert np.allclose(lse, l2, atol=1e-12), chunks
    # the sequence with one cached token returns that token's value
    assert np.allclose(o[1], vc[1, :, 0], atol=1e-14)


def pin_decode_is_last_causal_row():
    rng = np.random.default_rng(RNG_SEED + 9)
    B, H, N, d = 2, 3, 24, 8
    q = _rand(rng, B, H, N, d)
    k, v = _rand(rng, B, H, N, d), _rand(rng, B, H, N, d)
    o, lse = oracle.attention_fwd(q, k, v, 0.3, True)
    od, ld = oracle.decode(q[:, :, -1], k, v, np.array([N, N]), 0.3)
    assert np.allclose(o[:, :, -1], od, atol=1e-13)
    assert np.allclose(lse[:, :, -1], ld, atol=1e-12)
    # a shorter visible prefix equals the causal row at that position
    od2, ld2 = oracle.decode(q[:, :, 9], k, v, np.array([10, 10]), 0.3)
    assert np.allclose(o[:, :, 9], od2, atol=1e-13)


def pin_rows_helper_matches_full():
    rng = np.random.default_rng(RNG_SEED + 10)
    n, d = 40, 8
    q, k, v = _rand(rng, n, d), _rand(rng, n, d), _rand(rng, n, d)
    for causal in (False, True):
        o, lse = oracle.attention_fwd(q, k, v, 0.3, causal)
        orows, lrows = oracle.attention_fwd_rows(q, k, v, 0.3, causal, 13, 29)
        assert np.allclose(o[13:29], orows, atol=1e-14)
        assert np.allclose(lse[13:29], lrows, atol=1e-14)


def pin_against_library_sdpa():
    """Forward and backward against PyTorch's float64 implementation."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(RNG_SEED + 11)
    B, H, n, d = 2, 3, 33, 16
    q, k, v, do = (_rand(rng, B, H, n, d) for _ in range(4))
    for causal in (False, True):
        scale = 1.0 / math.sqrt(d)
        o, lse = oracle.attention_fwd(q, k, v, scale, causal)
        dq, dk, dv = oracle.attention_bwd(q, k, v, do, scale, causal)
        tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True)
                      for x in (q, k, v))
        to = torch.nn.functional.scaled_dot_product_attention(
            tq, tk, tv, is_causal=causal, scale=scale)
        to.backward(torch.tensor(do, dtype=torch.float64))
        assert np.allclose(o, to.detach().numpy(), atol=1e-12)
        assert np.allclose(dq, tq.grad.numpy(), atol=1e-11)
        assert np.allclose(dk, tk.grad.numpy(), atol=1e-11)
        assert np.allclose(dv, tv.grad.numpy(), atol=1e-11)
        s = torch.tensor(q) @ torch.tensor(k).transpose(-1, -2) * scale
        if causal:
            s = s.masked_fill(torch.ones(n, n).triu(1).bool(), float("-inf"))
        assert np.allclose(lse, torch.logsumexp(s, dim=-1).numpy(), atol=1e-12)


def _paged_from_contiguous(rng, kc, vc, page, spare=3):
    """Store contiguous caches [B, Hkv, L, d] in shuffled pages of `page`
    rows (L a multiple of page), plus `spare` pages of noise that no block
    table entry names. Returns kpages, vpages, block_table."""
    B, hkv, L, d = kc.shape
    per = L // page
    total = B * per + spare
    order = rng.permutation(total)
    kp = rng.standard_normal((total, hkv, page, d)) * 100.0
    vp = rng.standard_normal((total, hkv, page, d)) * 100.0
    table = np.empty((B, per), dtype=np.int64)
    for b in range(B):
        for i in range(per):
            pg = order[b * per + i]
            table[b, i] = pg
            kp[pg] = kc[b, :, i * page:(i + 1) * page]
            vp[pg] = vc[b, :, i * page:(i + 1) * page]
    return kp, vp, table


def pin_paged_gqa_is_repeated_contiguous_decode():
    rng = np.random.default_rng(RNG_SEED + 12)
    B, hq, hkv, L, d = 3, 6, 2, 48, 8
    q = _rand(rng, B, hq, d)
    kc, vc = _rand(rng, B, hkv, L, d), _rand(rng, B, hkv, L, d)
    lens = np.array([48, 1, 29])
    # each KV head repeated for the hq / hkv consecutive query heads it serves
    kr, vr = np.repeat(kc, hq // hkv, axis=1), np.repeat(vc, hq // hkv, axis=1)
    o_ref, l_ref = oracle.decode(q, kr, vr, lens, 0.4)
    for page in (1, 8, 16, 48):
        kp, vp, table = _paged_from_contiguous(rng, kc, vc, page)
        o, lse = oracle.decode_paged(q, kp, vp, table, lens, 0.4)
        assert np.allclose(o, o_ref, atol=1e-13), page
        assert np.allclose(lse, l_ref, atol=1e-13), page
    # multi-query: one KV head for every query head
    k1, v1 = kc[:, :1], vc[:, :1]
    kp, vp, table = _paged_from_contiguous(rng, k1, v1, 16)
    o, lse = oracle.decode_paged(q, kp, vp, table, lens, 0.4)
    o1, l1 = oracle.decode(q, np.repeat(k1, hq, axis=1), np.repeat(v1, hq, axis=1), lens, 0.4)
    assert np.allclose(o, o1, atol=1e-13) and np.allclose(lse, l1, atol=1e-13)


def pin_paged_empty_and_one_key():
    rng = np.random.default_rng(RNG_SEED + 13)
    B, hq, hkv, L, d = 2, 2, 1, 16, 4
    q = _rand(rng, B, hq, d)
    kc, vc = _rand(rng, B, hkv, L, d), _rand(rng, B, hkv, L, d)
    kp, vp, table = _paged_from_contiguous(rng, kc, vc, 8)
    o, lse = oracle.decode_paged(q, kp, vp, table, np.array([0, 1]), 0.5)
    assert np.all(o[0] == 0.0) and np.all(np.isneginf(lse[0]))
    # one visible key: O is that key's value, LSE its score
    assert np.allclose(o[1], vc[1, 0, 0][None, :], atol=1e-14)
    assert np.allclose(lse[1], 0.5 * (q[1] @ kc[1, 0, 0]), atol=1e-14)


PINS = [
    pin_rows_sum_to_one,
    pin_row_shift_invariance,
    pin_single_key,
    pin_identical_keys,
    pin_causal_first_and_prefix_rows,
    pin_closed_form_two_by_two,
    pin_online_equals_two_pass,
    pin_backward_finite_differences,
    pin_d_identity,
    pin_decode_split_merge,
    pin_decode_is_last_causal_row,
    pin_rows_helper_matches_full,
    pin_against_library_sdpa,
    pin_paged_gqa_is_repeated_contiguous_decode,
    pin_paged_empty_and_one_key,
]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()
