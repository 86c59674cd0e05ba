"""Plant plausible mistakes in the oracle (on the CPU) and check the pins
catch each one.

Every mutant below is a small, realistic slip: a dropped scale, a mask in
the wrong direction, a transposed operand, a wrong sign, a missing rescale,
an unnormalised merge weight. Each must make at least one pin of
``test_oracle_pins.py`` fail; otherwise the pins would not be pinning the
oracle to anything.
"""
import contextlib

import numpy as np
import pytest

import oracle
from oracle import attention as A

import test_oracle_pins as pins


def _mut_scores_no_scale(q, k, scale, causal, row_offset=0):
    return _orig["scores"](q, k, 1.0, causal, row_offset)


def _mut_scores_mask_flipped(q, k, scale, causal, row_offset=0):
    s = scale * (q @ k.T)
    if causal:
        i = np.arange(q.shape[0])[:, None] + row_offset
        j = np.arange(k.shape[0])[None, :]
        s = np.where(j >= i, s, -np.inf)
    return s


def _mut_scores_mask_zero(q, k, scale, causal, row_offset=0):
    s = scale * (q @ k.T)
    if causal:
        i = np.arange(q.shape[0])[:, None] + row_offset
        j = np.arange(k.shape[0])[None, :]
        s = np.where(j <= i, s, 0.0)
    return s


def _mut_softmax_lse_without_max(s):
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=1, keepdims=True)
    return e / l, np.log(l)[:, 0]


def _mut_softmax_divide_by_max(s):
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=1, keepdims=True)
    return e / np.max(e, axis=1, keepdims=True), (m + np.log(l))[:, 0]


def _mut_fwd_transposed_p(q, k, v, scale, causal):
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    lead = q.shape[:-2]
    qf = q.reshape(-1, *q.shape[-2:])
    kf = k.reshape(-1, *k.shape[-2:])
    vf = v.reshape(-1, *v.shape[-2:])
    o = np.empty((qf.shape[0], qf.shape[1], vf.shape[-1]))
    lse = np.empty(qf.shape[:2])
    for h in range(qf.shape[0]):
        p, lse[h] = A.softmax_rows(A.scores(qf[h], kf[h], scale, causal))
        if p.shape[0] == p.shape[1]:
            o[h] = p.T @ vf[h]
        else:
            o[h] = p @ vf[h]
    return o.reshape(*lead, *o.shape[1:]), lse.reshape(*lead, lse.shape[-1])


def _bwd_variant(kind):
    def bwd(q, k, v, do, scale, causal):
        q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
        lead = q.shape[:-2]
        qf, kf, vf, dof = (x.reshape(-1, *x.shape[-2:]) for x in (q, k, v, do))
        dq, dk, dv = (np.empty_like(x) for x in (qf, kf, vf))
        for h in range(qf.shape[0]):
            s = A.scores(qf[h], kf[h], scale, causal)
            p, lse = A.softmax_rows(s)
            o = p @ vf[h]
            dv[h] = p.T @ dof[h]
            dp = dof[h] @ vf[h].T
            dsum = np.sum(dof[h] * o, axis=1)
            if kind == "d_from_v":
                dsum = np.sum(dof[h] * vf[h], axis=1)
            ds = p * (dp - dsum[:, None])
            if kind == "ds_sign":
                ds = -ds
            dq[h] = scale * (ds @ kf[h])
            if kind == "dq_transposed":
                dq[h] = scale * (ds.T @ kf[h])
            dk[h] = scale * (ds.T @ qf[h])
            if kind == "dk_no_scale":
                dk[h] = ds.T @ qf[h]
        return (dq.reshape(*lead, *q.shape[-2:]), dk.reshape(*lead, *k.shape[-2:]),
                dv.reshape(*lead, *v.shape[-2:]))
    return bwd


def _mut_online_no_rescale(q, k, v, scale, causal, col_blocks):
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    nq = q.shape[0]
    m = np.full(nq, -np.inf)
    l = np.zeros(nq)
    acc = np.zeros((nq, v.shape[1]))
    start = 0
    for width in col_blocks:
        s = scale * (q @ k[start:start + width].T)
        if causal:
            i = np.arange(nq)[:, None]
            j = np.arange(start, start + width)[None, :]
            s = np.where(j <= i, s, -np.inf)
        m_new = np.maximum(m, np.max(s, axis=1))
        ref = np.where(np.isfinite(m_new), m_new, 0.0)
        alpha = np.where(np.isfinite(m), np.exp(m - ref), 0.0)
        p = np.exp(s - ref[:, None])
        l = alpha * l + np.sum(p, axis=1)
        acc = acc + p @ v[start:start + width]  # planted: acc not rescaled
        m = m_new
        start += width
    return acc / l[:, None], m + np.log(l)


def _mut_merge_unnormalised(o_parts, lse_parts):
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    mx = np.max(lse_parts)
    w = np.exp(lse_parts - mx)
    return w @ o_parts, mx + np.log(np.sum(w))


def _mut_decode_drop_last_key(q, kcache, vcache, seqlens, scale):
    return _orig["decode"](q, kcache, vcache, np.maximum(np.asarray(seqlens) - 1, 1),
                           scale)


def _mut_paged_head_modulo(q, kpages, vpages, block_table, seqlens, scale):
    # planted: query head h reads KV head h % Hkv instead of h // (Hq / Hkv)
    q = np.asarray(q, dtype=np.float64)
    hkv = kpages.shape[1]
    out_o = np.zeros((q.shape[0], q.shape[1], vpages.shape[-1]))
    out_l = np.full(q.shape[:2], -np.inf)
    for h in range(q.shape[1]):
        kp = np.repeat(kpages[:, h % hkv:h % hkv + 1], 1, axis=1)
        vp = np.repeat(vpages[:, h % hkv:h % hkv + 1], 1, axis=1)
        o, l = _orig["decode_paged"](q[:, h:h + 1], kp, vp, block_table, seqlens, scale)
        out_o[:, h], out_l[:, h] = o[:, 0], l[:, 0]
    return out_o, out_l


def _mut_paged_row_within_page(q, kpages, vpages, block_table, seqlens, scale):
    # planted: the row inside a page taken as t // page instead of t % page
    page = kpages.shape[2]
    q = np.asarray(q, dtype=np.float64)
    table = np.asarray(block_table)
    o = np.zeros((q.shape[0], q.shape[1], vpages.shape[-1]))
    lse = np.full(q.shape[:2], -np.inf)
    g = q.shape[1] // kpages.shape[1]
    for b in range(q.shape[0]):
        n = int(seqlens[b])
        if n == 0:
            continue
        t = np.arange(n)
        pg, row = table[b, t // page], np.minimum(t // page, page - 1)
        for h in range(q.shape[1]):
            kb, vb = kpages[pg, h // g, row], vpages[pg, h // g, row]
            p, l_row = A.softmax_rows(A.scores(q[b, h][None, :], kb, scale, False))
            o[b, h], lse[b, h] = (p @ vb)[0], l_row[0]
    return o, lse


_orig = {name: getattr(A, name) for name in
         ("scores", "softmax_rows", "attention_fwd", "attention_bwd",
          "online_attention_fwd", "merge_partials", "decode", "decode_paged")}

MUTANTS = {
    "scores_no_scale": {"scores": _mut_scores_no_scale},
    "mask_flipped": {"scores": _mut_scores_mask_flipped},
    "mask_zero_not_minus_inf": {"scores": _mut_scores_mask_zero},
    "lse_without_max": {"softmax_rows": _mut_softmax_lse_without_max},
    "softmax_divide_by_max": {"softmax_rows": _mut_softmax_divide_by_max},
    "pv_transposed": {"attention_fwd": _mut_fwd_transposed_p},
    "bwd_ds_sign": {"attention_bwd": _bwd_variant("ds_sign")},
    "bwd_dk_no_scale": {"attention_bwd": _bwd_variant("dk_no_scale")},
    "bwd_dq_transposed": {"attention_bwd": _bwd_variant("dq_transposed")},
    "bwd_d_from_v": {"attention_bwd": _bwd_variant("d_from_v")},
    "online_no_rescale": {"online_attention_fwd": _mut_online_no_rescale},
    "merge_unnormalised": {"merge_partials": _mut_merge_unnormalised},
    "decode_drops_last_key": {"decode": _mut_decode_drop_last_key},
    "paged_head_modulo": {"decode_paged": _mut_paged_head_modulo},
    "paged_row_within_page": {"decode_paged": _mut_paged_row_within_page},
}


@contextlib.contextmanager
def planted(patches):
    saved = []
    for name, fn in patches.items():
        for mod in (A, oracle):
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
        for pin in pins.PINS:
            try:
                pin()
            except Exception:  # AssertionError, or a shape error the slip causes
                caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {mutant}"
