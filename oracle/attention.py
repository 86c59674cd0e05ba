"""fp64 CPU oracle for exact scaled dot-product attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this
module: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` use it. It shares no code with the CUDA library.

Every function materialises the full score matrix S and probability matrix P
in float64 and follows the plain definition written out on the pages:

* "FlashAttention'i Anlamak Bolum 1" (blog.edumints.com), section 0.2
  Notasyon: S = Q K^T / sqrt(d) (+ B), P = softmax_row(S), O = P V, with
  N_q = N_k = N.
* "Bellek Duvarinin Fizigi" (webturing Principia), sections
  "Attention'in Cebiri" (the definition and the 1/sqrt(d_k) scale),
  "Softmax'in Kalesi" (subtracting the row maximum),
  "Online Softmax" (the running max / running sum recurrence),
  "Forward gecisin iskeleti" (the output accumulator recurrence and the
  final diag(l)^-1 normalisation),
  "Maskeleme ve Dropout" (causal: query i sees keys j <= i; masked scores
  are -inf before the row maximum),
  "Geri Yayilim" (saved log-sum-exp L, P = exp(S - L), D = rowsum(dO*O),
  dS = P * (dP - D)),
  "Decode Asamasi: Flash-Decoding" (split the key/value axis into chunks,
  each chunk gives (m, l, O~), merged by the rescale identity),
  "Duvarin Otesi" (the KV cache of decoding, and the inference-side methods
  it names: paged KV caches and grouped / multi-query attention).

Where those sections lost their display formulas in extraction, the reading
taken is the standard identity the surrounding prose describes; the readings
are listed with the build's design notes. The log-sum-exp is the natural
logarithm of sum_j exp(S_ij) with the scale already inside S.

Parity of every public function here is pinned by the CPU tests in
``tests/test_oracle_pins.py`` (closed forms, invariants, finite differences
and an independent library implementation), not by re-typing formulas.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "scores",
    "softmax_rows",
    "attention_fwd",
    "attention_fwd_rows",
    "attention_bwd",
    "online_attention_fwd",
    "decode",
    "decode_split",
    "merge_partials",
    "decode_paged",
]


# ---------------------------------------------------------------------------
# building blocks (one head at a time; every array float64)
# ---------------------------------------------------------------------------

def scores(q: np.ndarray, k: np.ndarray, scale: float, causal: bool,
           row_offset: int = 0) -> np.ndarray:
    """S = scale * q k^T with the causal mask applied as -inf.

    ``q`` is [Nq, d] (query rows ``row_offset ..``), ``k`` is [Nk, d].
    Causal ("Maskeleme ve Dropout"): query row i may look at key j only when
    j <= i; other entries are -inf, filled before any row maximum is taken.
    """
    s = scale * (q @ k.T)
    if causal:
        i = np.arange(q.shape[0])[:, None] + row_offset
        j = np.arange(k.shape[0])[None, :]
        s = np.where(j <= i, s, -np.inf)
    return s


def softmax_rows(s: np.ndarray):
    """Row softmax with the row maximum subtracted ("Softmax'in Kalesi").

    Returns (P, LSE) with LSE_i = m_i + ln sum_j exp(S_ij - m_i).
    Every row must contain at least one finite score.
    """
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=1, keepdims=True)
    p = e / l
    lse = (m + np.log(l))[:, 0]
    return p, lse


def _as_f64(x):
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# forward
# ---------------------------------------------------------------------------

def attention_fwd(q, k, v, scale: float, causal: bool):
    """O = softmax(scale * Q K^T [+ causal mask]) V and the per-row LSE.

    Shapes: q [..., Nq, d], k [..., Nk, d], v [..., Nk, dv]; leading axes
    are independent heads. Causal requires Nq == Nk. Returns
    (O [..., Nq, dv], LSE [..., Nq]) in float64.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    lead = q.shape[:-2]
    nq, nk = q.shape[-2], k.shape[-2]
    if causal and nq != nk:
        raise ValueError("causal attention here needs Nq == Nk")
    qf = q.reshape(-1, nq, q.shape[-1])
    kf = k.reshape(-1, nk, k.shape[-1])
    vf = v.reshape(-1, nk, v.shape[-1])
    o = np.empty((qf.shape[0], nq, vf.shape[-1]))
    lse = np.empty((qf.shape[0], nq))
    for h in range(qf.shape[0]):
        p, lse[h] = softmax_rows(scores(qf[h], kf[h], scale, causal))
        o[h] = p @ vf[h]
    return o.reshape(*lead, nq, vf.shape[-1]), lse.reshape(*lead, nq)


def attention_fwd_rows(q, k, v, scale: float, causal: bool, row0: int,
                       row1: int):
    """The rows row0..row1-1 of ``attention_fwd`` for one head.

    q [N, d], k [N, d], v [N, dv]. Only the needed score rows are formed, so
    a sampled row block of a long sequence costs O(rows * N * d).
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    s = scores(q[row0:row1], k, scale, causal, row_offset=row0)
    p, lse = softmax_rows(s)
    return p @ v, lse


def online_attention_fwd(q, k, v, scale: float, causal: bool, col_blocks):
    """One-pass forward over key/value blocks with the online recurrence.

    This is the streaming form the pages derive ("Online Softmax" and
    "Forward gecisin iskeleti"): for each key block b with scores S_b,
        m_new = max(m, rowmax(S_b))
        l     = exp(m - m_new) * l + rowsum(exp(S_b - m_new))
        O~    = exp(m - m_new) * O~ + exp(S_b - m_new) V_b
    and once all blocks are done O = diag(l)^-1 O~ and LSE = m + ln l.
    ``col_blocks`` is the list of block widths (summing to Nk). One head:
    q [Nq, d], k [Nk, d], v [Nk, dv]. It exists so the tests can check that
    the recurrence reaches the two-pass result (up to rounding order).
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    nq = q.shape[0]
    if sum(col_blocks) != k.shape[0]:
        raise ValueError("block widths must cover every key")
    m = np.full(nq, -np.inf)
    l = np.zeros(nq)
    acc = np.zeros((nq, v.shape[1]))
    start = 0
    for width in col_blocks:
        kb = k[start:start + width]
        vb = v[start:start + width]
        s = scale * (q @ kb.T)
        if causal:
            i = np.arange(nq)[:, None]
            j = np.arange(start, start + width)[None, :]
            s = np.where(j <= i, s, -np.inf)
        m_new = np.maximum(m, np.max(s, axis=1))
        # A row that has seen only masked keys keeps m = -inf. Its reference
        # is taken as 0 so that exp(-inf - (-inf)) never appears; nothing has
        # been accumulated for it, so its old-state factor is 0.
        ref = np.where(np.isfinite(m_new), m_new, 0.0)
        alpha = np.where(np.isfinite(m), np.exp(m - ref), 0.0)
        p = np.exp(s - ref[:, None])
        l = alpha * l + np.sum(p, axis=1)
        acc = alpha[:, None] * acc + p @ vb
        m = m_new
        start += width
    o = acc / l[:, None]
    lse = m + np.log(l)
    return o, lse


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------

def attention_bwd(q, k, v, do, scale: float, causal: bool):
    """Gradients of sum(O * dO) with respect to Q, K and V.

    Follows "Geri Yayilim": with the saved LSE, P = exp(S - LSE);
    dV = P^T dO; dP = dO V^T; D_i = sum_c dO_ic O_ic; dS = P * (dP - D);
    dQ = scale * dS K; dK = scale * dS^T Q. O and P are the oracle's own
    exact values. Shapes as in ``attention_fwd``; returns (dQ, dK, dV).
    """
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    lead = q.shape[:-2]
    n, d = q.shape[-2], q.shape[-1]
    qf, kf, vf, dof = (x.reshape(-1, x.shape[-2], x.shape[-1])
                       for x in (q, k, v, do))
    dq = np.empty_like(qf)
    dk = np.empty_like(kf)
    dv = np.empty_like(vf)
    for h in range(qf.shape[0]):
        s = scores(qf[h], kf[h], scale, causal)
        p, lse = softmax_rows(s)
        o = p @ vf[h]
        p_re = np.exp(s - lse[:, None])          # recomputed from LSE
        dv[h] = p_re.T @ dof[h]
        dp = dof[h] @ vf[h].T
        dsum = np.sum(dof[h] * o, axis=1)        # D
        ds = p_re * (dp - dsum[:, None])
        dq[h] = scale * (ds @ kf[h])
        dk[h] = scale * (ds.T @ qf[h])
    return (dq.reshape(*lead, n, d), dk.reshape(*lead, *k.shape[-2:]),
            dv.reshape(*lead, *v.shape[-2:]))


# ---------------------------------------------------------------------------
# decode (one query token per sequence and head)
# ---------------------------------------------------------------------------

def decode(q, kcache, vcache, seqlens, scale: float):
    """Single-token attention over a KV cache, computed directly.

    q [B, H, d]; kcache, vcache [B, H, Lmax, d]; seqlens [B] with
    1 <= seqlens[b] <= Lmax. Keys 0 .. seqlens[b]-1 are visible (no mask
    inside the cache). Returns (O [B, H, d], LSE [B, H]).
    """
    q = _as_f64(q)
    bsz, nh, d = q.shape
    o = np.empty((bsz, nh, vcache.shape[-1]))
    lse = np.empty((bsz, nh))
    for b in range(bsz):
        n = int(seqlens[b])
        if n < 1:
            raise ValueError("every sequence needs at least one cached token")
        for h in range(nh):
            kb = _as_f64(kcache[b, h, :n])
            vb = _as_f64(vcache[b, h, :n])
            p, l_row = softmax_rows(scores(q[b, h][None, :], kb, scale, False))
            o[b, h] = (p @ vb)[0]
            lse[b, h] = l_row[0]
    return o, lse


def merge_partials(o_parts, lse_parts):
    """Merge per-chunk results by log-sum-exp ("Decode Asamasi").

    Each chunk c gives its normalised output o_c and its lse_c; then
    LSE = ln sum_c exp(lse_c) and O = sum_c exp(lse_c - LSE) o_c.
    o_parts [C, dv], lse_parts [C].
    """
    o_parts = _as_f64(o_parts)
    lse_parts = _as_f64(lse_parts)
    mx = np.max(lse_parts)
    w = np.exp(lse_parts - mx)
    total = mx + math.log(float(np.sum(w)))
    weights = np.exp(lse_parts - total)
    return weights @ o_parts, total


def decode_split(q, kcache, vcache, seqlens, scale: float, num_chunks: int):
    """Flash-Decoding in the oracle: chunk the cache, solve, merge by LSE.

    Chunk c of sequence b covers keys [c*n/C, (c+1)*n/C) with n = seqlens[b]
    (integer division); empty chunks are skipped. Exists so the tests can
    check that split-and-merge equals the direct ``decode``.
    """
    q = _as_f64(q)
    bsz, nh, _ = q.shape
    o = np.empty((bsz, nh, vcache.shape[-1]))
    lse = np.empty((bsz, nh))
    for b in range(bsz):
        n = int(seqlens[b])
        bounds = [(c * n) // num_chunks for c in range(num_chunks + 1)]
        for h in range(nh):
            parts_o, parts_l = [], []
            for c in range(num_chunks):
                lo, hi = bounds[c], bounds[c + 1]
                if hi <= lo:
                    continue
                kb = _as_f64(kcache[b, h, lo:hi])
                vb = _as_f64(vcache[b, h, lo:hi])
                p, l_row = softmax_rows(scores(q[b, h][None, :], kb, scale,
                                               False))
                parts_o.append((p @ vb)[0])
                parts_l.append(l_row[0])
            o[b, h], lse[b, h] = merge_partials(np.array(parts_o),
                                                np.array(parts_l))
    return o, lse


def decode_paged(q, kpages, vpages, block_table, seqlens, scale: float):
    """Single-token attention over a paged KV cache with grouped query heads.

    The KV cache of "Duvarin Otesi", stored in fixed-size pages and shared by
    groups of query heads (the paged and grouped-query layouts that section
    names), computed directly by gathering each sequence's keys and values.

    q [B, Hq, d]. kpages, vpages [P, Hkv, page, d]: page p holds `page`
    consecutive cache positions of every KV head. block_table [B, M] (ints):
    cache position t of sequence b is row t % page of page
    block_table[b, t // page]. Hq is a multiple of Hkv, and query head h
    reads KV head h // (Hq // Hkv) (consecutive query heads share a KV head;
    Hkv = 1 is multi-query attention). Keys 0 .. seqlens[b]-1 are visible. A
    sequence with no visible key gets O = 0 and LSE = -inf (an empty sum).
    Returns (O [B, Hq, dv], LSE [B, Hq]).
    """
    q = _as_f64(q)
    bsz, hq, _ = q.shape
    _, hkv, page, _ = kpages.shape
    if hq % hkv:
        raise ValueError("the number of query heads must be a multiple of the KV heads")
    group = hq // hkv
    table = np.asarray(block_table)
    o = np.zeros((bsz, hq, vpages.shape[-1]))
    lse = np.full((bsz, hq), -np.inf)
    for b in range(bsz):
        n = int(seqlens[b])
        if n == 0:
            continue
        t = np.arange(n)
        pg, row = table[b, t // page], t % page
        for h in range(hq):
            kv = h // group
            kb = _as_f64(kpages[pg, kv, row])
            vb = _as_f64(vpages[pg, kv, row])
            p, l_row = softmax_rows(scores(q[b, h][None, :], kb, scale, False))
            o[b, h] = (p @ vb)[0]
            lse[b, h] = l_row[0]
    return o, lse
