"""Split-KV decode parity on the GPU against the fp64 oracle.

Cache positions at or past seqlens[b] hold NaN, so reading one would poison
the result. Tolerances: max |O - O_ref| <= 1e-2, max |LSE - LSE_ref| <= 1e-3.
"""
import numpy as np
import pytest
import torch

import exact_attention_130_b200 as fa
import inputgen
import oracle
from gpu_helpers import TOL_LSE, TOL_O, Guarded, bf16_device, f64, max_abs

pytestmark = pytest.mark.gpu


def small_workload(B, H, Lmax, d, lo, hi, index=40):
    return inputgen.Workload("decode_small", index, B=B, H=H, N=Lmax, d=d,
                             dtype="bf16", kind="decode", seqlen_range=(lo, hi))


def run_decode(x, num_splits=0, scale=None):
    B, H, d = x["q"].shape
    q = bf16_device(x["q"])
    kc = bf16_device(x["kcache"])
    vc = bf16_device(x["vcache"])
    lens = torch.from_numpy(x["seqlens"].astype(np.int32)).cuda()
    o = Guarded((B, H, d), torch.bfloat16)
    lse = Guarded((B, H), torch.float32)
    fa.fa_decode_splitkv(q, kc, vc, lens, scale=scale, num_splits=num_splits,
                         o=o.t, lse=lse.t)
    torch.cuda.synchronize()
    assert o.guards_intact() and lse.guards_intact()
    return o.t, lse.t



def _oracle(x, scale):
    B, H, d = x["q"].shape
    o = np.empty((B, H, d))
    lse = np.empty((B, H))
    for b in range(B):
        n = int(x["seqlens"][b])
        ob, lb = oracle.decode(f64(x["q"][b:b + 1]), f64(x["kcache"][b:b + 1, :, :n]),
                               f64(x["vcache"][b:b + 1, :, :n]), np.array([n]), scale)
        o[b], lse[b] = ob[0], lb[0]
    return o, lse


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("num_splits", [0, 1, 2, 7, 64])
def test_decode_small(d, num_splits):
    w = small_workload(3, 2, 300, d, 1, 300)
    x = inputgen.make_decode_inputs(w, seqlens=[300, 1, 137])
    o, lse = run_decode(x, num_splits)
    ro, rl = _oracle(x, w.scale)
    assert max_abs(o, ro) <= TOL_O
    assert max_abs(lse, rl) <= TOL_LSE


def test_decode_ragged_lengths_and_tails():
    w = small_workload(6, 3, 1000, 128, 1, 1000, index=41)
    x = inputgen.make_decode_inputs(w, seqlens=[1, 31, 32, 33, 999, 1000])
    for splits in (0, 3, 33):
        o, lse = run_decode(x, splits)
        ro, rl = _oracle(x, w.scale)
        assert max_abs(o, ro) <= TOL_O
        assert max_abs(lse, rl) <= TOL_LSE


def test_decode_workload_full():
    """B=8, H=32, d=128, cache lengths drawn from [16384, 32768]."""
    w = inputgen.WORKLOADS["decode"]
    x = inputgen.make_decode_inputs(w)
    o, lse = run_decode(x)
    ro, rl = _oracle(x, w.scale)
    assert max_abs(o, ro) <= TOL_O
    assert max_abs(lse, rl) <= TOL_LSE


def test_decode_split_count_invariance_and_determinism():
    w = small_workload(4, 4, 4096, 128, 1000, 4096, index=42)
    x = inputgen.make_decode_inputs(w)
    ref_o, ref_l = run_decode(x, 1)
    for splits in (2, 7, 0, 100):
        o, lse = run_decode(x, splits)
        assert float((o.float() - ref_o.float()).abs().max()) <= 2e-3
        assert float((lse - ref_l).abs().max()) <= 1e-5
    o1, l1 = run_decode(x, 0)
    o2, l2 = run_decode(x, 0)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)


def test_decode_matches_last_causal_row_of_forward():
    """decode(q_N-1, K, V, N) equals the causal forward's last row."""
    B, H, N, d = 2, 3, 700, 128
    x = inputgen.make_small_inputs(31, B, H, N, d)
    q, k, v = (bf16_device(x[n]) for n in ("q", "k", "v"))
    o_f, l_f = fa.fa_fwd(q, k, v, causal=True)
    lens = torch.full((B,), N, dtype=torch.int32, device="cuda")
    o_d, l_d = fa.fa_decode_splitkv(q[:, :, -1].contiguous(), k, v, lens)
    torch.cuda.synchronize()
    assert float((o_d.float() - o_f[:, :, -1].float()).abs().max()) <= 2e-2
    assert float((l_d - l_f[:, :, -1]).abs().max()) <= 2e-3


# ---------------------------------------------------------------------------
# paged KV cache with grouped query heads (fa_decode_paged)
# ---------------------------------------------------------------------------

def run_paged(x, num_splits=0, scale=None):
    B, Hq, d = x["q"].shape
    q = bf16_device(x["q"])
    kp, vp = bf16_device(x["kpages"]), bf16_device(x["vpages"])
    table = torch.from_numpy(x["block_table"]).cuda()
    lens = torch.from_numpy(x["seqlens"].astype(np.int32)).cuda()
    o = Guarded((B, Hq, d), torch.bfloat16)
    lse = Guarded((B, Hq), torch.float32)
    fa.fa_decode_paged(q, kp, vp, table, lens, scale=scale, num_splits=num_splits,
                       o=o.t, lse=lse.t)
    torch.cuda.synchronize()
    assert fa.fa_device_status()[0] == 0
    assert o.guards_intact() and lse.guards_intact()
    return o.t, lse.t


def _check_paged(x, o, lse, scale):
    ro, rl = oracle.decode_paged(f64(x["q"]), f64(x["kpages"]), f64(x["vpages"]),
                                 x["block_table"], x["seqlens"], scale)
    o_np, l_np = o.float().cpu().numpy(), lse.cpu().numpy()
    empty = x["seqlens"] == 0
    # a sequence with no key: O = 0 and LSE = -inf exactly
    assert np.all(o_np[empty] == 0.0) and np.all(np.isneginf(l_np[empty]))
    assert np.max(np.abs(o_np[~empty] - ro[~empty]), initial=0.0) <= TOL_O
    assert np.max(np.abs(l_np[~empty] - rl[~empty]), initial=0.0) <= TOL_LSE


@pytest.mark.parametrize("heads", [(4, 4), (8, 2), (6, 1)], ids=["mha", "gqa4", "mqa"])
@pytest.mark.parametrize("page", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("d", [64, 128])
def test_paged_decode_small(d, page, heads):
    hq, hkv = heads
    x = inputgen.make_paged_decode_inputs(500 + page + d + hq, 4, hq, hkv, d, page,
                                          seqlens=[0, 1, 300, 517])
    o, lse = run_paged(x)
    _check_paged(x, o, lse, 1 / np.sqrt(d))


@pytest.mark.parametrize("num_splits", [1, 2, 7, 64])
def test_paged_decode_split_counts(num_splits):
    x = inputgen.make_paged_decode_inputs(611, 3, 8, 2, 128, 64, seqlens=[2000, 63, 1025],
                                          max_pages=40)
    o, lse = run_paged(x, num_splits)
    _check_paged(x, o, lse, 1 / np.sqrt(128))


def test_paged_decode_workload():
    """B=8, Hq=32, Hkv=8, d=128, pages of 64 rows, cache lengths drawn from
    [16384, 32768] (the split-KV decode workload with grouped query heads and a
    paged cache), every head compared."""
    x = inputgen.make_paged_decode_inputs(20264, 8, 32, 8, 128, 64,
                                          seqlen_range=(16384, 32768))
    o, lse = run_paged(x)
    _check_paged(x, o, lse, 1 / np.sqrt(128))


def test_paged_decode_bad_page_is_reported_not_read():
    """A block-table entry outside the page pool is never dereferenced: the
    call reports FA_ERR_INVALID_ARG through fa_device_status, and the next
    call with a correct table gives correct results."""
    x = inputgen.make_paged_decode_inputs(612, 2, 4, 2, 128, 64, seqlens=[200, 130])
    q = bf16_device(x["q"])
    kp, vp = bf16_device(x["kpages"]), bf16_device(x["vpages"])
    lens = torch.from_numpy(x["seqlens"]).cuda()
    bad = x["block_table"].copy()
    bad[1, 1] = kp.shape[0] + 5      # past the pool
    bad[0, 2] = -3                   # negative
    assert fa.fa_device_status()[0] == 0
    fa.fa_decode_paged(q, kp, vp, torch.from_numpy(bad).cuda(), lens)
    st, word = fa.fa_device_status()
    assert st == 1, (st, word)                      # FA_ERR_INVALID_ARG
    assert (word >> 16) == 6 and (word & 0xff) == 2, hex(word)
    assert fa.fa_device_status()[0] == 0
    o, lse = run_paged(x)
    _check_paged(x, o, lse, 1 / np.sqrt(128))


@pytest.mark.parametrize("heads", [(16, 1), (64, 1), (128, 2), (4, 2), (6, 2), (10, 2), (256, 1)],
                         ids=["g16", "g64", "g128-2kv", "g2", "g3", "g5", "g256"])
def test_paged_decode_large_groups(heads):
    """Groups of 2 and 3 query heads per KV head (CUDA cores, two and one
    heads per CTA), 5, 16 and 64 (the tensor-core path with one and two
    softmax warps), and 256 (past the tensor-core path's 128 rows: CUDA
    cores); lengths leave partial last tiles over NaN-filled page rows."""
    hq, hkv = heads
    x = inputgen.make_paged_decode_inputs(620 + hq, 3, hq, hkv, 128, 64, seqlens=[1, 700, 4097])
    o, lse = run_paged(x)
    _check_paged(x, o, lse, 1 / np.sqrt(128))


@pytest.mark.parametrize("page", [16, 64, 128, 192, 256])
@pytest.mark.parametrize("heads", [(16, 4), (32, 4), (32, 2)], ids=["g4", "g8", "g16"])
def test_paged_decode_keys_as_rows(heads, page):
    """Groups of 4 and 8 query heads per KV head at d = 128 run with the keys
    as the tensor cores' M rows (128-key tiles; 192-row pages, whose tiles
    would straddle two pages, take the heads-as-rows kernel, as do groups of
    16); lengths leave partial last tiles over NaN-filled page rows, one
    sequence is empty, and one chunk count splits the cache into many short
    chunks."""
    hq, hkv = heads
    x = inputgen.make_paged_decode_inputs(640 + hq + page, 4, hq, hkv, 128, page,
                                          seqlens=[0, 129, 1000, 5000])
    for splits in (0, 9):
        o, lse = run_paged(x, splits)
        _check_paged(x, o, lse, 1 / np.sqrt(128))


@pytest.mark.parametrize("page", [64, 128])
@pytest.mark.parametrize("heads", [(16, 4), (12, 2), (16, 2)], ids=["g4", "g6", "g8"])
def test_paged_decode_balanced_split(heads, page):
    """The automatic split of groups of 4 to 8 query heads (d = 128) deals
    whole 128-key tiles out to persistent CTAs in equal ranges. 45 sequences
    (more than one warp's worth, for the CTAs' scan of the lengths), empty
    and one-key ones, lengths on and just off a tile boundary, the rest
    random: pieces start and end inside sequences, a sequence spans several
    CTAs, a CTA several sequences, and rows past each length are NaN."""
    hq, hkv = heads
    rng = np.random.default_rng(660 + hq + page)
    lens = rng.integers(0, 3000, size=45).astype(np.int32)
    lens[:6] = [0, 1, 127, 128, 129, 0]
    x = inputgen.make_paged_decode_inputs(660 + hq + page, 45, hq, hkv, 128, page, seqlens=lens)
    o, lse = run_paged(x)
    _check_paged(x, o, lse, 1 / np.sqrt(128))


@pytest.mark.parametrize("heads", [(8, 2), (16, 2)], ids=["g4", "g8"])
def test_paged_decode_balanced_many_short_pieces(heads):
    """600 short sequences (0 to 300 keys: one to three tiles each), so that
    a persistent CTA's range covers several whole segments: its pipeline
    runs across three or more pieces, reusing both O accumulators and the Q
    buffer, while other segments still span two CTAs."""
    hq, hkv = heads
    rng = np.random.default_rng(680 + hq)
    lens = rng.integers(0, 301, size=600).astype(np.int32)
    lens[:4] = [0, 1, 128, 129]
    x = inputgen.make_paged_decode_inputs(680 + hq, 600, hq, hkv, 128, 64, seqlens=lens)
    o, lse = run_paged(x)
    _check_paged(x, o, lse, 1 / np.sqrt(128))


def test_paged_decode_tensor_core_bad_page_is_reported_not_read():
    """As the bad-page test above, on the tensor-core path (4 query heads per
    KV head): no page outside the pool is read, the status says so."""
    x = inputgen.make_paged_decode_inputs(613, 2, 8, 2, 128, 32, seqlens=[200, 130])
    q = bf16_device(x["q"])
    kp, vp = bf16_device(x["kpages"]), bf16_device(x["vpages"])
    lens = torch.from_numpy(x["seqlens"]).cuda()
    bad = x["block_table"].copy()
    bad[1, 2] = kp.shape[0]          # one past the pool
    assert fa.fa_device_status()[0] == 0
    fa.fa_decode_paged(q, kp, vp, torch.from_numpy(bad).cuda(), lens)
    st, word = fa.fa_device_status()
    assert st == 1 and (word >> 16) == 6 and (word & 0xff) == 2, (st, hex(word))
    o, lse = run_paged(x)
    _check_paged(x, o, lse, 1 / np.sqrt(128))
