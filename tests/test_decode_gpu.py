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
