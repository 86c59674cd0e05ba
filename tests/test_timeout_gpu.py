"""Failure detection on the GPU without a fault.

With fa_debug_skip_load set, the next call has one CTA of the named kernel
(forward, backward dK/dV, backward dQ or decode split) leave out one load, so
a wait inside that CTA can never complete. Every device-side wait is
bounded in time: the kernel records the failure in the device status word and
returns, fa_device_status reports FA_ERR_TIMEOUT, and the context stays usable
(the next call gives correct results). No trap, no fault, no endless loop.
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_130_b200 as fa
import inputgen
import oracle
from gpu_helpers import TOL_GRAD_REL, TOL_LSE, TOL_O, bf16_device, f64, max_abs, rel_fro

pytestmark = pytest.mark.gpu


def test_missing_load_times_out_and_context_survives():
    x = inputgen.make_small_inputs(88, 1, 2, 512, 128)
    q, k, v = (bf16_device(x[n]) for n in ("q", "k", "v"))
    assert fa.fa_device_status()[0] == 0
    fa.fa_set_wait_limit(50_000_000)  # 50 ms
    try:
        fa.fa_debug_skip_load(True)
        fa.fa_fwd(q, k, v, causal=False)
        st, word = fa.fa_device_status()
        assert st == 6, (st, word)           # FA_ERR_TIMEOUT
        assert (word >> 16) == 1 and (word & 1)  # forward kernel, wait gave up
        assert fa.fa_device_status()[0] == 0  # the word was cleared
    finally:
        fa.fa_debug_skip_load(False)
        fa.fa_set_wait_limit(0)
    o, lse = fa.fa_fwd(q, k, v, causal=False)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_fwd(f64(x["q"]), f64(x["k"]), f64(x["v"]), 1 / math.sqrt(128), False)
    assert max_abs(o, ro) <= TOL_O and max_abs(lse, rl) <= TOL_LSE


def _expect_timeout(kernel_id, call):
    """Run `call` with the named kernel's load left out; the status word must
    name that kernel and a wait that gave up, and be cleared by the read."""
    assert fa.fa_device_status()[0] == 0
    fa.fa_set_wait_limit(50_000_000)  # 50 ms
    try:
        fa.fa_debug_skip_load(fa.KERNEL_NAMES[kernel_id])
        call()
        st, word = fa.fa_device_status()
        assert st == 6, (st, word)                     # FA_ERR_TIMEOUT
        assert (word >> 16) == kernel_id and (word & 1), hex(word)
        assert fa.fa_device_status()[0] == 0
    finally:
        fa.fa_debug_skip_load(0)
        fa.fa_set_wait_limit(0)


@pytest.mark.parametrize("kernel_id", [4, 5], ids=["dkdv", "dq"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_backward_missing_load_times_out(kernel_id, causal):
    x = inputgen.make_small_inputs(89, 2, 2, 640, 128, with_grad=True)
    q, k, v, do = (bf16_device(x[n]) for n in ("q", "k", "v", "do"))
    o, lse = fa.fa_fwd(q, k, v, causal=causal)
    _expect_timeout(kernel_id, lambda: fa.fa_bwd(q, k, v, o, lse, do, causal=causal))
    dq, dk, dv = fa.fa_bwd(q, k, v, o, lse, do, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_device_status()[0] == 0
    ref = oracle.attention_bwd(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["do"]),
                               1 / math.sqrt(128), causal)
    for g, r in zip((dq, dk, dv), ref):
        assert rel_fro(g, r) <= TOL_GRAD_REL


def test_decode_missing_load_times_out():
    w = inputgen.Workload("decode_small", 41, B=2, H=2, N=700, d=128, dtype="bf16",
                          kind="decode", seqlen_range=(1, 700))
    x = inputgen.make_decode_inputs(w, seqlens=[700, 333])
    q, kc, vc = (bf16_device(x[n]) for n in ("q", "kcache", "vcache"))
    lens = torch.from_numpy(x["seqlens"].astype(np.int32)).cuda()
    _expect_timeout(6, lambda: fa.fa_decode_splitkv(q, kc, vc, lens))
    o, lse = fa.fa_decode_splitkv(q, kc, vc, lens)
    torch.cuda.synchronize()
    assert fa.fa_device_status()[0] == 0
    for b in range(2):
        n = int(x["seqlens"][b])
        ro, rl = oracle.decode(f64(x["q"][b:b + 1]), f64(x["kcache"][b:b + 1, :, :n]),
                               f64(x["vcache"][b:b + 1, :, :n]), np.array([n]), w.scale)
        assert max_abs(o[b:b + 1], ro) <= TOL_O and max_abs(lse[b:b + 1], rl) <= TOL_LSE


def test_hook_is_consumed_by_the_next_call():
    """A hook naming another kernel is used up by the next call and has no
    effect on it; the call after that runs every load."""
    x = inputgen.make_small_inputs(90, 1, 1, 256, 64, with_grad=True)
    q, k, v, do = (bf16_device(x[n]) for n in ("q", "k", "v", "do"))
    fa.fa_set_wait_limit(50_000_000)
    try:
        fa.fa_debug_skip_load("bwd_dq")
        o, lse = fa.fa_fwd(q, k, v)
        fa.fa_bwd(q, k, v, o, lse, do)
        torch.cuda.synchronize()
        assert fa.fa_device_status()[0] == 0
    finally:
        fa.fa_debug_skip_load(0)
        fa.fa_set_wait_limit(0)


def test_paged_tensor_core_decode_missing_load_times_out():
    """The tensor-core paged decode (8 query heads per KV head): its first
    CTA leaves out a V tile, the wait runs out and reports the decode kernel."""
    x = inputgen.make_paged_decode_inputs(614, 2, 16, 2, 128, 64, seqlens=[500, 300])
    q = bf16_device(x["q"])
    kp, vp = bf16_device(x["kpages"]), bf16_device(x["vpages"])
    table = torch.from_numpy(x["block_table"]).cuda()
    lens = torch.from_numpy(x["seqlens"]).cuda()
    _expect_timeout(6, lambda: fa.fa_decode_paged(q, kp, vp, table, lens))
    o, lse = fa.fa_decode_paged(q, kp, vp, table, lens)
    torch.cuda.synchronize()
    assert fa.fa_device_status()[0] == 0
    ro, rl = oracle.decode_paged(f64(x["q"]), f64(x["kpages"]), f64(x["vpages"]),
                                 x["block_table"], x["seqlens"], 1 / math.sqrt(128))
    assert max_abs(o, ro) <= TOL_O and max_abs(lse, rl) <= TOL_LSE
