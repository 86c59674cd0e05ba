"""Backward parity on the GPU: fa_bwd against the fp64 oracle.

O and LSE come from fa_fwd (as the backward workload states). dQ, dK, dV
must be within 2e-2 relative Frobenius error of the oracle's gradients of
sum(O * dO), per tensor. Outputs carry NaN guard bands.
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_130_b200 as fa
import inputgen
import oracle
from gpu_helpers import TOL_GRAD_REL, Guarded, bf16_device, f64, rel_fro

pytestmark = pytest.mark.gpu

SMALL = [
    (1, 2, 128, 128), (1, 2, 256, 64), (2, 1, 384, 128), (1, 2, 200, 64),
    (1, 1, 1000, 128), (1, 1, 1, 128), (1, 3, 130, 128), (2, 2, 640, 64),
]


def run_bwd(x, causal, scale=None):
    B, H, N, d = x["q"].shape
    q, k, v, do = (bf16_device(x[n]) for n in ("q", "k", "v", "do"))
    o, lse = fa.fa_fwd(q, k, v, causal=causal, scale=scale)
    grads = [Guarded((B, H, N, d), torch.bfloat16) for _ in range(3)]
    fa.fa_bwd(q, k, v, o, lse, do, causal=causal, scale=scale,
              dq=grads[0].t, dk=grads[1].t, dv=grads[2].t)
    torch.cuda.synchronize()
    assert all(g.guards_intact() for g in grads)
    st, word = fa.fa_device_status()
    assert st == 0, word
    return [g.t for g in grads]


def check(x, causal, scale=None):
    d = x["q"].shape[-1]
    sc = 1 / math.sqrt(d) if scale is None else scale
    dq, dk, dv = run_bwd(x, causal, scale)
    rq, rk, rv = oracle.attention_bwd(f64(x["q"]), f64(x["k"]), f64(x["v"]),
                                      f64(x["do"]), sc, causal)
    errs = {}
    for name, g, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        if np.linalg.norm(ref) < 1e-9:
            # e.g. a single key: softmax is constant, the exact gradient is 0;
            # a relative error is undefined, so bound the absolute residue
            errs[name] = float(np.max(np.abs(g.float().cpu().numpy())))
            assert errs[name] <= 1e-3, (name, errs)
        else:
            errs[name] = rel_fro(g, ref)
            assert errs[name] <= TOL_GRAD_REL, (name, errs)
    return errs


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "x".join(map(str, s)))
def test_bwd_small(shape, causal):
    B, H, N, d = shape
    x = inputgen.make_small_inputs(2000 + N + d, B, H, N, d, with_grad=True)
    check(x, causal)


# more (head, tile) items than SMs, so every CTA of the persistent kernels
# walks several items: d = 64, a ragged last tile, and N = 256 (two tiles:
# under the mask half the items are a single block, so consecutive items
# stage their outputs in both slots before the producer stores them)
MULTI = [(2, 40, 512, 64), (1, 30, 700, 128), (4, 40, 256, 64)]


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("shape", MULTI, ids=lambda s: "x".join(map(str, s)))
def test_bwd_persistent_multi_item(shape, causal):
    B, H, N, d = shape
    x = inputgen.make_small_inputs(3000 + N + H, B, H, N, d, with_grad=True)
    check(x, causal)


def test_bwd_workload_every_head():
    """B=2, H=16, N=4096, d=128, causal; compared in full for every head."""
    w = inputgen.WORKLOADS["backward"]
    x = inputgen.make_attention_inputs(w, with_grad=True)
    check(x, True)


def test_bwd_nondefault_scale():
    x = inputgen.make_small_inputs(71, 1, 2, 300, 128, with_grad=True)
    check(x, True, scale=0.05)
    check(x, False, scale=0.2)


def test_bwd_deterministic():
    x = inputgen.make_small_inputs(72, 2, 2, 1000, 128, with_grad=True)
    a = run_bwd(x, True)
    b = run_bwd(x, True)
    for ga, gb in zip(a, b):
        assert torch.equal(ga.view(torch.int16), gb.view(torch.int16))
