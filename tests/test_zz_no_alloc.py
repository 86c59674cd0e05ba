"""fa_decode_splitkv_static: decode for callers that cannot allocate.

Some callers cannot hand the library a device workspace when they decode:
a serving loop whose allocator forbids cudaMalloc on its hot path
(cudaMalloc can synchronise the device and stall every other stream), or a
host framework that passes the library only its inputs and outputs and
keeps no memory pool for it. fa_decode_splitkv_static keeps the per-chunk
partials in an 8 MiB buffer built into the library instead.

This file checks, through the C ABI, on calls made one after another (so
each call finds the previous call's partials in the shared buffer):
  * O and LSE against the fp64 oracle's direct decode, within the decode
    tolerances (max |O - O_ref| <= 1e-2, max |LSE - LSE_ref| <= 1e-3);
  * the same outputs against fa_decode_splitkv with a caller workspace;
  * a sequence with no visible key (length 0) gives O = 0 and LSE = -inf
    exactly, whatever the buffer held before;
  * a shape too large for the buffer is refused before any launch.
It is named to be collected last, and passes on its own in a fresh process
as well.
"""
import ctypes

import numpy as np
import pytest
import torch

import exact_attention_130_b200 as fa
import inputgen
import oracle
from gpu_helpers import TOL_LSE, TOL_O, bf16_device, f64

pytestmark = pytest.mark.gpu


def _inputs(index, B, H, Lmax, d, lens):
    w = inputgen.Workload("no_alloc", index, B=B, H=H, N=Lmax, d=d, dtype="bf16",
                          kind="decode", seqlen_range=(1, Lmax))
    x = inputgen.make_decode_inputs(w, seqlens=lens)
    dev = (bf16_device(x["q"]), bf16_device(x["kcache"]), bf16_device(x["vcache"]),
           torch.from_numpy(np.asarray(lens, dtype=np.int32)).cuda())
    return x, dev


def _static_call(lib, q, kc, vc, lens, num_splits=0):
    B, H, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    P = ctypes.c_void_p
    st = lib.fa_decode_splitkv_static(
        P(q.data_ptr()), P(kc.data_ptr()), P(vc.data_ptr()), P(lens.data_ptr()),
        P(o.data_ptr()), P(lse.data_ptr()), B, H, kc.shape[2], d, 1.0 / d ** 0.5,
        num_splits, P(torch.cuda.current_stream().cuda_stream))
    return st, o, lse


def _oracle_decode(x, d):
    """fp64 oracle decode of the sequences with at least one key."""
    lens = np.asarray(x["seqlens"])
    live = lens > 0
    ro = np.zeros(x["q"].shape, dtype=np.float64)
    rl = np.full(lens.shape + (x["q"].shape[1],), -np.inf)
    if live.any():
        o, l = oracle.decode(f64(x["q"][live]), f64(x["kcache"][live]), f64(x["vcache"][live]),
                             lens[live], 1.0 / d ** 0.5)
        ro[live], rl[live] = o, l
    return ro, rl, live


def test_static_decode_matches_oracle_and_workspace_decode():
    lib = fa.load_library()
    cases = [
        (60, 4, 8, 3000, 128, [3000, 1, 1777, 64], 0),
        (61, 2, 16, 2048, 64, [2048, 999], 0),
        # a sequence with no key, after calls that left partials in the buffer
        (62, 3, 4, 700, 128, [0, 700, 5], 7),
    ]
    for index, B, H, Lmax, d, lens, splits in cases:  # calls one after another
        x, (q, kc, vc, dlens) = _inputs(index, B, H, Lmax, d, lens)
        st, o, lse = _static_call(lib, q, kc, vc, dlens, splits)
        assert st == 0, lib.fa_last_error()
        wo, wl = fa.fa_decode_splitkv(q, kc, vc, dlens, num_splits=splits)
        torch.cuda.synchronize()
        ro, rl, live = _oracle_decode(x, d)
        o_np = o.float().cpu().numpy().astype(np.float64)
        l_np = lse.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(o_np))
        assert np.max(np.abs(o_np[live] - ro[live])) <= TOL_O
        assert np.max(np.abs(l_np[live] - rl[live])) <= TOL_LSE
        assert np.all(o_np[~live] == 0.0) and np.all(np.isneginf(l_np[~live]))
        # the workspace entry point gives the same answer within the tolerance
        assert float((o.float() - wo.float()).abs().max()) <= TOL_O
        w_np = wl.cpu().numpy().astype(np.float64)
        assert np.max(np.abs(l_np[live] - w_np[live])) <= TOL_LSE
        assert np.all(np.isneginf(w_np[~live]))
    st, word = fa.fa_device_status()
    assert st == 0, word


def test_static_decode_refuses_shapes_beyond_its_buffer():
    lib = fa.load_library()
    P = ctypes.c_void_p
    # B*H*C*(d+1)*4 bytes of partials: 64 * 64 * 64 * 129 * 4 > 8 MiB. The
    # size check comes before any device work, so the placeholder pointers
    # (aligned, never dereferenced) are not touched.
    st = lib.fa_decode_splitkv_static(P(16), P(16), P(16), P(16), P(16), P(16),
                                      64, 64, 4096, 128, 0.088, 64, None)
    assert st == 4  # FA_ERR_WORKSPACE
    assert b"built into the library" in lib.fa_last_error()
