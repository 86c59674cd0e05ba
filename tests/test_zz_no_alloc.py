"""fa_decode_splitkv_static: decode for callers that cannot allocate.

Some callers cannot hand the library a device workspace when they decode
(a stream capture in progress, an allocator that forbids cudaMalloc on the
hot path, no memory pool of their own). fa_decode_splitkv_static keeps the
per-chunk partials in an 8 MiB buffer built into the library instead. This
file checks, through the C ABI, that two calls in a row give the same
answer as fa_decode_splitkv with a caller workspace, within the decode
tolerances (max |O - O_ref| <= 1e-2, max |LSE - LSE_ref| <= 1e-3), and that
a shape too large for the buffer is refused. It is named to be collected
last, and passes on its own in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest
import torch

import exact_attention_130_b200 as fa
import inputgen
from gpu_helpers import TOL_LSE, TOL_O, bf16_device

pytestmark = pytest.mark.gpu


def _inputs(index, B, H, Lmax, d, lens):
    w = inputgen.Workload("no_alloc", index, B=B, H=H, N=Lmax, d=d, dtype="bf16",
                          kind="decode", seqlen_range=(1, Lmax))
    x = inputgen.make_decode_inputs(w, seqlens=lens)
    return (bf16_device(x["q"]), bf16_device(x["kcache"]), bf16_device(x["vcache"]),
            torch.from_numpy(np.asarray(lens, dtype=np.int32)).cuda())


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


def test_static_decode_matches_workspace_decode_twice():
    lib = fa.load_library()
    cases = [
        _inputs(60, 4, 8, 3000, 128, [3000, 1, 1777, 64]),
        _inputs(61, 2, 16, 2048, 64, [2048, 999]),
    ]
    for q, kc, vc, lens in cases:  # two calls in a row, different shapes and data
        st, o, lse = _static_call(lib, q, kc, vc, lens)
        assert st == 0, lib.fa_last_error()
        ro, rl = fa.fa_decode_splitkv(q, kc, vc, lens)
        torch.cuda.synchronize()
        assert float((o.float() - ro.float()).abs().max()) <= TOL_O
        assert float((lse - rl).abs().max()) <= TOL_LSE
        assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    st, word = fa.fa_device_status()
    assert st == 0, word


def test_static_decode_refuses_shapes_beyond_its_buffer():
    lib = fa.load_library()
    P = ctypes.c_void_p
    # B*H*C*(d+1)*4 bytes of partials: 64 * 64 * 64 * 129 * 4 > 8 MiB
    st = lib.fa_decode_splitkv_static(P(16), P(16), P(16), P(16), P(16), P(16),
                                      64, 64, 4096, 128, 0.088, 64, None)
    assert st == 4  # FA_ERR_WORKSPACE
    assert b"built into the library" in lib.fa_last_error()
