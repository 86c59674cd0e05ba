"""Failure detection on the GPU without a fault.

With fa_debug_skip_load set, the next fa_fwd launch has one CTA skip one V-tile
load, so a wait inside that CTA can never complete. Every device-side wait is
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
from gpu_helpers import TOL_LSE, TOL_O, bf16_device, f64, max_abs

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
