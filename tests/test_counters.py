"""The bench's FLOP and byte counters against numbers the pages print.

Golden values: tests/golden/memory_wall_numbers.json, each entry citing the
section of "Bellek Duvarinin Fizigi" it is printed in.
"""
import json
import os

import pytest

from exact_attention_130_b200 import counters as C

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                   "memory_wall_numbers.json")))


@pytest.mark.parametrize("row", GOLD["prob_matrix_fp16"]["rows"],
                         ids=lambda r: f"N{r['N']}")
def test_prob_matrix_table(row):
    n = row["N"]
    assert abs(n * n - row["elements"]) / row["elements"] < row["rel_tol"]
    assert abs(C.prob_matrix_bytes(n) - row["bytes"]) / row["bytes"] < row["rel_tol"]


def test_prob_matrix_share_of_a100():
    share = C.prob_matrix_bytes(131072) / 80e9
    assert abs(share - GOLD["prob_matrix_fp16"]["a100_80gb_share_at_131072"]) < 0.005


def test_ridge_point():
    g = GOLD["a100_roofline"]
    r = C.ridge_point(g["peak_fp16_tensor_flops"], g["hbm_bytes_per_s"])
    assert abs(r - g["ridge_flop_per_byte"]) / g["ridge_flop_per_byte"] < g["ridge_rel_tol"]


def test_naive_intensity():
    g = GOLD["naive_intensity"]
    assert C.naive_intensity(g["d"]) == pytest.approx(g["flop_per_byte"])


def test_naive_time_estimate():
    g = GOLD["naive_time_estimate"]
    a = GOLD["a100_roofline"]
    t_mm = C.naive_matmul_time_s(g["N"], g["d"], a["peak_fp16_tensor_flops"]) * 1e3
    t_io = C.naive_io_time_s(g["N"], a["hbm_bytes_per_s"]) * 1e3
    assert abs(t_mm - g["matmul_ms"]) < g["abs_tol_ms"]
    assert abs(t_io - g["io_ms"]) < g["abs_tol_ms"]
    # the same 4 N^2 d count is the per-head forward count of the bench
    assert C.fwd_flops(1, 1, g["N"], g["d"], False) == 4.0 * g["N"] ** 2 * g["d"]


def test_softmax_share():
    g = GOLD["softmax_flop_share"]
    n = 4096
    share = 3.0 * n * n / (C.fwd_flops(1, 1, n, g["d"], False) + 3.0 * n * n)
    assert share < g["max_share"]


def test_kv_cache_example():
    g = GOLD["kv_cache"]
    per_tok = C.kv_cache_bytes_per_token(g["d_model"], g["layers"])
    assert abs(per_tok - g["bytes_per_token"]) / g["bytes_per_token"] < g["rel_tol"]
    assert abs(per_tok * g["tokens"] - g["session_bytes"]) / g["session_bytes"] < g["session_rel_tol"]


def test_workload_counts():
    # prefill: 4 B H N^2 d = 137.4 GFLOP, halved under the causal mask;
    # backward: 2.5x the causal forward of its own shape
    assert C.fwd_flops(4, 16, 2048, 128, False) == pytest.approx(137.44e9, rel=1e-3)
    assert C.fwd_flops(4, 16, 2048, 128, True) == pytest.approx(68.72e9, rel=1e-3)
    assert C.bwd_flops(2, 16, 4096, 128, True) == pytest.approx(343.6e9, rel=1e-3)
    assert C.fwd_flops(1, 32, 16384, 128, True) == pytest.approx(2.199e12, rel=1e-3)
    # decode bytes: every visible K and V row once (256 B each at d = 128)
    assert C.decode_bytes(32, [1000], 128) == 2 * 32 * 1000 * 256 + 2 * 32 * 256 + 4 * 32
