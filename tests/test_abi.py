"""The C ABI without a GPU: the library loads, exports every entry point the
header declares, and rejects bad arguments before touching the device."""
import ctypes
import subprocess

import pytest

import exact_attention_130_b200 as fa

EXPECTED = {
    "fa_status_string", "fa_last_error", "fa_abi_version", "fa_fwd",
    "fa_fwd_f32", "fa_fwd_tf32", "fa_bwd_workspace_size", "fa_bwd",
    "fa_decode_workspace_size", "fa_decode_splitkv", "fa_device_status",
    "fa_set_wait_limit", "fa_debug_skip_load", "fa_profile_begin",
    "fa_profile_end", "fa_decode_splitkv_static", "fa_decode_paged",
    "fa_fp8_vt_keys", "fa_fp8_prepare", "fa_fwd_fp8", "fa_fwd_ex", "fa_bwd_ex",
    "fa_dropout_keep_threshold", "fa_fwd_pair",
}


@pytest.fixture(scope="module")
def lib():
    return fa.load_library()


def test_header_declares_expected_entry_points():
    assert set(fa.exported_symbols()) == EXPECTED


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", fa.library_path()],
                         capture_output=True, text=True, check=True).stdout
    dyn = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in fa.exported_symbols():
        assert name in dyn, name
        assert getattr(lib, name) is not None


def test_status_strings(lib):
    for code, name in fa.STATUS.items():
        assert lib.fa_status_string(code).decode() == name
    assert lib.fa_abi_version() == 104


def _fwd(lib, q=16, k=16, v=16, o=16, lse=16, B=1, H=1, N=8, d=64,
         scale=0.125, causal=0):
    P = ctypes.c_void_p
    return lib.fa_fwd(P(q), P(k), P(v), P(o), P(lse), B, H, N, d, scale, causal,
                      None)


def test_fwd_argument_errors_need_no_device(lib):
    assert _fwd(lib, q=0) == 1                    # null pointer
    assert _fwd(lib, k=24) == 3                   # not 16-byte aligned
    assert b"16-byte" in lib.fa_last_error()
    assert _fwd(lib, N=0) == 1
    assert _fwd(lib, B=-1) == 1
    assert _fwd(lib, d=96) == 2                   # unsupported head dim
    assert _fwd(lib, scale=float("nan")) == 1
    assert _fwd(lib, scale=-1.0) == 1
    assert _fwd(lib, causal=2) == 1
    assert _fwd(lib, B=1 << 16, H=1 << 16, N=2) == 1   # B*H*N overflow


def test_bwd_and_decode_argument_errors(lib):
    P = ctypes.c_void_p
    # workspace too small
    st = lib.fa_bwd(P(16), P(16), P(16), P(16), P(16), P(16), P(16), P(16),
                    P(16), 1, 1, 8, 64, 0.125, 0, P(16), 8, None)
    assert st == 4
    st = lib.fa_decode_splitkv(P(16), P(16), P(16), P(16), P(16), P(16), 1, 1,
                               8, 64, 0.125, 0, P(16), 0, None)
    assert st == 4
    st = lib.fa_decode_splitkv(P(16), P(16), P(16), P(0), P(16), P(16), 1, 1,
                               8, 64, 0.125, 0, P(16), 1 << 20, None)
    assert st == 1
    st = lib.fa_decode_splitkv(P(16), P(16), P(16), P(16), P(16), P(16), 1, 1,
                               8, 64, 0.125, 2000, P(16), 1 << 20, None)
    assert st == 1


def _paged(lib, table=16, B=1, Hq=4, Hkv=2, num_pages=4, page=64, max_pages=2, d=64,
           scale=0.125, ws_bytes=1 << 20):
    P = ctypes.c_void_p
    return lib.fa_decode_paged(P(16), P(16), P(16), P(table), P(16), P(16), P(16), B, Hq, Hkv,
                               num_pages, page, max_pages, d, scale, 0, P(16), ws_bytes, None)


def test_paged_decode_argument_errors(lib):
    assert _paged(lib, table=0) == 1              # no block table
    assert _paged(lib, table=18) == 1             # block table not 4-byte aligned
    assert _paged(lib, Hq=6, Hkv=4) == 1          # Hq not a multiple of Hkv
    assert b"multiple" in lib.fa_last_error()
    assert _paged(lib, page=48) == 2              # unsupported page size
    assert _paged(lib, page=8) == 2
    assert _paged(lib, num_pages=0) == 1
    assert _paged(lib, d=96) == 2
    assert _paged(lib, ws_bytes=8) == 4           # workspace too small
    assert _paged(lib, max_pages=1 << 20, page=4096) == 1   # positions overflow


def test_fp8_argument_errors(lib):
    P = ctypes.c_void_p

    def prep(signs=None, B=1, H=1, N=8, d=128, q8=16):
        return lib.fa_fp8_prepare(P(16), P(16), P(16), P(signs) if signs else None, B, H, N, d,
                                  P(q8), P(16), P(16), P(16), P(16), P(16), None)

    def fwd(d=128, N=8, causal=0, scale=0.125, vt8=16):
        return lib.fa_fwd_fp8(P(16), P(16), P(vt8), P(16), P(16), P(16), P(16), P(16), 1, 1, N, d,
                              scale, causal, None)

    assert prep(d=64) == 2                         # FP8 path: d = 128 only
    assert prep(q8=0) == 1
    assert prep(q8=24) == 3
    assert prep(signs=18) == 3                     # signs not 4-byte aligned
    assert prep(B=300, H=300) == 1                 # B*H > 65535
    assert prep(N=0) == 1
    assert fwd(d=64) == 2
    assert fwd(vt8=0) == 1
    assert fwd(causal=3) == 1
    assert fwd(scale=0.0) == 1
    assert lib.fa_fp8_vt_keys(1) == 16 and lib.fa_fp8_vt_keys(32) == 32
    assert lib.fa_fp8_vt_keys(1000) == 1008 and lib.fa_fp8_vt_keys(0) == 0


def test_bias_dropout_argument_errors(lib):
    P = ctypes.c_void_p

    def fwd(bias=None, sb=0, sh=0, p=0.1):
        return lib.fa_fwd_ex(P(16), P(16), P(16), P(16), P(16), 1, 1, 8, 64, 0.125, 0,
                             P(bias) if bias else None, sb, sh, p, 1, 0, None)

    def bwd(p=0.1, ws=1 << 20):
        return lib.fa_bwd_ex(P(16), P(16), P(16), P(16), P(16), P(16), P(16), P(16), P(16),
                             1, 1, 8, 64, 0.125, 0, None, 0, 0, p, 1, 0, P(16), ws, None)

    assert fwd(p=1.0) == 1 and fwd(p=-0.1) == 1 and fwd(p=float("nan")) == 1
    assert fwd(bias=24) == 3                       # bias not 16-byte aligned
    assert fwd(bias=16, sb=-1) == 1                # negative stride
    assert bwd(p=1.5) == 1
    assert bwd(ws=8) == 4                          # workspace too small


def test_dropout_keep_threshold_matches_oracle(lib):
    """The host's t = round(256 (1 - p)) (ties to even, clamped) equals the
    oracle's for the float32 p the call receives, ties included."""
    import numpy as np
    import oracle
    ps = [0.0, 0.1, 0.25, 0.5, 0.997, 0.999, 0.9999, 1e-3, 0.3, 0.7]
    ps += [float(np.float32((2 * k + 1) / 512)) for k in range(0, 256, 7)]  # exact ties
    ps += list(np.random.default_rng(3).random(200).astype(np.float32).astype(float))
    for p in ps:
        p32 = float(np.float32(p))
        assert fa.fa_dropout_keep_threshold(p32) == oracle.keep_threshold(p32), p32
    assert fa.fa_dropout_keep_threshold(1.0) == -1 and fa.fa_dropout_keep_threshold(-0.5) == -1


def test_workspace_sizes(lib):
    # base-2 LSE and D (fp32 [B,H,Np], Np = N rounded up to 128), each
    # 256-aligned
    # two fp32 vectors and two rows of 16 bf16 per (batch, head, padded row)
    assert fa.fa_bwd_workspace_size(2, 16, 4096, 128) == 2 * (2 * 16 * 4096 * 4) + 2 * (2 * 16 * 4096 * 32)
    assert fa.fa_bwd_workspace_size(1, 1, 130, 64) == 2 * 1024 + 2 * 256 * 32
    assert fa.fa_bwd_workspace_size(1, 1, 0, 64) == 0
    # decode: C chunks of partial outputs and LSEs
    ws = fa.fa_decode_workspace_size(8, 32, 32768, 128, 16)
    assert ws == 8 * 32 * 16 * 128 * 4 + 8 * 32 * 16 * 4
    assert fa.fa_decode_workspace_size(8, 32, 32768, 128, 0) == ws  # auto = 16 here
    assert fa.fa_decode_workspace_size(1, 1, 100, 128, 0) > 0
    assert fa.fa_decode_workspace_size(1, 1, 100, 96, 0) == 0
    # the automatic split also covers the paged decode's balanced schedule:
    # B*H + 2368 partial rows of d + 1 floats and 8 bytes per (sequence, head),
    # each region 256-aligned; larger than the chunked need for small shapes
    a256 = lambda x: (x + 255) // 256 * 256
    for B, H, L in ((1, 8, 2048), (3, 12, 700), (8, 32, 32768)):
        rows = B * H + 2368
        balanced = a256(rows * 128 * 4) + a256(rows * 4) + a256(B * H * 8)
        auto = fa.fa_decode_workspace_size(B, H, L, 128, 0)
        assert auto >= balanced and auto >= fa.fa_decode_workspace_size(B, H, L, 128, 1)
    assert fa.fa_decode_workspace_size(1, 8, 2048, 128, 0) == a256((8 + 2368) * 512) + a256((8 + 2368) * 4) + a256(64)
