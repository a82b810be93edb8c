"""The C-ABI library loads without a GPU, exports every entry point of include/krea2.h, and
rejects bad arguments on the host before anything is launched."""
import ctypes

import numpy as np
import os
import re

import pytest

import krea2_inputs as KI

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "krea2.h")


@pytest.fixture(scope="module")
def K2():
    from flow_matching_stream_b200 import build
    build.build()
    import flow_matching_stream_b200 as K2
    return K2


def declared_entry_points():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(krea2_\w+)\s*\(", text)))


def test_header_declares_the_four_named_entry_points():
    names = declared_entry_points()
    for n in ("krea2_rope_tables", "krea2_gqa_attention", "krea2_block_forward", "krea2_backbone_forward"):
        assert n in names


def test_library_exports_every_declared_symbol(K2):
    lib = ctypes.CDLL(os.path.join(ROOT, "flow_matching_stream_b200", "libkrea2.so"))
    missing = [n for n in declared_entry_points() if not hasattr(lib, n)]
    assert not missing, missing
    from flow_matching_stream_b200 import _lib
    assert sorted(_lib.SIGNATURES) == declared_entry_points()


def test_workspace_size_and_dim_checks_on_host(K2):
    d = K2.dims_struct(KI.FULL)
    lib = K2.lib()
    ws = lib.krea2_workspace_size(ctypes.byref(d), 2, 512, 4096, K2.KREA2_BF16)
    assert ws > 0
    bad = K2.dims_struct(KI.FULL)
    bad.axes[2] = 40                      # sum(axes) != head_dim (the pages' ValueError)
    assert lib.krea2_workspace_size(ctypes.byref(bad), 2, 512, 4096, K2.KREA2_BF16) == 0
    assert lib.krea2_workspace_size(ctypes.byref(d), 2, 512, 0, K2.KREA2_BF16) == 0   # no image tokens
    rc = lib.krea2_rope_tables(ctypes.byref(bad), None, 10, None, None, None)
    assert rc == -1 and b"axes" in lib.krea2_last_error_string()
    rc = lib.krea2_rope_tables(ctypes.byref(d), None, 10, None, None, None)
    assert rc == -1 and b"NULL" in lib.krea2_last_error_string()
    bad2 = K2.dims_struct(KI.FULL)
    bad2.Hkv = 10
    assert lib.krea2_block_forward(ctypes.byref(bad2), 1, 8, 8, 0, None, None, None, None, None, None, None, 0,
                                   None) == -1
    assert lib.krea2_linear(K2.KREA2_BF16, 0, 128, 100, 64, 1, 1, 1, None, 1, 0, None) == -5   # Nw % 128
    assert lib.krea2_linear(K2.KREA2_BF16, 7, 128, 128, 64, 1, 1, 1, None, 1, 0, None) == -1   # epilogue
    assert lib.krea2_attention_workspace_size(ctypes.byref(d), 2, 512, 4096, K2.KREA2_BF16) == \
        2 * 4608 * (48 + 12) * 128 * 2


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    from flow_matching_stream_b200 import _lib
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        _lib.load()


def test_sigma_schedule_host_functions_match_oracle(K2):
    # host-side schedule of the library (C code) against the oracle's fp64 schedule
    from oracle import krea2_oracle as O
    for n in (28, 8, 1):
        for mu in (O.shift_mu(4096), 1.15, 0.0):
            got = K2.sigma_schedule(n, mu)
            ref = O.shifted_sigmas(n, mu)
            assert got.shape == ref.shape
            assert abs(float(got[-1])) == 0.0 and abs(float(got[0]) - 1.0) < 1e-7
            assert float(np.max(np.abs(got - ref))) < 1e-7
    for L in (256, 1024, 4096, 6400):
        assert abs(K2.shift_mu(L) - O.shift_mu(L)) < 1e-12
    assert K2.lib().krea2_sigma_schedule(0, 0.5, None) == -1


def test_block_causal_key_end_matches_the_oracle_pattern(K2):
    from oracle import krea2_oracle as O
    rng = np.random.default_rng(5)
    for _ in range(30):
        segs = [(("text", "image")[rng.integers(2)], int(rng.integers(1, 9))) for _ in range(rng.integers(1, 8))]
        ids = O.image_block_ids(segs)
        kend = K2.block_causal_key_end(ids)
        allowed = O.block_causal_allowed(ids)
        S = len(ids)
        assert all(allowed[q].tolist() == [k < kend[q] for k in range(S)] for q in range(S))
    bad = np.array([0, 0, -1, 0], dtype=np.int32)  # block 0 split in two runs
    with pytest.raises(K2.Krea2Error):
        K2.block_causal_key_end(bad)


def test_kv_cache_argument_checks_on_host(K2):
    # every rejection happens before anything is launched (the pointers are never touched)
    d = K2.dims_struct(KI.FULL)
    lib = K2.lib()
    fake = 1 << 20
    assert lib.krea2_kv_cache_attention_workspace_size(ctypes.byref(d), 2, 1024, K2.KREA2_BF16) == 2 * 1024 * 48 * 128 * 2
    assert lib.krea2_kv_cache_attention_workspace_size(ctypes.byref(d), 2, 1024, K2.KREA2_F32) == 0
    # rows [row0, row0 + n) must fit the capacity
    rc = lib.krea2_kv_cache_append(ctypes.byref(d), 2, 100, 950, 1000, K2.KREA2_BF16, fake, fake, fake, fake, fake,
                                   fake, None)
    assert rc == -1 and b"capacity" in lib.krea2_last_error_string()
    rc = lib.krea2_kv_cache_append(ctypes.byref(d), 2, 100, 0, 1000, K2.KREA2_F32, fake, fake, fake, fake, fake, fake,
                                   None)
    assert rc == -5
    rc = lib.krea2_kv_cache_append(ctypes.byref(d), 2, 100, 0, 1000, K2.KREA2_BF16, fake, fake, fake, fake, fake + 8,
                                   fake, None)
    assert rc == -1 and b"aligned" in lib.krea2_last_error_string()
    # the queries are the last Nq of L cached keys, and the cache must hold L rows
    for T, L, Nq, cap in ((0, 100, 101, 200), (120, 100, 10, 200), (0, 300, 10, 200)):
        rc = lib.krea2_gqa_attention_kv_cache(ctypes.byref(d), 2, T, L, Nq, K2.KREA2_BF16, fake, fake, fake, fake,
                                              None, fake, fake, cap, None, fake, fake, 1 << 30, None)
        assert rc == -1, (T, L, Nq, cap)
    rc = lib.krea2_gqa_attention_kv_cache(ctypes.byref(d), 2, 0, 300, 10, K2.KREA2_BF16, fake, fake, fake, fake, None,
                                          fake, fake, 300, None, fake, fake, 10, None)
    assert rc == -2  # workspace too small


def test_token_counts_that_overflow_int_are_rejected(K2):
    # T + N beyond 2^31 must be caught by the size checks, not wrap around
    d = K2.dims_struct(KI.FULL)
    lib = K2.lib()
    big = (1 << 31) - 10
    assert lib.krea2_workspace_size(ctypes.byref(d), 1, big, 100, K2.KREA2_BF16) == 0
    assert lib.krea2_attention_workspace_size(ctypes.byref(d), 1, big, 100, K2.KREA2_BF16) == 0
    fake = 1 << 20
    rc = lib.krea2_gqa_attention_block_causal(ctypes.byref(d), 1, big, 100, K2.KREA2_BF16, fake, fake, fake, fake,
                                              fake, None, fake, fake, fake, 1 << 40, None)
    assert rc == -1 and b"2^30" in lib.krea2_last_error_string()
    bad = K2.dims_struct(KI.FULL)
    bad.H = 1 << 30                       # H * D overflows int
    assert lib.krea2_workspace_size(ctypes.byref(bad), 1, 8, 8, K2.KREA2_BF16) == 0
