"""The C-ABI library without a GPU: it loads, exports every entry point that
include/kvq.h declares, reproduces the per-token byte table, and rejects bad
arguments on the host before any CUDA call."""
import ctypes
import json
import os
import re

import pytest

import oracle as O
import quantized_paged_kv_03_b200 as K
from quantized_paged_kv_03_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return K.lib()


def header_functions():
    src = open(os.path.join(ROOT, "include", "kvq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol(L):
    names = header_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n
    assert sorted(K.exported_symbols()) == names
    assert L.kvq_version() == 3


def test_token_bytes_table(L):
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "token_bytes.json")))
    for name, want in g["bytes_per_token"].items():
        assert K.token_bytes(name, 256) == want
    assert K.token_bytes("mxfp8_g32", 128) == 264
    assert K.token_bytes("fp8_tensor", 128) == 256
    assert K.token_bytes("bf16", 128) == 512
    assert K.token_bytes("fp8_row256", 128) == 0        # a 256-wide row needs D = 256
    assert K.token_bytes(9, 256) == 0


@pytest.mark.parametrize("fmt", sorted(K.FORMATS))
@pytest.mark.parametrize("D", [128, 256])
def test_row_bytes_agree_with_oracle(L, fmt, D):
    f = K.FORMATS[fmt]
    for is_v in (False, True):
        want = O.row_bytes(f, is_v, D)
        if K.token_bytes(fmt, D) == 0:
            continue
        assert K.row_bytes(fmt, D, is_v) == want


def test_cache_bytes_is_header_plus_slabs(L):
    # slab = 64 tokens x (K+V bytes per token) for formats whose regions are 16-byte multiples
    for fmt, D, P in (("int8_g64", 256, 64), ("nvfp4_g16", 256, 64), ("k8v4", 256, 64),
                      ("mxfp8_g32", 128, 128), ("bf16", 128, 64), ("fp8_tensor", 128, 64)):
        n = K.cache_bytes(fmt, D, n_kv_heads=3, page_size=P, num_pages=5, num_layers=2)
        assert n == 256 + 2 * 5 * 3 * P * K.token_bytes(fmt, D), fmt


def test_slab_regions_are_32_byte_aligned(L):
    """The prefill kernel reads a row's 16-byte code chunks in pairs with one
    32-byte load, and the pool starts 256-byte aligned: every code row, every
    region of a page slab (K codes, K scales, V codes, V scales) and the slab
    itself must then be whole multiples of 32 bytes, for every format, head_dim
    and page size the cache accepts.  The slab size is read back from the pool
    size (header + layers x pages x heads x slab)."""
    a16 = lambda x: (x + 15) // 16 * 16
    checked = 0
    for fmt in sorted(K.FORMATS):
        for D in (128, 256):
            if K.token_bytes(fmt, D) == 0:
                continue
            kc, ks = K.row_bytes(fmt, D, False)
            vc, vs = K.row_bytes(fmt, D, True)
            assert kc % 32 == 0 and vc % 32 == 0, (fmt, D)
            for P in range(16, 257, 16):
                regions = [a16(P * kc), a16(P * ks), a16(P * vc), a16(P * vs)]
                assert all(r % 32 == 0 for r in regions), (fmt, D, P, regions)
                slab = K.cache_bytes(fmt, D, n_kv_heads=1, page_size=P, num_pages=1, flags=K.FLAG_NO_ROTATE) - 256
                assert slab == sum(regions) and slab % 32 == 0, (fmt, D, P, slab)
                checked += 1
    assert checked >= 12 * 16


def _desc(**kw):
    base = dict(fmt=K.FORMATS["int8_g64"], D=256, H=2, P=64, pages=4, layers=1, flags=0)
    base.update(kw)
    return K._Desc(base["fmt"], base["D"], base["H"], base["P"], base["pages"], base["layers"],
                   base["flags"], None)


def test_create_validates_on_host(L):
    h = ctypes.c_void_p()
    fake = ctypes.c_void_p(1 << 20)          # never dereferenced by create
    ok = _desc()
    need = L.kvq_cache_bytes(ctypes.byref(ok))
    assert L.kvq_cache_create(ctypes.byref(ok), fake, need, ctypes.byref(h)) == 0
    assert L.kvq_cache_destroy(h) == 0
    assert L.kvq_cache_create(ctypes.byref(ok), fake, need - 1, ctypes.byref(h)) == 4
    assert L.kvq_cache_create(ctypes.byref(ok), ctypes.c_void_p((1 << 20) + 16), need,
                              ctypes.byref(h)) == 1
    assert L.kvq_cache_create(ctypes.byref(ok), None, need, ctypes.byref(h)) == 1
    assert L.kvq_cache_create(ctypes.byref(_desc(fmt=11)), fake, need, ctypes.byref(h)) == 2
    assert L.kvq_cache_create(ctypes.byref(_desc(D=128)), fake, need, ctypes.byref(h)) == 2   # rotated needs 256
    assert L.kvq_cache_create(ctypes.byref(_desc(D=128, flags=1)), fake, need, ctypes.byref(h)) == 0
    L.kvq_cache_destroy(h)
    assert L.kvq_cache_create(ctypes.byref(_desc(P=48 + 8)), fake, need, ctypes.byref(h)) == 3
    assert L.kvq_cache_create(ctypes.byref(_desc(H=0)), fake, need, ctypes.byref(h)) == 3
    assert L.kvq_cache_create(ctypes.byref(_desc(D=96)), fake, need, ctypes.byref(h)) == 2


def test_calls_reject_bad_arguments_before_launch(L):
    h = ctypes.c_void_p()
    fake = ctypes.c_void_p(1 << 20)
    d = _desc(H=2)
    assert L.kvq_cache_create(ctypes.byref(d), fake, L.kvq_cache_bytes(ctypes.byref(d)), ctypes.byref(h)) == 0
    p = ctypes.c_void_p(1 << 21)
    # layer out of range, negative count, zero tokens
    assert L.kvq_append(h, 1, p, p, p, 4, None) == 1
    assert L.kvq_append(h, 0, p, p, p, -1, None) == 1
    assert L.kvq_append(h, 0, p, p, p, 0, None) == 0
    assert L.kvq_append(h, 0, ctypes.c_void_p((1 << 21) + 2), p, p, 4, None) == 1   # misaligned
    # n_q_heads not a multiple of n_kv_heads
    assert L.kvq_decode_attention(h, 0, p, 5, p, 4, p, 2, 256, p, 1, 0.0, p, 1 << 20, None) == 3
    assert L.kvq_decode_workspace_bytes(h, 2, 5, 256) == 0
    # max_seq_len beyond the block table
    assert L.kvq_decode_attention(h, 0, p, 4, p, 2, p, 2, 256, p, 1, 0.0, p, 1 << 20, None) == 3
    # batch 0 is a no-op
    assert L.kvq_decode_attention(h, 0, p, 4, p, 4, p, 0, 256, p, 1, 0.0, p, 1 << 20, None) == 0
    # chunked prefill: layer out of range, heads not a multiple of kv-heads,
    # negative scale, misaligned q; max_q_len 0 and batch 0 are no-ops
    assert L.kvq_prefill_attention(h, 1, p, 4, p, 8, p, 4, p, 2, p, 1, 0.0, None) == 1
    assert L.kvq_prefill_attention(h, 0, p, 5, p, 8, p, 4, p, 2, p, 1, 0.0, None) == 3
    assert L.kvq_prefill_attention(h, 0, p, 4, p, 8, p, 4, p, 2, p, 1, -1.0, None) == 1
    assert L.kvq_prefill_attention(h, 0, ctypes.c_void_p((1 << 21) + 8), 4, p, 8, p, 4, p, 2, p, 1, 0.0,
                                   None) == 1
    assert L.kvq_prefill_attention(h, 0, p, 4, p, 0, p, 4, p, 2, p, 1, 0.0, None) == 0
    assert L.kvq_prefill_attention(h, 0, p, 4, p, 8, p, 4, p, 0, p, 1, 0.0, None) == 0
    assert L.kvq_encode(7, p, 4, p, None) == 1
    assert L.kvq_encode(0, p, 0, p, None) == 0
    assert L.kvq_read_rows(h, 0, p, 3, p, None, p, p, None) == 1     # K scales needed
    assert L.kvq_dequant(h, 3, p, 3, p, p, None) == 1
    assert L.kvq_status_string(4) == b"pool or workspace too small"
    L.kvq_cache_destroy(h)


def test_noalloc_decode_rejects_what_decode_rejects(L):
    """The allocation-free entry point validates through the same host checks
    as kvq_decode_attention and returns the same status codes, before any CUDA
    call (this runs without a GPU)."""
    h = ctypes.c_void_p()
    fake = ctypes.c_void_p(1 << 20)
    d = _desc(H=2)
    assert L.kvq_cache_create(ctypes.byref(d), fake, L.kvq_cache_bytes(ctypes.byref(d)), ctypes.byref(h)) == 0
    p = ctypes.c_void_p(1 << 21)
    odd = ctypes.c_void_p((1 << 21) + 8)
    #   (layer, q, n_q_heads, max_pages, batch, max_seq_len, out, scale) -> status
    cases = [((1, p, 4, 4, 2, 256, p, 0.0), 1),      # layer out of range
             ((0, p, 5, 4, 2, 256, p, 0.0), 3),      # heads not a multiple of kv-heads
             ((0, p, 0, 4, 2, 256, p, 0.0), 1),      # no query heads
             ((0, p, 4, 4, -1, 256, p, 0.0), 1),     # negative batch
             ((0, p, 4, 4, 5000, 256, p, 0.0), 3),   # batch beyond the limit
             ((0, p, 4, 2, 2, 256, p, 0.0), 3),      # max_seq_len beyond the block table
             ((0, odd, 4, 4, 2, 256, p, 0.0), 1),    # misaligned q
             ((0, p, 4, 4, 2, 256, odd, 0.0), 1),    # misaligned out
             ((0, None, 4, 4, 2, 256, p, 0.0), 1),   # null q
             ((0, p, 4, 4, 2, 256, p, -1.0), 1),     # negative scale
             ((0, p, 4, 4, 0, 256, p, 0.0), 0)]      # batch 0: nothing to do
    for (layer, q, hq, mp, B, ms, out, sc), want in cases:
        a = L.kvq_decode_attention(h, layer, q, hq, p, mp, p, B, ms, out, 1, sc, p, 1 << 20, None)
        b = L.kvq_decode_attention_noalloc(h, layer, q, hq, p, mp, p, B, ms, out, 1, sc, None)
        assert a == b == want, (layer, hq, mp, B, ms, sc, a, b)
    # a call that would launch without a workspace is an argument error
    assert L.kvq_decode_attention(h, 0, p, 4, p, 4, p, 2, 256, p, 1, 0.0, None, 1 << 20, None) == 1
    L.kvq_cache_destroy(h)


def test_wait_limit_setting_round_trips(L):
    prev = L.kvq_debug_set_wait_polls(7)
    assert L.kvq_debug_set_wait_polls(-1) == 7       # negative restores the default
    assert L.kvq_debug_set_wait_polls(-1) == prev == 1 << 22


def test_python_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(K, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(K, "_lib", None)
    with pytest.raises(K.KVQError):
        K.lib()
