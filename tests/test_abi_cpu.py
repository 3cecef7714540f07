"""The C-ABI library loads, exports every entry point the header declares, and
its host-only logic (sizes, argument checks) behaves as documented.  No
compute calls: these run without a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

import weight_shared_looped_b200 as tl
from oracle import tinyloop_oracle as o

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(tl_[a-z0-9_]+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert {"tl_pack_weights", "tl_block_create", "tl_prefill", "tl_decode_step"} <= names
    for n in sorted(names):
        assert hasattr(tl.lib, n), n


def test_only_tl_symbols_exported():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", tl.LIB_PATH], capture_output=True,
                         text=True).stdout
    syms = [line.split()[-1] for line in out.splitlines() if line.strip()]
    assert syms and all(s.startswith("tl_") or s.startswith("_") for s in syms), syms


def test_abi_version():
    assert tl.tl_abi_version() == 101


@pytest.mark.parametrize("K", [64, 256, 2048, 8192, 10, 11, 4000])
def test_words_per_row_matches_oracle(K):
    assert tl.tl_packed_words_per_row(K, 3) == o.int3_words_per_row(K)
    if K % 8 == 0:
        assert tl.tl_packed_words_per_row(K, 4) == K // 8


def test_packed_bytes_match_oracle_block_bytes():
    d, f = 2048, 8192
    for bits in (3, 4):
        total = 0
        for n, k in ((3 * d, d), (d, d), (f, d), (f, d), (d, f)):
            c, s = tl.tl_packed_bytes(n, k, bits, 128)
            total += c + s
        assert total == o.packed_block_bytes(d, f, bits, 128)


def test_kv_layer_bytes_match_pages_figures():
    # 10 layers (2 pre-blocks + L=8), max_seq 2048, 16 heads x 128
    fp16 = 10 * tl.tl_kv_layer_bytes(16, 128, 2048, tl.TL_KV_FP16)
    int8 = 10 * tl.tl_kv_layer_bytes(16, 128, 2048, tl.TL_KV_INT8)
    assert fp16 == o.kv_cache_bytes(10, 2048, 16, 128, "fp16")
    assert int8 == o.kv_cache_bytes(10, 2048, 16, 128, "int8")
    assert round(fp16 / 1e6, 1) == 167.8 and round(int8 / 1e6, 1) == 85.2


def test_store_h_slot_is_half_the_fp16_slot():
    # store-h keeps d fp16 values per position instead of the 2d of K and V
    # ("Current Status", KV cache mode table, Store-h (FP16): 43-50 % saving)
    h = 10 * tl.tl_kv_layer_bytes(16, 128, 2048, tl.TL_KV_H)
    fp16 = 10 * tl.tl_kv_layer_bytes(16, 128, 2048, tl.TL_KV_FP16)
    assert h * 2 == fp16 and h == 10 * 2048 * 2048 * 2


@pytest.mark.parametrize("args,status", [
    ((64, 128, 5, 64), tl.TL_ERR_UNSUPPORTED),     # bits
    ((64, 128, 4, 32), tl.TL_ERR_UNSUPPORTED),     # group
    ((64, 96, 4, 64), tl.TL_ERR_INVALID_ARG),      # K % group
    ((0, 128, 4, 64), tl.TL_ERR_INVALID_ARG),      # empty N
])
def test_pack_rejects_before_launch(args, status):
    n, k, bits, group = args
    rc = tl.lib.tl_pack_weights(ctypes.c_void_p(16), n, k, bits, group, ctypes.c_void_p(16),
                                ctypes.c_void_p(16), None)
    assert rc == status
    assert tl.lib.tl_last_error()


@pytest.mark.parametrize("T,H,hd,status", [
    (-1, 2, 64, tl.TL_ERR_INVALID_ARG),
    (8193, 2, 64, tl.TL_ERR_INVALID_ARG),
    (4, 0, 64, tl.TL_ERR_INVALID_ARG),
    (4, 257, 64, tl.TL_ERR_INVALID_ARG),
    (4, 2, 96, tl.TL_ERR_UNSUPPORTED),
    (4, 2, 32, tl.TL_ERR_UNSUPPORTED),
])
def test_attention_prefill_rejects_before_launch(T, H, hd, status):
    p = ctypes.c_void_p(16)
    assert tl.lib.tl_attention_prefill(p, p, p, T, H, hd, p, None) == status
    assert tl.lib.tl_last_error()


def test_attention_prefill_pointer_checks():
    p, odd = ctypes.c_void_p(16), ctypes.c_void_p(24)   # 24: 8-byte but not 16-byte aligned
    f = tl.lib.tl_attention_prefill
    assert f(None, p, p, 4, 2, 64, p, None) == tl.TL_ERR_INVALID_ARG
    assert f(p, p, p, 4, 2, 64, None, None) == tl.TL_ERR_INVALID_ARG
    assert f(p, odd, p, 4, 2, 128, p, None) == tl.TL_ERR_INVALID_ARG
    assert f(p, p, p, 4, 2, 64, odd, None) == tl.TL_ERR_INVALID_ARG
    assert f(None, None, None, 0, 2, 64, None, None) == tl.TL_OK   # empty: no-op


def test_null_pointers_rejected():
    assert tl.lib.tl_pack_weights(None, 8, 64, 4, 64, None, None, None) == tl.TL_ERR_INVALID_ARG
    assert tl.lib.tl_kv_quant_int8(None, 4, 128, None, None, None) == tl.TL_ERR_INVALID_ARG
    assert tl.lib.tl_kv_quant_int8(None, 0, 128, None, None, None) == tl.TL_OK   # empty: no-op
    assert tl.lib.tl_kv_quant_int8(None, 4, 0, None, None, None) == tl.TL_ERR_INVALID_ARG
    assert tl.lib.tl_prefill(None, None, None, 1, 1, None, 0, None, None, None) == tl.TL_ERR_INVALID_ARG
    assert tl.lib.tl_sync_status(None, None) == tl.TL_ERR_INVALID_ARG


def _desc(**over):
    cfg = dict(d_model=256, n_heads=4, head_dim=64, ffn=768, bits=4, group=64, eps=1e-5,
               rope_theta=1e4)
    cfg.update(over)
    ptrs = [16] * 12
    return tl.BlockDesc(cfg["d_model"], cfg["n_heads"], cfg["head_dim"], cfg["ffn"], cfg["bits"],
                        cfg["group"], cfg["eps"], cfg["rope_theta"], *ptrs)


@pytest.mark.parametrize("over,status", [
    ({"d_model": 200}, tl.TL_ERR_INVALID_ARG),
    ({"head_dim": 96, "n_heads": 2, "d_model": 192}, tl.TL_ERR_INVALID_ARG),
    ({"head_dim": 32, "n_heads": 8}, tl.TL_ERR_UNSUPPORTED),
    ({"n_heads": 3}, tl.TL_ERR_INVALID_ARG),
    ({"ffn": 700}, tl.TL_ERR_INVALID_ARG),
    ({"bits": 2}, tl.TL_ERR_UNSUPPORTED),
    ({"eps": 0.0}, tl.TL_ERR_INVALID_ARG),
])
def test_block_create_validation(over, status):
    out = ctypes.c_void_p()
    assert tl.lib.tl_block_create(ctypes.byref(_desc(**over)), ctypes.byref(out)) == status
    assert not out.value


def test_int4_block_wraps_without_device_work():
    out = ctypes.c_void_p()
    assert tl.lib.tl_block_create(ctypes.byref(_desc()), ctypes.byref(out)) == tl.TL_OK
    assert out.value
    assert tl.lib.tl_block_destroy(out) == tl.TL_OK


def test_model_create_validation():
    blk = ctypes.c_void_p()
    assert tl.lib.tl_block_create(ctypes.byref(_desc()), ctypes.byref(blk)) == tl.TL_OK
    bad = [dict(max_tokens=0), dict(max_lanes=9), dict(max_L=65), dict(max_ctx=4)]
    for b in bad:
        kw = dict(max_tokens=16, max_lanes=1, max_ctx=64, max_L=8)
        kw.update(b)
        d = tl.ModelDesc(None, 0, blk, None, 0, ctypes.c_void_p(16), kw["max_tokens"],
                         kw["max_lanes"], kw["max_ctx"], kw["max_L"])
        out = ctypes.c_void_p()
        assert tl.lib.tl_model_create(ctypes.byref(d), ctypes.byref(out)) == tl.TL_ERR_INVALID_ARG
    tl.lib.tl_block_destroy(blk)


@pytest.mark.parametrize("N,K,group,T,status", [
    (64, 192, 128, 1, tl.TL_ERR_INVALID_ARG),    # K % group == 64: half a scale group per row
    (64, 320, 128, 16, tl.TL_ERR_INVALID_ARG),
    (64, 96, 64, 1, tl.TL_ERR_INVALID_ARG),      # K % 64
    (96, 128, 64, 1, tl.TL_ERR_INVALID_ARG),     # N % 64
    (64, 128, 32, 1, tl.TL_ERR_UNSUPPORTED),     # group
    (64, 128, 64, 0, tl.TL_ERR_INVALID_ARG),     # T
    (64, 128, 64, 8193, tl.TL_ERR_INVALID_ARG),
])
def test_linear_entry_points_reject_before_launch(N, K, group, T, status):
    """Both linear-layer entry points reject a shape whose rows do not hold
    whole scale groups before anything is launched (no GPU is touched: the
    pointers are placeholders)."""
    p = ctypes.c_void_p(256)
    assert tl.lib.tl_linear(p, p, N, K, group, p, T, p, p, None) == status
    assert tl.lib.tl_last_error()
    assert tl.lib.tl_linear_noalloc(p, p, N, K, group, p, T, p, None) == status
    assert tl.lib.tl_last_error()


def test_read_probe_rejects_before_launch():
    p, odd = ctypes.c_void_p(256), ctypes.c_void_p(264)
    f = tl.lib.tl_read_probe
    assert f(None, 1024, 1, p, None) == tl.TL_ERR_INVALID_ARG
    assert f(p, 1024, 1, None, None) == tl.TL_ERR_INVALID_ARG
    assert f(odd, 1024, 1, p, None) == tl.TL_ERR_INVALID_ARG      # 8-byte aligned only
    assert f(p, 1000, 1, p, None) == tl.TL_ERR_INVALID_ARG        # not a multiple of 16
    assert f(p, 0, 1, p, None) == tl.TL_ERR_INVALID_ARG
    assert f(p, 1024, 0, p, None) == tl.TL_ERR_INVALID_ARG
    assert f(p, 1024, 4097, p, None) == tl.TL_ERR_INVALID_ARG


def test_int3_block_wraps_without_device_work():
    """An INT3 block is wrapped like an INT4 one: no copy, no device work, no
    library-owned bytes (every kernel reads the canonical INT3 words)."""
    out = ctypes.c_void_p()
    assert tl.lib.tl_block_create(ctypes.byref(_desc(bits=3)), ctypes.byref(out)) == tl.TL_OK
    n = ctypes.c_size_t(7)
    assert tl.lib.tl_block_device_bytes(out, ctypes.byref(n)) == tl.TL_OK
    assert n.value == 0
    assert tl.lib.tl_block_destroy(out) == tl.TL_OK


@pytest.mark.parametrize("N,K", [(1, 1), (3, 31), (48, 256), (6144, 2048), (2048, 8192), (5, 100)])
def test_sign_bits_bytes_match_oracle_plane(N, K):
    """The sign plane is the oracle's bit-plane layout: uint32 [N, ceil(K/32)]."""
    want = o.pack_bits(np.zeros((N, K), np.uint8)).nbytes
    assert tl.tl_sign_bits_bytes(N, K) == want == N * ((K + 31) // 32) * 4


def test_sign_plane_is_a_quarter_of_the_int4_codes():
    """One bit per weight on top of four: the pages' "+25 % storage" for the
    sign-of-frac channel ("Performance and Memory", "Cross-iteration stochastic
    rounding"), for every matrix of the 407M-shaped block."""
    d, f = 2048, 8192
    for n, k in ((3 * d, d), (d, d), (f, d), (f, d), (d, f)):
        codes, _ = tl.tl_packed_bytes(n, k, 4, 128)
        assert tl.tl_sign_bits_bytes(n, k) * 4 == codes


@pytest.mark.parametrize("args,status", [
    ((64, 128, 5, 64), tl.TL_ERR_UNSUPPORTED),     # bits
    ((64, 128, 4, 32), tl.TL_ERR_UNSUPPORTED),     # group
    ((64, 96, 4, 64), tl.TL_ERR_INVALID_ARG),      # K % group
    ((0, 128, 4, 64), tl.TL_ERR_INVALID_ARG),      # empty N
])
def test_pack_sign_bits_rejects_before_launch(args, status):
    n, k, bits, group = args
    p = ctypes.c_void_p(16)
    assert tl.lib.tl_pack_sign_bits(p, n, k, bits, group, p, p, None) == status
    assert tl.lib.tl_last_error()


def test_sign_bits_null_arguments_rejected():
    p = ctypes.c_void_p(16)
    assert tl.lib.tl_pack_sign_bits(None, 64, 128, 4, 64, p, p, None) == tl.TL_ERR_INVALID_ARG
    assert tl.lib.tl_pack_sign_bits(p, 64, 128, 4, 64, None, p, None) == tl.TL_ERR_INVALID_ARG
    assert tl.lib.tl_pack_sign_bits(p, 64, 128, 4, 64, p, None, None) == tl.TL_ERR_INVALID_ARG
    assert tl.lib.tl_sign_bits_bytes(64, 128, None) == tl.TL_ERR_INVALID_ARG
    assert tl.lib.tl_sign_bits_bytes(0, 128, ctypes.byref(ctypes.c_size_t())) == tl.TL_ERR_INVALID_ARG


def test_null_handles_rejected_before_any_work():
    """Every call on a model, block or cache handle checks the handle first
    (a NULL handle is TL_ERR_INVALID_ARG, nothing launched); destroying NULL
    is a no-op."""
    p = ctypes.c_void_p(16)
    sz = ctypes.c_size_t()
    i = ctypes.c_int()
    one = (ctypes.c_int * 1)(1)
    E = tl.TL_ERR_INVALID_ARG
    L = tl.lib
    calls = [
        L.tl_block_device_bytes(None, ctypes.byref(sz)),
        L.tl_model_device_bytes(None, ctypes.byref(sz)),
        L.tl_model_set_graphs(None, 1),
        L.tl_model_set_decode_chunks(None, 0),
        L.tl_model_set_exit_threshold(None, 1.0),
        L.tl_model_set_cross_iter(None, 1),
        L.tl_model_set_iteration_blocks(None, None, 0),
        L.tl_loops_used(None, p, 1, None),
        L.tl_kv_bytes(None, 1, 16, ctypes.cast(one, ctypes.c_void_p), 0, ctypes.byref(sz)),
        L.tl_kv_create(None, 1, 16, ctypes.cast(one, ctypes.c_void_p), 0, p, 1 << 20, None),
        L.tl_kv_reset(None, 0, None),
        L.tl_kv_position(None, 0, ctypes.byref(i)),
        L.tl_kv_set_position(None, 0, 0, None),
        L.tl_kv_layer_ptrs(None, 0, 0, ctypes.byref(ctypes.c_void_p()), ctypes.byref(ctypes.c_void_p()),
                           ctypes.byref(ctypes.c_void_p()), ctypes.byref(ctypes.c_void_p())),
        L.tl_decode_step(None, None, p, None, ctypes.cast(one, ctypes.c_void_p), 0, None, None, None),
        L.tl_extend(None, None, 0, p, None, 1, 1, None, None, None),
        L.tl_greedy_head(None, p, 1, p, None),
        L.tl_spec_step(None, None, 0, 1, 2, 1, 2, p, ctypes.byref(i), None),
        L.tl_check_bounded_wait(None, 1000, None),
        L.tl_sync_status(None, None),
    ]
    assert calls == [E] * len(calls), calls
    assert L.tl_block_destroy(None) == tl.TL_OK
    assert L.tl_model_destroy(None) == tl.TL_OK
    assert L.tl_kv_destroy(None) == tl.TL_OK
