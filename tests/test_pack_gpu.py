"""Packer and INT8 KV quantiser on the GPU: bit-exact against the oracle on
identical inputs (the integer parts of the hot path)."""
import numpy as np
import pytest
import torch

import synthetic as syn
import weight_shared_looped_b200 as tl
from oracle import tinyloop_oracle as o

pytestmark = pytest.mark.gpu


def _adversarial(n, k, group, seed):
    w = syn.normal((n, k), 0.02, seed, f"pack.{n}.{k}.{group}")
    rng = np.random.default_rng(seed)
    g = w.reshape(n, k // group, group)
    if n > 3:
        g[1, 0] = 0.0                                            # zero group
        g[2, 0] = np.float32(7e-3)                               # constant group
        g[3, 0, :8] = np.array([7, 2.5, -2.5, 3.5, -0.5, 0.5, 1.5, -7], np.float32)  # exact halves
        g[3, 0, 8:] = 0.0
    if n > 5:
        g[4, -1] *= np.float32(1e-5)                             # fp16-subnormal scale
        g[5, -1] *= np.float32(300.0)                            # large magnitudes
    # random exact ties: value = (m + 0.5) * s for an exactly representable s
    rows = rng.integers(0, n, size=min(n, 16))
    for r in rows:
        g[r, -1, :4] = np.array([3.5, -1.5, 0.5, 7.0], np.float32) * np.float32(0.25)
    return w


@pytest.mark.parametrize("bits,group,n,k", [
    (4, 64, 1, 64), (4, 128, 37, 1024), (4, 64, 300, 256), (4, 128, 6, 8192),
    (3, 128, 37, 1280), (3, 64, 5, 64), (3, 128, 129, 2048), (3, 64, 17, 1000 // 64 * 64),
])
def test_pack_bit_exact(bits, group, n, k):
    w = _adversarial(n, k, group, seed=n * 7 + k)
    codes, scales = o.quantize_groupwise(w, bits, group)
    words = o.pack_codes(codes, bits)
    cb, sb = tl.tl_packed_bytes(n, k, bits, group)
    assert cb == words.nbytes and sb == scales.nbytes
    pw = torch.full((cb // 4,), -1, dtype=torch.int32, device="cuda")
    ps = torch.full((sb // 2,), -1, dtype=torch.int16, device="cuda")
    tl.tl_pack_weights(torch.from_numpy(w).cuda(), bits, group, pw, ps)
    got_w = pw.cpu().numpy().view(np.uint32).reshape(words.shape)
    got_s = ps.cpu().numpy().view(np.uint16).reshape(scales.shape)
    assert np.array_equal(got_s, scales.view(np.uint16))
    assert np.array_equal(got_w, words)
    out = torch.zeros(n * k, dtype=torch.int8, device="cuda")
    tl.tl_unpack_codes(pw, n, k, bits, out)
    assert np.array_equal(out.cpu().numpy().reshape(n, k), codes)


@pytest.mark.parametrize("name", ["qkv", "o", "gate", "up", "down"])
@pytest.mark.parametrize("bits", [4, 3])
def test_pack_full_size_407m_loop_block(name, bits):
    w = syn.block_weights(syn.SHAPE_407M, 0, "loop")[f"w_{name}"]
    n, k = w.shape
    codes, scales = o.quantize_groupwise(w, bits, 128)
    words = o.pack_codes(codes, bits)
    cb, sb = tl.tl_packed_bytes(n, k, bits, 128)
    pw = torch.empty(cb // 4, dtype=torch.int32, device="cuda")
    ps = torch.empty(sb // 2, dtype=torch.int16, device="cuda")
    tl.tl_pack_weights(torch.from_numpy(w).cuda(), bits, 128, pw, ps)
    assert np.array_equal(ps.cpu().numpy().view(np.uint16), scales.view(np.uint16).ravel())
    assert np.array_equal(pw.cpu().numpy().view(np.uint32), words.ravel())


@pytest.mark.parametrize("rows,hd", [(0, 128), (1, 128), (1000, 128), (333, 64), (7, 5), (3, 256)])
def test_kv_quant_int8_bit_exact(rows, hd):
    x = (syn.normal((max(rows, 1), hd), 1.0, 0, f"kvq.{rows}.{hd}")[:rows]).astype(np.float16)
    if rows > 3:
        x[0] = 0                                            # zero row -> scale 0, codes 0
        x[1, : min(hd, 8)] = np.array([0.9921875, -0.5, 0.25, 0.00390625, 0.01171875,
                                       -0.9921875, 0.1, 0.0], np.float16)[: min(hd, 8)]
        x[1, 8:] = 0
        x[2] *= np.float16(1e-3)                            # small scale
        x[3] *= np.float16(100)                             # large values
    codes = torch.full((max(rows, 1) * hd,), 99, dtype=torch.int8, device="cuda")
    scales = torch.full((max(rows, 1),), -1, dtype=torch.int16, device="cuda")
    xt = torch.from_numpy(x.view(np.int16).copy()).cuda().reshape(rows, hd)
    tl.tl_kv_quant_int8(xt, codes, scales)
    if rows == 0:
        assert int(codes[0]) == 99 and int(scales[0]) == -1   # nothing written
        return
    rc, rs = o.kv_quant_int8(x)
    assert np.array_equal(scales.cpu().numpy()[:rows].view(np.uint16), rs.view(np.uint16))
    assert np.array_equal(codes.cpu().numpy()[: rows * hd].reshape(rows, hd), rc)
