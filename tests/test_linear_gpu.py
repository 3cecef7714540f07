"""The quantised-weight GEMM (tl_linear) against the oracle's dequantised
matrix product, element by element, for both kernels: the register-dequant
mma.sync kernel (T < 64) and the tcgen05 kernel (T >= 64), across several
tiles, ragged token tails and split-K."""
import numpy as np
import pytest
import torch

import synthetic as syn
import weight_shared_looped_b200 as tl
from oracle import tinyloop_oracle as o

pytestmark = pytest.mark.gpu


def _case(N, K, T, group, seed):
    w = syn.normal((N, K), 0.02, seed, f"lin.w.{N}.{K}")
    codes, scales = o.quantize_groupwise(w, 4, group)
    words = o.pack_codes(codes, 4)
    x = syn.normal((T, K), 1.0, seed, f"lin.x.{T}.{K}").astype(np.float16)
    ref = x.astype(np.float64) @ o.dequantize(codes, scales, group).T
    return words, scales, x, ref


def _run(words, scales, x, N, K, group):
    T = x.shape[0]
    y = torch.full((T, N), float("nan"), dtype=torch.float32, device="cuda")
    wsb = tl.tl_linear_workspace_bytes(N, K, T)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    tl.tl_linear(torch.from_numpy(words.view(np.int32)).cuda(),
                 torch.from_numpy(scales.view(np.int16)).cuda(), N, K, group,
                 torch.from_numpy(x.view(np.int16)).cuda(), y, ws)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("N,K,T,group", [
    (64, 64, 1, 64), (128, 256, 8, 64), (256, 2048, 5, 128), (6144, 2048, 3, 128),
    (2048, 8192, 8, 128), (768, 256, 37, 64), (1536, 256, 16, 64),
    # chunk counts that are not powers of two (3 and 5 chunks of 64 k; odd scale groups per row)
    (128, 192, 3, 64), (256, 320, 8, 64),
])
def test_linear_mma_kernel(N, K, T, group):
    words, scales, x, ref = _case(N, K, T, group, seed=N + K + T)
    y = _run(words, scales, x, N, K, group)
    # exact codes, fp32 scale and accumulation: only summation order differs
    assert np.abs(y - ref).max() <= 1e-5 * np.abs(ref).max() + 1e-6


@pytest.mark.parametrize("N,K,T,group", [
    (128, 64, 64, 64), (256, 256, 100, 64), (768, 256, 128, 64), (2048, 2048, 128, 128),
    (6144, 2048, 128, 128), (2048, 8192, 128, 128), (16384, 2048, 128, 128),
    (1024, 2048, 256, 128), (512, 1024, 300, 128), (2048, 2048, 1024, 128),
    # 64 tokens (64-wide token tile: its activation ring is deeper than the
    # TMEM weight ring) over many k blocks
    (2048, 8192, 64, 128), (6144, 2048, 64, 128),
])
def test_linear_tc_kernel(N, K, T, group):
    words, scales, x, ref = _case(N, K, T, group, seed=N + K + T)
    y = _run(words, scales, x, N, K, group)
    assert np.isfinite(y).all()
    # weights enter the tensor cores as fp16(code * scale): relative error
    # below 2^-11 per weight, accumulated in fp32
    err = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert err <= 1e-3, err
    assert np.abs(y - ref).max() <= 5e-3 * np.abs(ref).max()


@pytest.mark.parametrize("N,K,T,group", [
    (64, 128, 1, 64), (128, 256, 8, 64), (2048, 2048, 1, 128), (6144, 2048, 3, 128),
    (16384, 2048, 8, 128), (2048, 8192, 5, 128), (768, 1024, 7, 64), (192, 384, 2, 128),
])
def test_linear_decode_projection_kernel(N, K, T, group):
    """Decode-sized calls (T <= 8, K % 128 == 0) run the decode projection
    kernel: no split-K, the sixteen warps of a CTA split K and add in warp order;
    exact codes with the group scale applied to fp32 sums (G = 64: one sum per
    group), so only the summation order differs from the exact product."""
    assert tl.tl_linear_workspace_bytes(N, K, T) == 0
    words, scales, x, ref = _case(N, K, T, group, seed=N + K + T + 7)
    y = _run(words, scales, x, N, K, group)
    assert np.abs(y - ref).max() <= 1e-5 * np.abs(ref).max() + 1e-6


def test_linear_decode_projection_rows_independent():
    """A token's result does not depend on the other tokens of the call."""
    N, K, group = 2048, 2048, 128
    words, scales, x, _ = _case(N, K, 8, group, seed=99)
    y8 = _run(words, scales, x, N, K, group)
    for t in (0, 3, 7):
        y1 = _run(words, scales, x[t:t + 1], N, K, group)
        assert np.array_equal(y1[0], y8[t])
