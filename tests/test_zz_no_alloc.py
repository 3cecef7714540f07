"""tl_linear_noalloc, the linear layer for callers that cannot allocate device
memory while they run (a process whose memory another allocator reserved up
front, work issued inside an open stream capture, fixed real-time budgets).
Its output must match tl_linear's, which takes a caller-allocated scratch
buffer, on two calls in a row through the same built-in buffer.  This file is
collected last so that a failure here never hides the other tests."""
import ctypes

import numpy as np
import pytest
import torch

import synthetic as syn
import weight_shared_looped_b200 as tl
from oracle import tinyloop_oracle as o

pytestmark = pytest.mark.gpu


def _inputs(N, K, T, group, tag):
    w = syn.normal((N, K), 0.02, 0, f"noalloc.w.{N}.{K}")
    codes, scales = o.quantize_groupwise(w, 4, group)
    words = torch.from_numpy(o.pack_codes(codes, 4).view(np.int32)).cuda()
    sc = torch.from_numpy(scales.view(np.int16)).cuda()
    x = torch.from_numpy(syn.normal((T, K), 1.0, 0, f"noalloc.x.{tag}").astype(np.float16)
                         .view(np.int16)).cuda()
    return words, sc, x


def _with_workspace(words, sc, x, N, K, group):
    T = x.shape[0]
    y = torch.empty(T, N, dtype=torch.float32, device="cuda")
    ws = torch.empty(max(tl.tl_linear_workspace_bytes(N, K, T), 1), dtype=torch.uint8,
                     device="cuda")
    tl.tl_linear(words, sc, N, K, group, x, y, ws)
    return y


# token counts whose kernels write split-K partial sums (decode-sized calls,
# T <= 8, need no scratch at all and are covered by the linear-layer tests)
@pytest.mark.parametrize("N,K,T,group", [(6144, 2048, 16, 128), (2048, 8192, 12, 128),
                                         (768, 1024, 24, 64), (1024, 2048, 40, 128)])
def test_noalloc_matches_workspace_version_twice(N, K, T, group):
    assert tl.tl_linear_workspace_bytes(N, K, T) > 0          # the split-K scratch is in use
    words, sc, _ = _inputs(N, K, T, group, "a")
    for call, tag in enumerate(("first", "second")):
        _, _, x = _inputs(N, K, T, group, f"{tag}.{N}")
        y_ref = _with_workspace(words, sc, x, N, K, group)
        y = torch.full((T, N), float("nan"), dtype=torch.float32, device="cuda")
        tl.tl_linear_noalloc(words, sc, N, K, group, x, y)
        torch.cuda.synchronize()
        a, b = y.cpu().numpy(), y_ref.cpu().numpy()
        assert np.isfinite(a).all(), call
        assert np.abs(a - b).max() <= 1e-5 * np.abs(b).max() + 1e-6, call


def test_noalloc_rejects_sizes_beyond_its_buffer():
    # 128 tokens of a 6144 x 2048 projection need more than 4 MiB of partials
    words, sc, x = _inputs(6144, 2048, 128, 128, "big")
    y = torch.empty(128, 6144, dtype=torch.float32, device="cuda")
    with pytest.raises(tl.TLError) as e:
        tl.tl_linear_noalloc(words, sc, 6144, 2048, 128, x, y)
    assert e.value.status == tl.TL_ERR_INVALID_ARG
    assert "scratch" in str(e.value)
