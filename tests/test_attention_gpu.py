"""Parity of the prefill attention kernel, called on its own through the C ABI
(tl_attention_prefill), against the oracle's causal softmax attention in fp64
on the same fp16 inputs.

Tolerance from the arithmetic: scores, maxima, exponentials and sums are fp32;
two values are rounded to fp16 on the way (the softmax weights entering the
P.V product, and the output), each by at most 2^-11 relative.  An emulation of
exactly those two roundings gives a relative L2 error of about 2.5e-4 and a
largest error of about 4e-4 of max|out| on these inputs; the bounds below
leave a margin of about eight.  Where the result is exact (one key: the
output is that key's value row) the comparison is bit for bit."""
import numpy as np
import pytest
import torch

import synthetic as syn
import weight_shared_looped_b200 as tl
from oracle import tinyloop_oracle as o

from gpu_util import rel_l2

pytestmark = pytest.mark.gpu

REL_L2 = 2e-3
MAX_REL = 4e-3


def _qkv(T, H, hd, seed, q_std=1.0):
    q = syn.normal((T, H, hd), q_std, seed, "attn.q").astype(np.float16)
    k = syn.normal((T, H, hd), 1.0, seed, "attn.k").astype(np.float16)
    v = syn.normal((T, H, hd), 1.0, seed, "attn.v").astype(np.float16)
    return q, k, v


def _run(q, k, v):
    T, H, hd = q.shape
    dq, dk, dv = (torch.from_numpy(a.reshape(T, H * hd)).cuda() for a in (q, k, v))
    out = torch.full((T, H * hd), float("nan"), dtype=torch.float16, device="cuda")
    tl.tl_attention_prefill(dq, dk, dv, H, hd, out)
    torch.cuda.synchronize()
    return out.cpu().numpy().reshape(T, H, hd)


def _check(y, ref):
    y = y.astype(np.float64)
    assert np.isfinite(y).all()
    assert rel_l2(y, ref) <= REL_L2
    assert np.abs(y - ref).max() <= MAX_REL * np.abs(ref).max()


@pytest.mark.parametrize("T,H,hd,q_std", [
    (2, 2, 64, 1.0), (17, 4, 64, 1.0), (64, 4, 64, 1.0), (65, 2, 128, 1.0),
    (128, 16, 128, 1.0),            # the 407M-shaped model's prefill at 128 tokens
    (130, 16, 128, 1.0), (300, 2, 128, 4.0), (1000, 2, 64, 8.0), (1024, 2, 128, 1.0),
])
def test_attention_prefill_matches_oracle(T, H, hd, q_std):
    """Several query and key tiles (64 each) with ragged tails; q_std > 1 makes
    the softmax peaked, so the running maximum changes between key tiles."""
    q, k, v = _qkv(T, H, hd, seed=T * 31 + H * 7 + hd, q_std=q_std)
    y = _run(q, k, v)
    ref = o.causal_attention(q.astype(np.float64), k.astype(np.float64), v.astype(np.float64),
                             np.arange(T))
    _check(y, ref)


@pytest.mark.parametrize("hd", [64, 128])
def test_one_key_returns_its_value_row_exactly(hd):
    q, k, v = _qkv(1, 3, hd, seed=5)
    y = _run(q, k, v)
    assert np.array_equal(y, v)


def test_identical_keys_give_running_means():
    """With every key equal, each query weighs keys 0..t equally: out[t] is the
    mean of v[0..t] (a closed form independent of q)."""
    T, H, hd = 1000, 2, 128
    q, _, v = _qkv(T, H, hd, seed=11)
    k = np.broadcast_to(syn.normal((1, H, hd), 1.0, 11, "attn.k1").astype(np.float16),
                        (T, H, hd)).copy()
    y = _run(q, k, v)
    ref = np.cumsum(v.astype(np.float64), axis=0) / np.arange(1, T + 1)[:, None, None]
    _check(y, ref)


def test_largest_prefill_sampled_rows():
    """T = 8192 (the largest prefill a model takes), 16 heads of 128: the
    oracle computes sampled query rows one by one, first and last included."""
    T, H, hd = 8192, 16, 128
    q, k, v = _qkv(T, H, hd, seed=8192)
    y = _run(q, k, v)
    rows = np.array([0, 1, 63, 64, 65, 1000, 4095, 4096, 6000, 8127, 8128, 8190, 8191])
    ref = o.causal_attention(q[rows].astype(np.float64), k.astype(np.float64),
                             v.astype(np.float64), rows)
    _check(y[rows], ref)


def test_empty_prefill_is_a_no_op():
    out = torch.zeros((0, 128), dtype=torch.float16, device="cuda")
    tl.tl_attention_prefill(out, out, out, 2, 64, out)
    torch.cuda.synchronize()
