"""The INT8 KV codes the hot path itself writes -- the prefill cache append and
the decode cache append -- read back from the cache and compared bit for bit
with the oracle's quantisation of the same fp16 rows.

At layer 0 a token's K/V row depends only on that token's input: the layer's
input is the embedding (or the caller's hidden state), and its RMSNorm, QKV
projection and RoPE involve no cached entry.  So an FP16 cache and an INT8
cache filled from the same inputs see the same K/V values, and the FP16 cache
holds exactly the fp16 rows the INT8 path quantised.  The codes and scales in
the INT8 cache must then equal the oracle's per-(token, head) quantisation of
those rows ("Performance and Memory", "KV cache INT8": symmetric INT8, one FP16
scale per (token, head), scale = max|x| / 127)."""
import numpy as np
import pytest
import torch

import synthetic as syn
import weight_shared_looped_b200 as tl
from oracle import tinyloop_oracle as o

from gpu_util import device_model, to_dev

pytestmark = pytest.mark.gpu


def _raw(kv, ptr, shape, dtype):
    off = ptr - kv.buffer.data_ptr()
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    return kv.buffer[off:off + n].view(dtype).view(*shape)


def _layer0(kv, lane, H, hd, n):
    """K and V of layer 0 of one lane, positions 0..n-1: fp16 rows [n, H, hd]
    (FP16 cache) or (codes [n, H, hd], scales [n, H]) (INT8 cache)."""
    k, v, ks, vs = kv.layer_ptrs(lane, 0)
    out = []
    if ks is None or ks == 0:
        for p in (k, v):
            a = _raw(kv, p, (H, kv.max_ctx, hd), torch.int16)[:, :n]
            out.append(a.cpu().numpy().view(np.float16).transpose(1, 0, 2))
        return out
    for p, sp in ((k, ks), (v, vs)):
        c = _raw(kv, p, (H, kv.max_ctx, hd), torch.int8)[:, :n].cpu().numpy().transpose(1, 0, 2)
        s = _raw(kv, sp, (H, kv.max_ctx), torch.int16)[:, :n].cpu().numpy().view(np.float16).T
        out.append((c, s))
    return out


def _check_lane(kv16, kv8, lane, H, hd, n):
    k16, v16 = _layer0(kv16, lane, H, hd, n)
    (kc, ks), (vc, vs) = _layer0(kv8, lane, H, hd, n)
    for rows, codes, scales, name in ((k16, kc, ks, "K"), (v16, vc, vs, "V")):
        rc, rs = o.kv_quant_int8(rows)
        bad = np.argwhere(codes != rc)
        assert bad.size == 0, (name, lane, bad[:5])
        assert np.array_equal(scales.view(np.uint16), rs.view(np.uint16)), (name, lane)
    # the rows are not degenerate (every code zero would pass trivially)
    assert np.abs(kc).max() == 127 and np.abs(vc).max() == 127


def _fill(model, dtype, L_per_lane, prompts, steps, max_ctx, use_ids):
    kv = model.new_kv(L_per_lane, max_ctx=max_ctx, dtype=dtype)
    for b, p in enumerate(prompts):
        if use_ids:
            model.prefill(torch.from_numpy(p).cuda(), L=L_per_lane[b], kv=kv, lane=b)
        else:
            model.prefill(h_in=to_dev(p, torch.float16), L=L_per_lane[b], kv=kv, lane=b)
    for s in steps:
        if use_ids:
            model.decode(kv, torch.from_numpy(s).cuda(), L_per_lane=L_per_lane)
        else:
            model.decode(kv, h_in=to_dev(s, torch.float16), L_per_lane=L_per_lane)
    assert model.sync_status() == tl.TL_OK
    return kv


@pytest.mark.parametrize("graphs", [True, False])
def test_tiny_hot_path_int8_codes_bit_exact(graphs):
    """Tiny block (head_dim 64): a 37-token prefill (a ragged 64-key stage) and
    three decode steps on two lanes of different depth."""
    w = syn.WORKLOADS["tiny"]
    m = device_model("tiny", max_tokens=64, max_lanes=2, max_ctx=64)
    m.set_graphs(graphs)
    H, hd = w.shape.n_heads, w.shape.head_dim
    P, S, Ls = 37, 3, [2, 1]
    prompts = [syn.hidden_input(w, P, name=f"kvcodes.prompt{b}") for b in range(2)]
    steps = [np.stack([syn.hidden_input(w, 1, name=f"kvcodes.step{s}.{b}")[0] for b in range(2)])
             for s in range(S)]
    kv16 = _fill(m, "fp16", Ls, prompts, steps, 64, False)
    kv8 = _fill(m, "int8", Ls, prompts, steps, 64, False)
    for lane in range(2):
        _check_lane(kv16, kv8, lane, H, hd, P + S)
    kv16.close()
    kv8.close()
    m.close()


def test_407m_hot_path_int8_codes_bit_exact():
    """407M-shaped model (head_dim 128): a 128-token prefill through the
    tensor-core GEMM and the RoPE/KV kernel, then two decode steps through the
    decode GEMV and the fused decode attention append."""
    w = syn.WORKLOADS["prefill407m"]
    m = device_model("prefill407m", max_tokens=128, max_lanes=2, max_ctx=160)
    H, hd = w.shape.n_heads, w.shape.head_dim
    P, S, Ls = 128, 2, [2, 1]
    prompts = [syn.token_ids(P, w.seed, f"kvcodes.prompt{b}") for b in range(2)]
    steps = [syn.token_ids(2, w.seed, f"kvcodes.step{s}") for s in range(S)]
    kv16 = _fill(m, "fp16", Ls, prompts, steps, 160, True)
    kv8 = _fill(m, "int8", Ls, prompts, steps, 160, True)
    for lane in range(2):
        _check_lane(kv16, kv8, lane, H, hd, P + S)
    kv16.close()
    kv8.close()
    m.close()
