"""Self-speculative decode on the GPU ("Current Status", speculative and
adaptive decode table, self-speculative row: L=2 draft, L=8 verify, same
weights; "TinyLoop Framework", "What Makes It Different": draft and verify
reuse the same weights and cache).

* tl_extend (the verify pass: n tokens of one lane at its position) is
  bit-identical to n successive one-token steps, cache contents included, and
  matches the oracle's extend per block;
* the greedy head (tied embedding) picks the oracle's token;
* tl_spec_step emits exactly the tokens plain greedy decoding at the verify
  depth emits (the defining property of speculative decoding with an exact
  verify), accepts every draft when the draft depth is the verify depth, and
  matches the oracle's greedy tokens."""
import numpy as np
import pytest
import torch

import synthetic as syn
import weight_shared_looped_b200 as tl
from oracle import tinyloop_oracle as o
from oracle.workloads import packed_weights
from weight_shared_looped_b200.model import DeviceModel

from gpu_util import (BLOCK_REL_L2, FINAL_COSINE, cosine, device_blocks, device_model,
                      oracle_model, rel_l2, to_dev)

pytestmark = pytest.mark.gpu
W = syn.WORKLOADS["tiny"]
VOCAB_TINY = 1000


def _ids(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).cuda()


def _raw(kv, ptr, nbytes):
    off = ptr - kv.buffer.data_ptr()
    return kv.buffer[off:off + nbytes]


def _cache_bytes(kv, lane, layers, n_pos, int8):
    """The written positions 0..n_pos-1 of every head of a lane's K and V (and
    INT8 scales), layer by layer."""
    H, hd = W.shape.n_heads, W.shape.head_dim
    esz = 1 if int8 else 2
    out = []
    for layer in range(layers):
        k, v, ks, vs = kv.layer_ptrs(lane, layer)
        parts = []
        for ptr in (k, v):
            a = _raw(kv, ptr, H * kv.max_ctx * hd * esz).view(H, kv.max_ctx, hd * esz)
            parts.append(a[:, :n_pos].reshape(-1))
        if int8:
            for ptr in (ks, vs):
                a = _raw(kv, ptr, H * kv.max_ctx * 2).view(H, kv.max_ctx, 2)
                parts.append(a[:, :n_pos].reshape(-1))
        out.append(torch.cat(parts).cpu().numpy())
    return out


@pytest.fixture(scope="module")
def tiny_blocks():
    return device_blocks("tiny")


@pytest.fixture(scope="module")
def tiny_emb_model(tiny_blocks):
    """The tiny loop block with an fp16 N(0, 0.02) embedding (and tied head)."""
    emb = syn.normal((VOCAB_TINY, W.shape.d_model), 0.02, W.seed, "tiny.embed").astype(np.float16)
    m = DeviceModel([], tiny_blocks["loop"], syn.final_gain(W.shape, W.seed), emb,
                    max_tokens=64, max_lanes=8, max_ctx=160, max_L=8)
    m._emb = emb
    yield m
    m.close()


def _oracle_emb_model(emb):
    blk = o.Block(packed_weights("tiny")["loop"], o.block_cfg(W.shape, 4, W.group, W.eps, W.rope_theta))
    return o.LoopedModel([], blk, syn.final_gain(W.shape, W.seed), emb)


@pytest.mark.parametrize("dtype", ["fp16", "int8"])
@pytest.mark.parametrize("n", [1, 3, 8])
def test_extend_is_bit_exact_with_one_token_steps(tiny_emb_model, dtype, n):
    m, L, P = tiny_emb_model, 3, 21
    prompt = syn.token_ids(P + n, W.seed, "ext.prompt", VOCAB_TINY)
    kvs = []
    for _ in range(2):
        kv = m.new_kv([2, L], max_ctx=P + n + 1, dtype=dtype)
        m.prefill(_ids(prompt[:P]), L=L, kv=kv, lane=1)
        kvs.append(kv)
    ya = m.extend(kvs[0], _ids(prompt[P:]), lane=1, L=L)
    yb = torch.cat([m.extend(kvs[1], _ids(prompt[P + i:P + i + 1]), lane=1, L=L)
                    for i in range(n)])
    assert m.sync_status() == tl.TL_OK
    assert torch.equal(ya, yb)
    assert kvs[0].position(1) == kvs[1].position(1) == P + n
    for a, b in zip(_cache_bytes(kvs[0], 1, L, P + n, dtype == "int8"),
                    _cache_bytes(kvs[1], 1, L, P + n, dtype == "int8")):
        assert np.array_equal(a, b)
    for kv in kvs:
        kv.close()


def test_one_token_extend_is_the_decode_step(tiny_emb_model):
    m, L, P = tiny_emb_model, 2, 9
    prompt = syn.token_ids(P + 4, W.seed, "ext.dec", VOCAB_TINY)
    kva, kvb = m.new_kv([L], max_ctx=P + 4), m.new_kv([L], max_ctx=P + 4)
    for kv in (kva, kvb):
        m.prefill(_ids(prompt[:P]), L=L, kv=kv)
    for i in range(4):
        t = _ids(prompt[P + i:P + i + 1])
        assert torch.equal(m.extend(kva, t, L=L), m.decode(kvb, t, L_per_lane=[L]))
    kva.close()
    kvb.close()


def test_extend_matches_oracle_per_block(tiny_emb_model):
    m, L, P, n = tiny_emb_model, 3, 17, 5
    ids = syn.token_ids(P + n, W.seed, "ext.oracle", VOCAB_TINY)
    kv = m.new_kv([L], max_ctx=P + n)
    m.prefill(_ids(ids[:P]), L=L, kv=kv)
    tr = torch.empty(L, n, W.shape.d_model, dtype=torch.float32, device="cuda")
    y = m.extend(kv, _ids(ids[P:]), L=L, h_trace=tr).cpu().numpy()
    om = _oracle_emb_model(m._emb)
    okv = om.new_kv(L, "fp16")
    om.prefill(ids[:P], L, kv=okv)
    rtr = []
    ry = om.extend(ids[P:], L, okv, trace=rtr)
    trc = tr.cpu().numpy()
    for layer in range(L):
        assert rel_l2(trc[layer], rtr[layer]) <= BLOCK_REL_L2, layer
    for i in range(n):
        assert cosine(y[i], ry[i]) >= FINAL_COSINE
    kv.close()


def test_greedy_head_matches_oracle(tiny_emb_model):
    m = tiny_emb_model
    om = _oracle_emb_model(m._emb)
    y = syn.normal((8, W.shape.d_model), 1.0, W.seed, "head.y")
    got = m.greedy_head(torch.from_numpy(y).cuda()).cpu().numpy()
    want = om.greedy_head(y.astype(np.float64))
    logits = y.astype(np.float64) @ m._emb.astype(np.float64).T
    for r in range(8):
        if got[r] != want[r]:
            # the only admissible difference: a near-tie inside fp32 rounding
            assert logits[r, got[r]] >= logits[r, want[r]] - 1e-4 * np.abs(logits[r]).max(), r


def test_greedy_head_rejects_bad_calls(tiny_blocks):
    m = DeviceModel([], tiny_blocks["loop"], syn.final_gain(W.shape, W.seed), max_tokens=8)
    y = torch.zeros(2, W.shape.d_model, device="cuda")
    with pytest.raises(tl.TLError) as e:                         # no embedding to use as a head
        m.greedy_head(y)
    assert e.value.status == tl.TL_ERR_INVALID_ARG
    m.close()


def _greedy_by_steps(m, kv, token, n, L):
    out = []
    for _ in range(n):
        y = m.extend(kv, _ids([token]), L=L)
        token = int(m.greedy_head(y).item())
        out.append(token)
    return out


@pytest.mark.parametrize("K,L_draft", [(1, 1), (3, 1), (4, 2), (7, 1)])
def test_spec_step_emits_greedy_decode_tokens(tiny_emb_model, K, L_draft):
    m, L, P = tiny_emb_model, 3, 12
    prompt = syn.token_ids(P, W.seed, "spec.prompt", VOCAB_TINY)
    kv_s, kv_g = m.new_kv([L], max_ctx=80), m.new_kv([L], max_ctx=80)
    for kv in (kv_s, kv_g):
        m.prefill(_ids(prompt[:-1]), L=L, kv=kv)
    tok, got, steps = int(prompt[-1]), [], 0
    while len(got) < 24:
        out = m.spec_step(kv_s, tok, K=K, L_draft=L_draft, L_verify=L)
        assert 1 <= len(out) <= K + 1
        got += out
        tok = out[-1]
        steps += 1
        assert kv_s.position(0) == P - 1 + len(got)
    want = _greedy_by_steps(m, kv_g, int(prompt[-1]), len(got), L)
    assert got == want
    assert m.sync_status() == tl.TL_OK
    kv_s.close()
    kv_g.close()


def test_spec_step_accepts_every_draft_at_the_verify_depth(tiny_emb_model):
    m, L, K = tiny_emb_model, 2, 5
    kv = m.new_kv([L], max_ctx=64)
    m.prefill(_ids(syn.token_ids(10, W.seed, "spec.full", VOCAB_TINY)), L=L, kv=kv)
    tok = 7
    for _ in range(4):
        out = m.spec_step(kv, tok, K=K, L_draft=L, L_verify=L)
        assert len(out) == K + 1
        tok = out[-1]
    kv.close()


def test_spec_tokens_match_oracle_greedy(tiny_emb_model):
    m, L, P = tiny_emb_model, 2, 8
    prompt = syn.token_ids(P, W.seed, "spec.oracle", VOCAB_TINY)
    kv = m.new_kv([L], max_ctx=64)
    m.prefill(_ids(prompt[:-1]), L=L, kv=kv)
    tok, got = int(prompt[-1]), []
    while len(got) < 8:
        out = m.spec_step(kv, tok, K=3, L_draft=1, L_verify=L)
        got += out
        tok = out[-1]
    om = _oracle_emb_model(m._emb)
    okv = om.new_kv(L, "fp16")
    om.prefill(prompt[:-1], L, kv=okv)
    want = om.greedy_decode(int(prompt[-1]), len(got), L, okv)
    assert got[:8] == want[:8]
    kv.close()


def test_extend_and_spec_reject_bad_calls(tiny_emb_model):
    m = tiny_emb_model
    kv = m.new_kv([2], max_ctx=12)
    m.prefill(_ids([1, 2, 3, 4, 5, 6, 7, 8, 9, 10]), L=2, kv=kv)
    for kw in (dict(L=3), dict(L=0)):
        with pytest.raises(tl.TLError):
            m.extend(kv, _ids([1]), **kw)
    with pytest.raises(tl.TLError):                            # 10 + 3 > 12 positions
        m.extend(kv, _ids([1, 2, 3]), L=2)
    with pytest.raises(tl.TLError):                            # more than 8 tokens
        m.extend(kv, _ids(list(range(9))), L=2)
    with pytest.raises(tl.TLError):                            # K + 1 positions do not fit
        m.spec_step(kv, 1, K=3, L_draft=1, L_verify=2)
    with pytest.raises(tl.TLError):
        m.spec_step(kv, VOCAB_TINY, K=1, L_draft=1, L_verify=2)   # token outside the vocabulary
    assert kv.position(0) == 10
    kv.close()
