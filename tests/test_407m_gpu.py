"""Full-size parity on the 407M-shaped model (d 2048, 16 heads x 128, ffn 8192,
INT4 group 128, 2 pre-blocks + 1 loop block), in the launch configuration the
benchmark times (CUDA graphs on):

  * prefill, seq 128, L=8: every block output and the final hidden state
    against the oracle;
  * KV-cached decode: 256-token prompt + 128 teacher-forced steps, FP16 KV;
    every step against the oracle's uncached 384-token forward (causality makes
    position t of the uncached forward the cached step's reference);
  * long-context INT8 KV, batch 8, context 2048, 64 steps: oracle-derived
    caches, sampled steps against the oracle, a lane bit-exact with itself;
  * mixed-depth INT3 loop block, lanes L=[4, 16, 32], context 1024, 32 steps:
    each lane bit-exact with its own single-lane run; sampled oracle check at a
    shorter context.
"""
import numpy as np
import pytest
import torch

import synthetic as syn
import weight_shared_looped_b200 as tl
from oracle import tinyloop_oracle as o

from gpu_util import (BLOCK_REL_L2, FINAL_COSINE, cosine, device_blocks, device_model,
                      oracle_model, rel_l2, row_cosines, to_dev)

pytestmark = pytest.mark.gpu


def _ids(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).cuda()


@pytest.fixture(scope="module")
def m407():
    m = device_model("prefill407m", max_tokens=384, max_lanes=8, max_ctx=2048 + 64)
    yield m
    m.close()


def test_prefill_407m_matches_oracle(m407):
    w = syn.WORKLOADS["prefill407m"]
    L, seq = w.L[0], w.seq
    ids = syn.prompt_ids(w)
    trace = torch.empty(w.n_pre + L, seq, w.shape.d_model, dtype=torch.float32, device="cuda")
    y = m407.prefill(_ids(ids), L=L, h_trace=trace)
    assert m407.sync_status() == tl.TL_OK
    rtr = []
    ry = oracle_model("prefill407m").prefill(ids, L, trace=rtr)
    tr = trace.cpu().numpy()
    errs = [rel_l2(tr[i], rtr[i]) for i in range(len(rtr))]
    assert max(errs) <= BLOCK_REL_L2, errs
    yc = y.cpu().numpy()
    assert cosine(yc, ry) >= FINAL_COSINE
    assert row_cosines(yc, ry).min() >= FINAL_COSINE


def test_cached_decode_407m_matches_uncached(m407):
    w = syn.WORKLOADS["decode407m"]
    L = w.L[0]
    prompt, steps = syn.prompt_ids(w), syn.decode_ids(w)
    full = np.concatenate([prompt, steps])
    kv = m407.new_kv([L], max_ctx=w.max_ctx, dtype="fp16")
    m407.prefill(_ids(prompt), L=L, kv=kv, lane=0)
    ys = []
    for t in range(w.steps):
        ys.append(m407.decode(kv, _ids(steps[t:t + 1]), L_per_lane=[L]).clone())
    assert m407.sync_status() == tl.TL_OK
    y = torch.cat(ys).cpu().numpy()                      # [128, d]
    yu = m407.prefill(_ids(full), L=L).cpu().numpy()     # GPU uncached, [384, d]
    ry = oracle_model("prefill407m").prefill(full, L)    # oracle uncached
    cu = row_cosines(y, yu[w.seq:])
    co = row_cosines(y, ry[w.seq:])
    assert cu.min() >= FINAL_COSINE, cu.min()
    assert co.min() >= FINAL_COSINE, co.min()
    assert rel_l2(y, ry[w.seq:]) <= 2 * BLOCK_REL_L2
    kv.close()


def test_cached_decode_407m_per_block_traces(m407):
    """Every block output of the first decode steps after a 256-token prompt
    (FP16 KV) against the oracle's cached decode of the same prompt, at the
    per-block tolerance; both sides run free from the same ids."""
    w = syn.WORKLOADS["decode407m"]
    L, n_layers, S = w.L[0], w.n_pre + w.L[0], 3
    prompt, steps = syn.prompt_ids(w), syn.decode_ids(w)
    kv = m407.new_kv([L], max_ctx=w.max_ctx, dtype="fp16")
    m407.prefill(_ids(prompt), L=L, kv=kv, lane=0)
    om = oracle_model("prefill407m")
    okv = om.new_kv(L, "fp16")
    om.prefill(prompt, L, kv=okv)
    for s in range(S):
        tr = torch.empty(n_layers, 1, w.shape.d_model, dtype=torch.float32, device="cuda")
        y = m407.decode(kv, _ids(steps[s:s + 1]), L_per_lane=[L], h_trace=tr)
        assert m407.sync_status() == tl.TL_OK
        rtr = []
        ry = om.decode_step(np.int64(steps[s]), L, okv, trace=rtr)
        trc = tr.cpu().numpy()
        errs = [rel_l2(trc[i, 0], rtr[i][0]) for i in range(n_layers)]
        assert max(errs) <= BLOCK_REL_L2, (s, errs)
        assert cosine(y[0].cpu().numpy(), ry) >= FINAL_COSINE, s
    kv.close()


def _raw_view(kv, ptr, shape, dtype):
    """A torch view of one region of the caller-owned KV buffer."""
    off = ptr - kv.buffer.data_ptr()
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    return kv.buffer[off:off + n].view(dtype).view(*shape)


def _load_int8_context(kv, lane, ctx_codes):
    """Upload oracle-derived INT8 K/V codes [ctx, H, hd] and scales [ctx, H]
    for every layer of one lane into the device layout [H][max_ctx][hd]."""
    for layer, (kc, ks, vc, vs) in enumerate(ctx_codes):
        kp, vp, ksp, vsp = kv.layer_ptrs(lane, layer)
        T, H, hd = kc.shape
        for ptr, arr in ((kp, kc), (vp, vc)):
            src = torch.from_numpy(np.ascontiguousarray(arr.transpose(1, 0, 2))).cuda()
            _raw_view(kv, ptr, (H, kv.max_ctx, hd), torch.int8)[:, :T].copy_(src)
        for ptr, arr in ((ksp, ks), (vsp, vs)):
            src = torch.from_numpy(np.ascontiguousarray(arr.T).view(np.int16)).cuda()
            _raw_view(kv, ptr, (H, kv.max_ctx), torch.int16)[:, :T].copy_(src)
    kv.set_position(lane, ctx_codes[0][0].shape[0])


def test_long_context_int8_decode(m407):
    w = syn.WORKLOADS["longctx_int8"]
    om = oracle_model("prefill407m")            # same model, INT4 everywhere
    L = w.L[0]
    n_lanes = len(w.L)
    derived_lanes = (0, 3, 7)
    blocks = om.schedule(L)
    ctx = {}
    for lane in derived_lanes:
        ctx[lane] = [o.derive_context_kv(blocks[layer], syn.context_hidden(w, layer, lane))
                     for layer in range(len(blocks))]
    lane_src = [lane if lane in derived_lanes else 0 for lane in range(n_lanes)]
    kv = m407.new_kv(list(w.L), max_ctx=w.max_ctx, dtype="int8")
    for lane in range(n_lanes):
        _load_int8_context(kv, lane, ctx[lane_src[lane]])
    ids = np.stack([syn.decode_ids(w, lane) for lane in range(n_lanes)], axis=1)   # [steps, 8]
    ys = [m407.decode(kv, _ids(ids[s]), L_per_lane=list(w.L)).clone() for s in range(w.steps)]
    assert m407.sync_status() == tl.TL_OK
    y = torch.stack(ys).cpu().numpy()                    # [64, 8, d]
    assert np.isfinite(y).all()
    # the same lane alone, from the same cache content, bit for bit
    kv1 = m407.new_kv([L], max_ctx=w.max_ctx, dtype="int8")
    _load_int8_context(kv1, 0, ctx[3])
    y1 = torch.stack([m407.decode(kv1, _ids(ids[s, 3:4]), L_per_lane=[L]).clone()
                      for s in range(w.steps)]).cpu().numpy()
    assert np.array_equal(y1[:, 0], y[:, 3])
    # sampled steps of the derived lanes against the oracle
    for lane in derived_lanes:
        okv = om.new_kv(L, "int8")
        for layer, (kc, ks, vc, vs) in enumerate(ctx[lane]):
            okv[layer].load_stored(o.kv_dequant_int8(kc, ks), o.kv_dequant_int8(vc, vs))
        for s in range(4):
            r = om.decode_step(np.int64(ids[s, lane]), L, okv)
            assert cosine(y[s, lane], r) >= FINAL_COSINE, (lane, s)
            assert rel_l2(y[s, lane], r) <= 2 * BLOCK_REL_L2, (lane, s)
    kv.close()
    kv1.close()


@pytest.fixture(scope="module")
def m_int3():
    m = device_model("mixed_int3", max_tokens=1024, max_lanes=3, max_ctx=1024 + 32)
    yield m
    m.close()


def _mixed_run(model, L_per_lane, prompts, steps_ids, max_ctx):
    kv = model.new_kv(L_per_lane, max_ctx=max_ctx)
    for b, p in enumerate(prompts):
        model.prefill(_ids(p), L=L_per_lane[b], kv=kv, lane=b)
    ys = [model.decode(kv, _ids(steps_ids[s]), L_per_lane=L_per_lane).clone()
          for s in range(steps_ids.shape[0])]
    assert model.sync_status() == tl.TL_OK
    kv.close()
    return torch.stack(ys).cpu().numpy()


def test_mixed_depth_int3_lanes_bit_exact(m_int3):
    w = syn.WORKLOADS["mixed_int3"]
    Ls = list(w.L)
    prompts = [syn.prompt_ids(w, b) for b in range(3)]
    ids = np.stack([syn.decode_ids(w, b) for b in range(3)], axis=1)     # [32, 3]
    y = _mixed_run(m_int3, Ls, prompts, ids, w.max_ctx)
    assert np.isfinite(y).all()
    for b in range(3):
        y1 = _mixed_run(m_int3, [Ls[b]], [prompts[b]], ids[:, b:b + 1], w.max_ctx)
        assert np.array_equal(y1[:, 0], y[:, b]), b
    # depth changes the result
    assert not np.allclose(y[:, 0], y[:, 1])


def test_mixed_depth_int3_matches_oracle_short_context(m_int3):
    w = syn.WORKLOADS["mixed_int3"]
    Ls = list(w.L)
    P, S = 48, 2
    prompts = [syn.prompt_ids(w, b)[:P] for b in range(3)]
    ids = np.stack([syn.decode_ids(w, b)[:S] for b in range(3)], axis=1)
    y = _mixed_run(m_int3, Ls, prompts, ids, P + S)
    om = oracle_model("mixed_int3")
    for b, L in enumerate(Ls):
        kv = om.new_kv(L, "fp16")
        om.prefill(prompts[b], L, kv=kv)
        for s in range(S):
            r = om.decode_step(np.int64(ids[s, b]), L, kv)
            assert cosine(y[s, b], r) >= FINAL_COSINE, (b, s)
            assert rel_l2(y[s, b], r) <= 2 * BLOCK_REL_L2, (b, s)
