"""Looped forward on the GPU against the oracle, tiny FP32-checkable block
(d 256, 4 heads x 64, ffn 768, group 64, 0 pre-blocks + loop L=2, seq 16), plus
the invariants the pages fix: L copies = L iterations, weight memory
independent of L, cached = uncached, per-lane L bit-exact."""
import numpy as np
import pytest
import torch

import synthetic as syn
import weight_shared_looped_b200 as tl
from oracle import tinyloop_oracle as o
from weight_shared_looped_b200.model import DeviceBlock, DeviceModel

from gpu_util import (BLOCK_REL_L2, FINAL_COSINE, block_cfg, cosine, device_blocks, device_model,
                      oracle_model, rel_l2, row_cosines, to_dev)

pytestmark = pytest.mark.gpu
W = syn.WORKLOADS["tiny"]


@pytest.fixture(scope="module")
def blocks():
    return device_blocks("tiny")


@pytest.fixture(scope="module")
def model(blocks):
    m = device_model("tiny", max_tokens=64, max_lanes=8, max_ctx=128, blocks=blocks)
    yield m
    m.close()


def _oracle_trace(x, L, kv=None):
    trace = []
    y = oracle_model("tiny").prefill(np.asarray(x, np.float64), L, kv=kv, trace=trace)
    return y, trace


@pytest.mark.parametrize("seq", [16, 1, 37, 64])
@pytest.mark.parametrize("graphs", [True, False])
def test_tiny_prefill_matches_oracle(model, seq, graphs):
    model.set_graphs(graphs)
    L = W.L[0]
    x = syn.hidden_input(W, seq, name=f"h_in.{seq}")
    trace = torch.empty(L, seq, W.shape.d_model, dtype=torch.float32, device="cuda")
    y = model.prefill(h_in=to_dev(x, torch.float16), L=L, h_trace=trace)
    assert model.sync_status() == tl.TL_OK
    ry, rtrace = _oracle_trace(x.astype(np.float32), L)
    tr = trace.cpu().numpy()
    for layer in range(L):
        assert rel_l2(tr[layer], rtrace[layer]) <= BLOCK_REL_L2, layer
    assert cosine(y.cpu().numpy(), ry) >= FINAL_COSINE
    assert row_cosines(y.cpu().numpy(), ry).min() >= FINAL_COSINE
    model.set_graphs(True)


def test_graph_replay_is_deterministic(model):
    x = to_dev(syn.hidden_input(W), torch.float16)
    a = model.prefill(h_in=x, L=2).clone()
    b = model.prefill(h_in=x, L=2).clone()
    model.set_graphs(False)
    c = model.prefill(h_in=x, L=2).clone()
    model.set_graphs(True)
    assert torch.equal(a, b) and torch.equal(a, c)


def test_L_copies_equal_L_iterations(blocks):
    """L distinct copies of the block, applied as a plain deep stack, give the
    bit-identical result of the looped block applied L times."""
    L = 3
    loop = blocks["loop"]
    copies = []
    for _ in range(L):
        packed = {k: v.cpu().numpy() for k, v in loop.t.items()}
        packed = {k: (v.view(np.uint32) if k.startswith("w_") else
                      v.view(np.float16) if k.startswith("s_") else v) for k, v in packed.items()}
        copies.append(DeviceBlock(loop.cfg, packed=packed))
    x = to_dev(syn.hidden_input(W), torch.float16)
    looped = DeviceModel([], loop, syn.final_gain(W.shape, W.seed), max_tokens=16, max_L=L)
    deep = DeviceModel(copies[:-1], copies[-1], syn.final_gain(W.shape, W.seed), max_tokens=16,
                       max_L=1)
    a = looped.prefill(h_in=x, L=L)
    b = deep.prefill(h_in=x, L=1)
    assert torch.equal(a, b)
    for m in (looped, deep):
        m.close()
    for c in copies:
        c.close()


def test_weight_memory_independent_of_L(blocks):
    sizes = []
    for max_L in (1, 8, 64):
        m = DeviceModel([], blocks["loop"], syn.final_gain(W.shape, W.seed), max_tokens=16,
                        max_L=max_L)
        sizes.append(m.device_bytes())
        free0 = torch.cuda.mem_get_info()[0]
        x = to_dev(syn.hidden_input(W), torch.float16)
        for L in (1, max_L):
            m.prefill(h_in=x, L=L)
        torch.cuda.synchronize()
        m.close()
    assert sizes[0] == sizes[1] == sizes[2]


def _decode_run(model, L_per_lane, prompt_len, steps, dtype="fp16", lanes_inputs=None):
    """Prefill each lane with its own prompt, then decode `steps` steps.
    Returns y [steps, n_lanes, d]."""
    n = len(L_per_lane)
    kv = model.new_kv(L_per_lane, max_ctx=prompt_len + steps, dtype=dtype)
    for b in range(n):
        x = syn.hidden_input(W, prompt_len, name=f"prompt.{lanes_inputs[b]}")
        model.prefill(h_in=to_dev(x, torch.float16), L=L_per_lane[b], kv=kv, lane=b)
    ys = []
    for s in range(steps):
        hs = np.stack([syn.hidden_input(W, 1, name=f"step{s}.{lanes_inputs[b]}")[0]
                       for b in range(n)])
        ys.append(model.decode(kv, h_in=to_dev(hs, torch.float16), L_per_lane=L_per_lane).clone())
    assert model.sync_status() == tl.TL_OK
    for b in range(n):
        assert kv.position(b) == prompt_len + steps
    kv.close()
    return torch.stack(ys).cpu().numpy()


@pytest.mark.parametrize("dtype", ["fp16", "int8"])
def test_cached_decode_matches_uncached_and_oracle(model, dtype):
    P, S, L = 10, 6, 2
    y = _decode_run(model, [L], P, S, dtype, lanes_inputs=["c"])[:, 0]
    full = np.concatenate([syn.hidden_input(W, P, name="prompt.c")] +
                          [syn.hidden_input(W, 1, name=f"step{s}.c") for s in range(S)])
    # GPU uncached forward over all P + S tokens
    yu = model.prefill(h_in=to_dev(full, torch.float16), L=L).cpu().numpy()
    # oracle: uncached, and cached with the same storage dtype
    om = oracle_model("tiny")
    ry = om.prefill(full.astype(np.float64), L)
    kv = om.new_kv(L, dtype)
    om.prefill(full[:P].astype(np.float64), L, kv=kv)
    rc = np.stack([om.decode_step(full[P + s].astype(np.float64), L, kv) for s in range(S)])
    for s in range(S):
        assert cosine(y[s], yu[P + s]) >= FINAL_COSINE
        assert cosine(y[s], ry[P + s]) >= FINAL_COSINE
        assert cosine(y[s], rc[s]) >= FINAL_COSINE
        assert rel_l2(y[s], rc[s]) <= 2 * BLOCK_REL_L2


def test_decode_trace_matches_oracle(model):
    P, L = 12, 2
    kv = model.new_kv([L], max_ctx=P + 1)
    x = syn.hidden_input(W, P + 1, name="trace.dec")
    model.prefill(h_in=to_dev(x[:P], torch.float16), L=L, kv=kv, lane=0)
    tr = torch.empty(L, 1, W.shape.d_model, dtype=torch.float32, device="cuda")
    y = model.decode(kv, h_in=to_dev(x[P:], torch.float16), L_per_lane=[L], h_trace=tr)
    om = oracle_model("tiny")
    okv = om.new_kv(L, "fp16")
    om.prefill(x[:P].astype(np.float64), L, kv=okv)
    rtr = []
    ry = om.decode_step(x[P].astype(np.float64), L, okv, trace=rtr)
    for layer in range(L):
        assert rel_l2(tr[layer, 0].cpu().numpy(), rtr[layer][0]) <= BLOCK_REL_L2
    assert cosine(y[0].cpu().numpy(), ry) >= FINAL_COSINE
    kv.close()


def test_per_lane_L_bit_exact_with_single_lane_runs(model):
    L_per_lane = [1, 3, 2, 3]
    names = ["a", "b", "c", "d"]
    batched = _decode_run(model, L_per_lane, 9, 4, lanes_inputs=names)
    for b in range(4):
        single = _decode_run(model, [L_per_lane[b]], 9, 4, lanes_inputs=[names[b]])
        assert np.array_equal(batched[:, b], single[:, 0]), b


def test_decode_lanes_match_oracle(model):
    L_per_lane = [2, 1, 3]
    names = ["p", "q", "r"]
    P, S = 7, 3
    y = _decode_run(model, L_per_lane, P, S, lanes_inputs=names)
    om = oracle_model("tiny")
    for b, L in enumerate(L_per_lane):
        kv = om.new_kv(L, "fp16")
        om.prefill(syn.hidden_input(W, P, name=f"prompt.{names[b]}").astype(np.float64), L, kv=kv)
        for s in range(S):
            r = om.decode_step(syn.hidden_input(W, 1, name=f"step{s}.{names[b]}")[0].astype(np.float64),
                               L, kv)
            assert cosine(y[s, b], r) >= FINAL_COSINE
            assert rel_l2(y[s, b], r) <= 2 * BLOCK_REL_L2


def test_invalid_calls_rejected_before_launch(model):
    kv = model.new_kv([2], max_ctx=4)
    x = to_dev(syn.hidden_input(W, 4), torch.float16)
    with pytest.raises(tl.TLError) as e:
        model.prefill(h_in=x, L=3, kv=kv)                     # L above the lane's slots
    assert e.value.status == tl.TL_ERR_INVALID_ARG
    with pytest.raises(tl.TLError):
        model.prefill(h_in=to_dev(syn.hidden_input(W, 65), torch.float16), L=1)   # > max_tokens
    model.prefill(h_in=x, L=2, kv=kv)
    with pytest.raises(tl.TLError) as e:
        model.decode(kv, h_in=x[:1], L_per_lane=[2])          # cache full
    assert e.value.status == tl.TL_ERR_INVALID_ARG
    kv.set_position(0, 3)
    model.decode(kv, h_in=x[:1], L_per_lane=[2])
    assert kv.position(0) == 4
    with pytest.raises(tl.TLError):
        model.decode(kv, h_in=x[:1], L_per_lane=[0])
    with pytest.raises(tl.TLError) as e:
        model.prefill(h_in=x[:0], L=1)                        # empty prompt
    assert e.value.status == tl.TL_ERR_INVALID_ARG
    for bad in (-1, 9):                                       # chunks per decode-attention CTA
        with pytest.raises(tl.TLError) as e:
            model.set_decode_chunks(bad)
        assert e.value.status == tl.TL_ERR_INVALID_ARG
    model.set_decode_chunks(0)
    assert model.sync_status() == tl.TL_OK
    kv.close()


def test_non_finite_input_reports_numeric_status(model):
    x = syn.hidden_input(W, 4).copy()
    x[2, 5] = np.float16(np.inf)
    model.prefill(h_in=to_dev(x, torch.float16), L=1)
    assert model.sync_status() == tl.TL_ERR_NUMERIC
    assert model.sync_status() == tl.TL_OK           # the status word is cleared


def test_new_cache_after_destroy_uses_its_own_graphs(model):
    """A cache created after another was destroyed (possibly at the same host
    address) must not replay graphs captured for the old one."""
    x = to_dev(syn.hidden_input(W, 8, name="reuse.prompt"), torch.float16)
    step = to_dev(syn.hidden_input(W, 1, name="reuse.step"), torch.float16)
    outs = []
    for lanes in ([2, 1, 2], [2]):
        kv = model.new_kv(lanes, max_ctx=9)
        for b in range(len(lanes)):
            model.prefill(h_in=x, L=lanes[b], kv=kv, lane=b)
        outs.append(model.decode(kv, h_in=step.repeat(len(lanes), 1),
                                 L_per_lane=lanes).cpu().numpy())
        kv.close()
    assert np.array_equal(outs[0][0], outs[1][0])
    assert np.array_equal(outs[0][2], outs[1][0])


def test_bounded_wait_reports_timeout_and_context_survives(model):
    """A device wait that can never complete gives up after its limit and
    reports TL_ERR_TIMEOUT; the context keeps working afterwards."""
    import time
    t0 = time.perf_counter()
    tl.tl_check_bounded_wait(model.handle, 2000)          # 2 ms limit
    assert model.sync_status() == tl.TL_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    assert model.sync_status() == tl.TL_OK               # cleared
    x = to_dev(syn.hidden_input(W, 4), torch.float16)
    y = model.prefill(h_in=x, L=1)
    assert model.sync_status() == tl.TL_OK and torch.isfinite(y).all()
