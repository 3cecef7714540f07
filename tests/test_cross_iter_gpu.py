"""Cross-iteration rounding on the GPU ("Performance and Memory",
"Cross-iteration stochastic rounding": INT4 plus a 1-bit sign-of-frac channel;
"Current Status", architecture-unique features table, deterministic error
cancellation row: even iterations use the standard rounding, odd iterations
apply the sign correction).

* tl_pack_sign_bits writes the oracle's bit plane bit for bit (INT4 and INT3,
  both group sizes, an all-zero group, extreme elements);
* with the switch on, odd loop iterations of prefill (tensor-core GEMM) and of
  decode / extend (decode projection kernel) follow the oracle's odd-iteration
  weights per block, for INT4 and INT3 loop blocks;
* L = 1 (no odd iteration) is bit-identical to the switch off, and a model
  without sign bits refuses the switch."""
import numpy as np
import pytest
import torch

import synthetic as syn
import weight_shared_looped_b200 as tl
from oracle import tinyloop_oracle as o
from weight_shared_looped_b200.model import DeviceBlock, DeviceModel

from gpu_util import (BLOCK_REL_L2, FINAL_COSINE, cosine, rel_l2, row_cosines, to_dev)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits", [4, 3])
@pytest.mark.parametrize("group", [64, 128])
def test_pack_sign_bits_is_bit_exact(bits, group):
    rng = np.random.default_rng(100 * bits + group)
    N, K = 48, 4 * group
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[5, :group] = 0.0                                  # an all-zero group: s = 0, no bits
    w[7, 3] = 0.5                                       # the group maximum: code +qmax, bit 0
    w[9, group + 1] = -0.5                              # the group minimum
    w[11, 2 * group:3 * group] = np.linspace(-1, 1, group, dtype=np.float32)   # exact quotients
    wd = torch.from_numpy(w).cuda()
    cb, sb = tl.tl_packed_bytes(N, K, bits, group)
    packed = torch.empty(cb // 4, dtype=torch.int32, device="cuda")
    scales = torch.empty(sb // 2, dtype=torch.int16, device="cuda")
    tl.tl_pack_weights(wd, bits, group, packed, scales)
    sign = torch.empty(tl.tl_sign_bits_bytes(N, K) // 4, dtype=torch.int32, device="cuda")
    tl.tl_pack_sign_bits(wd, bits, group, scales, sign)
    torch.cuda.synchronize()
    want = o.pack_bits(o.sign_of_frac(w, group, bits))
    got = sign.cpu().numpy().view(np.uint32).reshape(N, -1)
    assert np.array_equal(got, want)
    assert not got[5, :group // 32].any()


def _cfg(bits):
    w = syn.WORKLOADS["tiny"]
    return o.block_cfg(w.shape, bits, w.group, w.eps, w.rope_theta)


def _weights(seed_name):
    w = syn.WORKLOADS["tiny"]
    return syn.block_weights(w.shape, w.seed, seed_name)


@pytest.fixture(scope="module", params=[4, 3], ids=["int4", "int3"])
def pair(request):
    """A tiny looped model (no pre-block, loop block with sign bits) on the GPU
    and the same model in the oracle, cross-iteration rounding on in both."""
    bits = request.param
    cfg = _cfg(bits)
    w = _weights(f"xiter.loop{bits}")
    packed = o.pack_block(w, bits, cfg["group"], sign=True)
    gpu_blk = DeviceBlock(cfg, weights=w, sign=True)             # packed on the GPU
    for m in ("qkv", "o", "gate", "up", "down"):
        assert np.array_equal(gpu_blk.t[f"sign_{m}"].cpu().numpy().view(np.uint32),
                              packed[f"sign_{m}"]), m
    shape = syn.WORKLOADS["tiny"].shape
    gam = syn.final_gain(shape, 7)
    dm = DeviceModel([], gpu_blk, gam, max_tokens=64, max_lanes=4, max_ctx=96, max_L=8)
    dm.set_cross_iter(True)
    om = o.LoopedModel([], o.Block(packed, cfg), gam)
    om.cross_iter = True
    yield dm, om, bits
    dm.close()
    gpu_blk.close()


@pytest.mark.parametrize("seq", [1, 6, 16, 37])
def test_prefill_odd_iterations_per_block(pair, seq):
    dm, om, bits = pair
    L = 4
    x = syn.hidden_input(syn.WORKLOADS["tiny"], seq, name=f"xiter.p{bits}.{seq}")
    trace = torch.empty(L, seq, 256, dtype=torch.float32, device="cuda")
    y = dm.prefill(h_in=to_dev(x, torch.float16), L=L, h_trace=trace)
    assert dm.sync_status() == tl.TL_OK
    rtr = []
    ry = om.prefill(x.astype(np.float64), L, trace=rtr)
    tr = trace.cpu().numpy()
    errs = [rel_l2(tr[i], rtr[i]) for i in range(L)]
    assert max(errs) <= BLOCK_REL_L2, errs
    assert row_cosines(y.cpu().numpy(), ry).min() >= FINAL_COSINE


def test_decode_and_extend_odd_iterations_per_block(pair):
    dm, om, bits = pair
    L, P, S = 3, 9, 4
    x = syn.hidden_input(syn.WORKLOADS["tiny"], P + S + 3, name=f"xiter.d{bits}")
    kv = dm.new_kv([L], max_ctx=P + S + 3)
    dm.prefill(h_in=to_dev(x[:P], torch.float16), L=L, kv=kv)
    okv = om.new_kv(L, "fp16")
    om.prefill(x[:P].astype(np.float64), L, kv=okv)
    for s in range(S):
        tr = torch.empty(L, 1, 256, dtype=torch.float32, device="cuda")
        y = dm.decode(kv, h_in=to_dev(x[P + s:P + s + 1], torch.float16), L_per_lane=[L],
                      h_trace=tr)
        rtr = []
        ry = om.decode_step(x[P + s].astype(np.float64), L, okv, trace=rtr)
        trc = tr.cpu().numpy()
        for layer in range(L):
            assert rel_l2(trc[layer, 0], rtr[layer][0]) <= BLOCK_REL_L2, (s, layer)
        assert cosine(y[0].cpu().numpy(), ry) >= FINAL_COSINE
    # three more tokens through the cached extend (decode rows of one lane)
    tr = torch.empty(L, 3, 256, dtype=torch.float32, device="cuda")
    y = dm.extend(kv, h_in=to_dev(x[P + S:], torch.float16), L=L, h_trace=tr)
    rtr = []
    ry = om.extend(x[P + S:].astype(np.float64), L, okv, trace=rtr)
    trc = tr.cpu().numpy()
    for layer in range(L):
        assert rel_l2(trc[layer], rtr[layer]) <= BLOCK_REL_L2, layer
    assert row_cosines(y.cpu().numpy(), ry).min() >= FINAL_COSINE
    assert dm.sync_status() == tl.TL_OK
    kv.close()


def test_single_iteration_is_unchanged(pair):
    """Iteration 0 is even: with L = 1 the switch changes nothing, bit for bit;
    with L = 2 the odd iteration changes the result."""
    dm, om, bits = pair
    x = to_dev(syn.hidden_input(syn.WORKLOADS["tiny"], 12, name=f"xiter.one{bits}"), torch.float16)
    on = {L: dm.prefill(h_in=x, L=L).clone() for L in (1, 2)}
    dm.set_cross_iter(False)
    off = {L: dm.prefill(h_in=x, L=L).clone() for L in (1, 2)}
    dm.set_cross_iter(True)
    assert torch.equal(on[1], off[1])
    assert not torch.equal(on[2], off[2])


def test_switch_needs_sign_bits():
    blk = DeviceBlock(_cfg(4), weights=_weights("xiter.nosign"))
    m = DeviceModel([], blk, syn.final_gain(syn.WORKLOADS["tiny"].shape, 7), max_tokens=8)
    with pytest.raises(tl.TLError) as e:
        m.set_cross_iter(True)
    assert e.value.status == tl.TL_ERR_INVALID_ARG
    m.set_cross_iter(False)
    m.close()
    blk.close()


def test_407m_decode_odd_iterations():
    """The 407M-shaped loop block (d 2048, ffn 8192: every decode projection
    shape, K = 8192 included) with sign bits: one prompt, two decode steps at
    L = 3 (iteration 1 odd), per block against the oracle."""
    w = syn.WORKLOADS["decode407m"]
    cfg = o.block_cfg(w.shape, 4, w.group, w.eps, w.rope_theta)
    wl = syn.block_weights(w.shape, w.seed, "loop")
    packed = o.pack_block(wl, 4, w.group, sign=True)
    blk = DeviceBlock(cfg, weights=wl, sign=True)
    for m in ("qkv", "down"):
        assert np.array_equal(blk.t[f"sign_{m}"].cpu().numpy().view(np.uint32), packed[f"sign_{m}"])
    gam = syn.final_gain(w.shape, w.seed)
    dm = DeviceModel([], blk, gam, max_tokens=16, max_lanes=1, max_ctx=32, max_L=4)
    dm.set_cross_iter(True)
    om = o.LoopedModel([], o.Block(packed, cfg), gam)
    om.cross_iter = True
    L, P = 3, 12
    x = syn.normal((P + 2, w.shape.d_model), 1.0, w.seed, "xiter.407m").astype(np.float16)
    kv = dm.new_kv([L], max_ctx=P + 2)
    dm.prefill(h_in=to_dev(x[:P], torch.float16), L=L, kv=kv)
    okv = om.new_kv(L, "fp16")
    om.prefill(x[:P].astype(np.float64), L, kv=okv)
    for s in range(2):
        tr = torch.empty(L, 1, w.shape.d_model, dtype=torch.float32, device="cuda")
        dm.decode(kv, h_in=to_dev(x[P + s:P + s + 1], torch.float16), L_per_lane=[L], h_trace=tr)
        rtr = []
        om.decode_step(x[P + s].astype(np.float64), L, okv, trace=rtr)
        trc = tr.cpu().numpy()
        for layer in range(L):
            assert rel_l2(trc[layer, 0], rtr[layer][0]) <= BLOCK_REL_L2, (s, layer)
    assert dm.sync_status() == tl.TL_OK
    kv.close()
    dm.close()
    blk.close()
