"""Per-iteration weight variants on the GPU ("Current Status",
architecture-unique features table, dual-bit and triple-bit weight swap rows:
a low-bit copy of the loop block for the early iterations, the higher-bit copy
later, optionally another copy for iteration 0).

* prefill, decode and extend with variants follow the oracle's schedule per
  block (INT3 copies for early iterations of an INT4 loop block, and an
  iteration-0 variant of other weights);
* the loop block itself as the variant is bit-identical to no variant;
* cross-iteration rounding uses the sign bits of the block an odd iteration runs;
* blocks of another shape and out-of-range counts are refused."""
import numpy as np
import pytest
import torch

import synthetic as syn
import weight_shared_looped_b200 as tl
from oracle import tinyloop_oracle as o
from weight_shared_looped_b200.model import DeviceBlock, DeviceModel

from gpu_util import BLOCK_REL_L2, FINAL_COSINE, cosine, rel_l2, row_cosines, to_dev

pytestmark = pytest.mark.gpu
W = syn.WORKLOADS["tiny"]


def _cfg(bits):
    return o.block_cfg(W.shape, bits, W.group, W.eps, W.rope_theta)


@pytest.fixture(scope="module")
def setup():
    w_loop = syn.block_weights(W.shape, W.seed, "iv.loop")
    w_first = syn.block_weights(W.shape, W.seed, "iv.first")
    pk = {"loop4": o.pack_block(w_loop, 4, W.group, sign=True),
          "loop3": o.pack_block(w_loop, 3, W.group, sign=True),
          "first4": o.pack_block(w_first, 4, W.group)}
    dev = {"loop4": DeviceBlock(_cfg(4), packed=pk["loop4"]),
           "loop3": DeviceBlock(_cfg(3), packed=pk["loop3"]),
           "first4": DeviceBlock(_cfg(4), packed=pk["first4"])}
    orc = {"loop4": o.Block(pk["loop4"], _cfg(4)), "loop3": o.Block(pk["loop3"], _cfg(3)),
           "first4": o.Block(pk["first4"], _cfg(4))}
    gam = syn.final_gain(W.shape, 3)
    dm = DeviceModel([], dev["loop4"], gam, max_tokens=64, max_lanes=4, max_ctx=96, max_L=8)
    om = o.LoopedModel([], orc["loop4"], gam)
    yield dm, om, dev, orc
    dm.close()
    for b in dev.values():
        b.close()


SCHEDULES = {"dual": ["loop3", "loop3"], "triple": ["first4", "loop3", "loop3"],
             "odd_gap": [None, "loop3", None, "loop3"]}


def _apply(dm, om, dev, orc, names):
    dm.set_iteration_blocks([dev[n] if n else None for n in names])
    om.iter_blocks = [orc[n] if n else None for n in names]


@pytest.mark.parametrize("sched", list(SCHEDULES))
@pytest.mark.parametrize("seq", [5, 16, 33])
def test_prefill_with_variants_per_block(setup, sched, seq):
    dm, om, dev, orc = setup
    _apply(dm, om, dev, orc, SCHEDULES[sched])
    L = 5
    x = syn.hidden_input(W, seq, name=f"iv.p.{sched}.{seq}")
    trace = torch.empty(L, seq, 256, dtype=torch.float32, device="cuda")
    y = dm.prefill(h_in=to_dev(x, torch.float16), L=L, h_trace=trace)
    assert dm.sync_status() == tl.TL_OK
    rtr = []
    ry = om.prefill(x.astype(np.float64), L, trace=rtr)
    tr = trace.cpu().numpy()
    errs = [rel_l2(tr[i], rtr[i]) for i in range(L)]
    assert max(errs) <= BLOCK_REL_L2, errs
    assert row_cosines(y.cpu().numpy(), ry).min() >= FINAL_COSINE


@pytest.mark.parametrize("cross_iter", [False, True])
@pytest.mark.parametrize("sched", ["dual", "triple"])
def test_decode_and_extend_with_variants_per_block(setup, sched, cross_iter):
    dm, om, dev, orc = setup
    _apply(dm, om, dev, orc, SCHEDULES[sched])
    dm.set_cross_iter(cross_iter)
    om.cross_iter = cross_iter
    L, P, S = 4, 10, 3
    x = syn.hidden_input(W, P + S + 2, name=f"iv.d.{sched}")
    kv = dm.new_kv([L], max_ctx=P + S + 2)
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
    y = dm.extend(kv, h_in=to_dev(x[P + S:], torch.float16), L=L)
    ry = om.extend(x[P + S:].astype(np.float64), L, okv)
    assert row_cosines(y.cpu().numpy(), ry).min() >= FINAL_COSINE
    assert dm.sync_status() == tl.TL_OK
    dm.set_cross_iter(False)
    om.cross_iter = False
    kv.close()


def test_loop_block_as_variant_is_bit_identical(setup):
    dm, om, dev, orc = setup
    x = to_dev(syn.hidden_input(W, 20, name="iv.same"), torch.float16)
    dm.set_iteration_blocks([])
    want = dm.prefill(h_in=x, L=3).clone()
    dm.set_iteration_blocks([dev["loop4"], None, dev["loop4"]])
    assert torch.equal(dm.prefill(h_in=x, L=3), want)
    dm.set_iteration_blocks([dev["loop3"]])
    assert not torch.equal(dm.prefill(h_in=x, L=3), want)
    dm.set_iteration_blocks([])


def test_variants_are_checked(setup):
    dm, om, dev, orc = setup
    other = syn.BlockShape(256, 2, 128, 768)                 # heads differ
    cfg = o.block_cfg(other, 4, W.group, W.eps, W.rope_theta)
    blk = DeviceBlock(cfg, weights=syn.block_weights(other, W.seed, "iv.other"))
    for bad in ([blk], [None] * 9):
        with pytest.raises(tl.TLError) as e:
            dm.set_iteration_blocks(bad)
        assert e.value.status == tl.TL_ERR_INVALID_ARG
    blk.close()
