"""The per-iteration residual-norm check on the GPU ("Current Status",
architecture-unique features table, per-iteration safety check row: the
residual stream's L2 norm every iteration, the loop stops above a
threshold), against the oracle's reading of it: prefill (tokens), decode and
extend (lanes), loop counts exact and outputs within the block tolerance;
lanes stay bit-exact with their single-lane runs; tau < 0 changes nothing.

The threshold is placed between the oracle's per-iteration norms, at the
middle of a gap far wider than the GPU/oracle difference of the streams, so
the integer decision does not hinge on rounding."""
import numpy as np
import pytest
import torch

import synthetic as syn
import weight_shared_looped_b200 as tl

from gpu_util import (BLOCK_REL_L2, FINAL_COSINE, cosine, device_model, oracle_model, rel_l2,
                      row_cosines, to_dev)

pytestmark = pytest.mark.gpu
W = syn.WORKLOADS["tiny"]


@pytest.fixture(scope="module")
def model():
    m = device_model("tiny", max_tokens=64, max_lanes=8, max_ctx=128)
    yield m
    m.set_exit_threshold(-1.0)
    m.close()


def _pick_tau(norms, rel_margin=0.005):
    """A threshold in the middle of the widest gap between sorted norms (away
    from the extremes), so that the GPU/oracle difference of a row's norm
    (~1e-4 relative: a norm averages the elementwise errors) cannot move a
    decision."""
    v = np.sort(np.asarray(norms).ravel())
    lo, hi = len(v) // 10, len(v) - 1 - len(v) // 10
    gaps = (v[lo + 1:hi + 1] - v[lo:hi]) / v[lo:hi]
    i = lo + int(np.argmax(gaps))
    assert gaps.max() > rel_margin, gaps.max()
    return float((v[i] + v[i + 1]) / 2)


def test_prefill_exit_matches_oracle(model):
    L, seq = 6, 29
    x = syn.hidden_input(W, seq, name="exit.prefill").astype(np.float64)
    om = oracle_model("tiny")
    trace = []
    om.prefill(x, L, trace=trace)
    tau = _pick_tau([np.linalg.norm(trace[j], axis=-1) for j in range(L - 1)])
    info = {}
    ry = om.prefill(x, L, exit_tau=tau, info=info)
    assert 1 < len(set(info["loops"])), info["loops"]
    model.set_exit_threshold(tau)
    y = model.prefill(h_in=to_dev(x.astype(np.float16), torch.float16), L=L).cpu().numpy()
    loops = model.loops_used(seq)
    model.set_exit_threshold(-1.0)
    assert model.sync_status() == tl.TL_OK
    assert loops == [int(v) for v in info["loops"]]
    assert row_cosines(y, ry).min() >= FINAL_COSINE
    assert rel_l2(y, ry) <= 2 * BLOCK_REL_L2


def _lanes_run(model, Ls, prompts, steps, tau):
    model.set_exit_threshold(tau)
    kv = model.new_kv(Ls, max_ctx=len(prompts[0]) + len(steps))
    for b, p in enumerate(prompts):
        model.prefill(h_in=to_dev(p, torch.float16), L=Ls[b], kv=kv, lane=b)
    ys, loops = [], []
    for st in steps:
        ys.append(model.decode(kv, h_in=to_dev(st, torch.float16), L_per_lane=Ls).cpu().numpy())
        loops.append(model.loops_used(len(Ls)))
    kv.close()
    model.set_exit_threshold(-1.0)
    return np.stack(ys), loops


def test_decode_exit_matches_oracle_and_lanes_stay_bit_exact(model):
    Ls, P, S = [5, 3, 5], 9, 3
    names = ["ea", "eb", "ec"]
    prompts = [syn.hidden_input(W, P, name=f"exit.p.{n}") for n in names]
    steps = [np.stack([syn.hidden_input(W, 1, name=f"exit.s{s}.{n}")[0] for n in names])
             for s in range(S)]
    om = oracle_model("tiny")
    # the norms the oracle's lanes see entering each iteration, exit-free
    norms = []
    for b, L in enumerate(Ls):
        kv = om.new_kv(L, "fp16")
        om.prefill(prompts[b].astype(np.float64), L, kv=kv)
        for s in range(S):
            tr = []
            om.decode_step(steps[s][b].astype(np.float64), L, kv, trace=tr)
            norms += [np.linalg.norm(tr[1 + j][0]) for j in range(L - 1)]
    tau = _pick_tau(norms)
    y, loops = _lanes_run(model, Ls, prompts, steps, tau)
    seen = set()
    for b, L in enumerate(Ls):
        kv = om.new_kv(L, "fp16")
        om.prefill(prompts[b].astype(np.float64), L, kv=kv, exit_tau=tau)
        for s in range(S):
            info = {}
            r = om.decode_step(steps[s][b].astype(np.float64), L, kv, exit_tau=tau, info=info)
            assert loops[s][b] == int(info["loops"][0]), (s, b)
            seen.add(loops[s][b])
            assert cosine(y[s, b], r) >= FINAL_COSINE, (s, b)
            assert rel_l2(y[s, b], r) <= 2 * BLOCK_REL_L2, (s, b)
    assert len(seen) > 1, seen
    for b in range(len(Ls)):
        y1, l1 = _lanes_run(model, [Ls[b]], [prompts[b]], [st[b:b + 1] for st in steps], tau)
        assert np.array_equal(y1[:, 0], y[:, b]), b
        assert [l[0] for l in l1] == [l[b] for l in loops]


def test_negative_threshold_changes_nothing(model):
    x = to_dev(syn.hidden_input(W, 12, name="exit.off"), torch.float16)
    a = model.prefill(h_in=x, L=4).clone()
    model.set_exit_threshold(1e30)
    b = model.prefill(h_in=x, L=4).clone()
    assert model.loops_used(12) == [4] * 12
    model.set_exit_threshold(-1.0)
    c = model.prefill(h_in=x, L=4).clone()
    assert torch.equal(a, b) and torch.equal(a, c)
    with pytest.raises(tl.TLError):
        model.set_exit_threshold(float("nan"))


def test_zero_threshold_is_the_one_iteration_forward(model):
    x = to_dev(syn.hidden_input(W, 10, name="exit.zero"), torch.float16)
    one = model.prefill(h_in=x, L=1).clone()
    model.set_exit_threshold(0.0)
    y = model.prefill(h_in=x, L=5).clone()
    assert model.loops_used(10) == [1] * 10
    model.set_exit_threshold(-1.0)
    assert torch.equal(y, one)
