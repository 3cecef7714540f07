"""INT3 blocks read natively (10 codes per 32-bit word: "Current Status", core
inference table, INT3 GEMM row) by every kernel: the tensor-core prefill GEMM
at every token count and the decode projection kernel, against the oracle's
INT3 dequantisation, per block; and an INT3 block costs fewer device bytes
than an INT4 one (no library-owned copy of its codes)."""
import numpy as np
import pytest
import torch

import synthetic as syn
import weight_shared_looped_b200 as tl
from oracle import tinyloop_oracle as o

from gpu_util import (BLOCK_REL_L2, FINAL_COSINE, cosine, device_blocks, device_model,
                      oracle_model, rel_l2, row_cosines, to_dev)

pytestmark = pytest.mark.gpu
W = syn.WORKLOADS["tiny_int3"]


@pytest.fixture(scope="module")
def model():
    m = device_model("tiny_int3", max_tokens=64, max_lanes=4, max_ctx=96)
    yield m
    m.close()


@pytest.mark.parametrize("seq", [1, 5, 16, 37, 64])
def test_tiny_int3_prefill_per_block(model, seq):
    L = 3
    x = syn.hidden_input(W, seq, name=f"int3.h_in.{seq}")
    trace = torch.empty(L, seq, W.shape.d_model, dtype=torch.float32, device="cuda")
    y = model.prefill(h_in=to_dev(x, torch.float16), L=L, h_trace=trace)
    assert model.sync_status() == tl.TL_OK
    rtr = []
    ry = oracle_model("tiny_int3").prefill(x.astype(np.float64), L, trace=rtr)
    tr = trace.cpu().numpy()
    errs = [rel_l2(tr[i], rtr[i]) for i in range(L)]
    assert max(errs) <= BLOCK_REL_L2, errs
    assert row_cosines(y.cpu().numpy(), ry).min() >= FINAL_COSINE


def test_tiny_int3_decode_per_block(model):
    L, P, S = 2, 11, 4
    kv = model.new_kv([L], max_ctx=P + S)
    x = syn.hidden_input(W, P + S, name="int3.dec")
    model.prefill(h_in=to_dev(x[:P], torch.float16), L=L, kv=kv, lane=0)
    om = oracle_model("tiny_int3")
    okv = om.new_kv(L, "fp16")
    om.prefill(x[:P].astype(np.float64), L, kv=okv)
    for s in range(S):
        tr = torch.empty(L, 1, W.shape.d_model, dtype=torch.float32, device="cuda")
        y = model.decode(kv, h_in=to_dev(x[P + s:P + s + 1], torch.float16), L_per_lane=[L],
                         h_trace=tr)
        rtr = []
        ry = om.decode_step(x[P + s].astype(np.float64), L, okv, trace=rtr)
        trc = tr.cpu().numpy()
        for layer in range(L):
            assert rel_l2(trc[layer, 0], rtr[layer][0]) <= BLOCK_REL_L2, (s, layer)
        assert cosine(y[0].cpu().numpy(), ry) >= FINAL_COSINE
    assert model.sync_status() == tl.TL_OK
    kv.close()


def test_int3_block_costs_fewer_bytes_than_int4():
    d, f = 2048, 8192
    shapes = ((3 * d, d), (d, d), (f, d), (f, d), (d, f))
    by = {bits: sum(sum(tl.tl_packed_bytes(n, k, bits, 128)) for n, k in shapes) for bits in (3, 4)}
    assert by[3] < by[4]
    blocks = device_blocks("mixed_int3", check_packing=False)
    for name, blk in blocks.items():
        assert tl.tl_block_device_bytes(blk.handle) == 0, name   # nothing beyond the caller's words
        held = sum(t.numel() * t.element_size() for k, t in blk.t.items() if k[0] in "ws")
        bits = 3 if name == "loop" else 4
        assert held == by[bits], (name, held)
    for blk in blocks.values():
        blk.close()
