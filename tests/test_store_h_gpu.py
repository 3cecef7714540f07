"""Store-h KV on the GPU ("Current Status", KV cache mode table, Store-h
(FP16) and tensor-core reconstruction rows; "Claims & Data Sources", h-mode
KV reconstruction from shared W_k / W_v).

* the cache keeps the fp16 QKV-input rows (half the bytes of K and V per
  position) and every decode step rebuilds K and V from them with the
  quantised-weight GEMM; decode follows the oracle's store-h slots per block,
  for INT4 and INT3 loop blocks, several lanes of different depth, with
  cross-iteration rounding, and at the 407M shape (tensor-core rebuild);
* the slots hold exactly the rows the prefill normalised (bit for bit with
  the model's own fp16 activations), and a store-h decode stays close to the
  fp16-KV decode of the same model;
* extend and speculative steps refuse a store-h cache."""
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


def _cfg(shape, bits):
    return o.block_cfg(shape, bits, W.group, W.eps, W.rope_theta)


@pytest.fixture(scope="module", params=[4, 3], ids=["int4", "int3"])
def pair(request):
    bits = request.param
    shape = W.shape
    w_pre = syn.block_weights(shape, W.seed, "sh.pre")
    w_loop = syn.block_weights(shape, W.seed, "sh.loop")
    pk_pre = o.pack_block(w_pre, 4, W.group)
    pk_loop = o.pack_block(w_loop, bits, W.group, sign=True)
    pre = DeviceBlock(_cfg(shape, 4), packed=pk_pre)
    loop = DeviceBlock(_cfg(shape, bits), packed=pk_loop)
    gam = syn.final_gain(shape, 5)
    dm = DeviceModel([pre], loop, gam, max_tokens=96, max_lanes=4, max_ctx=160, max_L=8)
    om = o.LoopedModel([o.Block(pk_pre, _cfg(shape, 4))], o.Block(pk_loop, _cfg(shape, bits)), gam)
    yield dm, om, bits
    dm.close()
    pre.close()
    loop.close()


@pytest.mark.parametrize("cross_iter", [False, True])
def test_store_h_decode_per_block(pair, cross_iter):
    dm, om, bits = pair
    dm.set_cross_iter(cross_iter)
    om.cross_iter = cross_iter
    Ls, P, S = [3, 1, 2], [70, 9, 33], 3             # lanes of different depth and context
    n_layers = [1 + L for L in Ls]
    kv = dm.new_kv(Ls, max_ctx=80, dtype="h")
    okvs = []
    xs = [syn.hidden_input(W, P[b] + S, name=f"sh.x{b}") for b in range(3)]
    for b in range(3):
        dm.prefill(h_in=to_dev(xs[b][:P[b]], torch.float16), L=Ls[b], kv=kv, lane=b)
        okv = om.new_kv(Ls[b], "h")
        om.prefill(xs[b][:P[b]].astype(np.float64), Ls[b], kv=okv)
        okvs.append(okv)
    for s in range(S):
        hin = np.stack([xs[b][P[b] + s] for b in range(3)])
        tr = torch.empty(max(n_layers), 3, 256, dtype=torch.float32, device="cuda")
        y = dm.decode(kv, h_in=to_dev(hin, torch.float16), L_per_lane=Ls, h_trace=tr).cpu().numpy()
        trc = tr.cpu().numpy()
        for b in range(3):
            rtr = []
            ry = om.decode_step(xs[b][P[b] + s].astype(np.float64), Ls[b], okvs[b], trace=rtr)
            for layer in range(n_layers[b]):
                assert rel_l2(trc[layer, b], rtr[layer][0]) <= BLOCK_REL_L2, (s, b, layer)
            assert cosine(y[b], ry) >= FINAL_COSINE
    assert dm.sync_status() == tl.TL_OK
    assert [kv.position(b) for b in range(3)] == [P[b] + S for b in range(3)]
    dm.set_cross_iter(False)
    om.cross_iter = False
    kv.close()


def test_store_h_slots_hold_the_prefill_rows(pair):
    """The slot of a layer holds the fp16 rows the layer's QKV projection read:
    for layer 0 (after the embedding), fp16(RMSNorm(h_in) * gamma_attn) as the
    model's own norm kernel forms it, i.e. the prefill's x rows."""
    dm, om, bits = pair
    P = 12
    x = syn.hidden_input(W, P, name="sh.rows")
    kvh = dm.new_kv([2], max_ctx=16, dtype="h")
    dm.prefill(h_in=to_dev(x, torch.float16), L=2, kv=kvh)
    kptr, vptr, ks, vs = kvh.layer_ptrs(0, 0)
    assert vptr is None and ks is None and vs is None
    off = kptr - kvh.buffer.data_ptr()
    rows = kvh.buffer[off:off + P * 256 * 2].view(torch.float16).view(P, 256).cpu().numpy()
    want = o.rmsnorm(x.astype(np.float64), om.pre[0].gamma_attn, W.eps)
    assert np.abs(rows.astype(np.float64) - want).max() <= 2e-3 * np.abs(want).max()
    kvh.close()


def test_store_h_decode_close_to_fp16_cache(pair):
    dm, om, bits = pair
    P, L = 40, 3
    x = syn.hidden_input(W, P + 4, name="sh.cmp")
    outs = {}
    for dtype in ("fp16", "h"):
        kv = dm.new_kv([L], max_ctx=P + 4, dtype=dtype)
        dm.prefill(h_in=to_dev(x[:P], torch.float16), L=L, kv=kv)
        outs[dtype] = np.stack([dm.decode(kv, h_in=to_dev(x[P + s:P + s + 1], torch.float16),
                                          L_per_lane=[L]).cpu().numpy()[0] for s in range(4)])
        kv.close()
    assert row_cosines(outs["h"], outs["fp16"]).min() >= 0.999


def test_store_h_bytes_and_refusals(pair):
    dm, om, bits = pair
    fp16 = tl.tl_kv_bytes(dm.handle, 160, [8, 8], tl.TL_KV_FP16)
    h = tl.tl_kv_bytes(dm.handle, 160, [8, 8], tl.TL_KV_H)
    slots = 2 * 9 * tl.tl_kv_layer_bytes(4, 64, 160, tl.TL_KV_H)
    assert slots * 2 == fp16 - 4096
    assert h > 4096 + slots          # the slots, then the rebuild workspace
    kv = dm.new_kv([2], max_ctx=16, dtype="h")
    dm.prefill(h_in=to_dev(syn.hidden_input(W, 4, name="sh.ref"), torch.float16), L=2, kv=kv)
    with pytest.raises(tl.TLError) as e:
        dm.extend(kv, h_in=to_dev(syn.hidden_input(W, 2, name="sh.ext"), torch.float16), L=2)
    assert e.value.status == tl.TL_ERR_UNSUPPORTED
    assert kv.position(0) == 4
    kv.close()


def test_store_h_407m_decode():
    """The 407M-shaped loop block: a 96-token prompt (rebuild GEMM on the
    tensor cores) and a 20-token one (register-dequant GEMM), two decode steps
    as two lanes, against the oracle's store-h slots per block."""
    w = syn.WORKLOADS["decode407m"]
    cfg = o.block_cfg(w.shape, 4, w.group, w.eps, w.rope_theta)
    wl = syn.block_weights(w.shape, w.seed, "loop")
    blk = DeviceBlock(cfg, weights=wl)
    gam = syn.final_gain(w.shape, w.seed)
    dm = DeviceModel([], blk, gam, max_tokens=96, max_lanes=2, max_ctx=128, max_L=4)
    om = o.LoopedModel([], o.Block(o.pack_block(wl, 4, w.group), cfg), gam)
    L, P = 2, [96, 20]
    xs = [syn.normal((P[b] + 2, w.shape.d_model), 1.0, w.seed, f"sh.407m.{b}").astype(np.float16)
          for b in range(2)]
    kv = dm.new_kv([L, L], max_ctx=128, dtype="h")
    okvs = []
    for b in range(2):
        dm.prefill(h_in=to_dev(xs[b][:P[b]], torch.float16), L=L, kv=kv, lane=b)
        okv = om.new_kv(L, "h")
        om.prefill(xs[b][:P[b]].astype(np.float64), L, kv=okv)
        okvs.append(okv)
    for s in range(2):
        tr = torch.empty(L, 2, w.shape.d_model, dtype=torch.float32, device="cuda")
        hin = np.stack([xs[b][P[b] + s] for b in range(2)])
        dm.decode(kv, h_in=to_dev(hin, torch.float16), L_per_lane=[L, L], h_trace=tr)
        trc = tr.cpu().numpy()
        for b in range(2):
            rtr = []
            om.decode_step(xs[b][P[b] + s].astype(np.float64), L, okvs[b], trace=rtr)
            for layer in range(L):
                assert rel_l2(trc[layer, b], rtr[layer][0]) <= BLOCK_REL_L2, (s, b, layer)
    assert dm.sync_status() == tl.TL_OK
    kv.close()
    dm.close()
    blk.close()
