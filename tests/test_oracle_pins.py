"""Pins of the CPU oracle to facts fixed outside the oracle itself: the pages'
printed memory figures, hand-worked closed forms, brute force on tiny inputs
and the invariants the pages state.  CPU only."""
import math
import os

import numpy as np
import pytest

import synthetic as syn
from oracle import tinyloop_oracle as o

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_memory():
    out = {}
    with open(os.path.join(GOLDEN, "memory_numbers.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, val, unit = line.split("|")[0].split()
            out[key] = (float(val), unit)
    return out


# ---------------------------------------------------------------- quantisation

def _f16_hex(x):
    return np.float16(x).view(np.uint16).item()


@pytest.mark.parametrize("bits,weights,scale_hex,codes", [
    # absmax 0.7: 0.7/7 rounds to fp16 0x2E66 = 0.0999755859375; the ratios
    # w/s are 7.0017, -3.5009, 1.0002, 0, 2.4996, -7.0017, 0.50012, 3.5009
    (4, [0.7, -0.35, 0.1, 0, 0.2499, -0.7, 0.05, 0.35], 0x2E66, [7, -4, 1, 0, 2, -7, 1, 4]),
    # absmax 7 gives scale 1.0 exactly; exact halves round to even
    (4, [7, 2.5, -2.5, 3.5, -0.5, 0.5, 1.5, 0], 0x3C00, [7, 2, -2, 4, 0, 0, 2, 0]),
    # an all-zero group has scale 0 and codes 0
    (4, [0] * 8, 0x0000, [0] * 8),
    # INT3: absmax 3 gives scale 1.0, codes stay in [-4, 3]
    (3, [3, 1.5, -1.5, 2.5, -0.5, 0.5, -3, 0], 0x3C00, [3, 2, -2, 2, 0, 0, -3, 0]),
    # negative absmax element maps to -qmax, never to -qmax-1; scale fp16(0.1),
    # ratios -3.0007, 1.0002, 0.50012
    (3, [-0.3, 0.1, 0.05, 0, 0, 0, 0, 0], 0x2E66, [-3, 1, 1, 0, 0, 0, 0, 0]),
])
def test_quantize_hand_worked(bits, weights, scale_hex, codes):
    w = np.array([weights], dtype=np.float32)
    c, s = o.quantize_groupwise(w, bits, group=8)
    assert s.view(np.uint16)[0, 0] == scale_hex
    assert c[0].tolist() == codes


def test_pack_layout_int4_nibble_order():
    # offset binary u = code + 8, lowest k in the lowest nibble
    codes = np.array([[-8, -7, -6, -5, -4, -3, -2, -1, 0, 1, 2, 3, 4, 5, 6, 7]], np.int8)
    words = o.pack_codes(codes, 4)
    assert words.tolist() == [[0x76543210, 0xFEDCBA98]]


def test_pack_layout_int3_ten_per_word():
    # u = code + 4 at bits 3i: the octal digits of the word are u9..u0
    codes = np.array([[-4, -3, -2, -1, 0, 1, 2, 3, -4, -3, 3]], np.int8)
    words = o.pack_codes(codes, 3)
    pad = int("4444444444", 8)
    assert words.shape == (1, 4)                  # ceil(11/10) = 2 words, padded to 4
    assert words[0, 0] == 0o1076543210
    assert words[0, 1] == int("4444444447", 8)    # k=10 holds u=7, the rest padding u=4
    assert words[0, 2] == pad and words[0, 3] == pad
    assert int(words.max()) < (1 << 30)           # bits 30-31 zero


def test_int3_words_per_row():
    assert o.int3_words_per_row(2048) == 208       # 205 words padded to 208
    assert o.int3_words_per_row(8192) == 820
    assert o.int3_words_per_row(10) == 4


@pytest.mark.parametrize("bits,group", [(4, 64), (4, 128), (3, 128), (3, 64)])
def test_quantize_properties(bits, group):
    rng = np.random.default_rng(1)
    w = (rng.standard_normal((37, 4 * group)) * 0.02).astype(np.float32)
    w[3, :group] = 0.0                                   # all-zero group
    w[5, group:2 * group] = 1e-3                         # constant group
    codes, s16 = o.quantize_groupwise(w, bits, group)
    qmax = o.QMAX[bits]
    assert codes.min() >= -qmax and codes.max() <= qmax     # -qmax-1 never produced
    # round trip through the packed words
    assert np.array_equal(o.unpack_codes(o.pack_codes(codes, bits), w.shape[1], bits), codes)
    s = np.repeat(s16.astype(np.float64), group, axis=1)
    err = np.abs(w.astype(np.float64) - codes * s)
    assert np.all(err <= s / 2 * (1 + 1e-6) + 1e-12)
    # the largest-magnitude element of each group maps to +-qmax
    g = np.abs(w).reshape(37, -1, group)
    am = g.argmax(axis=2)
    cg = codes.reshape(37, -1, group)
    top = np.take_along_axis(np.abs(cg), am[..., None], axis=2)[..., 0]
    nz = s16 != 0
    assert np.all(top[nz] == qmax)
    assert np.all(s16[3, 0] == 0) and np.all(codes[3, :group] == 0)


def test_dequantize_uses_group_of_each_column():
    codes = np.ones((1, 8), np.int8)
    s16 = np.array([[1.0, 2.0, 4.0, 8.0]], np.float16)
    assert o.dequantize(codes, s16, 2).tolist() == [[1, 1, 2, 2, 4, 4, 8, 8]]


# ---------------------------------------------------------------- INT8 KV

def test_kv_int8_hand_worked():
    # absmax 127 * 2^-7: scale = 2^-7 exactly, codes = 128 x; fp16(0.1) = 0.0999755859375
    x = np.array([[0.9921875, -0.5, 0.25, 0.00390625, 0.01171875, -0.9921875, 0.1, 0.0]], np.float16)
    c, s = o.kv_quant_int8(x)
    assert s[0] == np.float16(2.0 ** -7)
    assert c[0].tolist() == [127, -64, 32, 0, 2, -127, 13, 0]


def test_kv_int8_properties():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 16, 128)).astype(np.float16)
    x[0, 0] = 0
    c, s = o.kv_quant_int8(x)
    assert c.shape == x.shape and s.shape == (64, 16)
    assert s[0, 0] == 0 and np.all(c[0, 0] == 0)
    am = np.abs(x.astype(np.float32)).max(-1)
    assert np.array_equal(s, (am / np.float32(127)).astype(np.float16))   # one scale per (token, head)
    err = np.abs(x.astype(np.float64) - o.kv_dequant_int8(c, s))
    assert np.all(err <= s.astype(np.float64)[..., None] / 2 * (1 + 1e-6) + 1e-12)
    assert np.all(np.abs(c).max(-1)[s != 0] == 127)


# ---------------------------------------------------------------- memory figures

def test_kv_bytes_match_pages():
    g = _golden_memory()
    fp16 = o.kv_cache_bytes(10, 2048, 16, 128, "fp16")
    int8 = o.kv_cache_bytes(10, 2048, 16, 128, "int8")
    assert round(fp16 / 1e6, 1) == g["kv_fp16_max_seq_2048_10_layers"][0]
    assert round(int8 / 1e6, 1) == g["kv_int8_max_seq_2048_10_layers"][0]
    assert round((int8 / fp16 - 1) * 100, 1) == g["kv_int8_delta_percent"][0]


def test_weight_counts_match_pages():
    g = _golden_memory()
    per_block = o.block_weight_count(2048, 8192)
    assert per_block == 64 * 2 ** 20
    params = 3 * per_block + 2 * syn.VOCAB * 2048               # 3 blocks + embedding + head
    assert round(params / 1e6) == g["model_params"][0]
    # the FP16 body cache adds 2 bytes per body weight: 216 -> 619 MB
    delta = g["weight_vram_int4_plus_fp16_body"][0] - g["weight_vram_int4"][0]
    assert abs(3 * per_block * 2 / 1e6 - delta) < 1.0
    # weight bytes of one packed INT4 block (group 128) and INT3 block
    assert o.packed_block_bytes(2048, 8192, 4, 128) == 32 * 2 ** 20 + 2 ** 20
    assert o.packed_block_bytes(2048, 8192, 3, 128) < o.packed_block_bytes(2048, 8192, 4, 128)


# ---------------------------------------------------------------- RMSNorm / RoPE / SwiGLU

def test_rmsnorm_closed_form():
    rng = np.random.default_rng(3)
    h = rng.standard_normal((5, 64)) * 3
    gam = 1 + 0.1 * rng.standard_normal(64)
    y = o.rmsnorm(h, gam, 1e-5)
    ms = (h * h).mean(-1)
    rms_unscaled = np.sqrt(((y / gam) ** 2).mean(-1))
    assert np.allclose(rms_unscaled, np.sqrt(ms / (ms + 1e-5)), rtol=1e-12)
    # per element, against a plain loop
    for t in range(5):
        s = sum(float(v) * float(v) for v in h[t]) / 64
        for i in range(64):
            assert abs(y[t, i] - h[t, i] / math.sqrt(s + 1e-5) * gam[i]) < 1e-12


def test_rope_hand_values():
    # hd = 2: inv_freq = 1, so pos 1 rotates the pair by 1 rad
    y = o.rope(np.array([[[1.0, 0.0]]]), np.array([1]), 10000.0)
    assert np.allclose(y[0, 0], [math.cos(1), math.sin(1)], atol=1e-15)
    y = o.rope(np.array([[[0.0, 1.0]]]), np.array([2]), 10000.0)
    assert np.allclose(y[0, 0], [-math.sin(2), math.cos(2)], atol=1e-15)
    # hd = 4: pair (1, 3) has inv_freq 10000^(-2/4) = 0.01, so pos 100 turns it by 1 rad
    y = o.rope(np.array([[[0.0, 1.0, 0.0, 0.0]]]), np.array([100]), 10000.0)
    assert np.allclose(y[0, 0], [0, math.cos(1), 0, math.sin(1)], atol=1e-12)


def test_rope_properties():
    rng = np.random.default_rng(4)
    hd = 64
    q = rng.standard_normal((1, 3, hd))
    k = rng.standard_normal((1, 3, hd))
    assert np.array_equal(o.rope(q, np.array([0]), 1e4), q)             # pos 0 is identity
    r = o.rope(q, np.array([777]), 1e4)
    half = hd // 2
    assert np.allclose(r[..., :half] ** 2 + r[..., half:] ** 2, q[..., :half] ** 2 + q[..., half:] ** 2)
    # <R_m q, R_n k> depends only on m - n
    dots = [np.sum(o.rope(q, np.array([m]), 1e4) * o.rope(k, np.array([m - 5]), 1e4)) for m in (5, 40, 900)]
    assert np.allclose(dots, dots[0], rtol=1e-9)
    # complex-number form: z_i = x_i + j x_{i+hd/2} multiplied by exp(j pos theta^(-2i/hd))
    z = q[..., :half] + 1j * q[..., half:]
    w = z * np.exp(1j * 321 * 1e4 ** (-2 * np.arange(half) / hd))
    r = o.rope(q, np.array([321]), 1e4)
    assert np.allclose(r[..., :half], w.real) and np.allclose(r[..., half:], w.imag)


def test_silu_identities():
    z = np.linspace(-30, 30, 121)
    s = o.silu(z)
    assert o.silu(np.array([0.0]))[0] == 0
    assert np.allclose(s - o.silu(-z), z)                      # silu(x) - silu(-x) = x
    assert np.allclose(o.silu(np.array([40.0])), 40.0)
    assert abs(o.silu(np.array([1.0]))[0] - 1 / (1 + math.exp(-1))) < 1e-15


# ---------------------------------------------------------------- attention

def _attention_brute(q, k, v, q_pos):
    tq, nh, hd = q.shape
    out = np.zeros_like(q, dtype=np.float64)
    for t in range(tq):
        for h in range(nh):
            sc = [sum(q[t, h, e] * k[j, h, e] for e in range(hd)) / math.sqrt(hd) for j in range(q_pos[t] + 1)]
            m = max(sc)
            p = [math.exp(x - m) for x in sc]
            z = sum(p)
            for e in range(hd):
                out[t, h, e] = sum(p[j] * v[j, h, e] for j in range(len(p))) / z
    return out


@pytest.mark.parametrize("t,nh,hd", [(1, 1, 4), (5, 2, 4), (9, 3, 8), (16, 1, 16)])
def test_attention_brute_force(t, nh, hd):
    rng = np.random.default_rng(t * 100 + hd)
    q, k, v = (rng.standard_normal((t, nh, hd)) for _ in range(3))
    pos = np.arange(t)
    assert np.allclose(o.causal_attention(q, k, v, pos), _attention_brute(q, k, v, pos), atol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(5)
    k, v = rng.standard_normal((7, 2, 8)), rng.standard_normal((7, 2, 8))
    # a single key returns its value
    assert np.allclose(o.causal_attention(rng.standard_normal((1, 2, 8)), k[:1], v[:1], np.array([0])), v[:1])
    # q = 0 gives the mean of the visible values (causal prefix means)
    out = o.causal_attention(np.zeros((7, 2, 8)), k, v, np.arange(7))
    pref = np.cumsum(v, axis=0) / np.arange(1, 8)[:, None, None]
    assert np.allclose(out, pref)
    # a decode query at position p sees keys 0..p
    out = o.causal_attention(rng.standard_normal((1, 2, 8)), k, v, np.array([3]))
    out2 = o.causal_attention(out * 0 + 0, k[:4], v[:4], np.array([3]))
    assert np.allclose(out2[0], v[:4].mean(0))


# ---------------------------------------------------------------- whole block, brute force

def _tiny_cfg():
    return {"d_model": 8, "n_heads": 2, "head_dim": 4, "ffn": 16, "bits": 4, "group": 8,
            "eps": 1e-5, "rope_theta": 10000.0}


def _tiny_weights(seed):
    shape = syn.BlockShape(8, 2, 4, 16)
    w = syn.block_weights(shape, seed, "tiny")
    for k in list(w):
        if k.startswith("w_"):
            w[k] = (w[k] * 10).astype(np.float32)
    return w


def _block_brute(blk, h, pos0=0, kv_from_fp16_x=False):
    """One block by explicit loops over indices, from the dequantised weights.
    With kv_from_fp16_x, K and V are projected from the fp16 rounding of the
    normalised input (the store-h cache's stored rows), q from the input
    itself."""
    c = blk.cfg
    d, nh, hd, f = c["d_model"], c["n_heads"], c["head_dim"], c["ffn"]
    W = blk.W
    t = len(h)

    def norm(row, g):
        ms = sum(x * x for x in row) / d
        return [row[i] / math.sqrt(ms + c["eps"]) * g[i] for i in range(d)]

    def mv(m, x):
        return [sum(m[n][kk] * x[kk] for kk in range(len(x))) for n in range(len(m))]

    q = [[[0.0] * hd for _ in range(nh)] for _ in range(t)]
    k = [[[0.0] * hd for _ in range(nh)] for _ in range(t)]
    v = [[[0.0] * hd for _ in range(nh)] for _ in range(t)]
    for ti in range(t):
        x = norm(list(h[ti]), blk.gamma_attn)
        y = mv(W["qkv"], x)
        ykv = mv(W["qkv"], [float(np.float16(e)) for e in x]) if kv_from_fp16_x else y
        for hh in range(nh):
            for e in range(hd):
                q[ti][hh][e] = y[hh * hd + e]
                k[ti][hh][e] = ykv[d + hh * hd + e]
                v[ti][hh][e] = ykv[2 * d + hh * hd + e]
        for arr in (q, k):
            for hh in range(nh):
                vec = list(arr[ti][hh])
                for i in range(hd // 2):
                    a = (pos0 + ti) * c["rope_theta"] ** (-2.0 * i / hd)
                    arr[ti][hh][i] = vec[i] * math.cos(a) - vec[i + hd // 2] * math.sin(a)
                    arr[ti][hh][i + hd // 2] = vec[i + hd // 2] * math.cos(a) + vec[i] * math.sin(a)
    out = []
    for ti in range(t):
        att = []
        for hh in range(nh):
            sc = [sum(q[ti][hh][e] * k[j][hh][e] for e in range(hd)) / math.sqrt(hd) for j in range(ti + 1)]
            m = max(sc)
            p = [math.exp(s - m) for s in sc]
            z = sum(p)
            att += [sum(p[j] * v[j][hh][e] for j in range(ti + 1)) / z for e in range(hd)]
        o1 = mv(W["o"], att)
        r = [h[ti][i] + o1[i] for i in range(d)]
        x = norm(r, blk.gamma_ffn)
        g = mv(W["gate"], x)
        u = mv(W["up"], x)
        a = [g[i] / (1 + math.exp(-g[i])) * u[i] for i in range(f)]
        dn = mv(W["down"], a)
        out.append([r[i] + dn[i] for i in range(d)])
    return np.array(out)


def _apply_block(blk, h):
    pos = np.arange(len(h))
    q, k, v = blk.qkv(h, pos)
    return blk.finish(h, o.causal_attention(q, k, v, pos))


def test_block_brute_force():
    blk = o.Block.from_fp32(_tiny_weights(7), _tiny_cfg())
    h = np.random.default_rng(8).standard_normal((3, 8))
    assert np.allclose(_apply_block(blk, h), _block_brute(blk, h), atol=1e-12)


def test_zero_weights_block_is_identity():
    w = _tiny_weights(9)
    for k in list(w):
        if k.startswith("w_"):
            w[k] = np.zeros_like(w[k])
    blk = o.Block.from_fp32(w, _tiny_cfg())
    h = np.random.default_rng(10).standard_normal((4, 8))
    assert np.array_equal(_apply_block(blk, h), h)


# ---------------------------------------------------------------- model invariants

def _tiny_model(L_seed=11, n_pre=1):
    cfg = _tiny_cfg()
    pre = [o.Block.from_fp32(_tiny_weights(L_seed + i), cfg) for i in range(n_pre)]
    loop = o.Block.from_fp32(_tiny_weights(L_seed + 50), cfg)
    gam = 1 + 0.1 * np.random.default_rng(L_seed).standard_normal(8)
    emb = (np.random.default_rng(L_seed + 1).standard_normal((20, 8))).astype(np.float16)
    return o.LoopedModel(pre, loop, gam, emb)


def test_schedule_reuses_loop_block():
    m = _tiny_model()
    sched = m.schedule(5)
    assert len(sched) == 6 and all(b is m.loop for b in sched[1:])


def test_L_copies_equal_L_iterations():
    m = _tiny_model()
    ids = np.array([1, 5, 7, 2, 19])
    for L in (1, 3, 6):
        looped = m.prefill(ids, L)
        deep = o.unrolled_copy(m, L).prefill(ids, L)
        assert np.array_equal(looped, deep)


def test_cached_decode_matches_uncached_forward():
    m = _tiny_model()
    ids = np.array([3, 1, 4, 1, 5, 9, 2, 6, 5, 3])
    L = 3
    full = m.prefill(ids, L)
    kv = m.new_kv(L, "exact")
    m.prefill(ids[:4], L, kv=kv)
    for t in range(4, 10):
        y = m.decode_step(ids[t], L, kv)
        assert np.allclose(y, full[t], atol=1e-12)
    # with FP16 storage the cached path stays within the float tolerance
    kv16 = m.new_kv(L, "fp16")
    m.prefill(ids[:4], L, kv=kv16)
    for t in range(4, 10):
        y = m.decode_step(ids[t], L, kv16)
        cos = y @ full[t] / np.linalg.norm(y) / np.linalg.norm(full[t])
        assert cos > 0.9999


def test_per_lane_L_is_its_own_run():
    m = _tiny_model()
    ids = np.array([4, 8, 15, 16])
    outs = {}
    for L in (1, 2, 4):
        kv = m.new_kv(L, "fp16")
        m.prefill(ids, L, kv=kv)
        outs[L] = m.decode_step(np.int64(7), L, kv)
    assert not np.allclose(outs[1], outs[4])          # depth changes the result
    kv = m.new_kv(2, "fp16")
    m.prefill(ids, 2, kv=kv)
    assert np.array_equal(m.decode_step(np.int64(7), 2, kv), outs[2])


def test_kv_slot_count_is_pre_plus_L():
    m = _tiny_model(n_pre=2)
    kv = m.new_kv(5, "fp16")
    m.prefill(np.array([1, 2, 3]), 5, kv=kv)
    assert len(kv) == 7 and all(len(s) == 3 for s in kv)


# ---------------------------------------------------------------- planted mistakes

def _pins_pass():
    """Run the cheap pins; returns False if any fails."""
    checks = [test_block_brute_force, test_rope_hand_values, test_rope_properties,
              lambda: test_attention_brute_force(5, 2, 4), test_attention_special_cases,
              test_rmsnorm_closed_form, test_cached_decode_matches_uncached_forward,
              test_zero_weights_block_is_identity, test_dequantize_uses_group_of_each_column]
    for c in checks:
        try:
            c()
        except AssertionError:
            return False
    return True


def _mutants():
    orig_rope, orig_attn, orig_finish, orig_norm, orig_deq = (
        o.rope, o.causal_attention, o.Block.finish, o.rmsnorm, o.dequantize)

    def rope_sign(x, pos, theta):             # wrong sign of the sine term
        return orig_rope(x, -np.asarray(pos), theta)

    def rope_pairs(x, pos, theta):            # interleaved instead of rotate-half pairing
        y = np.asarray(x, float)
        hd = y.shape[-1]
        perm = np.concatenate([np.arange(0, hd, 2), np.arange(1, hd, 2)])
        inv = np.argsort(perm)
        return orig_rope(y[..., perm], pos, theta)[..., inv]

    def attn_no_mask(q, k, v, q_pos):         # causal mask dropped
        return orig_attn(q, k, v, np.full(len(q_pos), k.shape[0] - 1))

    def attn_no_scale(q, k, v, q_pos):        # 1/sqrt(hd) dropped
        return orig_attn(np.asarray(q) * math.sqrt(q.shape[-1]), k, v, q_pos)

    def finish_no_residual(self, h, attn):    # residual add dropped
        return orig_finish(self, h, attn) - h

    def finish_transposed_o(self, h, attn):   # W_o used transposed
        w = self.W["o"]
        self.W["o"] = w.T
        try:
            return orig_finish(self, h, attn)
        finally:
            self.W["o"] = w

    def norm_no_gain(h, gamma, eps):          # gain ignored
        return orig_norm(h, np.ones_like(gamma), eps)

    def norm_no_eps(h, gamma, eps):           # mean of squares replaced by mean of abs
        hh = np.asarray(h, float)
        return hh / np.mean(np.abs(hh), axis=-1, keepdims=True) * gamma

    def deq_wrong_group(codes, s, g):         # group index k % n_groups instead of k // g
        return codes.astype(float) * np.tile(s.astype(float), (1, codes.shape[1] // s.shape[1]))

    return [("rope", rope_sign), ("rope", rope_pairs), ("causal_attention", attn_no_mask),
            ("causal_attention", attn_no_scale), ("finish", finish_no_residual),
            ("finish", finish_transposed_o), ("rmsnorm", norm_no_gain), ("rmsnorm", norm_no_eps),
            ("dequantize", deq_wrong_group)]


@pytest.mark.parametrize("idx", range(9))
def test_planted_mistake_is_caught(monkeypatch, idx):
    """Each plausible mistake planted in the oracle makes at least one pin fail."""
    # the pins compare against brute force built on the (possibly mutated) Block
    # weights, so mutate the module-level functions the oracle itself calls
    name, fn = _mutants()[idx]
    if name == "finish":
        monkeypatch.setattr(o.Block, "finish", fn)
    else:
        monkeypatch.setattr(o, name, fn)
    assert not _pins_pass()


# ---------------------------------------------------------------- cached extend (verify pass)

def test_extend_equals_sequential_decode_steps():
    """n tokens in one cached call equal n single-token steps: the causal mask
    by absolute position and the append-then-attend order are the same."""
    m = _tiny_model()
    ids = np.array([3, 17, 5, 11, 0, 19, 8], np.int64)
    for dtype in ("exact", "fp16", "int8"):
        kv_a, kv_b = m.new_kv(3, dtype), m.new_kv(3, dtype)
        m.prefill(ids[:3], 3, kv=kv_a)
        m.prefill(ids[:3], 3, kv=kv_b)
        ya = m.extend(ids[3:], 3, kv_a)
        yb = np.stack([m.decode_step(np.int64(t), 3, kv_b) for t in ids[3:]])
        assert np.allclose(ya, yb, rtol=0, atol=1e-12), dtype
        for sa, sb in zip(kv_a, kv_b):
            assert len(sa) == len(sb) == len(ids)
            assert np.allclose(sa.k, sb.k, atol=1e-12) and np.allclose(sa.v, sb.v, atol=1e-12)


def test_extend_from_empty_exact_cache_is_the_uncached_forward():
    m = _tiny_model()
    ids = np.array([1, 2, 3, 4, 5, 6], np.int64)
    y = m.extend(ids, 2, m.new_kv(2, "exact"))
    assert np.allclose(y, m.prefill(ids, 2), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- per-iteration residual-norm exit

def test_exit_threshold_infinite_changes_nothing():
    m = _tiny_model()
    ids = np.array([4, 9, 13, 2], np.int64)
    info = {}
    a = m.prefill(ids, 4, exit_tau=float("inf"), info=info)
    assert np.array_equal(a, m.prefill(ids, 4))
    assert list(info["loops"]) == [4, 4, 4, 4]


def test_exit_threshold_zero_stops_after_the_first_iteration():
    """Every norm is above 0: each token keeps the stream of its first loop
    iteration, so the output is the L = 1 forward's."""
    m = _tiny_model()
    ids = np.array([4, 9, 13, 2, 7], np.int64)
    info = {}
    y = m.prefill(ids, 5, exit_tau=0.0, info=info)
    assert np.array_equal(y, m.prefill(ids, 1))
    assert list(info["loops"]) == [1] * 5


def test_exit_loop_counts_are_the_first_norm_crossings():
    """Before a token freezes its stream is the exit-free one, so its loop
    count is the first iteration j >= 1 whose input (the stream leaving
    iteration j - 1) has an L2 norm above the threshold; checked against the
    exit-free trace by brute force, with a threshold between the norms."""
    m = _tiny_model(n_pre=1)
    ids = np.array([4, 9, 13, 2, 7, 1, 18], np.int64)
    L = 6
    trace = []
    m.prefill(ids, L, trace=trace)
    norms = np.array([[math.sqrt(sum(x * x for x in row)) for row in trace[1 + j]] for j in range(L)])
    flat = np.sort(norms[:L - 1].ravel())
    tau = float((flat[len(flat) // 2] + flat[len(flat) // 2 + 1]) / 2)
    want = []
    for t in range(len(ids)):
        cross = [j for j in range(1, L) if norms[j - 1, t] > tau]
        want.append(cross[0] if cross else L)
    info = {}
    m.prefill(ids, L, exit_tau=tau, info=info)
    assert list(info["loops"]) == want
    assert 1 < len(set(want))          # the threshold splits the tokens


def test_exit_in_decode_equals_the_shallower_step():
    """A decode token frozen after j iterations outputs what a depth-j step
    from the same cache outputs (only its own stream reaches the output)."""
    m = _tiny_model()
    ids = np.array([3, 17, 5, 11], np.int64)
    L = 5
    for tau in (0.5, 2.0, 4.0, 1e9):
        kv = m.new_kv(L, "fp16")
        m.prefill(ids, L, kv=kv)
        snap = [(s.k.copy(), s.v.copy()) for s in kv]
        info = {}
        y = m.decode_step(np.int64(6), L, kv, exit_tau=tau, info=info)
        j = int(info["loops"][0])
        kv2 = m.new_kv(j, "fp16")
        for slot, (k, v) in zip(kv2, snap):
            slot.load_stored(k, v)
        assert np.array_equal(y, m.decode_step(np.int64(6), j, kv2)), tau


# ---------------------------------------------------------------- greedy head and self-speculative step

def test_greedy_head_brute_force():
    m = _tiny_model()
    y = np.random.default_rng(3).standard_normal((5, 8))
    E = m.embed16.astype(np.float64)
    for r in range(5):
        scores = [sum(y[r, i] * E[v, i] for i in range(8)) for v in range(E.shape[0])]
        assert m.greedy_head(y[r:r + 1])[0] == max(range(len(scores)), key=lambda v: (scores[v], -v))


def _spec_model():
    """The tiny model with its projections five times stronger, so that the
    block, not the token's own embedding, decides the greedy token: greedy
    decoding then moves between tokens and shallow drafts get rejected."""
    cfg = _tiny_cfg()

    def wts(seed):
        w = _tiny_weights(seed)
        return {k: ((v * 5).astype(np.float32) if k.startswith("w_") else v) for k, v in w.items()}
    pre = [o.Block.from_fp32(wts(11), cfg)]
    loop = o.Block.from_fp32(wts(61), cfg)
    gam = 1 + 0.1 * np.random.default_rng(11).standard_normal(8)
    emb = (np.random.default_rng(12).standard_normal((20, 8))).astype(np.float16)
    return o.LoopedModel(pre, loop, gam, emb)


@pytest.mark.parametrize("K,L_draft", [(1, 1), (3, 1), (4, 2), (7, 2), (3, 3)])
def test_spec_step_emits_the_greedy_decode_tokens(K, L_draft):
    """Greedy self-speculative decoding with an exact verify emits exactly the
    tokens greedy decoding at the verify depth emits, whatever the draft; a
    shallower draft gets some of its tokens rejected on the way, a draft at
    the verify depth none."""
    L = 3
    m = _spec_model()
    prompt = np.array([3, 17, 5, 11], np.int64)
    kv_s, kv_g = m.new_kv(L, "fp16"), m.new_kv(L, "fp16")
    m.prefill(prompt[:-1], L, kv=kv_s)
    m.prefill(prompt[:-1], L, kv=kv_g)
    tok, got, lens = int(prompt[-1]), [], []
    while len(got) < 12:
        out = m.spec_step(tok, K, L_draft, L, kv_s)
        assert 1 <= len(out) <= K + 1
        got += out
        lens.append(len(out))
        tok = out[-1]
        assert len(kv_s[0]) == len(prompt) - 1 + len(got)
    want = m.greedy_decode(int(prompt[-1]), len(got), L, kv_g)
    assert got == want
    assert len(set(want)) > 2                   # greedy decoding is not stuck on one token
    if L_draft < L:
        assert min(lens) < K + 1                # some draft was rejected
    else:                                       # the draft is the verify model: all accepted
        assert lens == [K + 1] * len(lens)


# ---------------------------------------------------------------- cross-iteration rounding (sign of frac)

def test_sign_of_frac_hand_worked():
    """One group of eight weights with absmax 3.5, so s = fp16(3.5 / 7) = 0.5
    exactly and w / s = 7, 2.4, -2.4, 0.52, -0.48, 0, 5.5, -6.5: codes round to
    nearest (ties to even), the bit says the quotient lies above its code, and
    odd iterations take the other neighbour."""
    w = np.array([[3.5, 1.2, -1.2, 0.26, -0.24, 0.0, 2.75, -3.25]], np.float32)
    codes, scales = o.quantize_groupwise(w, 4, 8)
    assert float(scales[0, 0]) == 0.5
    assert codes.tolist() == [[7, 2, -2, 1, 0, 0, 6, -6]]
    bits = o.sign_of_frac(w, 8)
    assert bits.tolist() == [[0, 1, 0, 0, 0, 0, 0, 0]]
    assert o.odd_iteration_codes(codes, bits).tolist() == [[6, 3, -3, 0, -1, -1, 5, -7]]


@pytest.mark.parametrize("group", [64, 128])
def test_odd_codes_bracket_the_quotient(group):
    rng = np.random.default_rng(21)
    w = (rng.standard_normal((16, 512)) * 0.02).astype(np.float32)
    w[3, :group] = 0.0                                     # an all-zero group: s = 0
    codes, scales = o.quantize_groupwise(w, 4, group)
    bits = o.sign_of_frac(w, group)
    odd = o.odd_iteration_codes(codes, bits)
    s = np.repeat(scales.astype(np.float32), group, axis=1)
    nz = s != 0
    r = (w[nz] / s[nz]).astype(np.float32)
    assert np.all(np.abs(odd[nz] - codes[nz]) == 1)
    assert np.all(np.minimum(codes[nz], odd[nz]) <= r) and np.all(r <= np.maximum(codes[nz], odd[nz]))
    assert not bits[~nz].any()
    # both roundings dequantise to zero in an all-zero group
    assert np.all(o.dequantize(odd, scales, group)[3, :group] == 0)


def test_bit_plane_layout():
    bits = np.zeros((2, 64), np.uint8)
    bits[0, 0] = bits[0, 33] = bits[1, 31] = 1
    words = o.pack_bits(bits)
    assert words.tolist() == [[1, 2], [1 << 31, 0]]
    assert np.array_equal(o.unpack_bits(words, 64), bits)


def _sign_model():
    cfg = _tiny_cfg()
    pre = [o.Block.from_fp32(_tiny_weights(31), cfg)]
    w = _tiny_weights(32)
    loop = o.Block(o.pack_block(w, 4, cfg["group"], sign=True), cfg)
    gam = 1 + 0.1 * np.random.default_rng(33).standard_normal(8)
    emb = (np.random.default_rng(34).standard_normal((20, 8))).astype(np.float16)
    return o.LoopedModel(pre, loop, gam, emb), w


def test_cross_iteration_rounding_model():
    m, w = _sign_model()
    ids = np.array([3, 9, 14, 2, 7], np.int64)
    base = {L: m.prefill(ids, L) for L in (1, 2, 3)}
    m.cross_iter = True
    assert np.array_equal(m.prefill(ids, 1), base[1])     # no odd iteration yet
    assert not np.allclose(m.prefill(ids, 2), base[2])
    # an unrolled stack: pre-block, loop, odd-weight loop, loop
    packed = o.pack_block(w, 4, m.loop.cfg["group"], sign=True)
    odd_blk = o.Block(packed, m.loop.cfg)
    odd_blk.W = odd_blk.W_odd
    plain = o.Block(o.pack_block(w, 4, m.loop.cfg["group"]), m.loop.cfg)
    deep = o.LoopedModel(m.pre + [plain, odd_blk], plain, m.gamma_final, m.embed16)
    assert np.allclose(m.prefill(ids, 3), deep.prefill(ids, 1), rtol=0, atol=1e-12)
    # without a sign channel the switch changes nothing
    m2 = _tiny_model()
    y = m2.prefill(ids, 3)
    m2.cross_iter = True
    assert np.array_equal(m2.prefill(ids, 3), y)


# ---------------------------------------------------------------- per-iteration weight variants

def test_iteration_variants_are_an_unrolled_stack():
    """Dual-bit weight swap ("Current Status", architecture-unique features
    table: a low-bit copy of the loop block for the early iterations, the
    higher-bit one later): with variants for iterations 0 and 1 the model is
    the unrolled stack pre, v0, v1, loop, loop; without variants, or with the
    loop block itself as the variant, nothing changes."""
    m = _tiny_model()
    ids = np.array([4, 1, 19, 7], np.int64)
    base = m.prefill(ids, 4)
    w = _tiny_weights(61)                        # the loop block's own weights at INT3
    cfg3 = dict(_tiny_cfg(), bits=3)
    low = o.Block.from_fp32(_tiny_weights(11 + 50), cfg3)
    other = o.Block.from_fp32(w, _tiny_cfg())
    m.iter_blocks = [low, other]
    got = m.prefill(ids, 4)
    deep = o.LoopedModel(m.pre + [low, other, m.loop], m.loop, m.gamma_final, m.embed16)
    assert np.allclose(got, deep.prefill(ids, 1), rtol=0, atol=1e-12)
    assert not np.allclose(got, base)
    m.iter_blocks = [None, m.loop]
    assert np.array_equal(m.prefill(ids, 4), base)
    m.iter_blocks = [low] * 6                    # variants past L are never reached
    assert np.allclose(m.prefill(ids, 2),
                       o.LoopedModel(m.pre + [low], low, m.gamma_final, m.embed16).prefill(ids, 1),
                       rtol=0, atol=1e-12)


# ---------------------------------------------------------------- store-h KV

def test_store_h_decode_brute_force():
    """Store-h ("Current Status", KV cache mode table, Store-h rows): a
    one-block model caches the fp16 rows x of each position; a decode step
    rebuilds every position's K and V from them.  Against explicit loops over
    the whole sequence with K, V projected from fp16(x) (q from x itself)."""
    cfg = _tiny_cfg()
    blk = o.Block.from_fp32(_tiny_weights(71), cfg)
    gam = 1 + 0.1 * np.random.default_rng(72).standard_normal(8)
    m = o.LoopedModel([], blk, gam)
    h = np.random.default_rng(73).standard_normal((6, 8))
    kv = m.new_kv(1, "h")
    m.prefill(h[:5], 1, kv=kv)
    tr = []
    m.decode_step(h[5], 1, kv, trace=tr)
    want = _block_brute(blk, h, kv_from_fp16_x=True)[5]
    assert np.allclose(tr[0][0], want, rtol=0, atol=1e-12)
    # the rounding of x is what the mode stores: the exact-cache result differs
    kv_exact = m.new_kv(1, "exact")
    m.prefill(h[:5], 1, kv=kv_exact)
    tr_exact = []
    m.decode_step(h[5], 1, kv_exact, trace=tr_exact)
    assert np.allclose(tr_exact[0][0], _block_brute(blk, h)[5], rtol=0, atol=1e-12)
    assert not np.array_equal(tr[0][0], tr_exact[0][0])
    assert np.allclose(tr[0][0], tr_exact[0][0], rtol=0, atol=1e-2)
    # the slot holds d fp16 values per position (K and V would take 2d)
    assert kv[0]._x.dtype == np.float16 and kv[0]._x[:kv[0].n].shape == (6, 8)


def test_store_h_cross_iteration_uses_odd_weights():
    """An odd loop iteration's slot rebuilds K and V with that iteration's
    weights."""
    m, w = _sign_model()
    m.cross_iter = True
    ids = np.array([2, 5, 8, 13], np.int64)
    kv_h, kv_e = m.new_kv(2, "h"), m.new_kv(2, "exact")
    m.prefill(ids[:3], 2, kv=kv_h)
    m.prefill(ids[:3], 2, kv=kv_e)
    a = m.decode_step(ids[3], 2, kv_h)
    b = m.decode_step(ids[3], 2, kv_e)
    assert np.allclose(a, b, rtol=0, atol=5e-2)
    for layer in (1, 2):
        k_h = kv_h[layer].k
        x16 = kv_h[layer]._x[:4].astype(np.float64)
        _, k_want, _ = (m.loop.qkv_from_x(x16, np.arange(4), odd=(layer == 2)))
        assert np.array_equal(k_h, k_want), layer


# ---------------------------------------------------------------- planted mistakes, loop variants

def _variant_pins_pass():
    """The pins of cross-iteration rounding, the iteration variants, store-h
    and the residual-norm check; returns False if any fails."""
    checks = [test_sign_of_frac_hand_worked, lambda: test_odd_codes_bracket_the_quotient(64),
              test_bit_plane_layout, test_cross_iteration_rounding_model,
              test_iteration_variants_are_an_unrolled_stack, test_store_h_decode_brute_force,
              test_store_h_cross_iteration_uses_odd_weights, test_exit_threshold_infinite_changes_nothing,
              test_exit_threshold_zero_stops_after_the_first_iteration,
              test_exit_loop_counts_are_the_first_norm_crossings]
    for c in checks:
        try:
            c()
        except AssertionError:
            return False
    return True


def _variant_mutants():
    orig_sof, orig_odd_codes, orig_pack_bits = o.sign_of_frac, o.odd_iteration_codes, o.pack_bits

    def sof_ties_up(w, group, bits=4):            # a quotient equal to its code counts as above
        w = np.asarray(w, np.float32)
        codes, s16 = o.quantize_groupwise(w, bits, group)
        s = np.repeat(s16.astype(np.float32), group, axis=1)
        with np.errstate(divide="ignore", invalid="ignore"):
            r = (w / s).astype(np.float32)
        return ((s != 0) & (r >= codes.astype(np.float32))).astype(np.uint8)

    def sof_inverted(w, group, bits=4):           # the bit says the rounding went up
        return (1 - orig_sof(w, group, bits)).astype(np.uint8)

    def odd_codes_swapped(codes, bits):           # -1 where set, +1 where clear
        return orig_odd_codes(codes, 1 - (np.asarray(bits) != 0))

    def pack_bits_reversed(bits):                 # element 32j + i in bit 31 - i
        b = np.asarray(bits)
        n, k = b.shape
        nw = (k + 31) // 32
        b = np.concatenate([b, np.zeros((n, nw * 32 - k), b.dtype)], axis=1).reshape(n, nw, 32)
        return orig_pack_bits(b[:, :, ::-1].reshape(n, nw * 32))

    def odd_even_parity(self, layer):             # even loop iterations take the odd weights
        it = layer - len(self.pre)
        return self.cross_iter and it >= 0 and it % 2 == 0

    def schedule_no_variants(self, L):            # the variants ignored
        return self.pre + [self.loop] * L

    def exit_check_from_zero(self, h, layer, frozen, loops, exit_tau):   # also before iteration 0
        it = layer - len(self.pre)
        if exit_tau is None or it < 0:
            return
        newly = ~frozen & (np.sqrt(np.sum(h * h, axis=-1)) > exit_tau)
        loops[newly] = it
        frozen |= newly

    def exit_count_plus_one(self, h, layer, frozen, loops, exit_tau):    # loop count off by one
        it = layer - len(self.pre)
        if exit_tau is None or it < 1:
            return
        newly = ~frozen & (np.sqrt(np.sum(h * h, axis=-1)) > exit_tau)
        loops[newly] = it + 1
        frozen |= newly

    def append_x_unrounded(self, x, blk, odd):    # store-h rows kept in fp64
        x = np.asarray(x, np.float64)
        self._x = x if self._x is None else np.concatenate([self._x[:self.n], x])
        self._blk, self._odd = blk, odd
        self.n += x.shape[0]

    def rebuild_even_weights(self):               # odd iterations rebuilt with the even weights
        _, k, v = self._blk.qkv_from_x(self._x[:self.n].astype(np.float64), np.arange(self.n), False)
        return k, v

    return [("sign_of_frac", sof_ties_up), ("sign_of_frac", sof_inverted),
            ("odd_iteration_codes", odd_codes_swapped), ("pack_bits", pack_bits_reversed),
            ("LoopedModel.odd", odd_even_parity), ("LoopedModel.schedule", schedule_no_variants),
            ("LoopedModel._exit_check", exit_check_from_zero),
            ("LoopedModel._exit_check", exit_count_plus_one),
            ("KVSlot.append_x", append_x_unrounded), ("KVSlot._rebuild", rebuild_even_weights)]


def test_variant_pins_pass_unmutated():
    assert _variant_pins_pass()


@pytest.mark.parametrize("idx", range(10))
def test_planted_variant_mistake_is_caught(monkeypatch, idx):
    """Each plausible mistake planted in the oracle's cross-iteration rounding,
    iteration variants, store-h cache or residual-norm check makes at least
    one of their pins fail."""
    name, fn = _variant_mutants()[idx]
    if "." in name:
        cls, attr = name.split(".")
        monkeypatch.setattr(getattr(o, cls), attr, fn)
    else:
        monkeypatch.setattr(o, name, fn)
    assert not _variant_pins_pass()



# ---------------------------------------------------------------- planted mistakes, speculative step

def _spec_pins_pass():
    checks = [test_greedy_head_brute_force, lambda: test_spec_step_emits_the_greedy_decode_tokens(3, 1),
              lambda: test_spec_step_emits_the_greedy_decode_tokens(4, 2),
              lambda: test_spec_step_emits_the_greedy_decode_tokens(3, 3)]
    for c in checks:
        try:
            c()
        except AssertionError:
            return False
    return True


def _spec_step_with(accept_mismatch: bool, keep: int):
    """The self-speculative step with one planted mistake: accept the first
    mismatching draft too, or keep `keep` entries fewer in the cache."""
    def spec_step(self, token, K, L_draft, L_verify, kv):
        p = len(kv[0])
        drafts, t = [], token
        for _ in range(K):
            t = int(self.greedy_head(self.decode_step(np.int64(t), L_draft, kv))[0])
            drafts.append(t)
        for slot in kv:
            slot.truncate(p)
        ver = [int(v) for v in self.greedy_head(self.extend(np.array([token] + drafts, np.int64),
                                                            L_verify, kv))]
        m = 0
        while m < K and drafts[m] == ver[m]:
            m += 1
        if accept_mismatch and m < K:
            m += 1
        for slot in kv:
            slot.truncate(p + m + 1 - keep)
        return drafts[:m] + [ver[m]]
    return spec_step


@pytest.mark.parametrize("mutant", ["argmin_head", "accept_mismatch", "cache_short"])
def test_planted_spec_mistake_is_caught(monkeypatch, mutant):
    """Each plausible mistake planted in the greedy head or the speculative
    step makes at least one of their pins fail."""
    assert _spec_pins_pass()
    if mutant == "argmin_head":
        def head(self, y):
            logits = np.asarray(y, np.float64).reshape(-1, self.cfg["d_model"]) @ self.embed16.astype(np.float64).T
            return np.argmin(logits, axis=-1)
        monkeypatch.setattr(o.LoopedModel, "greedy_head", head)
    elif mutant == "accept_mismatch":
        monkeypatch.setattr(o.LoopedModel, "spec_step", _spec_step_with(True, 0))
    else:
        monkeypatch.setattr(o.LoopedModel, "spec_step", _spec_step_with(False, 1))
    assert not _spec_pins_pass()


# ---------------------------------------------------------------- planted mistakes, integer outputs

_HAND = [(4, [0.7, -0.35, 0.1, 0, 0.2499, -0.7, 0.05, 0.35], 0x2E66, [7, -4, 1, 0, 2, -7, 1, 4]),
         (4, [7, 2.5, -2.5, 3.5, -0.5, 0.5, 1.5, 0], 0x3C00, [7, 2, -2, 4, 0, 0, 2, 0]),
         (3, [3, 1.5, -1.5, 2.5, -0.5, 0.5, -3, 0], 0x3C00, [3, 2, -2, 2, 0, 0, -3, 0]),
         (3, [-0.3, 0.1, 0.05, 0, 0, 0, 0, 0], 0x2E66, [-3, 1, 1, 0, 0, 0, 0, 0])]


def _integer_pins_pass():
    """The pins of the bit-exact outputs: quantisers, word layouts, INT8 KV."""
    checks = [lambda h=h: test_quantize_hand_worked(*h) for h in _HAND]
    checks += [test_pack_layout_int4_nibble_order, test_pack_layout_int3_ten_per_word,
               lambda: test_quantize_properties(4, 64), lambda: test_quantize_properties(3, 128),
               test_kv_int8_hand_worked, test_kv_int8_properties]
    for c in checks:
        try:
            c()
        except AssertionError:
            return False
    return True


def _quantizer(scale_fn, round_fn, qmax_of):
    """quantize_groupwise with its scale and rounding steps replaceable."""
    def q(w, bits, group):
        w = np.asarray(w, np.float32)
        n, k = w.shape
        qmax = np.float32(qmax_of(bits))
        g = w.reshape(n, k // group, group)
        absmax = np.max(np.abs(g), axis=2)
        scale16 = (absmax / qmax).astype(np.float32).astype(np.float16)
        s = scale_fn(absmax, qmax, scale16)[:, :, None]
        with np.errstate(divide="ignore", invalid="ignore"):
            ratio = (g / s).astype(np.float32)
        ratio = np.where(s == 0, np.float32(0), ratio)
        codes = np.clip(round_fn(ratio), -qmax - 1, qmax).astype(np.int8)
        return codes.reshape(n, k), scale16
    return q


def _kv_quantizer(div, use_rounded):
    def q(x16):
        x = np.asarray(x16, np.float16).astype(np.float32)
        absmax = np.max(np.abs(x), axis=-1)
        scale16 = (absmax / np.float32(div)).astype(np.float32).astype(np.float16)
        s = (scale16.astype(np.float32) if use_rounded else (absmax / np.float32(127)))[..., None]
        with np.errstate(divide="ignore", invalid="ignore"):
            ratio = (x / s).astype(np.float32)
        ratio = np.where(s == 0, np.float32(0), ratio)
        return np.clip(np.rint(ratio), -127, 127).astype(np.int8), scale16
    return q


def _integer_mutants():
    rounded = lambda absmax, qmax, s16: s16.astype(np.float32)               # noqa: E731
    unrounded = lambda absmax, qmax, s16: (absmax / qmax).astype(np.float32)  # noqa: E731
    half_away = lambda r: np.sign(r) * np.floor(np.abs(r) + np.float32(0.5))   # noqa: E731
    orig_pack = o.pack_codes

    def pack_high_nibble_first(codes, bits):
        if bits != 4:
            return orig_pack(codes, bits)
        c = np.asarray(codes).reshape(codes.shape[0], -1, 8)[:, :, ::-1]
        return orig_pack(c.reshape(codes.shape), bits)

    def pack_int3_zero_padding(codes, bits):
        words = orig_pack(codes, bits)
        if bits != 3:
            return words
        k = codes.shape[1]
        w = words.astype(np.uint64)
        for slot in range(k, words.shape[1] * 10):     # clear the padding slots (u = 4 -> 0)
            j, i = divmod(slot, 10)
            w[:, j] &= ~np.uint64(7 << (3 * i))
        return w.astype(np.uint32)

    return [("quantize_groupwise", _quantizer(unrounded, np.rint, o.QMAX.get)),
            ("quantize_groupwise", _quantizer(rounded, half_away, o.QMAX.get)),
            ("quantize_groupwise", _quantizer(rounded, np.rint, lambda b: o.QMAX[b] + 1)),
            ("pack_codes", pack_high_nibble_first), ("pack_codes", pack_int3_zero_padding),
            ("kv_quant_int8", _kv_quantizer(128, True)), ("kv_quant_int8", _kv_quantizer(127, False))]


def test_integer_pins_pass_unmutated():
    assert _integer_pins_pass()


@pytest.mark.parametrize("idx", range(7))
def test_planted_integer_mistake_is_caught(monkeypatch, idx):
    """Each plausible mistake planted in a quantiser or a word layout (the
    unrounded scale, round half away from zero, the wrong level count, the
    nibble order, the INT3 padding code, the INT8 divisor, the unrounded INT8
    scale) makes at least one pin of the bit-exact outputs fail."""
    name, fn = _integer_mutants()[idx]
    monkeypatch.setattr(o, name, fn)
    assert not _integer_pins_pass()
