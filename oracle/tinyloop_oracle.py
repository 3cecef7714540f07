"""CPU oracle for the weight-shared looped-block hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only the tests, the smoke check and the benchmark's CPU-baseline leg may call
it.  It shares no code with the CUDA library; the only module both sides use
is ``synthetic`` (seeded random inputs, no arithmetic of the method).

What it computes, in the order the TinyLoop pages give it ("TinyLoop
Framework", the four-step list of the architectural family): embed tokens, run
the pre-blocks once each, run the one shared loop block L times with the same
weights, then normalise.  No output head ("Performance and Memory",
"Benchmark Shape Matters": no logits materialisation).

Precision
  * Floating-point math is fp64 (numpy float64, BLAS matmul as a library
    step).  The pages make the FP32 residual stream the default ("Current
    Status", core inference table, FP16 residual-stream row: FP16 is opt-in);
    fp64 is at least that precise.
  * Wherever floating point decides an integer (a weight code, an FP16 scale,
    an INT8 KV code) the decision is taken in IEEE fp32 exactly as written
    below, so that codes are comparable bit for bit with any implementation
    that follows the same reading.
  * Storage precisions the pages fix are modelled: the FP16 KV cache rounds K
    and V to fp16; the INT8 KV cache stores int8 codes with one fp16 scale per
    (token, head) ("Performance and Memory", "KV cache INT8" table and the
    sentence under it).

Readings where the pages are silent (each is repeated in the design notes):
  R1  INT4 group-wise symmetric: s = fp16(absmax/7), code = clamp(rint(w/s),
      -8, 7) with w/s an fp32 division by the fp16-rounded scale; s = 0 gives
      code 0.  Stored offset-binary u = code + 8, eight per uint32 word, the
      element with the lowest k in the lowest nibble.
  R2  INT3 ("8 levels, 3 bits/weight, 10 values per 32-bit word", "Current
      Status", INT3 GEMM row): s = fp16(absmax/3), code in [-4, 3], u =
      code + 4 at bits 3i of word k//10 (i = k % 10), bits 30-31 zero, row
      padded to a multiple of 4 words with u = 4 (code 0) in unused slots.
  R3  INT8 KV: s = fp16(max|x|/127) over one head's hd values of one token,
      code = clamp(rint(x/s), -127, 127), x the fp16 value the FP16 cache
      would hold; dequantised value code * s.
  R4  RoPE rotate-half: pairs (i, i + hd/2), angle = pos * theta^(-2i/hd),
      applied to q and k; K is cached after RoPE.
  R5  Fused QKV rows [Q; K; V], head-major; separate gate and up matrices;
      SwiGLU = silu(gate) * up; no biases; pre-norm RMSNorm with gain.
  R6  Prefill attention uses the call's own K/V; the cache keeps them in its
      storage dtype for later decode steps, which attend over the stored
      values (including the entry just appended).
"""
from __future__ import annotations

import copy
from typing import Dict, List, Optional, Sequence

import numpy as np

F64 = np.float64

# --------------------------------------------------------------------------
# Weight quantisation and packing (readings R1, R2)
# --------------------------------------------------------------------------

QMAX = {4: 7, 3: 3}


def quantize_groupwise(w: np.ndarray, bits: int, group: int):
    """Group-wise symmetric quantisation along K of an fp32 [N, K] matrix.

    Returns (codes int8 [N, K], scales fp16 [N, K/group]).  Every step is an
    fp32 operation: absmax (exact), absmax / qmax rounded to fp32 then to fp16
    (round to nearest even), w / float(scale) rounded to fp32, then rint
    (ties to even) and clamp."""
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    assert k % group == 0
    qmax = np.float32(QMAX[bits])
    g = w.reshape(n, k // group, group)
    absmax = np.max(np.abs(g), axis=2)
    scale16 = (absmax / qmax).astype(np.float32).astype(np.float16)
    s = scale16.astype(np.float32)[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = (g / s).astype(np.float32)
    ratio = np.where(s == 0, np.float32(0), ratio)
    codes = np.clip(np.rint(ratio), -qmax - 1, qmax).astype(np.int8)
    return codes.reshape(n, k), scale16


def int3_words_per_row(k: int) -> int:
    """uint32 words per packed INT3 row: ceil(K/10) rounded up to 4 words."""
    w = (k + 9) // 10
    return (w + 3) // 4 * 4


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Pack int8 codes [N, K] into uint32 words (readings R1, R2)."""
    codes = np.asarray(codes, dtype=np.int64)
    n, k = codes.shape
    if bits == 4:
        assert k % 8 == 0
        u = (codes + 8).reshape(n, k // 8, 8)
        word = np.zeros((n, k // 8), dtype=np.uint64)
        for i in range(8):
            word |= u[:, :, i].astype(np.uint64) << np.uint64(4 * i)
        return word.astype(np.uint32)
    if bits == 3:
        nw = int3_words_per_row(k)
        u = np.full((n, nw * 10), 4, dtype=np.int64)    # padding slots hold code 0
        u[:, :k] = codes + 4
        u = u.reshape(n, nw, 10)
        word = np.zeros((n, nw), dtype=np.uint64)
        for i in range(10):
            word |= u[:, :, i].astype(np.uint64) << np.uint64(3 * i)
        return word.astype(np.uint32)
    raise ValueError("bits must be 3 or 4")


def unpack_codes(packed: np.ndarray, k: int, bits: int) -> np.ndarray:
    """Inverse of pack_codes: uint32 words -> int8 codes [N, K]."""
    packed = np.asarray(packed, dtype=np.uint64)
    n = packed.shape[0]
    if bits == 4:
        out = np.zeros((n, packed.shape[1], 8), dtype=np.int64)
        for i in range(8):
            out[:, :, i] = (packed >> np.uint64(4 * i)) & np.uint64(15)
        return (out.reshape(n, -1)[:, :k] - 8).astype(np.int8)
    if bits == 3:
        out = np.zeros((n, packed.shape[1], 10), dtype=np.int64)
        for i in range(10):
            out[:, :, i] = (packed >> np.uint64(3 * i)) & np.uint64(7)
        return (out.reshape(n, -1)[:, :k] - 4).astype(np.int8)
    raise ValueError("bits must be 3 or 4")


def sign_of_frac(w: np.ndarray, group: int, bits: int = 4) -> np.ndarray:
    """The 1-bit sign-of-frac channel of group-wise quantised weights
    ("Performance and Memory", "Cross-iteration stochastic rounding": INT4 +
    1-bit sign-of-frac, +25 % storage; "Current Status", architecture-unique
    features table, deterministic error cancellation row: even iterations use
    the standard rounding, odd iterations apply the sign correction).
    bit[n, k] = 1 when w / s lies above its code (the rounding went down), else
    0; with the same fp32 quotient as quantize_groupwise.  Returns uint8 [N, K]."""
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    codes, scale16 = quantize_groupwise(w, bits, group)
    s = np.repeat(scale16.astype(np.float32), group, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = (w / s).astype(np.float32)
    return ((s != 0) & (ratio > codes.astype(np.float32))).astype(np.uint8)


def pack_bits(bits: np.ndarray) -> np.ndarray:
    """[N, K] bits -> uint32 [N, ceil(K/32)]; element 32j + i in bit i of word j
    (bits past K are zero)."""
    b = np.asarray(bits, dtype=np.uint64)
    n, k = b.shape
    nw = (k + 31) // 32
    b = np.concatenate([b, np.zeros((n, nw * 32 - k), np.uint64)], axis=1).reshape(n, nw, 32)
    word = np.zeros((n, nw), dtype=np.uint64)
    for i in range(32):
        word |= b[:, :, i] << np.uint64(i)
    return word.astype(np.uint32)


def unpack_bits(words: np.ndarray, k: int) -> np.ndarray:
    w = np.asarray(words, dtype=np.uint64)
    out = np.zeros((w.shape[0], w.shape[1], 32), dtype=np.uint8)
    for i in range(32):
        out[:, :, i] = (w >> np.uint64(i)) & np.uint64(1)
    return out.reshape(w.shape[0], -1)[:, :k]


def odd_iteration_codes(codes: np.ndarray, bits: np.ndarray) -> np.ndarray:
    """The codes an odd loop iteration uses: each moved to its other rounding
    neighbour, code + 1 where the bit is set, code - 1 where it is clear (so the
    two neighbours bracket w / s; a code exactly equal to w / s moves down).
    May leave the storage range by one (-9 .. 8): it is an arithmetic value,
    never stored."""
    return codes.astype(np.int16) + np.where(np.asarray(bits) != 0, 1, -1).astype(np.int16)


def dequantize(codes: np.ndarray, scales16: np.ndarray, group: int) -> np.ndarray:
    """W[n, k] = code[n, k] * float(scale[n, k // group]), in fp64 (exact)."""
    s = np.repeat(scales16.astype(F64), group, axis=1)
    return codes.astype(F64) * s


# --------------------------------------------------------------------------
# INT8 KV quantisation (reading R3)
# --------------------------------------------------------------------------

def kv_quant_int8(x16: np.ndarray):
    """Per-row symmetric INT8 of fp16 rows [rows, hd]: one fp16 scale per row,
    scale = max|x| / 127 ("Performance and Memory", "KV cache INT8")."""
    x = np.asarray(x16, dtype=np.float16).astype(np.float32)
    absmax = np.max(np.abs(x), axis=-1)
    scale16 = (absmax / np.float32(127.0)).astype(np.float32).astype(np.float16)
    s = scale16.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = (x / s).astype(np.float32)
    ratio = np.where(s == 0, np.float32(0), ratio)
    codes = np.clip(np.rint(ratio), -127, 127).astype(np.int8)
    return codes, scale16


def kv_dequant_int8(codes: np.ndarray, scale16: np.ndarray) -> np.ndarray:
    return codes.astype(F64) * scale16.astype(F64)[..., None]


# --------------------------------------------------------------------------
# Byte sizes (closed forms the pages' memory numbers pin)
# --------------------------------------------------------------------------

def kv_cache_bytes(n_layers: int, max_seq: int, n_heads: int, head_dim: int, kv_dtype: str) -> int:
    """K and V for every layer (each pre-block and each loop iteration keeps
    its own slot).  INT8 adds one fp16 scale per (token, head) for K and V."""
    elems = 2 * n_layers * max_seq * n_heads * head_dim
    if kv_dtype == "fp16":
        return 2 * elems
    if kv_dtype == "int8":
        return elems + 2 * (2 * n_layers * max_seq * n_heads)
    raise ValueError(kv_dtype)


def block_weight_count(d: int, ffn: int) -> int:
    """Weights of one block: QKV (3d x d), O (d x d), gate and up (ffn x d
    each), down (d x ffn)."""
    return 3 * d * d + d * d + 2 * ffn * d + d * ffn


def packed_block_bytes(d: int, ffn: int, bits: int, group: int) -> int:
    """Packed bytes (codes + fp16 scales) of one block."""
    total = 0
    for n, k in ((3 * d, d), (d, d), (ffn, d), (ffn, d), (d, ffn)):
        words = k // 8 if bits == 4 else int3_words_per_row(k)
        total += n * words * 4 + n * (k // group) * 2
    return total


# --------------------------------------------------------------------------
# Elementwise / normalisation / rotary / attention (fp64)
# --------------------------------------------------------------------------

def rmsnorm(h: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """y = h / sqrt(mean(h^2) + eps) * gamma, per row."""
    h = np.asarray(h, dtype=F64)
    ms = np.mean(h * h, axis=-1, keepdims=True)
    return h / np.sqrt(ms + eps) * np.asarray(gamma, dtype=F64)


def rope_angles(positions: np.ndarray, head_dim: int, theta: float) -> np.ndarray:
    """angle[p, i] = pos_p * theta^(-2i/hd) for i < hd/2 (reading R4)."""
    i = np.arange(head_dim // 2, dtype=F64)
    inv_freq = theta ** (-2.0 * i / head_dim)
    return np.asarray(positions, dtype=F64)[:, None] * inv_freq[None, :]


def rope(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half RoPE of x [T, H, hd] at absolute positions [T]."""
    x = np.asarray(x, dtype=F64)
    hd = x.shape[-1]
    half = hd // 2
    ang = rope_angles(positions, hd, theta)[:, None, :]      # [T, 1, hd/2]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def causal_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, q_pos: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(hd)) v per head, query at absolute position q_pos[t]
    seeing keys 0..q_pos[t].  q [Tq, H, hd], k/v [Tk, H, hd] with key j at
    position j.  Max-subtracted softmax in fp64."""
    q = np.asarray(q, F64)
    k = np.asarray(k, F64)
    v = np.asarray(v, F64)
    tq, n_heads, hd = q.shape
    tk = k.shape[0]
    scores = np.einsum("thd,jhd->htj", q, k) / np.sqrt(hd)           # [H, Tq, Tk]
    mask = np.arange(tk)[None, :] <= np.asarray(q_pos)[:, None]       # [Tq, Tk]
    scores = np.where(mask[None], scores, -np.inf)
    scores = scores - scores.max(axis=-1, keepdims=True)
    p = np.exp(scores)
    p = p / p.sum(axis=-1, keepdims=True)
    return np.einsum("htj,jhd->thd", p, v)


# --------------------------------------------------------------------------
# Blocks, KV storage and the looped model
# --------------------------------------------------------------------------

class Block:
    """One transformer block from its packed form: codes are unpacked to
    integers and dequantised to fp64 once."""

    def __init__(self, packed: Dict[str, np.ndarray], cfg: Dict):
        self.cfg = dict(cfg)
        d, f, g, bits = cfg["d_model"], cfg["ffn"], cfg["group"], cfg["bits"]
        shapes = {"qkv": (3 * d, d), "o": (d, d), "gate": (f, d), "up": (f, d), "down": (d, f)}
        self.W = {}
        self.W_odd = None
        for name, (n, k) in shapes.items():
            codes = unpack_codes(packed[f"w_{name}"], k, bits)
            self.W[name] = dequantize(codes, packed[f"s_{name}"], g)
            if f"sign_{name}" in packed:
                # the cross-iteration rounding channel: odd loop iterations'
                # weights (odd_iteration_codes x the same scales)
                if self.W_odd is None:
                    self.W_odd = {}
                odd = odd_iteration_codes(codes, unpack_bits(packed[f"sign_{name}"], k))
                self.W_odd[name] = dequantize(odd, packed[f"s_{name}"], g)
        self.gamma_attn = np.asarray(packed["gamma_attn"], F64)
        self.gamma_ffn = np.asarray(packed["gamma_ffn"], F64)

    @classmethod
    def from_fp32(cls, weights: Dict[str, np.ndarray], cfg: Dict) -> "Block":
        return cls(pack_block(weights, cfg["bits"], cfg["group"]), cfg)

    def weights(self, odd: bool = False) -> Dict[str, np.ndarray]:
        """The weights of a loop iteration: the odd-iteration set when asked for
        and present, else the standard one."""
        return self.W_odd if odd and self.W_odd is not None else self.W

    def x_in(self, h: np.ndarray) -> np.ndarray:
        """The input of the QKV projection: RMSNorm(h) * gamma_attn."""
        return rmsnorm(h, self.gamma_attn, self.cfg["eps"])

    def qkv_from_x(self, x: np.ndarray, positions: np.ndarray, odd: bool = False):
        """QKV projection of x -> RoPE on q and k."""
        c = self.cfg
        t = x.shape[0]
        qkv = x @ self.weights(odd)["qkv"].T
        d, nh, hd = c["d_model"], c["n_heads"], c["head_dim"]
        q = qkv[:, :d].reshape(t, nh, hd)
        k = qkv[:, d:2 * d].reshape(t, nh, hd)
        v = qkv[:, 2 * d:].reshape(t, nh, hd)
        return rope(q, positions, c["rope_theta"]), rope(k, positions, c["rope_theta"]), v

    def qkv(self, h: np.ndarray, positions: np.ndarray, odd: bool = False):
        """RMSNorm -> QKV projection -> RoPE on q and k."""
        return self.qkv_from_x(self.x_in(h), positions, odd)

    def finish(self, h: np.ndarray, attn: np.ndarray, odd: bool = False) -> np.ndarray:
        """O projection + residual, then RMSNorm -> SwiGLU MLP + residual."""
        c = self.cfg
        t = h.shape[0]
        W = self.weights(odd)
        h = h + attn.reshape(t, c["d_model"]) @ W["o"].T
        x = rmsnorm(h, self.gamma_ffn, c["eps"])
        u = silu(x @ W["gate"].T) * (x @ W["up"].T)
        return h + u @ W["down"].T


def pack_block(weights: Dict[str, np.ndarray], bits: int, group: int,
               sign: bool = False) -> Dict[str, np.ndarray]:
    """Quantise and pack the five matrices of one block (with the 1-bit
    sign-of-frac channel of each when `sign`)."""
    out = {}
    for name in ("qkv", "o", "gate", "up", "down"):
        codes, scales = quantize_groupwise(weights[f"w_{name}"], bits, group)
        out[f"w_{name}"] = pack_codes(codes, bits)
        out[f"s_{name}"] = scales
        if sign:
            out[f"sign_{name}"] = pack_bits(sign_of_frac(weights[f"w_{name}"], group, bits))
    out["gamma_attn"] = weights["gamma_attn"]
    out["gamma_ffn"] = weights["gamma_ffn"]
    return out


class KVSlot:
    """K/V of one layer (one pre-block or one loop iteration) for one lane, in
    the cache's storage dtype: "fp16", "int8", "exact" (fp64, used only to
    check the cached path against the uncached one without storage rounding)
    or "h".  Stored values are kept dequantised, positions 0..len-1.

    "h" is the store-h mode ("Current Status", KV cache mode table, Store-h
    (FP16) and tensor-core reconstruction rows; "Claims & Data Sources", the
    h-mode KV reconstruction from shared W_k / W_v row).  Reading: the slot
    keeps, per position, the fp16 rounding of the input the layer's QKV
    projection reads (x = RMSNorm(h) * gamma_attn: d values instead of the 2d
    of K and V); K and V are rebuilt from those rows with the layer's own
    W_k, W_v and RoPE whenever they are read, with no further rounding."""

    def __init__(self, dtype: str):
        self.dtype = dtype
        self._k: Optional[np.ndarray] = None
        self._v: Optional[np.ndarray] = None
        self.n = 0
        self._x: Optional[np.ndarray] = None   # "h": the stored fp16 input rows
        self._blk: Optional["Block"] = None
        self._odd = False

    def _store(self, x: np.ndarray) -> np.ndarray:
        if self.dtype == "exact":
            return np.asarray(x, F64)
        x16 = np.asarray(x, F64).astype(np.float16)
        if self.dtype == "fp16":
            return x16.astype(F64)
        if self.dtype == "int8":
            codes, scale = kv_quant_int8(x16)
            return kv_dequant_int8(codes, scale)
        raise ValueError(self.dtype)

    def _reserve(self, n: int, shape) -> None:
        if self._k is None or self._k.shape[0] < n:
            cap = max(n, 2 * (0 if self._k is None else self._k.shape[0]), 16)
            k = np.empty((cap,) + tuple(shape), F64)
            v = np.empty((cap,) + tuple(shape), F64)
            if self._k is not None:
                k[:self.n] = self._k[:self.n]
                v[:self.n] = self._v[:self.n]
            self._k, self._v = k, v

    def append(self, k: np.ndarray, v: np.ndarray) -> None:
        """Append T positions: k, v [T, H, hd], stored in the cache dtype."""
        t = k.shape[0]
        self._reserve(self.n + t, k.shape[1:])
        self._k[self.n:self.n + t] = self._store(k)
        self._v[self.n:self.n + t] = self._store(v)
        self.n += t

    def load_stored(self, k_values: np.ndarray, v_values: np.ndarray) -> None:
        """Set the slot to already-stored (dequantised) values [T, H, hd]."""
        self._k = self._v = None
        self.n = 0
        self._reserve(k_values.shape[0] + 64, k_values.shape[1:])
        self._k[:k_values.shape[0]] = k_values
        self._v[:v_values.shape[0]] = v_values
        self.n = k_values.shape[0]

    def append_x(self, x: np.ndarray, blk: "Block", odd: bool) -> None:
        """Store-h: append T input rows x [T, d] (kept as fp16), to be projected
        by `blk` (odd-iteration weights when `odd`)."""
        x16 = np.asarray(x, F64).astype(np.float16)
        self._x = x16 if self._x is None else np.concatenate([self._x[:self.n], x16])
        self._blk, self._odd = blk, odd
        self.n += x16.shape[0]

    def _rebuild(self):
        _, k, v = self._blk.qkv_from_x(self._x[:self.n].astype(F64), np.arange(self.n), self._odd)
        return k, v

    def truncate(self, n: int) -> None:
        """Keep positions 0..n-1 (entries past them are dropped)."""
        self.n = min(self.n, n)

    @property
    def k(self) -> np.ndarray:
        if self.dtype == "h":
            return self._rebuild()[0]
        return self._k[:self.n]

    @property
    def v(self) -> np.ndarray:
        if self.dtype == "h":
            return self._rebuild()[1]
        return self._v[:self.n]

    def __len__(self) -> int:
        return self.n


class LoopedModel:
    """embed -> pre-blocks once each -> loop block L times -> final RMSNorm."""

    def __init__(self, pre: Sequence[Block], loop: Block, gamma_final: np.ndarray,
                 embed16: Optional[np.ndarray] = None):
        self.pre = list(pre)
        self.loop = loop
        self.gamma_final = np.asarray(gamma_final, F64)
        self.embed16 = embed16
        self.cfg = loop.cfg
        self.cross_iter = False   # odd loop iterations use the loop block's odd weights
        # per-iteration weight variants ("Current Status", architecture-unique
        # features table, dual-bit and triple-bit weight swap rows): loop
        # iteration i < len(iter_blocks) runs iter_blocks[i] (None: the loop block)
        self.iter_blocks: List[Optional[Block]] = []

    def odd(self, layer: int) -> bool:
        """Whether layer `layer` is an odd loop iteration run with the odd
        weights (cross-iteration rounding on, and the loop block has them)."""
        it = layer - len(self.pre)
        return self.cross_iter and it >= 0 and it % 2 == 1

    def schedule(self, L: int) -> List[Block]:
        """Block applied at each layer index: the pre-blocks, then the same
        loop block object L times (weights shared, not copied), except the
        iterations given a variant."""
        its = [self.iter_blocks[i] if i < len(self.iter_blocks) and self.iter_blocks[i] is not None
               else self.loop for i in range(L)]
        return self.pre + its

    def embed(self, ids: np.ndarray) -> np.ndarray:
        return self.embed16[np.asarray(ids)].astype(F64)

    def _exit_check(self, h: np.ndarray, layer: int, frozen: np.ndarray, loops: np.ndarray,
                    exit_tau: Optional[float]) -> None:
        """Per-iteration safety check ("Current Status", architecture-unique
        features table, per-iteration safety check row: the residual stream's
        L2 norm is computed every iteration and the loop stops above a
        threshold, L checkpoints per token).  Reading: the check looks at the
        residual stream leaving each loop iteration; a token whose norm exceeds
        the threshold runs no further residual updates (its stream is frozen,
        and the later iterations' K/V slots receive what the frozen stream
        produces); its loop count is the iterations it ran."""
        it = layer - len(self.pre)          # the loop iteration about to run
        if exit_tau is None or it < 1:
            return
        norms = np.sqrt(np.sum(h * h, axis=-1))
        newly = ~frozen & (norms > exit_tau)
        loops[newly] = it
        frozen |= newly

    def prefill(self, x_in: np.ndarray, L: int, kv: Optional[List[KVSlot]] = None,
                trace: Optional[List[np.ndarray]] = None, exit_tau: Optional[float] = None,
                info: Optional[dict] = None) -> np.ndarray:
        """Causal forward over T tokens at positions 0..T-1.  ``x_in`` is int ids
        [T] or hidden states [T, d].  With ``kv`` (one KVSlot per layer) the
        K/V of every layer are appended.  ``trace`` receives the residual
        stream after every block application.  ``exit_tau`` enables the
        per-iteration residual-norm check (``info["loops"]`` receives each
        token's loop count).  Returns the final-norm output."""
        x_in = np.asarray(x_in)
        h = self.embed(x_in) if x_in.ndim == 1 else x_in.astype(F64)
        pos = np.arange(h.shape[0])
        frozen = np.zeros(h.shape[0], bool)
        loops = np.full(h.shape[0], L)
        for layer, blk in enumerate(self.schedule(L)):
            self._exit_check(h, layer, frozen, loops, exit_tau)
            odd = self.odd(layer)
            q, k, v = blk.qkv(h, pos, odd)
            if kv is not None:
                if kv[layer].dtype == "h":
                    kv[layer].append_x(blk.x_in(h), blk, odd)
                else:
                    kv[layer].append(k, v)
            h = np.where(frozen[:, None], h, blk.finish(h, causal_attention(q, k, v, pos), odd))
            if trace is not None:
                trace.append(h.copy())
        if info is not None:
            info["loops"] = loops
        return rmsnorm(h, self.gamma_final, self.cfg["eps"])

    def extend(self, x_in, L: int, kv: List[KVSlot], trace: Optional[List[np.ndarray]] = None,
               exit_tau: Optional[float] = None, info: Optional[dict] = None) -> np.ndarray:
        """Cached forward of n tokens of one lane at positions p .. p+n-1, p =
        len(kv[0]) (the verify pass of self-speculative decode: "Current
        Status", speculative and adaptive decode table, self-speculative row:
        L=2 draft, L=8 verify, same weights).  Every layer appends the n
        tokens' K/V in the cache's storage dtype, then each token attends over
        the stored entries up to its own position.  ``x_in``: ids [n] or
        hidden states [n, d].  Returns the final-norm outputs [n, d]."""
        x_in = np.asarray(x_in)
        h = self.embed(x_in) if x_in.ndim == 1 else x_in.reshape(-1, self.cfg["d_model"]).astype(F64)
        pos = np.arange(len(kv[0]), len(kv[0]) + h.shape[0])
        frozen = np.zeros(h.shape[0], bool)
        loops = np.full(h.shape[0], L)
        for layer, blk in enumerate(self.schedule(L)):
            self._exit_check(h, layer, frozen, loops, exit_tau)
            odd = self.odd(layer)
            q, k, v = blk.qkv(h, pos, odd)
            slot = kv[layer]
            if slot.dtype == "h":
                slot.append_x(blk.x_in(h), blk, odd)
            else:
                slot.append(k, v)
            h = np.where(frozen[:, None], h,
                         blk.finish(h, causal_attention(q, slot.k, slot.v, pos), odd))   # keys 0..pos
            if trace is not None:
                trace.append(h.copy())
        if info is not None:
            info["loops"] = loops
        return rmsnorm(h, self.gamma_final, self.cfg["eps"])

    def decode_step(self, x_in, L: int, kv: List[KVSlot],
                    trace: Optional[List[np.ndarray]] = None, exit_tau: Optional[float] = None,
                    info: Optional[dict] = None) -> np.ndarray:
        """One cached decode step for one lane at position len(kv[0]): append
        this token's K/V to every layer's slot, attend over the stored
        entries.  Returns the final-norm output [d]."""
        x_in = np.asarray(x_in)
        x1 = x_in.reshape(1) if x_in.ndim == 0 else x_in.reshape(1, -1)
        return self.extend(x1, L, kv, trace=trace, exit_tau=exit_tau, info=info)[0]

    def greedy_head(self, y: np.ndarray) -> np.ndarray:
        """Greedy next tokens from final-norm outputs y [n, d] through the tied
        embedding (logits = y . E^T, the head a self-speculative step needs to
        compare draft and verify tokens); the lowest id wins a tie."""
        logits = np.asarray(y, F64).reshape(-1, self.cfg["d_model"]) @ self.embed16.astype(F64).T
        return np.argmax(logits, axis=-1)

    def greedy_decode(self, token: int, n: int, L: int, kv: List[KVSlot]) -> List[int]:
        """n greedy decode steps at depth L from the input token `token`;
        returns the n generated tokens."""
        out = []
        for _ in range(n):
            token = int(self.greedy_head(self.decode_step(np.int64(token), L, kv))[0])
            out.append(token)
        return out

    def spec_step(self, token: int, K: int, L_draft: int, L_verify: int,
                  kv: List[KVSlot]) -> List[int]:
        """One greedy self-speculative step with one weight set and one cache
        ("TinyLoop Framework", "What Makes It Different": draft and verify
        reuse the same weights; "Current Status", self-speculative row: L=2
        draft, L=8 verify).  From the input token x at position p:
          draft   K decode steps at L_draft: d_1 .. d_K (each the greedy head
                  of the previous step's output; they write positions
                  p .. p+K-1 of the first n_pre + L_draft slots);
          verify  rewind to p, extend [x, d_1 .. d_K] at L_verify (positions
                  p .. p+K of every slot), greedy head: v_1 .. v_{K+1};
          accept  m = the longest prefix with d_i == v_i; the emitted tokens
                  are d_1 .. d_m, v_{m+1}; the cache keeps positions up to
                  p + m (the entries past it are dropped).
        The emitted tokens equal m + 1 greedy decode steps at L_verify."""
        p = len(kv[0])
        drafts, t = [], token
        for _ in range(K):
            t = int(self.greedy_head(self.decode_step(np.int64(t), L_draft, kv))[0])
            drafts.append(t)
        for slot in kv:
            slot.truncate(p)
        y = self.extend(np.array([token] + drafts, np.int64), L_verify, kv)
        ver = [int(v) for v in self.greedy_head(y)]
        m = 0
        while m < K and drafts[m] == ver[m]:
            m += 1
        for slot in kv:
            slot.truncate(p + m + 1)
        return drafts[:m] + [ver[m]]

    def new_kv(self, L: int, dtype: str) -> List[KVSlot]:
        return [KVSlot(dtype) for _ in range(len(self.pre) + L)]


def derive_context_kv(block: Block, h: np.ndarray, dtype=np.float32):
    """Synthetic long-context cache entries for one layer: hidden states h
    [T, d] go through the block's RMSNorm, K and V projections and RoPE at
    positions 0..T-1, are rounded to fp16 and INT8-quantised per (token, head).
    Returns (k_codes, k_scales, v_codes, v_scales) with codes int8 [T, H, hd]
    and scales fp16 [T, H].  ``dtype`` is the float type of this input
    synthesis; the codes are inputs to both sides, not an expected value."""
    c = block.cfg
    d, nh, hd = c["d_model"], c["n_heads"], c["head_dim"]
    t = h.shape[0]
    x = rmsnorm(h, block.gamma_attn, c["eps"]).astype(dtype)
    wk = block.W["qkv"][d:2 * d].astype(dtype)
    wv = block.W["qkv"][2 * d:].astype(dtype)
    k = (x @ wk.T).reshape(t, nh, hd)
    v = (x @ wv.T).reshape(t, nh, hd)
    k = rope(k, np.arange(t), c["rope_theta"])
    kc, ks = kv_quant_int8(k.astype(np.float16))
    vc, vs = kv_quant_int8(v.astype(np.float16))
    return kc, ks, vc, vs


def unrolled_copy(model: LoopedModel, L: int) -> LoopedModel:
    """A plain deep stack of n_pre + L distinct block objects, each holding its
    own copy of the weights it would share in the looped model."""
    blocks = [copy.deepcopy(b) for b in model.pre] + [copy.deepcopy(model.loop) for _ in range(L)]
    deep = LoopedModel(blocks, model.loop, model.gamma_final, model.embed16)
    deep.schedule = lambda _L: blocks        # type: ignore[assignment]
    return deep


def block_cfg(shape, bits: int, group: int, eps: float = 1e-5, rope_theta: float = 10000.0) -> Dict:
    return {"d_model": shape.d_model, "n_heads": shape.n_heads, "head_dim": shape.head_dim,
            "ffn": shape.ffn, "bits": bits, "group": group, "eps": eps, "rope_theta": rope_theta}
