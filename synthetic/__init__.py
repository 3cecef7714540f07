"""Seeded synthetic inputs for the looped-block hot path.

This module is the only code shared by the CPU oracle tests, the GPU parity
tests and the benchmark.  It draws random numbers and names workloads; it holds
none of the method's arithmetic (no quantisation, no normalisation, no
attention).  Every tensor gets its own generator stream, keyed by the run seed
and the tensor's name, so that any tensor can be regenerated on its own.

Generator: numpy's PCG64 seeded through SeedSequence([seed, crc32(name)]).
Normals come from ``Generator.standard_normal(dtype=float32)``.

Workload shapes follow the TinyLoop pages:
  * the forward order (embed, a few pre-blocks, one shared block run L times,
    final norm) is "TinyLoop Framework", list under the opening paragraph;
  * the 407M-shaped model (2 pre-blocks + 1 loop block, d 2048, 16 heads,
    ffn 8192, L=8, seq 128, no logits) is "Performance and Memory",
    "Benchmark Shape Matters" and the "FP16 body cache" table;
  * INT8 KV per (token, head) with one FP16 scale is "Performance and Memory",
    "KV cache INT8" table;
  * INT3 (8 levels, 10 values per 32-bit word) is "Current Status", core
    inference table, INT3 GEMM row;
  * per-lane loop counts [4, 16, 32] are "Current Status", architecture-unique
    features table, L-aware batching row.
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Dict, List, Optional, Tuple

import numpy as np

VOCAB = 50257


def _gen(seed: int, name: str) -> np.random.Generator:
    key = zlib.crc32(name.encode("utf-8"))
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), key])))


def normal(shape, std: float, seed: int, name: str) -> np.ndarray:
    """fp32 N(0, std^2) samples of the given shape."""
    z = _gen(seed, name).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        z *= np.float32(std)
    return z


def token_ids(n: int, seed: int, name: str, vocab: int = VOCAB) -> np.ndarray:
    """int32 token ids uniform over [0, vocab)."""
    return _gen(seed, name).integers(0, vocab, size=n, dtype=np.int64).astype(np.int32)


def gain(d: int, seed: int, name: str) -> np.ndarray:
    """Norm gains 1 + 0.1 N(0,1): far enough from 1 that a kernel ignoring the
    gain fails parity."""
    return (np.float32(1.0) + normal((d,), 0.1, seed, name)).astype(np.float32)


@dataclasses.dataclass(frozen=True)
class BlockShape:
    d_model: int
    n_heads: int
    head_dim: int
    ffn: int


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload.  ``bits_pre``/``bits_loop`` are the weight
    bit-widths of the pre-blocks and of the shared loop block."""
    name: str
    shape: BlockShape
    n_pre: int
    group: int
    bits_pre: int
    bits_loop: int
    L: Tuple[int, ...]          # one loop count per lane
    seq: int                    # prefill tokens (prompt length for decode workloads)
    steps: int                  # decode steps (0 = prefill only)
    kv_dtype: str               # "fp16" | "int8" | "none"
    input_kind: str             # "hidden" (fp16 N(0,1) hidden states) | "ids"
    max_ctx: int
    eps: float = 1e-5
    rope_theta: float = 10000.0
    seed: int = 0


SHAPE_TINY = BlockShape(256, 4, 64, 768)
SHAPE_407M = BlockShape(2048, 16, 128, 8192)

WORKLOADS: Dict[str, Workload] = {
    # tiny looped block, FP32-checkable
    "tiny": Workload("tiny", SHAPE_TINY, n_pre=0, group=64, bits_pre=4, bits_loop=4,
                     L=(2,), seq=16, steps=0, kv_dtype="none", input_kind="hidden",
                     max_ctx=16),
    # the tiny block with an INT3 loop block (10 codes per word, group 64)
    "tiny_int3": Workload("tiny_int3", SHAPE_TINY, n_pre=0, group=64, bits_pre=4, bits_loop=3,
                          L=(2,), seq=16, steps=0, kv_dtype="none", input_kind="hidden",
                          max_ctx=16),
    # 407M-shaped prefill, seq 128, L=8, no logits
    "prefill407m": Workload("prefill407m", SHAPE_407M, n_pre=2, group=128, bits_pre=4,
                            bits_loop=4, L=(8,), seq=128, steps=0, kv_dtype="none",
                            input_kind="ids", max_ctx=128),
    # KV-cached decode: 256-token prompt then 128 teacher-forced steps, FP16 KV
    "decode407m": Workload("decode407m", SHAPE_407M, n_pre=2, group=128, bits_pre=4,
                           bits_loop=4, L=(8,), seq=256, steps=128, kv_dtype="fp16",
                           input_kind="ids", max_ctx=384),
    # long-context batched decode, static batch 8, ctx 2048, INT8 KV, 64 steps
    "longctx_int8": Workload("longctx_int8", SHAPE_407M, n_pre=2, group=128, bits_pre=4,
                             bits_loop=4, L=(8,) * 8, seq=2048, steps=64, kv_dtype="int8",
                             input_kind="ids", max_ctx=2048 + 64),
    # mixed-depth batched decode, INT3 loop block, lanes L=[4,16,32], ctx 1024
    "mixed_int3": Workload("mixed_int3", SHAPE_407M, n_pre=2, group=128, bits_pre=4,
                           bits_loop=3, L=(4, 16, 32), seq=1024, steps=32, kv_dtype="fp16",
                           input_kind="ids", max_ctx=1024 + 32),
}


def block_names(w: Workload) -> List[str]:
    return [f"pre{i}" for i in range(w.n_pre)] + ["loop"]


def block_weights(shape: BlockShape, seed: int, block: str) -> Dict[str, np.ndarray]:
    """fp32 weights of one transformer block, N(0, 0.02) for the matrices.

    Matrices are [out_features, in_features].  ``w_qkv`` rows are ordered
    [Q; K; V], head-major inside each third."""
    d, f = shape.d_model, shape.ffn
    return {
        "w_qkv": normal((3 * d, d), 0.02, seed, f"{block}.w_qkv"),
        "w_o": normal((d, d), 0.02, seed, f"{block}.w_o"),
        "w_gate": normal((f, d), 0.02, seed, f"{block}.w_gate"),
        "w_up": normal((f, d), 0.02, seed, f"{block}.w_up"),
        "w_down": normal((d, f), 0.02, seed, f"{block}.w_down"),
        "gamma_attn": gain(d, seed, f"{block}.gamma_attn"),
        "gamma_ffn": gain(d, seed, f"{block}.gamma_ffn"),
    }


def final_gain(shape: BlockShape, seed: int) -> np.ndarray:
    return gain(shape.d_model, seed, "final.gamma")


def embedding(shape: BlockShape, seed: int, vocab: int = VOCAB) -> np.ndarray:
    """fp16 [vocab, d_model] embedding table, N(0, 0.02)."""
    return normal((vocab, shape.d_model), 0.02, seed, "embed").astype(np.float16)


def hidden_input(w: Workload, n_tokens: Optional[int] = None, name: str = "h_in") -> np.ndarray:
    """fp16 N(0,1) input hidden states [n_tokens, d_model]."""
    t = w.seq if n_tokens is None else n_tokens
    return normal((t, w.shape.d_model), 1.0, w.seed, name).astype(np.float16)


def prompt_ids(w: Workload, lane: int = 0) -> np.ndarray:
    return token_ids(w.seq, w.seed, f"prompt.lane{lane}")


def decode_ids(w: Workload, lane: int = 0) -> np.ndarray:
    """Teacher-forced ids for the decode steps of one lane."""
    return token_ids(w.steps, w.seed, f"decode.lane{lane}")


def context_hidden(w: Workload, slot: int, lane: int = 0) -> np.ndarray:
    """fp32 N(0,1) hidden states from which a synthetic long-context KV slot is
    derived (the long-context INT8 workload)."""
    return normal((w.seq, w.shape.d_model), 1.0, w.seed, f"ctx.lane{lane}.slot{slot}")
