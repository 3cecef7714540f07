"""Oracle models for the named synthetic workloads (test infrastructure only).

Weights come from ``synthetic`` (fp32 N(0, 0.02)); quantisation, packing and
dequantisation are the oracle's own (readings R1, R2 of tinyloop_oracle)."""
from __future__ import annotations

import functools
from typing import Dict, List

import synthetic as syn
from . import tinyloop_oracle as o


@functools.lru_cache(maxsize=8)
def packed_weights(workload_name: str) -> Dict[str, Dict]:
    """{block name: packed dict} for a workload, quantised by the oracle."""
    w = syn.WORKLOADS[workload_name]
    out = {}
    for i, name in enumerate(syn.block_names(w)):
        bits = w.bits_loop if name == "loop" else w.bits_pre
        out[name] = o.pack_block(syn.block_weights(w.shape, w.seed, name), bits, w.group)
    return out


@functools.lru_cache(maxsize=4)
def build_oracle_model(workload_name: str) -> o.LoopedModel:
    w = syn.WORKLOADS[workload_name]
    packed = packed_weights(workload_name)
    blocks: List[o.Block] = []
    for name in syn.block_names(w):
        bits = w.bits_loop if name == "loop" else w.bits_pre
        blocks.append(o.Block(packed[name], o.block_cfg(w.shape, bits, w.group, w.eps, w.rope_theta)))
    embed = syn.embedding(w.shape, w.seed) if w.input_kind == "ids" else None
    return o.LoopedModel(blocks[:-1], blocks[-1], syn.final_gain(w.shape, w.seed), embed)
