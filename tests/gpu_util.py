"""Helpers shared by the GPU parity tests: build device models from the seeded
synthetic weights (packed on the GPU by tl_pack_weights) and compare tensors."""
from __future__ import annotations

import functools

import numpy as np
import torch

import synthetic as syn
from oracle import tinyloop_oracle as o
from oracle.workloads import build_oracle_model, packed_weights
from weight_shared_looped_b200.model import DeviceBlock, DeviceModel

# float tolerances of the hot path: per block output and final hidden state
BLOCK_REL_L2 = 5e-3
FINAL_COSINE = 0.999


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def cosine(a, b) -> float:
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / np.linalg.norm(a) / np.linalg.norm(b))


def row_cosines(a, b) -> np.ndarray:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return (a * b).sum(-1) / np.linalg.norm(a, axis=-1) / np.linalg.norm(b, axis=-1)


def block_cfg(w: syn.Workload, name: str):
    bits = w.bits_loop if name == "loop" else w.bits_pre
    return o.block_cfg(w.shape, bits, w.group, w.eps, w.rope_theta)


def device_blocks(workload: str, check_packing: bool = True):
    """Blocks packed on the GPU from the fp32 synthetic weights; packing is
    checked bit for bit against the oracle's packing of the same weights."""
    w = syn.WORKLOADS[workload]
    ref = packed_weights(workload) if check_packing else None
    blocks = {}
    for name in syn.block_names(w):
        cfg = block_cfg(w, name)
        blk = DeviceBlock(cfg, weights=syn.block_weights(w.shape, w.seed, name))
        if check_packing:
            for m in ("qkv", "o", "gate", "up", "down"):
                got_w = blk.t[f"w_{m}"].cpu().numpy().view(np.uint32)
                got_s = blk.t[f"s_{m}"].cpu().numpy().view(np.uint16)
                assert np.array_equal(got_w, ref[name][f"w_{m}"]), (name, m)
                assert np.array_equal(got_s, ref[name][f"s_{m}"].view(np.uint16)), (name, m)
        blocks[name] = blk
    return blocks


def device_model(workload: str, *, max_tokens: int, max_lanes: int = 1, max_ctx: int = 0,
                 max_L: int = 64, blocks=None) -> DeviceModel:
    w = syn.WORKLOADS[workload]
    blocks = blocks or device_blocks(workload)
    names = syn.block_names(w)
    embed = syn.embedding(w.shape, w.seed) if w.input_kind == "ids" else None
    m = DeviceModel([blocks[n] for n in names[:-1]], blocks["loop"],
                    syn.final_gain(w.shape, w.seed), embed, max_tokens=max_tokens,
                    max_lanes=max_lanes, max_ctx=max_ctx, max_L=max_L)
    m._blocks = blocks
    return m


def oracle_model(workload: str):
    return build_oracle_model(workload)


def to_dev(x, dtype):
    if dtype == torch.float16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda()
    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype).cuda()
