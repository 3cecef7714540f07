"""Device-side model handle: owns the PyTorch device buffers that the C library
references (packed weights, scales, gains, embedding, KV storage) and wraps
the tl_* calls.  Packing runs on the GPU through tl_pack_weights; nothing here
computes any part of the forward."""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

from . import (TL_KV_FP16, TL_KV_INT8, TL_KV_H, tl_block_create, tl_block_destroy, tl_decode_step,
               tl_kv_bytes, tl_kv_create, tl_kv_destroy, tl_kv_layer_ptrs, tl_kv_position,
               tl_kv_reset, tl_kv_set_position, tl_model_create, tl_model_destroy,
               tl_model_device_bytes, tl_model_set_decode_chunks, tl_model_set_graphs,
               tl_pack_weights, tl_packed_bytes, tl_prefill, tl_sync_status, tl_extend,
               tl_greedy_head, tl_spec_step, tl_model_set_exit_threshold, tl_loops_used,
               tl_sign_bits_bytes, tl_pack_sign_bits, tl_model_set_cross_iter,
               tl_model_set_iteration_blocks)

MATRICES = ("qkv", "o", "gate", "up", "down")


def _dev(x, dtype=None, device="cuda"):
    t = torch.as_tensor(np.ascontiguousarray(x)) if isinstance(x, np.ndarray) else x
    if dtype is not None:
        t = t.to(dtype)
    return t.to(device).contiguous()


class DeviceBlock:
    """One block packed on the device from fp32 weights (or from canonical
    packed words and scales).  With `sign` (fp32 weights) or sign_* arrays in
    `packed`, the block also carries the sign-of-frac bits of cross-iteration
    rounding."""

    def __init__(self, cfg: Dict, weights: Optional[Dict] = None, packed: Optional[Dict] = None,
                 stream=None, sign: bool = False):
        self.cfg = dict(cfg)
        self.t: Dict[str, torch.Tensor] = {}
        bits, group = cfg["bits"], cfg["group"]
        for name in MATRICES:
            if packed is not None:
                self.t[f"w_{name}"] = _dev(packed[f"w_{name}"].view(np.int32), torch.int32)
                self.t[f"s_{name}"] = _dev(packed[f"s_{name}"].view(np.int16), torch.int16)
                if f"sign_{name}" in packed:
                    self.t[f"sign_{name}"] = _dev(packed[f"sign_{name}"].view(np.int32), torch.int32)
            else:
                w = _dev(weights[f"w_{name}"], torch.float32)
                n, k = w.shape
                cb, sb = tl_packed_bytes(n, k, bits, group)
                pw = torch.empty(cb // 4, dtype=torch.int32, device="cuda")
                ps = torch.empty(sb // 2, dtype=torch.int16, device="cuda")
                tl_pack_weights(w, bits, group, pw, ps, stream)
                self.t[f"w_{name}"] = pw.view(n, -1)
                self.t[f"s_{name}"] = ps.view(n, -1)
                if sign:
                    sg = torch.empty(tl_sign_bits_bytes(n, k) // 4, dtype=torch.int32, device="cuda")
                    tl_pack_sign_bits(w, bits, group, ps, sg, stream)
                    self.t[f"sign_{name}"] = sg.view(n, -1)
                del w
        src = packed if packed is not None else weights
        self.t["gamma_attn"] = _dev(src["gamma_attn"], torch.float32)
        self.t["gamma_ffn"] = _dev(src["gamma_ffn"], torch.float32)
        torch.cuda.synchronize()
        self.handle = tl_block_create(self.cfg, self.t)

    def close(self):
        if self.handle:
            tl_block_destroy(self.handle)
            self.handle = 0


class DeviceModel:
    def __init__(self, pre: Sequence[DeviceBlock], loop: DeviceBlock, gamma_final,
                 embed=None, *, max_tokens: int, max_lanes: int = 1, max_ctx: int = 0,
                 max_L: int = 64):
        self.pre, self.loop = list(pre), loop
        self.cfg = loop.cfg
        self.gamma_final = _dev(gamma_final, torch.float32)
        self.embed = None if embed is None else _dev(np.asarray(embed).view(np.int16), torch.int16)
        vocab = 0 if embed is None else self.embed.shape[0]
        self.max_ctx = max(max_ctx, max_tokens)
        self.handle = tl_model_create([b.handle for b in self.pre], loop.handle, self.embed, vocab,
                                      self.gamma_final, max_tokens, max_lanes, self.max_ctx, max_L)
        self.d = self.cfg["d_model"]

    def device_bytes(self) -> int:
        return tl_model_device_bytes(self.handle)

    def set_graphs(self, on: bool) -> None:
        tl_model_set_graphs(self.handle, on)

    def set_decode_chunks(self, chunks_per_cta: int) -> None:
        """Context chunks one decode-attention CTA streams (0 = automatic)."""
        tl_model_set_decode_chunks(self.handle, chunks_per_cta)

    def set_cross_iter(self, on: bool) -> None:
        """Cross-iteration rounding: odd loop iterations take the other rounding
        neighbour of every loop-block weight (needs a loop block with sign bits)."""
        tl_model_set_cross_iter(self.handle, on)

    def set_iteration_blocks(self, blocks: Sequence[Optional[DeviceBlock]]) -> None:
        """Per-iteration weight variants: loop iteration i < len(blocks) runs
        blocks[i] (None keeps the loop block)."""
        tl_model_set_iteration_blocks(self.handle, [b.handle if b else None for b in blocks])
        self._iter_blocks = list(blocks)   # referenced by the library: keep them alive

    def set_exit_threshold(self, tau: float) -> None:
        """Per-iteration residual-norm check threshold (< 0: off)."""
        tl_model_set_exit_threshold(self.handle, tau)

    def loops_used(self, n: int):
        return tl_loops_used(self.handle, n)

    def new_kv(self, L_per_lane: Sequence[int], max_ctx: int, dtype: str = "fp16") -> "DeviceKV":
        return DeviceKV(self, L_per_lane, max_ctx, dtype)

    def prefill(self, ids=None, h_in=None, *, L: int, kv: "DeviceKV" = None, lane: int = 0,
                y_out=None, h_trace=None, stream=None) -> torch.Tensor:
        x = ids if ids is not None else h_in
        seq = x.shape[0]
        if y_out is None:
            y_out = torch.empty(seq, self.d, dtype=torch.float32, device="cuda")
        tl_prefill(self.handle, ids, h_in, L=L, y_out=y_out, kv=kv.handle if kv else None,
                   lane=lane, h_trace=h_trace, stream=stream)
        return y_out

    def decode(self, kv: "DeviceKV", ids=None, h_in=None, *, L_per_lane: Sequence[int],
               y_out=None, h_trace=None, stream=None) -> torch.Tensor:
        n = len(L_per_lane)
        if y_out is None:
            y_out = torch.empty(n, self.d, dtype=torch.float32, device="cuda")
        tl_decode_step(self.handle, kv.handle, ids, h_in, L_per_lane=L_per_lane, y_out=y_out,
                       h_trace=h_trace, stream=stream)
        return y_out

    def extend(self, kv: "DeviceKV", ids=None, h_in=None, *, lane: int = 0, L: int, y_out=None,
               h_trace=None, stream=None) -> torch.Tensor:
        n = (ids if ids is not None else h_in).shape[0]
        if y_out is None:
            y_out = torch.empty(n, self.d, dtype=torch.float32, device="cuda")
        tl_extend(self.handle, kv.handle, lane, ids, h_in, L=L, y_out=y_out, h_trace=h_trace,
                  stream=stream)
        return y_out

    def greedy_head(self, y, stream=None) -> torch.Tensor:
        ids = torch.empty(y.shape[0], dtype=torch.int32, device="cuda")
        tl_greedy_head(self.handle, y, ids, stream=stream)
        return ids

    def spec_step(self, kv: "DeviceKV", token: int, *, lane: int = 0, K: int, L_draft: int,
                  L_verify: int, stream=None):
        return tl_spec_step(self.handle, kv.handle, lane, token, K, L_draft, L_verify,
                            stream=stream)

    def sync_status(self, stream=None) -> int:
        return tl_sync_status(self.handle, stream)

    def close(self):
        if self.handle:
            tl_model_destroy(self.handle)
            self.handle = 0


class DeviceKV:
    def __init__(self, model: DeviceModel, L_per_lane: Sequence[int], max_ctx: int,
                 dtype: str = "fp16"):
        self.model = model
        self.dtype = {"int8": TL_KV_INT8, "h": TL_KV_H}.get(dtype, TL_KV_FP16)
        self.L = list(L_per_lane)
        self.max_ctx = max_ctx
        nbytes = tl_kv_bytes(model.handle, max_ctx, self.L, self.dtype)
        self.buffer = torch.empty((nbytes + 255) // 256 * 256, dtype=torch.uint8, device="cuda")
        self.handle = tl_kv_create(model.handle, max_ctx, self.L, self.dtype, self.buffer)

    def position(self, lane: int) -> int:
        return tl_kv_position(self.handle, lane)

    def set_position(self, lane: int, pos: int) -> None:
        tl_kv_set_position(self.handle, lane, pos)

    def reset(self, lane: int = -1) -> None:
        tl_kv_reset(self.handle, lane)

    def layer_ptrs(self, lane: int, layer: int):
        return tl_kv_layer_ptrs(self.handle, lane, layer)

    def close(self):
        if self.handle:
            tl_kv_destroy(self.handle)
            self.handle = 0
