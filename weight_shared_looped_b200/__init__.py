"""Python binding of libtinyloop_b200.so (the looped-block library).

Argument marshalling only: every function here has the name of the C entry
point it calls, converts torch tensors to raw pointers and sizes, and raises
``TLError`` on a non-zero status.  All computation happens in the library's
CUDA kernels.  There is no fallback: if the shared library is missing the
import fails.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtinyloop_b200.so")

TL_OK, TL_ERR_INVALID_ARG, TL_ERR_CUDA, TL_ERR_OOM, TL_ERR_TIMEOUT, TL_ERR_UNSUPPORTED, \
    TL_ERR_NUMERIC = range(7)
TL_KV_FP16, TL_KV_INT8, TL_KV_H = 0, 1, 2
STATUS_NAMES = {0: "TL_OK", 1: "TL_ERR_INVALID_ARG", 2: "TL_ERR_CUDA", 3: "TL_ERR_OOM",
                4: "TL_ERR_TIMEOUT", 5: "TL_ERR_UNSUPPORTED", 6: "TL_ERR_NUMERIC"}


class TLError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing; build it with weight_shared_looped_b200.build")

lib = ctypes.CDLL(LIB_PATH)

P = ctypes.c_void_p
I = ctypes.c_int
SZ = ctypes.c_size_t
F = ctypes.c_float


class BlockDesc(ctypes.Structure):
    _fields_ = [("d_model", I), ("n_heads", I), ("head_dim", I), ("ffn", I), ("bits", I),
                ("group", I), ("eps", F), ("rope_theta", F),
                ("w_qkv", P), ("s_qkv", P), ("w_o", P), ("s_o", P), ("w_gate", P), ("s_gate", P),
                ("w_up", P), ("s_up", P), ("w_down", P), ("s_down", P),
                ("gamma_attn", P), ("gamma_ffn", P),
                ("sign_qkv", P), ("sign_o", P), ("sign_gate", P), ("sign_up", P), ("sign_down", P)]


class ModelDesc(ctypes.Structure):
    _fields_ = [("pre", P), ("n_pre", I), ("loop", P), ("embed", P), ("vocab", I),
                ("gamma_final", P), ("max_tokens", I), ("max_lanes", I), ("max_ctx", I),
                ("max_L", I)]


_SIGS = {
    "tl_last_error": ([], ctypes.c_char_p),
    "tl_abi_version": ([], I),
    "tl_packed_words_per_row": ([I, I, ctypes.POINTER(I)], I),
    "tl_packed_bytes": ([I, I, I, I, ctypes.POINTER(SZ), ctypes.POINTER(SZ)], I),
    "tl_pack_weights": ([P, I, I, I, I, P, P, P], I),
    "tl_unpack_codes": ([P, I, I, I, P, P], I),
    "tl_sign_bits_bytes": ([I, I, ctypes.POINTER(SZ)], I),
    "tl_pack_sign_bits": ([P, I, I, I, I, P, P, P], I),
    "tl_kv_quant_int8": ([P, I, I, P, P, P], I),
    "tl_attention_prefill": ([P, P, P, I, I, I, P, P], I),
    "tl_block_create": ([ctypes.POINTER(BlockDesc), ctypes.POINTER(P)], I),
    "tl_block_destroy": ([P], I),
    "tl_block_device_bytes": ([P, ctypes.POINTER(SZ)], I),
    "tl_model_create": ([ctypes.POINTER(ModelDesc), ctypes.POINTER(P)], I),
    "tl_model_destroy": ([P], I),
    "tl_model_device_bytes": ([P, ctypes.POINTER(SZ)], I),
    "tl_model_set_graphs": ([P, I], I),
    "tl_model_set_decode_chunks": ([P, I], I),
    "tl_model_set_exit_threshold": ([P, F], I),
    "tl_model_set_cross_iter": ([P, I], I),
    "tl_model_set_iteration_blocks": ([P, P, I], I),
    "tl_loops_used": ([P, P, I, P], I),
    "tl_kv_layer_bytes": ([I, I, I, I, ctypes.POINTER(SZ)], I),
    "tl_kv_bytes": ([P, I, I, P, I, ctypes.POINTER(SZ)], I),
    "tl_kv_create": ([P, I, I, P, I, P, SZ, ctypes.POINTER(P)], I),
    "tl_kv_destroy": ([P], I),
    "tl_kv_reset": ([P, I, P], I),
    "tl_kv_position": ([P, I, ctypes.POINTER(I)], I),
    "tl_kv_set_position": ([P, I, I, P], I),
    "tl_kv_layer_ptrs": ([P, I, I, ctypes.POINTER(P), ctypes.POINTER(P), ctypes.POINTER(P),
                          ctypes.POINTER(P)], I),
    "tl_prefill": ([P, P, P, I, I, P, I, P, P, P], I),
    "tl_decode_step": ([P, P, P, P, P, I, P, P, P], I),
    "tl_sync_status": ([P, P], I),
    "tl_extend": ([P, P, I, P, P, I, I, P, P, P], I),
    "tl_greedy_head": ([P, P, I, P, P], I),
    "tl_spec_step": ([P, P, I, ctypes.c_int32, I, I, I, P, ctypes.POINTER(I), P], I),
    "tl_linear_workspace_bytes": ([I, I, I, ctypes.POINTER(SZ)], I),
    "tl_linear": ([P, P, I, I, I, P, I, P, P, P], I),
    "tl_linear_noalloc": ([P, P, I, I, I, P, I, P, P], I),
    "tl_check_bounded_wait": ([P, ctypes.c_uint, P], I),
    "tl_read_probe": ([P, SZ, I, P, P], I),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res


def _check(status: int) -> None:
    if status != TL_OK:
        raise TLError(status, lib.tl_last_error().decode(errors="replace"))


def _ptr(t) -> Optional[int]:
    """Raw address of a tensor (host or device), or None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream or None
        return None
    if isinstance(stream, int):
        return stream or None
    return stream.cuda_stream or None


# --------------------------------------------------------------------- packing

def tl_abi_version() -> int:
    return lib.tl_abi_version()


def tl_packed_words_per_row(K: int, bits: int) -> int:
    w = I()
    _check(lib.tl_packed_words_per_row(K, bits, ctypes.byref(w)))
    return w.value


def tl_packed_bytes(N: int, K: int, bits: int, group: int):
    c, s = SZ(), SZ()
    _check(lib.tl_packed_bytes(N, K, bits, group, ctypes.byref(c), ctypes.byref(s)))
    return c.value, s.value


def tl_pack_weights(w, bits: int, group: int, packed, scales, stream=None) -> None:
    N, K = w.shape
    _check(lib.tl_pack_weights(_ptr(w), N, K, bits, group, _ptr(packed), _ptr(scales),
                               _stream(stream)))


def tl_sign_bits_bytes(N: int, K: int) -> int:
    b = SZ()
    _check(lib.tl_sign_bits_bytes(N, K, ctypes.byref(b)))
    return b.value


def tl_pack_sign_bits(w, bits: int, group: int, scales, sign, stream=None) -> None:
    """Sign-of-frac bits of fp32 w [N, K] with the scales tl_pack_weights wrote."""
    N, K = w.shape
    _check(lib.tl_pack_sign_bits(_ptr(w), N, K, bits, group, _ptr(scales), _ptr(sign),
                                 _stream(stream)))


def tl_unpack_codes(packed, N: int, K: int, bits: int, codes, stream=None) -> None:
    _check(lib.tl_unpack_codes(_ptr(packed), N, K, bits, _ptr(codes), _stream(stream)))


def tl_kv_quant_int8(x, codes, scales, stream=None) -> None:
    rows, hd = (x.shape[0], x.shape[1]) if x.dim() == 2 else (0, x.shape[-1])
    _check(lib.tl_kv_quant_int8(_ptr(x), rows, hd, _ptr(codes), _ptr(scales), _stream(stream)))


def tl_attention_prefill(q, k, v, H: int, hd: int, out, stream=None) -> None:
    """q, k, v, out: fp16 [T, H * hd] (or [T, H, hd]) device tensors."""
    T = q.shape[0]
    _check(lib.tl_attention_prefill(_ptr(q), _ptr(k), _ptr(v), T, H, hd, _ptr(out),
                                    _stream(stream)))


# --------------------------------------------------------------------- blocks / model

def tl_block_create(cfg: dict, packed: dict) -> int:
    """cfg: d_model, n_heads, head_dim, ffn, bits, group, eps, rope_theta;
    packed: device tensors w_qkv, s_qkv, ..., gamma_attn, gamma_ffn, and optionally
    sign_qkv, ..., sign_down (the sign-of-frac bits of cross-iteration rounding)."""
    d = BlockDesc(cfg["d_model"], cfg["n_heads"], cfg["head_dim"], cfg["ffn"], cfg["bits"],
                  cfg["group"], cfg["eps"], cfg["rope_theta"],
                  *[_ptr(packed[k]) for k in ("w_qkv", "s_qkv", "w_o", "s_o", "w_gate", "s_gate",
                                              "w_up", "s_up", "w_down", "s_down", "gamma_attn",
                                              "gamma_ffn")],
                  *[_ptr(packed.get(k)) for k in ("sign_qkv", "sign_o", "sign_gate", "sign_up",
                                                  "sign_down")])
    out = P()
    _check(lib.tl_block_create(ctypes.byref(d), ctypes.byref(out)))
    return out.value


def tl_block_destroy(block: int) -> None:
    _check(lib.tl_block_destroy(block))


def tl_block_device_bytes(block: int) -> int:
    b = SZ()
    _check(lib.tl_block_device_bytes(block, ctypes.byref(b)))
    return b.value


def tl_model_create(pre: Sequence[int], loop: int, embed, vocab: int, gamma_final,
                    max_tokens: int, max_lanes: int, max_ctx: int, max_L: int) -> int:
    arr = (P * max(1, len(pre)))(*pre)
    d = ModelDesc(ctypes.cast(arr, P) if pre else None, len(pre), loop, _ptr(embed), vocab,
                  _ptr(gamma_final), max_tokens, max_lanes, max_ctx, max_L)
    out = P()
    _check(lib.tl_model_create(ctypes.byref(d), ctypes.byref(out)))
    return out.value


def tl_model_destroy(model: int) -> None:
    _check(lib.tl_model_destroy(model))


def tl_model_device_bytes(model: int) -> int:
    b = SZ()
    _check(lib.tl_model_device_bytes(model, ctypes.byref(b)))
    return b.value


def tl_model_set_graphs(model: int, enable: bool) -> None:
    _check(lib.tl_model_set_graphs(model, 1 if enable else 0))


def tl_model_set_decode_chunks(model: int, chunks_per_cta: int) -> None:
    _check(lib.tl_model_set_decode_chunks(model, chunks_per_cta))


def tl_model_set_exit_threshold(model: int, tau: float) -> None:
    _check(lib.tl_model_set_exit_threshold(model, tau))


def tl_model_set_cross_iter(model: int, on: bool) -> None:
    _check(lib.tl_model_set_cross_iter(model, 1 if on else 0))


def tl_model_set_iteration_blocks(model: int, blocks: Sequence[Optional[int]]) -> None:
    """Loop iteration i < len(blocks) runs blocks[i] (None: the loop block)."""
    arr = (P * max(1, len(blocks)))(*[b or None for b in blocks])
    _check(lib.tl_model_set_iteration_blocks(model, ctypes.cast(arr, P) if blocks else None,
                                             len(blocks)))


def tl_loops_used(model: int, n: int, stream=None):
    arr = (I * n)()
    _check(lib.tl_loops_used(model, ctypes.cast(arr, P), n, _stream(stream)))
    return list(arr)


# --------------------------------------------------------------------- KV cache

def _int_array(vals: Sequence[int]):
    return (I * len(vals))(*vals)


def tl_kv_layer_bytes(n_heads: int, head_dim: int, max_ctx: int, dtype: int) -> int:
    b = SZ()
    _check(lib.tl_kv_layer_bytes(n_heads, head_dim, max_ctx, dtype, ctypes.byref(b)))
    return b.value


def tl_kv_bytes(model: int, max_ctx: int, L_per_lane: Sequence[int], dtype: int) -> int:
    b = SZ()
    arr = _int_array(L_per_lane)
    _check(lib.tl_kv_bytes(model, len(L_per_lane), max_ctx, ctypes.cast(arr, P), dtype,
                           ctypes.byref(b)))
    return b.value


def tl_kv_create(model: int, max_ctx: int, L_per_lane: Sequence[int], dtype: int, buffer) -> int:
    arr = _int_array(L_per_lane)
    out = P()
    nbytes = buffer.numel() * buffer.element_size()
    _check(lib.tl_kv_create(model, len(L_per_lane), max_ctx, ctypes.cast(arr, P), dtype,
                            _ptr(buffer), nbytes, ctypes.byref(out)))
    return out.value


def tl_kv_destroy(kv: int) -> None:
    _check(lib.tl_kv_destroy(kv))


def tl_kv_reset(kv: int, lane: int = -1, stream=None) -> None:
    _check(lib.tl_kv_reset(kv, lane, _stream(stream)))


def tl_kv_position(kv: int, lane: int) -> int:
    p = I()
    _check(lib.tl_kv_position(kv, lane, ctypes.byref(p)))
    return p.value


def tl_kv_set_position(kv: int, lane: int, pos: int, stream=None) -> None:
    _check(lib.tl_kv_set_position(kv, lane, pos, _stream(stream)))


def tl_kv_layer_ptrs(kv: int, lane: int, layer: int):
    k, v, ks, vs = P(), P(), P(), P()
    _check(lib.tl_kv_layer_ptrs(kv, lane, layer, ctypes.byref(k), ctypes.byref(v),
                                ctypes.byref(ks), ctypes.byref(vs)))
    return k.value, v.value, ks.value, vs.value


# --------------------------------------------------------------------- forward

def tl_prefill(model: int, ids=None, h_in=None, *, L: int, y_out, kv: Optional[int] = None,
               lane: int = 0, h_trace=None, stream=None) -> None:
    seq = (ids if ids is not None else h_in).shape[0]
    _check(lib.tl_prefill(model, _ptr(ids), _ptr(h_in), seq, L, kv, lane, _ptr(y_out),
                          _ptr(h_trace), _stream(stream)))


def tl_decode_step(model: int, kv: int, ids=None, h_in=None, *, L_per_lane: Sequence[int],
                   y_out, h_trace=None, stream=None) -> None:
    arr = _int_array(L_per_lane)
    _check(lib.tl_decode_step(model, kv, _ptr(ids), _ptr(h_in), ctypes.cast(arr, P),
                              len(L_per_lane), _ptr(y_out), _ptr(h_trace), _stream(stream)))


def tl_extend(model: int, kv: int, lane: int, ids=None, h_in=None, *, L: int, y_out,
              h_trace=None, stream=None) -> None:
    n = (ids if ids is not None else h_in).shape[0]
    _check(lib.tl_extend(model, kv, lane, _ptr(ids), _ptr(h_in), n, L, _ptr(y_out),
                         _ptr(h_trace), _stream(stream)))


def tl_greedy_head(model: int, y, ids, stream=None) -> None:
    _check(lib.tl_greedy_head(model, _ptr(y), y.shape[0], _ptr(ids), _stream(stream)))


def tl_spec_step(model: int, kv: int, lane: int, token: int, K: int, L_draft: int,
                 L_verify: int, stream=None):
    """Returns the emitted tokens (a list of 1 .. K + 1 ids)."""
    out = (ctypes.c_int32 * (K + 1))()
    n = I()
    _check(lib.tl_spec_step(model, kv, lane, token, K, L_draft, L_verify,
                            ctypes.cast(out, P), ctypes.byref(n), _stream(stream)))
    return list(out[:n.value])


def tl_linear_workspace_bytes(N: int, K: int, T: int) -> int:
    b = SZ()
    _check(lib.tl_linear_workspace_bytes(N, K, T, ctypes.byref(b)))
    return b.value


def tl_linear(packed, scales, N: int, K: int, group: int, x, y, workspace=None,
              stream=None) -> None:
    T = x.shape[0]
    _check(lib.tl_linear(_ptr(packed), _ptr(scales), N, K, group, _ptr(x), T, _ptr(y),
                         _ptr(workspace), _stream(stream)))


def tl_linear_noalloc(packed, scales, N: int, K: int, group: int, x, y, stream=None) -> None:
    T = x.shape[0]
    _check(lib.tl_linear_noalloc(_ptr(packed), _ptr(scales), N, K, group, _ptr(x), T, _ptr(y),
                                 _stream(stream)))


def tl_read_probe(buf, passes: int, sink, stream=None) -> None:
    """Read `buf` (a 16-byte aligned device tensor) `passes` times."""
    nbytes = buf.numel() * buf.element_size()
    _check(lib.tl_read_probe(_ptr(buf), nbytes, passes, _ptr(sink), _stream(stream)))


def tl_check_bounded_wait(model: int, limit_us: int, stream=None) -> None:
    _check(lib.tl_check_bounded_wait(model, limit_us, _stream(stream)))


def tl_sync_status(model: int, stream=None) -> int:
    """Returns the status code (does not raise) so callers can test for it."""
    return lib.tl_sync_status(model, _stream(stream))
