"""Flint MoE layer decode on B200: Python binding of libflint_moe.so.

Each function below has the name and arguments of the C entry point it wraps
(see include/flint_moe.h); it only turns torch tensors into device pointers,
passes the current CUDA stream, and raises FlintError on a non-zero status.
Every step of the layer runs in the library's CUDA kernels: there is no CPU or
PyTorch fallback, and importing this package on a machine without the built
library raises.
"""
from __future__ import annotations

import ctypes
import os

from .build import SO as _SO_PATH

__all__ = [
    "FlintError", "Shape", "Weights", "Options", "lib",
    "FLINT_W_NVFP4", "FLINT_W_BF16", "FLINT_PATH_AUTO", "FLINT_PATH_GEMV", "FLINT_PATH_MMA",
    "flint_packed_bytes", "flint_block_scale_bytes", "flint_tensor_scale_bytes",
    "flint_moe_workspace_bytes", "flint_moe_workspace_init", "flint_pack_nvfp4", "flint_pack_bf16", "flint_moe_route",
    "flint_moe_forward", "flint_moe_forward_ex", "flint_moe_forward_noalloc", "flint_moe_noalloc_get_status",
    "flint_moe_get_status", "flint_last_error", "flint_debug_noalloc_scratch",
    "flint_pack_nvfp4_dense", "flint_lm_head",
    "flint_debug_dequant", "flint_debug_decode", "flint_debug_group", "flint_debug_wait_timeout", "flint_version",
    "flint_qk_norm_rope_kv", "flint_decode_attention", "flint_decode_attention_workspace_bytes",
    "flint_moe_forward_routed", "flint_ep_dispatch", "flint_ep_combine",
]

FLINT_W_NVFP4, FLINT_W_BF16 = 0, 1
FLINT_PATH_AUTO, FLINT_PATH_GEMV, FLINT_PATH_MMA = 0, 1, 2
FLINT_LAYER_AUTO, FLINT_LAYER_FMA, FLINT_LAYER_MMA, FLINT_LAYER_CLUSTER = 0, 1, 2, 3
FLINT_DEVCHECK_EXPERT_ID, FLINT_DEVCHECK_NONFINITE, FLINT_DEVCHECK_WAIT, FLINT_DEVCHECK_MMA = 1, 2, 4, 8
FLINT_DEVCHECK_INDEX = 16
FLINT_ERR_DEVICE_CHECK, FLINT_ERR_TIMEOUT = -6, -7
STATUS_NAMES = {0: "FLINT_OK", -1: "FLINT_ERR_INVALID_ARG", -2: "FLINT_ERR_UNSUPPORTED_SHAPE",
                -3: "FLINT_ERR_MISALIGNED", -4: "FLINT_ERR_WORKSPACE", -5: "FLINT_ERR_CUDA",
                -6: "FLINT_ERR_DEVICE_CHECK", -7: "FLINT_ERR_TIMEOUT"}


class FlintError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


class Shape(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("inter", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("n_shared", ctypes.c_int32), ("wdtype", ctypes.c_int32)]


class Weights(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p), ("block_scales", ctypes.c_void_p),
                ("tensor_scales", ctypes.c_void_p)]


class Options(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("use_pdl", ctypes.c_int32),
                ("topk_ids", ctypes.c_void_p), ("topk_weights", ctypes.c_void_p),
                ("split_kernels", ctypes.c_int32), ("input_rmsnorm", ctypes.c_int32),
                ("profile_events", ctypes.c_void_p), ("layer_variant", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_SO_PATH):
            raise FlintError(-5, f"{_SO_PATH} is missing: run nvfp4_weight_only_flint_b200.build.build()")
        L = ctypes.CDLL(_SO_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        P = ctypes.POINTER
        L.flint_packed_bytes.argtypes = [P(Shape)]
        L.flint_packed_bytes.restype = sz
        L.flint_block_scale_bytes.argtypes = [P(Shape)]
        L.flint_block_scale_bytes.restype = sz
        L.flint_tensor_scale_bytes.argtypes = [P(Shape)]
        L.flint_tensor_scale_bytes.restype = sz
        L.flint_moe_workspace_bytes.argtypes = [P(Shape), i32]
        L.flint_moe_workspace_bytes.restype = sz
        L.flint_pack_nvfp4.argtypes = [vp, i32, P(Shape), vp, vp, vp, vp, sz, vp]
        L.flint_pack_nvfp4.restype = i32
        L.flint_pack_bf16.argtypes = [vp, P(Shape), vp, vp]
        L.flint_pack_bf16.restype = i32
        L.flint_moe_route.argtypes = [vp, i32, vp, P(Shape), vp, vp, vp, sz, vp]
        L.flint_moe_route.restype = i32
        L.flint_moe_forward.argtypes = [vp, i32, vp, P(Weights), P(Shape), vp, vp, vp, sz, vp]
        L.flint_moe_forward.restype = i32
        L.flint_moe_forward_ex.argtypes = [vp, i32, vp, P(Weights), P(Shape), vp, vp, vp, sz,
                                           P(Options), vp]
        L.flint_moe_forward_ex.restype = i32
        L.flint_moe_forward_noalloc.argtypes = [vp, i32, vp, P(Weights), P(Shape), vp, vp, vp]
        L.flint_moe_forward_noalloc.restype = i32
        L.flint_moe_noalloc_get_status.argtypes = [P(i32), vp]
        L.flint_moe_noalloc_get_status.restype = i32
        L.flint_debug_noalloc_scratch.argtypes = [P(vp)]
        L.flint_debug_noalloc_scratch.restype = i32
        L.flint_pack_nvfp4_dense.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, sz, vp]
        L.flint_pack_nvfp4_dense.restype = i32
        L.flint_lm_head.argtypes = [vp, i32, vp, vp, vp, i32, i32, vp, vp, sz, vp]
        L.flint_lm_head.restype = i32
        L.flint_qk_norm_rope_kv.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, i32, vp, i32, ctypes.c_float, vp,
                                            ctypes.c_int64, vp, vp, vp, vp, vp]
        L.flint_qk_norm_rope_kv.restype = i32
        L.flint_decode_attention_workspace_bytes.argtypes = [i32, i32, i32]
        L.flint_decode_attention_workspace_bytes.restype = sz
        L.flint_decode_attention.argtypes = [vp, vp, vp, ctypes.c_int64, vp, vp, i32, i32, i32, i32, i32,
                                             ctypes.c_float, vp, vp, sz, vp, vp]
        L.flint_decode_attention.restype = i32
        L.flint_moe_forward_routed.argtypes = [vp, i32, vp, vp, P(Weights), P(Shape), vp, vp, vp, sz, vp]
        L.flint_moe_forward_routed.restype = i32
        L.flint_ep_dispatch.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, vp, i32, vp, vp, vp, vp, vp, vp, vp,
                                        vp]
        L.flint_ep_dispatch.restype = i32
        L.flint_ep_combine.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp]
        L.flint_ep_combine.restype = i32
        L.flint_moe_workspace_init.argtypes = [vp, sz, vp]
        L.flint_moe_workspace_init.restype = i32
        L.flint_moe_get_status.argtypes = [vp, P(i32), vp]
        L.flint_moe_get_status.restype = i32
        L.flint_last_error.argtypes = []
        L.flint_last_error.restype = ctypes.c_char_p
        L.flint_debug_dequant.argtypes = [P(Weights), P(Shape), i32, i32, i32, i32, vp, vp, vp]
        L.flint_debug_dequant.restype = i32
        L.flint_debug_decode.argtypes = [P(Weights), P(Shape), i32, i32, i32, i32, i32, i32, i32, vp, vp]
        L.flint_debug_decode.restype = i32
        L.flint_debug_group.argtypes = [vp, i32, P(Shape), i32, vp, vp, vp, vp, vp, sz, vp]
        L.flint_debug_group.restype = i32
        L.flint_debug_wait_timeout.argtypes = [vp, ctypes.c_int64, vp]
        L.flint_debug_wait_timeout.restype = i32
        L.flint_version.argtypes = []
        L.flint_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


# ------------------------------------------------------------------ marshalling helpers
def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise FlintError(-1, "expected a CUDA tensor")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int):
    if rc != 0:
        raise FlintError(rc, lib().flint_last_error().decode())


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def flint_last_error() -> str:
    return lib().flint_last_error().decode()


def flint_version() -> str:
    return lib().flint_version().decode()


def flint_packed_bytes(shape: Shape) -> int:
    return lib().flint_packed_bytes(ctypes.byref(shape))


def flint_block_scale_bytes(shape: Shape) -> int:
    return lib().flint_block_scale_bytes(ctypes.byref(shape))


def flint_tensor_scale_bytes(shape: Shape) -> int:
    return lib().flint_tensor_scale_bytes(ctypes.byref(shape))


def flint_moe_workspace_bytes(shape: Shape, max_tokens: int) -> int:
    return lib().flint_moe_workspace_bytes(ctypes.byref(shape), int(max_tokens))


def flint_moe_workspace_init(workspace, stream=None) -> None:
    _check(lib().flint_moe_workspace_init(_ptr(workspace), _nbytes(workspace), _stream(stream)))


def flint_pack_nvfp4(w, w_is_bf16: int, shape: Shape, packed, block_scales, tensor_scales,
                     workspace, stream=None) -> None:
    _check(lib().flint_pack_nvfp4(_ptr(w), int(w_is_bf16), ctypes.byref(shape), _ptr(packed),
                                  _ptr(block_scales), _ptr(tensor_scales), _ptr(workspace),
                                  _nbytes(workspace), _stream(stream)))


def flint_pack_bf16(w, shape: Shape, packed, stream=None) -> None:
    _check(lib().flint_pack_bf16(_ptr(w), ctypes.byref(shape), _ptr(packed), _stream(stream)))


def flint_moe_route(x, T: int, router_w, shape: Shape, topk_ids, topk_weights, workspace,
                    stream=None) -> None:
    _check(lib().flint_moe_route(_ptr(x), int(T), _ptr(router_w), ctypes.byref(shape),
                                 _ptr(topk_ids), _ptr(topk_weights), _ptr(workspace),
                                 _nbytes(workspace), _stream(stream)))


def flint_moe_forward(x, T: int, router_w, weights: Weights, shape: Shape, residual, out,
                      workspace, stream=None) -> None:
    _check(lib().flint_moe_forward(_ptr(x), int(T), _ptr(router_w), ctypes.byref(weights),
                                   ctypes.byref(shape), _ptr(residual), _ptr(out),
                                   _ptr(workspace), _nbytes(workspace), _stream(stream)))


def flint_moe_forward_ex(x, T: int, router_w, weights: Weights, shape: Shape, residual, out,
                         workspace, options: Options | None, stream=None) -> None:
    _check(lib().flint_moe_forward_ex(_ptr(x), int(T), _ptr(router_w), ctypes.byref(weights),
                                      ctypes.byref(shape), _ptr(residual), _ptr(out),
                                      _ptr(workspace), _nbytes(workspace),
                                      ctypes.byref(options) if options is not None else None,
                                      _stream(stream)))


def flint_moe_forward_noalloc(x, T: int, router_w, weights: Weights, shape: Shape, residual, out,
                              stream=None) -> None:
    _check(lib().flint_moe_forward_noalloc(_ptr(x), int(T), _ptr(router_w), ctypes.byref(weights),
                                           ctypes.byref(shape), _ptr(residual), _ptr(out),
                                           _stream(stream)))


def flint_moe_noalloc_get_status(stream=None) -> tuple[int, int]:
    """Status of the built-in scratch of flint_moe_forward_noalloc: (status,
    device_flags) without raising."""
    flags = ctypes.c_int32(0)
    rc = lib().flint_moe_noalloc_get_status(ctypes.byref(flags), _stream(stream))
    return rc, flags.value


def flint_debug_noalloc_scratch() -> int:
    """Device address of the built-in scratch in the current context."""
    addr = ctypes.c_void_p(0)
    _check(lib().flint_debug_noalloc_scratch(ctypes.byref(addr)))
    return addr.value


def flint_pack_nvfp4_dense(w, w_is_bf16: int, rows: int, cols: int, codes, scales, tensor_scale, workspace,
                           stream=None) -> None:
    _check(lib().flint_pack_nvfp4_dense(_ptr(w), int(w_is_bf16), int(rows), int(cols), _ptr(codes), _ptr(scales),
                                        _ptr(tensor_scale), _ptr(workspace), _nbytes(workspace), _stream(stream)))


def flint_lm_head(x, T: int, codes, scales, tensor_scale, rows: int, cols: int, out, workspace,
                  stream=None) -> None:
    _check(lib().flint_lm_head(_ptr(x), int(T), _ptr(codes), _ptr(scales), _ptr(tensor_scale), int(rows),
                               int(cols), _ptr(out), _ptr(workspace), _nbytes(workspace), _stream(stream)))


def flint_qk_norm_rope_kv(qkv, T: int, n_q_heads: int, n_kv_heads: int, q_norm_w, k_norm_w, cos_sin, max_pos: int,
                          positions, rope: bool, eps: float, slots, n_slots: int, q_out, k_cache, v_cache,
                          status=None, head_dim: int = 128, stream=None) -> None:
    _check(lib().flint_qk_norm_rope_kv(_ptr(qkv), int(T), int(n_q_heads), int(n_kv_heads), int(head_dim),
                                       _ptr(q_norm_w), _ptr(k_norm_w), _ptr(cos_sin), int(max_pos), _ptr(positions),
                                       int(bool(rope)), float(eps), _ptr(slots), int(n_slots), _ptr(q_out),
                                       _ptr(k_cache), _ptr(v_cache), _ptr(status), _stream(stream)))


def flint_decode_attention_workspace_bytes(T: int, n_kv_heads: int, max_len: int) -> int:
    return int(lib().flint_decode_attention_workspace_bytes(int(T), int(n_kv_heads), int(max_len)))


def flint_decode_attention(q, k_cache, v_cache, n_rows: int, start, length, T: int, n_q_heads: int,
                           n_kv_heads: int, max_len: int, scale: float, out, workspace=None, status=None,
                           head_dim: int = 128, stream=None) -> None:
    _check(lib().flint_decode_attention(_ptr(q), _ptr(k_cache), _ptr(v_cache), int(n_rows), _ptr(start),
                                        _ptr(length), int(T), int(n_q_heads), int(n_kv_heads), int(head_dim),
                                        int(max_len), float(scale), _ptr(out), _ptr(workspace),
                                        _nbytes(workspace), _ptr(status), _stream(stream)))


def flint_moe_forward_routed(x, T: int, topk_ids, topk_weights, weights: Weights, shape: Shape, residual, out,
                             workspace, stream=None) -> None:
    _check(lib().flint_moe_forward_routed(_ptr(x), int(T), _ptr(topk_ids), _ptr(topk_weights), ctypes.byref(weights),
                                          ctypes.byref(shape), _ptr(residual), _ptr(out), _ptr(workspace),
                                          _nbytes(workspace), _stream(stream)))


def flint_ep_dispatch(topk_ids, topk_weights, T: int, top_k: int, n_shared: int, n_experts: int, n_ranks: int,
                      rank: int, x, d: int, send_x, send_ids, send_gates, send_token, send_counts, pair_pos,
                      status=None, stream=None) -> None:
    _check(lib().flint_ep_dispatch(_ptr(topk_ids), _ptr(topk_weights), int(T), int(top_k), int(n_shared),
                                   int(n_experts), int(n_ranks), int(rank), _ptr(x), int(d), _ptr(send_x),
                                   _ptr(send_ids), _ptr(send_gates), _ptr(send_token), _ptr(send_counts),
                                   _ptr(pair_pos), _ptr(status), _stream(stream)))


def flint_ep_combine(y, pair_pos, T: int, slots: int, d: int, residual, out, stream=None) -> None:
    _check(lib().flint_ep_combine(_ptr(y), _ptr(pair_pos), int(T), int(slots), int(d), _ptr(residual), _ptr(out),
                                  _stream(stream)))


def flint_moe_get_status(workspace, stream=None) -> tuple[int, int]:
    """Returns (status, device_flags) without raising."""
    flags = ctypes.c_int32(0)
    rc = lib().flint_moe_get_status(_ptr(workspace), ctypes.byref(flags), _stream(stream))
    return rc, flags.value


def flint_debug_dequant(weights: Weights, shape: Shape, expert: int, matrix: int, row0: int,
                        rows: int, out, stream=None) -> tuple[float, ...]:
    ts = (ctypes.c_float * 2)()
    _check(lib().flint_debug_dequant(ctypes.byref(weights), ctypes.byref(shape), int(expert),
                                     int(matrix), int(row0), int(rows), _ptr(out), ts,
                                     _stream(stream)))
    return (ts[0], ts[1]) if matrix == 0 else (ts[0],)


def flint_debug_decode(weights: Weights, shape: Shape, expert: int, matrix: int, decoder: int, row0: int,
                       rows: int, k0: int, kn: int, out, stream=None) -> None:
    _check(lib().flint_debug_decode(ctypes.byref(weights), ctypes.byref(shape), int(expert), int(matrix),
                                    int(decoder), int(row0), int(rows), int(k0), int(kn), _ptr(out),
                                    _stream(stream)))


def flint_debug_group(ids, T: int, shape: Shape, impl: int, act, off, pair, counts, workspace,
                      stream=None) -> None:
    _check(lib().flint_debug_group(_ptr(ids), int(T), ctypes.byref(shape), int(impl), _ptr(act), _ptr(off),
                                   _ptr(pair), _ptr(counts), _ptr(workspace), _nbytes(workspace),
                                   _stream(stream)))


def flint_debug_wait_timeout(workspace, cycles: int, stream=None) -> None:
    _check(lib().flint_debug_wait_timeout(_ptr(workspace), int(cycles), _stream(stream)))
