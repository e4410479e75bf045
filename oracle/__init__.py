"""ctypes front end of the fp64 CPU oracle (``flint_oracle.cpp``).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference leg may import this package. The
product (``nvfp4_weight_only_flint_b200``) never imports it, and this package
imports nothing from the product. Functions here only marshal numpy arrays in
and out; every step of the arithmetic is in the C++ file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "flint_oracle.cpp")
_HDR = os.path.join(_HERE, "flint_oracle.h")
_SO = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (IEEE fp32/fp64, no fused multiply-add)."""
    newest_src = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if not force and os.path.exists(_SO) and os.path.getmtime(_SO) >= newest_src:
        return _SO
    tmp = _SO + f".tmp{os.getpid()}"
    cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
           "-ffp-contract=off", "-fno-fast-math", _SRC, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _SO)
    return _SO


class OracleMatrix(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_int32),
        ("rows", ctypes.c_int32),
        ("cols", ctypes.c_int32),
        ("tensor_scale", ctypes.c_float),
        ("codes", ctypes.c_void_p),
        ("scales", ctypes.c_void_p),
        ("bf16", ctypes.c_void_p),
    ]


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        u8, i32, f32, f64, vp = (ctypes.c_uint8, ctypes.c_int32, ctypes.c_float,
                                 ctypes.c_double, ctypes.c_void_p)
        L.oracle_e2m1_decode.argtypes = [u8]
        L.oracle_e2m1_decode.restype = f64
        L.oracle_e4m3_decode.argtypes = [u8]
        L.oracle_e4m3_decode.restype = f64
        L.oracle_e2m1_encode.argtypes = [f32]
        L.oracle_e2m1_encode.restype = u8
        L.oracle_e4m3_encode.argtypes = [f32]
        L.oracle_e4m3_encode.restype = u8
        L.oracle_bf16_from_double.argtypes = [f64]
        L.oracle_bf16_from_double.restype = ctypes.c_uint16
        L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_double.restype = f64
        L.oracle_quantize_nvfp4.argtypes = [vp, i32, i32, vp, vp, vp]
        L.oracle_quantize_nvfp4.restype = i32
        L.oracle_quantize_nvfp4_rows.argtypes = [vp, i32, i32, f32, vp, vp, vp]
        L.oracle_quantize_nvfp4_rows.restype = i32
        L.oracle_decode_matrix.argtypes = [ctypes.POINTER(OracleMatrix), vp]
        L.oracle_decode_matrix.restype = i32
        L.oracle_pack_layout.argtypes = [ctypes.POINTER(OracleMatrix), i32, i32, i32, vp, vp, vp]
        L.oracle_pack_layout.restype = i32
        L.oracle_pack_layout_bf16.argtypes = [ctypes.POINTER(OracleMatrix), i32, i32, i32, vp]
        L.oracle_pack_layout_bf16.restype = i32
        L.oracle_router_logits.argtypes = [vp, i32, vp, i32, i32, vp]
        L.oracle_router_logits.restype = i32
        L.oracle_topk.argtypes = [vp, i32, i32, i32, vp, vp, vp]
        L.oracle_topk.restype = i32
        L.oracle_expert_ffn.argtypes = [ctypes.POINTER(OracleMatrix), i32, i32, vp, vp]
        L.oracle_expert_ffn.restype = i32
        L.oracle_moe_forward.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp,
                                         ctypes.POINTER(OracleMatrix), vp, vp, i32, i32,
                                         vp, vp, vp, vp, vp]
        L.oracle_moe_forward.restype = i32
        L.oracle_dense_gemv.argtypes = [ctypes.POINTER(OracleMatrix), vp, i32, vp, i32, vp]
        L.oracle_dense_gemv.restype = i32
        L.oracle_group.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp]
        L.oracle_group.restype = i32
        L.oracle_ep_plan.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp]
        L.oracle_ep_plan.restype = i32
        L.oracle_qk_norm_rope_kv.argtypes = [i32, i32, i32, i32, vp, vp, vp, vp, i32, vp, i32, f64, vp, vp, vp]
        L.oracle_qk_norm_rope_kv.restype = i32
        L.oracle_decode_attention.argtypes = [i32, i32, i32, i32, vp, vp, vp, ctypes.c_int64, vp, vp, f64, vp]
        L.oracle_decode_attention.restype = i32
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


# ---------------------------------------------------------------- codecs
def e2m1_decode(code: int) -> float:
    return lib().oracle_e2m1_decode(code)


def e4m3_decode(code: int) -> float:
    return lib().oracle_e4m3_decode(code)


def e2m1_encode(v: float) -> int:
    return lib().oracle_e2m1_encode(float(np.float32(v)))


def e4m3_encode(v: float) -> int:
    return lib().oracle_e4m3_encode(float(np.float32(v)))


def bf16_from_double(v: float) -> int:
    return lib().oracle_bf16_from_double(float(v))


def bf16_round_array(a: np.ndarray) -> np.ndarray:
    """fp64 array -> bf16 bit patterns (uint16), round to nearest even."""
    f = lib().oracle_bf16_from_double
    flat = np.asarray(a, dtype=np.float64).ravel()
    return np.array([f(float(v)) for v in flat], dtype=np.uint16).reshape(np.shape(a))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- quantiser
@dataclass
class NVFP4Matrix:
    """Natural-layout NVFP4 planes of one [rows][cols] matrix."""
    codes: np.ndarray   # uint8 [rows][cols/2]
    scales: np.ndarray  # uint8 [rows][cols/16]
    tensor_scale: float
    rows: int
    cols: int


@dataclass
class BF16Matrix:
    bits: np.ndarray  # uint16 [rows][cols]
    rows: int
    cols: int


def quantize(w: np.ndarray) -> NVFP4Matrix:
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, cols = w.shape
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    scales = np.zeros((rows, cols // 16), dtype=np.uint8)
    ts = np.zeros(1, dtype=np.float32)
    rc = lib().oracle_quantize_nvfp4(_ptr(w), rows, cols, _ptr(codes), _ptr(scales), _ptr(ts))
    if rc != 0:
        raise ValueError("oracle_quantize_nvfp4 rejected the input")
    return NVFP4Matrix(codes, scales, float(ts[0]), rows, cols)


def quantize_with_tensor_scale(w: np.ndarray, amax: float) -> NVFP4Matrix:
    """Rows of a larger tensor whose largest |w| is amax (its tensor scale is
    amax / 2688), quantised with the same recipe."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, cols = w.shape
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    scales = np.zeros((rows, cols // 16), dtype=np.uint8)
    ts = np.zeros(1, dtype=np.float32)
    if lib().oracle_quantize_nvfp4_rows(_ptr(w), rows, cols, float(np.float32(amax)), _ptr(codes), _ptr(scales),
                                        _ptr(ts)) != 0:
        raise ValueError("oracle_quantize_nvfp4_rows rejected the input")
    return NVFP4Matrix(codes, scales, float(ts[0]), rows, cols)


def _as_struct(m) -> OracleMatrix:
    s = OracleMatrix()
    if m is None:
        return s
    if isinstance(m, NVFP4Matrix):
        s.kind, s.rows, s.cols, s.tensor_scale = 0, m.rows, m.cols, m.tensor_scale
        s.codes, s.scales = m.codes.ctypes.data, m.scales.ctypes.data
    else:
        s.kind, s.rows, s.cols = 1, m.rows, m.cols
        s.bf16 = m.bits.ctypes.data
    return s


def _struct_array(mats):
    arr = (OracleMatrix * len(mats))()
    for i, m in enumerate(mats):
        arr[i] = _as_struct(m)
    return arr


def decode(m) -> np.ndarray:
    out = np.zeros((m.rows, m.cols), dtype=np.float64)
    s = _as_struct(m)
    if lib().oracle_decode_matrix(ctypes.byref(s), _ptr(out)) != 0:
        raise ValueError("oracle_decode_matrix failed")
    return out


def pack_layout(experts, d: int, inter: int):
    """experts: list of (gate, up, down) NVFP4Matrix triples -> (codes, scales, tensor_scales)."""
    mats = [m for trip in experts for m in trip]
    arr = _struct_array(mats)
    n = len(experts)
    codes = np.zeros(n * 3 * inter * d // 2, dtype=np.uint8)
    scales = np.zeros(n * 3 * inter * d // 16, dtype=np.uint8)
    ts = np.zeros(n * 3, dtype=np.float32)
    if lib().oracle_pack_layout(arr, n, d, inter, _ptr(codes), _ptr(scales), _ptr(ts)) != 0:
        raise ValueError("oracle_pack_layout failed")
    return codes, scales, ts


def pack_layout_bf16(experts, d: int, inter: int) -> np.ndarray:
    mats = [m for trip in experts for m in trip]
    arr = _struct_array(mats)
    n = len(experts)
    out = np.zeros(n * 3 * inter * d, dtype=np.uint16)
    if lib().oracle_pack_layout_bf16(arr, n, d, inter, _ptr(out)) != 0:
        raise ValueError("oracle_pack_layout_bf16 failed")
    return out


# ---------------------------------------------------------------- routing / forward
def router_logits(x_bits: np.ndarray, wr_bits: np.ndarray) -> np.ndarray:
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    wr_bits = np.ascontiguousarray(wr_bits, dtype=np.uint16)
    T, d = x_bits.shape
    E = wr_bits.shape[0]
    out = np.zeros((T, E), dtype=np.float64)
    lib().oracle_router_logits(_ptr(x_bits), T, _ptr(wr_bits), d, E, _ptr(out))
    return out


def topk(logits: np.ndarray, k: int):
    logits = np.ascontiguousarray(logits, dtype=np.float64)
    T, E = logits.shape
    ids = np.zeros((T, k), dtype=np.int32)
    gates = np.zeros((T, k), dtype=np.float64)
    gap = np.zeros(T, dtype=np.float64)
    if lib().oracle_topk(_ptr(logits), T, E, k, _ptr(ids), _ptr(gates), _ptr(gap)) != 0:
        raise ValueError("oracle_topk failed")
    return ids, gates, gap


def dense_gemv(m: NVFP4Matrix, x_bits: np.ndarray, rows=None) -> np.ndarray:
    """out [T][len(rows)] = decoded m[rows] . x in fp64 (all rows when None)."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    T = x_bits.shape[0]
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    n = m.rows if r is None else r.size
    out = np.zeros((T, n), dtype=np.float64)
    s = _as_struct(m)
    if lib().oracle_dense_gemv(ctypes.byref(s), _ptr(x_bits), T, _ptr(r), n, _ptr(out)) != 0:
        raise ValueError("oracle_dense_gemv failed")
    return out


def qk_norm_rope_kv(qkv_bits: np.ndarray, n_q_heads: int, n_kv_heads: int, q_w_bits, k_w_bits, cos_sin=None,
                    positions=None, rope: bool = False, eps: float = 1e-6):
    """Attention prologue of one layer in fp64 (see oracle_qk_norm_rope_kv):
    qkv_bits bf16 [T][Hq + 2*Hkv][Dh]; returns (q [T][Hq][Dh], k, v [T][Hkv][Dh])."""
    qkv = np.ascontiguousarray(qkv_bits, dtype=np.uint16)
    T, H, Dh = qkv.shape
    assert H == n_q_heads + 2 * n_kv_heads
    qw = np.ascontiguousarray(q_w_bits, dtype=np.uint16)
    kw = np.ascontiguousarray(k_w_bits, dtype=np.uint16)
    cs = None if cos_sin is None else np.ascontiguousarray(cos_sin, dtype=np.float32)
    pos = None if positions is None else np.ascontiguousarray(positions, dtype=np.int32)
    max_pos = 0 if cs is None else cs.shape[0]
    q = np.zeros((T, n_q_heads, Dh), dtype=np.float64)
    k = np.zeros((T, n_kv_heads, Dh), dtype=np.float64)
    v = np.zeros((T, n_kv_heads, Dh), dtype=np.float64)
    rc = lib().oracle_qk_norm_rope_kv(T, n_q_heads, n_kv_heads, Dh, _ptr(qkv), _ptr(qw), _ptr(kw), _ptr(cs), max_pos,
                                      _ptr(pos), int(bool(rope)), float(eps), _ptr(q), _ptr(k), _ptr(v))
    if rc != 0:
        raise ValueError("oracle_qk_norm_rope_kv failed")
    return q, k, v


def decode_attention(q_bits, k_bits, v_bits, start, length, scale=None):
    """fp64 decode attention: q_bits [T][Hq][Dh], k/v_bits [rows][Hkv][Dh]
    (bf16 bits), start int64 [T], length int32 [T]; returns [T][Hq][Dh]."""
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v = np.ascontiguousarray(v_bits, dtype=np.uint16)
    T, Hq, Dh = q.shape
    rows, Hkv, _ = k.shape
    st = np.ascontiguousarray(start, dtype=np.int64)
    ln = np.ascontiguousarray(length, dtype=np.int32)
    out = np.zeros((T, Hq, Dh), dtype=np.float64)
    sc = 1.0 / np.sqrt(Dh) if scale is None else float(scale)
    if lib().oracle_decode_attention(T, Hq, Hkv, Dh, _ptr(q), _ptr(k), _ptr(v), rows, _ptr(st), _ptr(ln), sc,
                                     _ptr(out)) != 0:
        raise ValueError("oracle_decode_attention failed")
    return out


def group(ids: np.ndarray, E: int, S: int):
    """Grouping by expert of ids [T][k]: (act, off, pair, n_routed), or None
    when an id lies outside [0, E)."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    act = np.zeros(E + S, dtype=np.int32)
    off = np.zeros(E + S + 1, dtype=np.int32)
    pair = np.zeros(max(1, T * (k + S)), dtype=np.int32)
    nr = np.zeros(1, dtype=np.int32)
    n = lib().oracle_group(_ptr(ids), T, k, E, S, _ptr(act), _ptr(off), _ptr(pair), _ptr(nr))
    if n < 0:
        return None
    return act[:n].copy(), off[:n + 1].copy(), pair[:T * (k + S)].copy(), int(nr[0])


def ep_plan(ids: np.ndarray, gates: np.ndarray, S: int, E: int, R: int, rank: int):
    """Expert-parallel dispatch plan of ids/gates [T][k] on rank `rank` of R:
    dict with send_ids, send_gates, send_token (send order), counts [R],
    pair_pos [T][k+S], dropped."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    gates = np.ascontiguousarray(gates, dtype=np.float32)
    T, k = ids.shape
    P = T * (k + S)
    send_ids = np.full(max(P, 1), -7, np.int32)
    send_gates = np.zeros(max(P, 1), np.float32)
    send_token = np.full(max(P, 1), -7, np.int32)
    counts = np.zeros(R, np.int32)
    pair_pos = np.zeros(max(P, 1), np.int32)
    dropped = lib().oracle_ep_plan(_ptr(ids), _ptr(gates), T, k, S, E, R, rank, _ptr(send_ids), _ptr(send_gates),
                                   _ptr(send_token), _ptr(counts), _ptr(pair_pos))
    if dropped < 0:
        raise ValueError("oracle_ep_plan: bad sizes")
    n = int(counts.sum())
    return {"send_ids": send_ids[:n].copy(), "send_gates": send_gates[:n].copy(), "send_token": send_token[:n].copy(),
            "counts": counts, "pair_pos": pair_pos[:P].reshape(T, k + S).copy(), "dropped": int(dropped)}


def expert_ffn(trip, x: np.ndarray) -> np.ndarray:
    gate, up, down = trip
    d, inter = gate.cols, gate.rows
    arr = _struct_array([gate, up, down])
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.zeros(d, dtype=np.float64)
    if lib().oracle_expert_ffn(arr, d, inter, _ptr(x), _ptr(y)) != 0:
        raise ValueError("oracle_expert_ffn failed")
    return y


def moe_forward(x_bits, wr_bits, experts, *, d, inter, E, k, S, residual_bits=None,
                ids_override=None, input_norm=False, n_threads=1):
    """experts: list of length E+S; entry e is a (gate, up, down) triple or None (unused)."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    wr_bits = np.ascontiguousarray(wr_bits, dtype=np.uint16)
    T = x_bits.shape[0]
    mats = []
    for trip in experts:
        mats.extend(trip if trip is not None else (None, None, None))
    arr = _struct_array(mats)
    res = None if residual_bits is None else np.ascontiguousarray(residual_bits, dtype=np.uint16)
    ovr = None if ids_override is None else np.ascontiguousarray(ids_override, dtype=np.int32)
    out = np.zeros((T, d), dtype=np.float64)
    ids = np.zeros((T, k), dtype=np.int32)
    gates = np.zeros((T, k), dtype=np.float64)
    gap = np.zeros(T, dtype=np.float64)
    logits = np.zeros((T, E), dtype=np.float64)
    rc = lib().oracle_moe_forward(T, d, inter, E, k, S, _ptr(x_bits), _ptr(wr_bits), arr,
                                  _ptr(res), _ptr(ovr), int(bool(input_norm)), int(n_threads),
                                  _ptr(ids), _ptr(gates),
                                  _ptr(gap), _ptr(logits), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_moe_forward failed")
    return {"out": out, "ids": ids, "gates": gates, "gap": gap, "logits": logits}
