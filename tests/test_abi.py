"""The C ABI library loads, exports every entry point include/*.h declares, and
rejects bad arguments on the host before touching the GPU (no compute calls)."""
import ctypes
import glob
import os
import re

import pytest

import nvfp4_weight_only_flint_b200 as fm
from nvfp4_weight_only_flint_b200 import build as fbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(flint_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def L():
    fbuild.build()
    return fm.lib()


def test_header_declares_the_layer_calls():
    names = _declared_functions()
    for required in ("flint_pack_nvfp4", "flint_moe_route", "flint_moe_forward"):
        assert required in names
    assert len(names) >= 12


def test_every_declared_symbol_is_exported(L):
    missing = [n for n in _declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def _shape(d=2048, inter=512, E=256, k=6, S=1, wd=0):
    return fm.Shape(d, inter, E, k, S, wd)


def test_sizes(L):
    s = _shape()
    assert fm.flint_packed_bytes(s) == 257 * 3 * 512 * 2048 // 2
    assert fm.flint_block_scale_bytes(s) == 257 * 3 * 512 * 2048 // 16
    assert fm.flint_tensor_scale_bytes(s) == 257 * 3 * 4
    sb = _shape(wd=1)
    assert fm.flint_packed_bytes(sb) == 257 * 3 * 512 * 2048 * 2
    assert fm.flint_block_scale_bytes(sb) == 0
    assert fm.flint_moe_workspace_bytes(s, 8) > fm.flint_moe_workspace_bytes(s, 1) > 0
    # the single-kernel path's tagged regions are sized for its largest batch
    # whatever max_tokens is: 8 tokens x 8 replicas x E tagged logits and
    # 8 x (k+S) x inter tagged SwiGLU values, 8 bytes each, after the 1 KiB
    # control block
    tagged = 8 * 8 * 256 * 8 + 8 * (6 + 1) * 512 * 8
    assert fm.flint_moe_workspace_bytes(s, 1) >= 1024 + tagged
    sizes = [fm.flint_moe_workspace_bytes(s, t) for t in (1, 2, 8, 32, 128)]
    assert sizes == sorted(sizes)


@pytest.mark.parametrize("bad", [dict(d=1000), dict(d=8192), dict(inter=96), dict(E=0), dict(E=513),
                                 dict(k=0), dict(k=9), dict(E=4, k=5), dict(S=2), dict(wd=7)])
def test_unsupported_shapes(L, bad):
    s = _shape(**bad)
    assert fm.flint_packed_bytes(s) == 0
    rc = L.flint_moe_forward(None, 1, None, None, ctypes.byref(s), None, None, None, 0, None)
    assert rc in (-1, -2)
    assert fm.flint_last_error()


def _weights(p=0x10000, b=0x20000, t=0x30000):
    return fm.Weights(p, b, t)


def test_host_validation_errors(L):
    s = _shape()
    ws_need = fm.flint_moe_workspace_bytes(s, 4)
    w = _weights()
    # NULL pointers
    assert L.flint_moe_forward(None, 4, 0x40000, ctypes.byref(w), ctypes.byref(s), None, 0x50000,
                               0x60000, ws_need, None) == -1
    # misaligned activations
    assert L.flint_moe_forward(0x40008, 4, 0x40000, ctypes.byref(w), ctypes.byref(s), None, 0x50000,
                               0x60000, ws_need, None) == -3
    # workspace too small (flint_moe_workspace_bytes covers every path; a call
    # needs at least its path's regions, always more than the control block)
    assert L.flint_moe_forward(0x40000, 4, 0x40000, ctypes.byref(w), ctypes.byref(s), None, 0x50000,
                               0x60000, 1024, None) == -4
    assert "workspace" in fm.flint_last_error()
    # negative token count; zero tokens is a no-op
    assert L.flint_moe_forward(0x40000, -1, 0x40000, ctypes.byref(w), ctypes.byref(s), None, 0x50000,
                               0x60000, ws_need, None) == -1
    assert L.flint_moe_forward(0x40000, 0, 0x40000, ctypes.byref(w), ctypes.byref(s), None, 0x50000,
                               0x60000, ws_need, None) == 0
    # bad path option
    opt = fm.Options(9, 1, None, None)
    assert L.flint_moe_forward_ex(0x40000, 4, 0x40000, ctypes.byref(w), ctypes.byref(s), None, 0x50000,
                                  0x60000, ws_need, ctypes.byref(opt), None) == -1
    # bad layer variant option
    opt = fm.Options(path=0, use_pdl=1, layer_variant=4)
    assert L.flint_moe_forward_ex(0x40000, 4, 0x40000, ctypes.byref(w), ctypes.byref(s), None, 0x50000,
                                  0x60000, ws_need, ctypes.byref(opt), None) == -1
    assert "layer_variant" in fm.flint_last_error()
    # the cluster kernels take at most 8 tokens (refused before any launch)
    opt = fm.Options(path=0, use_pdl=1, layer_variant=fm.FLINT_LAYER_CLUSTER)
    assert L.flint_moe_forward_ex(0x40000, 9, 0x40000, ctypes.byref(w), ctypes.byref(s), None, 0x50000,
                                  0x60000, ws_need, ctypes.byref(opt), None) == -2
    assert "cluster" in fm.flint_last_error()
    # NVFP4 weights without scales
    w2 = fm.Weights(0x10000, None, None)
    assert L.flint_moe_forward(0x40000, 4, 0x40000, ctypes.byref(w2), ctypes.byref(s), None, 0x50000,
                               0x60000, ws_need, None) == -1
    # route: NULL outputs
    assert L.flint_moe_route(0x40000, 4, 0x40000, ctypes.byref(s), None, None, 0x60000, ws_need, None) == -1
    # packer: wrong weight type
    sb = _shape(wd=1)
    assert L.flint_pack_nvfp4(0x40000, 0, ctypes.byref(sb), 0x10000, 0x20000, 0x30000, 0x60000,
                              ws_need, None) == -1
    # status without workspace
    assert L.flint_moe_get_status(None, None, None) == -1


def test_decode_attention_host_validation(L):
    # workspace: none when every context fits one chunk, else per-chunk partials
    assert fm.flint_decode_attention_workspace_bytes(64, 4, 4096) == 0
    assert fm.flint_decode_attention_workspace_bytes(1, 4, 32768) > 0
    assert fm.flint_decode_attention_workspace_bytes(0, 4, 32768) == 0
    need = fm.flint_decode_attention_workspace_bytes(1, 4, 32768)
    a = 0x100000

    def call(T=1, hq=32, hkv=4, dh=128, max_len=32768, scale=0.088, q=a, ws=a, ws_bytes=need):
        return L.flint_decode_attention(q, a, a, 1 << 20, a, a, T, hq, hkv, dh, max_len, scale, a, ws, ws_bytes,
                                        None, None)
    assert call(dh=64) == -2
    assert call(hq=64) == -2          # 16 query heads per kv head
    assert call(hq=30) == -2          # not a multiple of the kv heads
    assert call(T=-1) == -1
    assert call(scale=0.0) == -1
    assert call(T=0) == 0             # no-op
    assert call(q=None) == -1
    assert call(q=a + 8) == -3
    assert call(ws_bytes=need - 16) == -4
    assert call(ws=None) == -4
    assert call(max_len=(1 << 30) + 1) == -2
    assert fm.flint_decode_attention_workspace_bytes(1, 4, (1 << 30) + 1) == 0


def test_expert_parallel_host_validation(L):
    a = 0x100000
    # dispatch: sizes, rank counts, alignment; T = 0 still writes the counts (needs the pointer)
    def disp(T=4, k=6, S=1, E=256, R=8, rank=0, d=2048, x=a, counts=a):
        return L.flint_ep_dispatch(a, a, T, k, S, E, R, rank, x, d, a, a, a, a, counts, a, None, None)
    assert disp(R=9) == -2            # more than 8 ranks
    assert disp(E=250) == -2          # experts not a multiple of the ranks
    assert disp(rank=8) == -1
    assert disp(k=9) == -1
    assert disp(S=2) == -1
    assert disp(d=2044) == -1         # rows of whole 16-byte vectors
    assert disp(counts=None) == -1
    assert disp(x=a + 8) == -3
    # combine
    assert L.flint_ep_combine(a, a, 4, 10, 2048, None, a, None) == -1   # at most 9 slots
    assert L.flint_ep_combine(a, a, 0, 7, 2048, None, a, None) == 0     # no-op
    assert L.flint_ep_combine(a + 8, a, 4, 7, 2048, None, a, None) == -3
    assert L.flint_ep_combine(None, a, 4, 7, 2048, None, a, None) == -1
    # routed forward: the tensor-core path's limits
    s = _shape()
    w = _weights()
    ws_need = fm.flint_moe_workspace_bytes(s, 4)
    assert L.flint_moe_forward_routed(a, 4, None, a, ctypes.byref(w), ctypes.byref(s), None, a, a, ws_need,
                                      None) == -1
    assert L.flint_moe_forward_routed(a, 4, a + 2, a, ctypes.byref(w), ctypes.byref(s), None, a, a, ws_need,
                                      None) == -3
    assert L.flint_moe_forward_routed(a, 4, a, a, ctypes.byref(w), ctypes.byref(s), None, a, a, 64, None) == -4
    assert L.flint_moe_forward_routed(a, 0, a, a, ctypes.byref(w), ctypes.byref(s), None, a, a, ws_need, None) == 0
    assert L.flint_moe_forward_routed(a, 20000, a, a, ctypes.byref(w), ctypes.byref(s), None, a, a, ws_need,
                                      None) == -2


def test_version(L):
    assert "sm_100a" in fm.flint_version()
