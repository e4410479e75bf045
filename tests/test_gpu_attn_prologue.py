"""The attention prologue kernel (fused Q/K RMS normalisation + rotary
embedding + KV-cache write) against the fp64 oracle at the pages' head shape
(32 query, 4 key/value heads of dimension 128): query outputs and cache rows
within one bf16 rounding of the exact values, value heads copied bit for bit,
cache rows outside the tokens' slots untouched, rotary on and off, and the
out-of-range slot / position checks."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_flint_b200 as fm
import oracle
import synth

pytestmark = pytest.mark.gpu

HQ, HKV, DH = 32, 4, 128
SENTINEL = 0x1234


def _table(max_pos, theta=10000.0):
    inv = theta ** (-np.arange(0, DH, 2, dtype=np.float64) / DH)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * inv[None, :]
    return np.concatenate([np.cos(ang), np.sin(ang)], axis=1).astype(np.float32)


def _case(T, rope, seed, n_slots=1000, max_pos=4096, scale=1.0, hq=HQ, hkv=HKV):
    rng = np.random.default_rng(seed)
    qkv = synth.to_bf16_bits((rng.standard_normal((T, hq + 2 * hkv, DH)) * scale).astype(np.float32))
    qw = synth.to_bf16_bits((1.0 + 0.1 * rng.standard_normal(DH)).astype(np.float32))
    kw = synth.to_bf16_bits((1.0 + 0.1 * rng.standard_normal(DH)).astype(np.float32))
    cs = _table(max_pos)
    pos = rng.integers(0, max_pos, T).astype(np.int32)
    slots = rng.permutation(n_slots)[:T].astype(np.int32)
    return qkv, qw, kw, cs, pos, slots


def _run(qkv, qw, kw, cs, pos, slots, rope, n_slots=1000, eps=1e-6, hq=HQ, hkv=HKV):
    T = qkv.shape[0]
    d = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a).view(dt)).cuda()
    q_out = torch.zeros((T, hq, DH), dtype=torch.int16, device="cuda")
    kc = torch.full((n_slots, hkv, DH), SENTINEL, dtype=torch.int16, device="cuda")
    vc = torch.full((n_slots, hkv, DH), SENTINEL, dtype=torch.int16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    fm.flint_qk_norm_rope_kv(d(qkv, np.int16), T, hq, hkv, d(qw, np.int16), d(kw, np.int16), d(cs, np.float32),
                             cs.shape[0], d(pos, np.int32), rope, eps, d(slots, np.int32), n_slots, q_out, kc, vc,
                             status)
    torch.cuda.synchronize()
    u16 = lambda t: t.cpu().numpy().view(np.uint16)
    return u16(q_out), u16(kc), u16(vc), int(status.item())


def _close(got_bits, ref, what):
    got = synth.bf16_bits_to_f64(got_bits)
    rms = np.sqrt(np.mean(ref ** 2, axis=-1, keepdims=True)) + 1e-30
    # one bf16 rounding of the exact value (8 significant bits), plus fp32
    # arithmetic; an absolute floor relative to the head's rms for values
    # the rotation brings near zero
    tol = 2.0 ** -8 * np.abs(ref) + 2.0 ** -14 * rms
    bad = np.abs(got - ref) > tol
    assert not bad.any(), f"{what}: {bad.sum()} elements off, worst {np.max(np.abs(got - ref) - tol)}"


@pytest.mark.parametrize("T,rope", [(1, True), (1, False), (7, True), (64, True), (333, True), (333, False)])
def test_attn_prologue_matches_oracle(T, rope):
    qkv, qw, kw, cs, pos, slots = _case(T, rope, seed=T + (7 if rope else 0))
    q_g, kc, vc, st = _run(qkv, qw, kw, cs, pos, slots, rope)
    assert st == 0
    q_r, k_r, v_r = oracle.qk_norm_rope_kv(qkv, HQ, HKV, qw, kw, cs, pos, rope=rope)
    _close(q_g, q_r, "q")
    _close(kc[slots], k_r, "k cache rows")
    assert np.array_equal(vc[slots], qkv[:, HQ + HKV:])
    untouched = np.setdiff1d(np.arange(kc.shape[0]), slots)
    assert (kc[untouched] == SENTINEL).all() and (vc[untouched] == SENTINEL).all()


@pytest.mark.parametrize("hq,hkv,T", [(7, 3, 37), (5, 1, 3), (1, 2, 11)])
def test_attn_prologue_odd_head_counts(hq, hkv, T):
    # odd head counts put a value head and a query/key head in the two halves
    # of one warp, and an odd task count leaves the last half-warp alone
    qkv, qw, kw, cs, pos, slots = _case(T, True, seed=hq * 100 + hkv, hq=hq, hkv=hkv)
    q_g, kc, vc, st = _run(qkv, qw, kw, cs, pos, slots, True, hq=hq, hkv=hkv)
    assert st == 0
    q_r, k_r, v_r = oracle.qk_norm_rope_kv(qkv, hq, hkv, qw, kw, cs, pos, rope=True)
    _close(q_g, q_r, "q")
    _close(kc[slots], k_r, "k cache rows")
    assert np.array_equal(vc[slots], qkv[:, hq + hkv:])


def test_attn_prologue_large_and_small_magnitudes():
    for scale in (300.0, 1e-3):
        qkv, qw, kw, cs, pos, slots = _case(16, True, seed=int(scale * 10) + 1, scale=scale)
        q_g, kc, vc, st = _run(qkv, qw, kw, cs, pos, slots, True)
        q_r, k_r, _ = oracle.qk_norm_rope_kv(qkv, HQ, HKV, qw, kw, cs, pos, rope=True)
        _close(q_g, q_r, f"q at scale {scale}")
        _close(kc[slots], k_r, f"k at scale {scale}")


def test_attn_prologue_prefill_sized():
    T = 8192
    qkv, qw, kw, cs, pos, _ = _case(T, True, seed=5, n_slots=T, max_pos=T)
    pos = np.arange(T, dtype=np.int32)
    slots = np.arange(T, dtype=np.int32)
    q_g, kc, vc, st = _run(qkv, qw, kw, cs, pos, slots, True, n_slots=T)
    assert st == 0
    rows = np.random.default_rng(2).choice(T, 64, replace=False)
    q_r, k_r, _ = oracle.qk_norm_rope_kv(qkv[rows], HQ, HKV, qw, kw, cs, pos[rows], rope=True)
    _close(q_g[rows], q_r, "q (sampled tokens of 8192)")
    _close(kc[rows], k_r, "k (sampled tokens of 8192)")
    assert np.array_equal(vc, qkv[:, HQ + HKV:])


def test_attn_prologue_index_checks():
    qkv, qw, kw, cs, pos, slots = _case(4, True, seed=9)
    slots[2] = 5000  # outside the 1000-row cache: that token's key and value are skipped
    _, kc, vc, st = _run(qkv, qw, kw, cs, pos, slots, True)
    assert st & fm.FLINT_DEVCHECK_INDEX
    assert (kc[slots[[0, 1, 3]]] != SENTINEL).any()
    qkv, qw, kw, cs, pos, slots = _case(4, True, seed=10)
    pos[1] = cs.shape[0] + 7
    _, _, _, st = _run(qkv, qw, kw, cs, pos, slots, True)
    assert st & fm.FLINT_DEVCHECK_INDEX


def test_attn_prologue_rejects_other_head_dims():
    x = torch.zeros(64, dtype=torch.int16, device="cuda")
    with pytest.raises(fm.FlintError) as ei:
        fm.flint_qk_norm_rope_kv(x, 1, 1, 1, x, x, None, 0, None, False, 1e-6, x, 1, x, x, x, head_dim=64)
    assert ei.value.code == -2
