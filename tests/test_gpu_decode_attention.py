"""The decode attention kernels (split-K over the context on the register-
fragment tensor cores, then the chunk combine) against the fp64 oracle at the
pages' head shape (32 query, 4 key/value heads of dimension 128): one token
and batches, contexts from one key to 32K rows, ragged lengths and offsets,
peaked and flat score distributions, empty ranges, the index checks, and the
multi-chunk split against the single-chunk path.

Tolerance: the weights enter the value sum rounded to bf16 (2^-9 relative
each) and are normalised by the sum of the rounded weights, so each output is
a convex combination of the values with weights off by at most about 2^-8
relative: |err| <= 2^-8 sum_j w_j |v_j| (computed by the oracle on |v|), plus
the final bf16 rounding 2^-9 |out|; the test allows 2^-8 (|ref| + 1.25 A)."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_flint_b200 as fm
import oracle
import synth

pytestmark = pytest.mark.gpu

HQ, HKV, DH = 32, 4, 128
SCALE = 1.0 / np.sqrt(DH)


def _bits(rng, shape, scale=1.0):
    return synth.to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def _run(q, k, v, start, length, max_len=None, status=None):
    T = q.shape[0]
    rows = k.shape[0]
    if max_len is None:
        max_len = max(1, int(np.max(length)) if T else 1)
    d = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a).view(dt)).cuda()
    out = torch.full((T, HQ, DH), 0x7FC0, dtype=torch.int16, device="cuda")  # NaN sentinel
    nb = fm.flint_decode_attention_workspace_bytes(T, HKV, max_len)
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda") if nb else None
    fm.flint_decode_attention(d(q, np.int16), d(k, np.int16), d(v, np.int16), rows, d(start, np.int64),
                              d(length, np.int32), T, HQ, HKV, max_len, SCALE, out, ws, status)
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint16)


def _check(got_bits, q, k, v, start, length, what=""):
    ref = oracle.decode_attention(q, k, v, start, length, scale=SCALE)
    a = oracle.decode_attention(q, k, v & np.uint16(0x7FFF), start, length, scale=SCALE)
    got = synth.bf16_bits_to_f64(got_bits)
    tol = 2.0 ** -8 * (np.abs(ref) + 1.25 * a) + 1e-30
    err = np.abs(got - ref)
    bad = ~(err <= tol)
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} off, worst excess {np.nanmax(err - tol)}"
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert rel < 5e-3, f"{what}: rel-L2 {rel}"


def _case(seed, lengths, q_scale=1.0, gap=0):
    """One cache region per token, back to back (gap rows between them)."""
    rng = np.random.default_rng(seed)
    lengths = np.asarray(lengths, np.int32)
    T = len(lengths)
    start = np.zeros(T, np.int64)
    pos = 0
    for t in range(T):
        start[t] = pos
        pos += int(lengths[t]) + gap
    rows = max(pos, 1)
    return (_bits(rng, (T, HQ, DH), q_scale), _bits(rng, (rows, HKV, DH)), _bits(rng, (rows, HKV, DH)), start,
            lengths)


@pytest.mark.parametrize("lengths", [[1], [17], [64], [65], [1000], [4096], [32768]])
def test_decode_attention_one_token(lengths):
    q, k, v, start, length = _case(lengths[0], lengths)
    _check(_run(q, k, v, start, length), q, k, v, start, length, f"L={lengths[0]}")


@pytest.mark.parametrize("T,max_len", [(2, 3000), (8, 2048), (64, 4096), (200, 700)])
def test_decode_attention_ragged_batch(T, max_len):
    rng = np.random.default_rng(T)
    lengths = rng.integers(1, max_len + 1, T)
    lengths[0] = max_len
    q, k, v, start, length = _case(T + 100, lengths, gap=3)
    _check(_run(q, k, v, start, length, max_len=max_len), q, k, v, start, length, f"T={T}")


def test_decode_attention_shared_prefix_rows():
    # tokens reading overlapping row ranges of one cache (a shared prefix)
    rng = np.random.default_rng(5)
    rows = 3000
    q = _bits(rng, (4, HQ, DH))
    k, v = _bits(rng, (rows, HKV, DH)), _bits(rng, (rows, HKV, DH))
    start = np.array([0, 0, 100, 2999], np.int64)
    length = np.array([3000, 1500, 2900, 1], np.int32)
    _check(_run(q, k, v, start, length), q, k, v, start, length, "overlapping ranges")


@pytest.mark.parametrize("q_scale", [8.0, 30.0])
def test_decode_attention_peaked_scores(q_scale):
    # scores with spreads of tens to hundreds: the running max moves often and
    # most weights underflow to zero
    q, k, v, start, length = _case(int(q_scale), [5000, 300], q_scale=q_scale)
    _check(_run(q, k, v, start, length), q, k, v, start, length, f"q x{q_scale}")


def test_decode_attention_empty_ranges_and_single_chunk_path():
    q, k, v, start, length = _case(9, [0, 50, 0, 2000])
    got = _run(q, k, v, start, length)
    assert not synth.bf16_bits_to_f64(got[[0, 2]]).any()  # zeros, not the NaN sentinel
    _check(got, q, k, v, start, length, "with empty ranges")
    # a large max_len bound changes the chunking, not the result beyond rounding
    got2 = _run(q, k, v, start, length, max_len=60000)
    _check(got2, q, k, v, start, length, "max_len 60000")
    # batch of 300 tokens: one chunk per (token, kv head), finished in place
    q, k, v, start, length = _case(10, np.full(300, 130))
    assert fm.flint_decode_attention_workspace_bytes(300, HKV, 130) == 0
    _check(_run(q, k, v, start, length), q, k, v, start, length, "single-chunk path")


def test_decode_attention_index_checks():
    q, k, v, start, length = _case(11, [100, 200, 50])
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    bad_len = length.copy()
    bad_len[1] = 250  # above max_len 200: clamped to 200 and flagged
    got = _run(q, k, v, start, bad_len, max_len=200, status=st)
    assert int(st.item()) & fm.FLINT_DEVCHECK_INDEX
    clamp = bad_len.copy()
    clamp[1] = 200
    _check(got, q, k, v, start, clamp, "clamped length")
    st.zero_()
    bad_start = start.copy()
    bad_start[2] = k.shape[0] - 10  # range runs past the cache: that token gives zeros
    got = _run(q, k, v, bad_start, length, status=st)
    assert int(st.item()) & fm.FLINT_DEVCHECK_INDEX
    assert not synth.bf16_bits_to_f64(got[2]).any()
    _check(got[:2], q[:2], k, v, start[:2], length[:2], "valid tokens beside a bad one")


def test_decode_attention_rejects_unsupported():
    x = torch.zeros(64, dtype=torch.int64, device="cuda")
    with pytest.raises(fm.FlintError) as ei:
        fm.flint_decode_attention(x, x, x, 1, x, x, 1, HQ, HKV, 1, SCALE, x, head_dim=64)
    assert ei.value.code == -2
