"""Host-side helpers of the expert-parallel layer (no GPU): the per-rank
shapes and the slicing of a layer's weights into a rank's experts (its E/R
routed experts, then the shared expert)."""
import pytest
import torch

import nvfp4_weight_only_flint_b200 as fm
from nvfp4_weight_only_flint_b200 import ep


def test_local_and_packing_shapes():
    s = fm.Shape(2048, 512, 256, 6, 1, fm.FLINT_W_NVFP4)
    ls = ep.local_shape(s, 8)
    assert (ls.d, ls.inter, ls.n_experts, ls.top_k, ls.n_shared, ls.wdtype) == (2048, 512, 33, 1, 0, 0)
    ps = ep.packing_shape(s, 8)
    assert (ps.n_experts, ps.top_k, ps.n_shared) == (32, 6, 1)
    # the packed layout of E/R + S experts is the local shape's layout
    assert fm.flint_packed_bytes(ps) == fm.flint_packed_bytes(ls)
    assert fm.flint_block_scale_bytes(ps) == fm.flint_block_scale_bytes(ls)
    with pytest.raises(ValueError):
        ep.local_shape(fm.Shape(2048, 512, 250, 6, 1, 0), 8)


def test_slice_rank_weights():
    E, S, R = 8, 1, 4
    s = fm.Shape(512, 256, E, 2, S, fm.FLINT_W_NVFP4)
    full = torch.arange(E + S, dtype=torch.float32).reshape(E + S, 1, 1).expand(E + S, 3, 4).contiguous()
    for r in range(R):
        part = ep.slice_rank_weights(full, s, r, R)
        assert part.shape == (E // R + S, 3, 4)
        assert part[:, 0, 0].tolist() == [float(r * 2), float(r * 2 + 1), float(E)]
