"""Shared set-up for the GPU parity tests: a layer's synthetic inputs on the
device, packed by the CUDA library, and the oracle's view of the same inputs.

Inputs come from `synth` (seeded); the oracle quantises the same fp32 weights
itself (copied from the device), so no oracle input comes from the CUDA path.
"""
from __future__ import annotations

import numpy as np
import torch

import nvfp4_weight_only_flint_b200 as fm
import oracle
import synth

# Tolerances of the layer contract (outputs in bf16 against the fp64 oracle).
REL_L2_TOL = 5e-3
MAX_ABS_TOL_RMS = 2e-2
NEAR_TIE = 1e-6  # 6th/7th softmax gap below which routed ids are reported, not compared


def bits_to_cuda(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def cuda_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class GpuLayer:
    """One MoE layer's weights on the GPU (fp32 draws + packed NVFP4 or bf16)."""

    def __init__(self, w: synth.Workload, seed: int = 0, layer: int = 0, max_tokens: int = 64,
                 keep_f32: bool = True, wdtype: str | None = None, weights_f32: torch.Tensor | None = None):
        self.w = w
        self.seed, self.layer = seed, layer
        self.wdtype = wdtype or w.wdtype
        d, I, E, S = w.d, w.inter, w.E, w.S
        self.shape = fm.Shape(d, I, E, w.k, S, fm.FLINT_W_NVFP4 if self.wdtype == "nvfp4" else fm.FLINT_W_BF16)
        if weights_f32 is None:
            weights_f32 = synth.layer_weights_torch(seed, layer, E + S, d, I, w.std, device="cuda")
        self.wf32 = weights_f32
        self.ws = torch.empty(fm.flint_moe_workspace_bytes(self.shape, max_tokens), dtype=torch.uint8,
                              device="cuda")
        fm.flint_moe_workspace_init(self.ws)
        if self.wdtype == "nvfp4":
            self.packed = torch.empty(fm.flint_packed_bytes(self.shape), dtype=torch.uint8, device="cuda")
            self.scales = torch.empty(fm.flint_block_scale_bytes(self.shape), dtype=torch.uint8, device="cuda")
            self.tscales = torch.empty((E + S) * 3, dtype=torch.float32, device="cuda")
            fm.flint_pack_nvfp4(self.wf32, 0, self.shape, self.packed, self.scales, self.tscales, self.ws)
            self.weights = fm.Weights(self.packed.data_ptr(), self.scales.data_ptr(), self.tscales.data_ptr())
        else:
            self.wbf16 = self.wf32.to(torch.bfloat16)
            self.packed = torch.empty(fm.flint_packed_bytes(self.shape) // 2, dtype=torch.int16, device="cuda")
            fm.flint_pack_bf16(self.wbf16.view(torch.int16), self.shape, self.packed)
            self.weights = fm.Weights(self.packed.data_ptr(), None, None)
        torch.cuda.synchronize()
        if not keep_f32 and self.wdtype == "nvfp4":
            self.wf32 = None
        self._oracle_cache = {}

    # ------------------------------------------------------------- oracle side
    def expert_f32(self, e: int):
        d, I = self.w.d, self.w.inter
        if self.wf32 is None:
            wl = synth.layer_weights_torch(self.seed, self.layer, self.w.E + self.w.S, d, I, self.w.std)
            m = wl[e].cpu().numpy()
            del wl
        else:
            m = self.wf32[e].cpu().numpy()
        return m[0].reshape(I, d), m[1].reshape(I, d), m[2].reshape(d, I)

    def oracle_expert(self, e: int):
        if e not in self._oracle_cache:
            g, u, dn = self.expert_f32(e)
            if self.wdtype == "nvfp4":
                self._oracle_cache[e] = (oracle.quantize(g), oracle.quantize(u), oracle.quantize(dn))
            else:
                self._oracle_cache[e] = tuple(
                    oracle.BF16Matrix(synth.to_bf16_bits(m), m.shape[0], m.shape[1]) for m in (g, u, dn))
        return self._oracle_cache[e]

    def oracle_forward(self, x_bits, wr_bits, ids, residual_bits=None, n_threads=8, input_norm=False):
        E, S = self.w.E, self.w.S
        need = set(int(e) for e in np.asarray(ids).ravel()) | set(range(E, E + S))
        experts = [self.oracle_expert(e) if e in need else None for e in range(E + S)]
        return oracle.moe_forward(x_bits, wr_bits, experts, d=self.w.d, inter=self.w.inter, E=E, k=self.w.k,
                                  S=S, residual_bits=residual_bits, ids_override=np.asarray(ids, np.int32),
                                  input_norm=input_norm, n_threads=n_threads)

    # ------------------------------------------------------------- GPU side
    def forward(self, x: torch.Tensor, wr: torch.Tensor, residual=None, path=fm.FLINT_PATH_AUTO, pdl=True,
                out=None, input_norm=False, split=False, variant=fm.FLINT_LAYER_AUTO):
        T = x.shape[0]
        out = torch.empty_like(x) if out is None else out
        ids = torch.empty((T, self.w.k), dtype=torch.int32, device="cuda")
        gates = torch.empty((T, self.w.k), dtype=torch.float32, device="cuda")
        opt = fm.Options(path=path, use_pdl=1 if pdl else 0, topk_ids=ids.data_ptr(),
                         topk_weights=gates.data_ptr(), input_rmsnorm=1 if input_norm else 0,
                         split_kernels=1 if split else 0, layer_variant=variant)
        fm.flint_moe_forward_ex(x, T, wr, self.weights, self.shape, residual, out, self.ws, opt)
        return out, ids, gates


def check_routing(ids_gpu, gates_gpu, logits_f64, k):
    """Routed ids bit-exact except near-tie tokens (reported); gates close."""
    ids_o, gates_o, gap = oracle.topk(logits_f64, k)
    near = np.where(gap < NEAR_TIE)[0]
    for t in range(ids_o.shape[0]):
        if t in near:
            continue
        assert ids_gpu[t].tolist() == ids_o[t].tolist(), (t, ids_gpu[t], ids_o[t])
        np.testing.assert_allclose(gates_gpu[t], gates_o[t], rtol=0, atol=2e-6)
        assert abs(float(gates_gpu[t].sum()) - 1.0) <= 1e-6
    return near


def check_output(out_bits, ref_f64, what=""):
    got = synth.bf16_bits_to_f64(out_bits)
    diff = got - ref_f64
    norm = np.linalg.norm(ref_f64)
    rel = np.linalg.norm(diff) / norm if norm > 0 else np.linalg.norm(diff)
    rms = np.sqrt(np.mean(ref_f64 ** 2))
    mx = np.abs(diff).max()
    assert rel <= REL_L2_TOL, f"{what}: rel L2 {rel:.3e} > {REL_L2_TOL}"
    assert mx <= MAX_ABS_TOL_RMS * rms + 1e-30, f"{what}: max abs {mx:.3e} > {MAX_ABS_TOL_RMS}*rms ({rms:.3e})"
    return rel, mx / rms if rms > 0 else 0.0
