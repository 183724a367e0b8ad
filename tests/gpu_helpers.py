"""Shared helpers of the GPU parity tests: input placement, tolerances, comparisons."""
from __future__ import annotations

import numpy as np
import torch

from routed_grouped_gemm_softmax_b200.inputs import MoEConfig, make_inputs

# Output tolerances for bf16 outputs against the fp64 oracle: max-abs error and
# relative L2 error.  Gates (fp32 on the GPU, fp64 in the oracle) to a relative 1e-5.
MAX_ABS = 2e-2
REL_L2 = 5e-3
GATE_RTOL = 1e-5


def device_inputs(cfg: MoEConfig, zero_router: bool = False):
    """The config's seeded inputs, drawn on the GPU when large, on both devices."""
    big = cfg.E * cfg.I * cfg.H > (1 << 24)
    inp = make_inputs(cfg, device="cuda" if big else "cpu")
    if zero_router:
        inp.router_w = torch.zeros_like(inp.router_w)
    g = {k: (v.cuda() if v is not None else None) for k, v in
         dict(x=inp.x, router_w=inp.router_w, bias=inp.bias, w_gate=inp.w_gate, w_up=inp.w_up,
              w_down=inp.w_down).items()}
    c = {k: (v.cpu() if v is not None else None) for k, v in g.items()}
    return g, c


def compare_out(out_gpu: torch.Tensor, ref: np.ndarray, what: str = ""):
    o = out_gpu.float().cpu().double().numpy()
    err = o - ref
    max_abs = float(np.abs(err).max()) if err.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(err) / denom) if denom > 0 else float(np.linalg.norm(err))
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


def compare_routing(idx_gpu, w_gpu, idx_ref, gate_ref, what=""):
    ig = idx_gpu.cpu().numpy()
    assert np.array_equal(ig, idx_ref), f"{what}: expert indices differ at " \
        f"{np.argwhere(ig != idx_ref)[:5].tolist()}"
    wg = w_gpu.cpu().double().numpy()
    assert np.allclose(wg, gate_ref, rtol=GATE_RTOL, atol=0), \
        f"{what}: gates max rel err {np.max(np.abs(wg - gate_ref) / np.abs(gate_ref)):.2e}"


def compare_permute(res_gpu: dict, ref: dict, what=""):
    A = ref["sorted_to_flat"].size
    nt = int(res_gpu["num_tiles"].item())
    assert nt == ref["num_tiles"], f"{what}: num_tiles {nt} vs {ref['num_tiles']}"
    assert np.array_equal(res_gpu["offsets"].cpu().numpy(), ref["offsets"]), f"{what}: offsets"
    assert np.array_equal(res_gpu["sorted_to_flat"].cpu().numpy()[:A], ref["sorted_to_flat"]), f"{what}: s2f"
    assert np.array_equal(res_gpu["flat_to_sorted"].cpu().numpy()[:A], ref["flat_to_sorted"]), f"{what}: f2s"
    assert np.array_equal(res_gpu["tile_list"].cpu().numpy()[:nt], ref["tile_list"]), f"{what}: tiles"


def sample_tokens(T: int, n: int, seed: int = 0) -> np.ndarray:
    """First, last and a seeded random sample of token ids."""
    rng = np.random.default_rng(seed)
    s = set([0, T - 1]) | set(rng.choice(T, size=min(n, T), replace=False).tolist())
    return np.array(sorted(s), dtype=np.int32)


def hot_expert_tokens(idx_ref: np.ndarray, n: int, seed: int = 0) -> np.ndarray:
    """A seeded sample of n tokens routed to the most popular expert (its group spans
    the most m-tiles, and on deep groups the pair-of-CTA tiles)."""
    hot = int(np.bincount(idx_ref.reshape(-1)).argmax())
    toks = np.nonzero((idx_ref == hot).any(axis=1))[0]
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(toks, size=min(n, toks.size), replace=False)).astype(np.int32)
