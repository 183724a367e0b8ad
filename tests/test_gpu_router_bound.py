"""The certified router's error bound, audited over every (token, expert) pair.

For batches of more than 32 tokens the router computes its logits on the tensor
cores and evaluates the defining fp32 chain only for experts within a bound d of
the k-th choice; experts it excludes are never re-evaluated.  That is safe only if
|chain - tensor-core logit| <= d holds for every pair, chosen or not.  The audit
hook makes the router write every tensor-core logit and its bound; each is checked
here against the oracle's fp32 chain value of the same (t, e).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import compare_routing, device_inputs
from routed_grouped_gemm_softmax_b200 import api
from routed_grouped_gemm_softmax_b200.inputs import CONFIGS, make_inputs

pytestmark = pytest.mark.gpu

CASES = ["prefill", "skewed", "fp8", "ties", "ragged_bias"]


def _inputs(name):
    if name == "fp8":  # the fp8 config's router is the bf16 router over its bf16 x
        cfg = CONFIGS["fp8"]
        inp = make_inputs(cfg, device="cuda", weights=False)
        return cfg, inp.x, inp.router_w, inp.bias
    if name == "ties":  # zero router: every logit is 0 -> all ties, experts 0..k-1 chosen
        cfg = CONFIGS["prefill"].replace(name="ties", T=1000, seed=41)
        g, _ = device_inputs(cfg, zero_router=True)
        return cfg, g["x"], g["router_w"], g["bias"]
    if name == "ragged_bias":
        cfg = CONFIGS["tiny"].replace(name="ragged_bias", T=517, H=320, E=12, top_k=3, I=320, seed=12, zipf_s=1.2)
    else:
        cfg = CONFIGS[name]
    g, _ = device_inputs(cfg)
    return cfg, g["x"], g["router_w"], g["bias"]


@pytest.mark.parametrize("name", CASES)
def test_router_bound_holds_for_every_pair(name):
    cfg, x, rw, bias = _inputs(name)
    T, E, k = cfg.T, cfg.E, cfg.top_k
    assert T > 32  # the certified router
    lt = torch.full((T * E,), float("nan"), dtype=torch.float32, device="cuda")
    bd = torch.full((T * E,), float("nan"), dtype=torch.float32, device="cuda")
    ws = api.workspace(T, cfg.H, cfg.I, E, k, "cuda")
    try:
        api.set_router_audit(lt, bd)
        idx, w = api.moe_route(x, rw, bias, k, ws=ws)
        assert api.moe_get_device_status(ws) == api.MOE_OK
    finally:
        api.set_router_audit(None, None)
    idx_ref, gate_ref, l32, _ = oracle.get().route(x.cpu(), rw.cpu(), None if bias is None else bias.cpu(), k,
                                                   want_logits=True)
    compare_routing(idx, w, idx_ref, gate_ref, name)
    v = lt.view(T, E).cpu().numpy().astype(np.float64)
    d = bd.view(T, E).cpu().numpy().astype(np.float64)
    assert np.isfinite(v).all() and np.isfinite(d).all() and (d > 0).all(), f"{name}: pairs left unwritten"
    gap = np.abs(v - l32.astype(np.float64))
    ratio = gap / d
    worst = np.unravel_index(int(np.argmax(ratio)), ratio.shape)
    rec = {"case": name, "T": T, "H": cfg.H, "E": E, "pairs": int(T * E), "max_gap_over_bound": float(ratio.max()),
           "worst_pair": [int(worst[0]), int(worst[1])], "max_gap": float(gap.max()),
           "median_bound": float(np.median(d))}
    print("router bound audit:", json.dumps(rec))
    out_dir = os.environ.get("MOE_AUDIT_DIR")
    if out_dir:
        with open(os.path.join(out_dir, f"router_bound_{name}.json"), "w") as f:
            json.dump(rec, f)
    bad = np.argwhere(gap > d)
    assert bad.size == 0, f"{name}: |chain - tensor-core logit| > bound at {bad[:5].tolist()} " \
                          f"(max ratio {ratio.max():.3f})"


STAGING = [(8, 2, 4), (8, 4, 4), (8, 2, 2), (1, 1, 1), (2, 2, 1), (3, 2, 8), (2, 2, 8), (1, 1, 8)]


@pytest.mark.parametrize("name", ["prefill", "fp8", "ragged_bias"])
def test_router_staging_policies_route_identically(name):
    """The exact chains do not depend on how their operands are staged: every staging
    policy (chunks in flight, chunk width) gives the default's experts and gates bit for
    bit, and the default matches the oracle."""
    cfg, x, rw, bias = _inputs(name)
    T, E, k = cfg.T, cfg.E, cfg.top_k
    ws = api.workspace(T, cfg.H, cfg.I, E, k, "cuda")
    idx0, w0 = api.moe_route(x, rw, bias, k, ws=ws)
    assert api.moe_get_device_status(ws) == api.MOE_OK
    idx_ref, gate_ref = oracle.get().route(x.cpu(), rw.cpu(), None if bias is None else bias.cpu(), k)[:2]
    compare_routing(idx0, w0, idx_ref, gate_ref, name)
    try:
        for pol in STAGING:
            api.set_cert_staging(*pol)
            idx, w = api.moe_route(x, rw, bias, k, ws=ws)
            assert api.moe_get_device_status(ws) == api.MOE_OK, pol
            assert torch.equal(idx, idx0), pol
            assert torch.equal(w, w0), pol
    finally:
        api.set_cert_staging()
