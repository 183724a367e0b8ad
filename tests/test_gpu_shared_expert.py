"""The layer with a shared expert (moe_forward_shared) against the oracle.

Every token passes through the shared SwiGLU expert with weight 1 besides its k
routed experts: out = combine_ffn(...) + shared_ffn(...) (the oracle's two
functions, in fp64).  The shared expert's intermediate width is a multiple of I
and runs as that many extra expert slices inside the same grouped GEMM launches;
the outputs are checked with the bf16 layer's tolerances.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import compare_out, device_inputs
from routed_grouped_gemm_softmax_b200 import api
from routed_grouped_gemm_softmax_b200.inputs import CONFIGS, make_shared_weights

pytestmark = pytest.mark.gpu

CASES = {
    # name: (config, shared_I as a multiple of I)
    "tiny_x1": (CONFIGS["tiny"], 1),
    "tiny_x2": (CONFIGS["tiny"], 2),
    # I = 192: a 128-feature gate/up tile of slice 0 reaches into slice 1's rows (masked)
    "ragged_x2": (CONFIGS["tiny"].replace(name="sh_ragged", T=300, H=512, E=16, top_k=4, I=192, seed=61), 2),
    "bias_x1": (CONFIGS["tiny"].replace(name="sh_bias", T=517, H=320, E=12, top_k=3, I=320, seed=62,
                                        zipf_s=1.2), 1),
    # decode-sized: the fused router/grouping kernels and the combine inside the down GEMM
    "decode_x2": (CONFIGS["decode"], 2),
    "one_token_x3": (CONFIGS["tiny"].replace(name="sh_one", T=1, seed=63), 3),
}


def _oracle(c, idx_ref, gate_ref, sw):
    routed = oracle.combine_ffn(c["x"], idx_ref, gate_ref, c["w_gate"], c["w_up"], c["w_down"])
    return routed + oracle.shared_ffn(c["x"], *[t.cpu() for t in sw])


@pytest.mark.parametrize("name", list(CASES))
def test_shared_expert_layer(name):
    cfg, mult = CASES[name]
    g, c = device_inputs(cfg)
    sw = [t.cuda() for t in make_shared_weights(cfg, mult * cfg.I)]
    k = cfg.top_k
    n = api.moe_workspace_size_shared(cfg.T, cfg.H, cfg.I, cfg.E, k, mult * cfg.I)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    out = api.moe_forward_shared(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], *sw, k, ws=ws)
    assert api.moe_get_device_status(ws) == api.MOE_OK
    idx_ref, gate_ref = oracle.route(c["x"], c["router_w"], c["bias"], k)
    compare_out(out, _oracle(c, idx_ref, gate_ref, sw), name)


def test_shared_expert_pairs_and_schedules():
    # Deep groups (pair-of-CTA tiles, forced) and the one-CTA kernels over grid sizes
    # and every claim order: one result, bitwise, equal to the oracle's within tolerance.
    cfg = CONFIGS["tiny"].replace(name="sh_deep", T=2048, H=256, E=4, top_k=2, I=256, seed=64)
    g, c = device_inputs(cfg)
    sw = [t.cuda() for t in make_shared_weights(cfg, 2 * cfg.I)]
    outs = []
    try:
        for pair, ctas, mode, fused in [("always", 0, False, "never"), ("always", 6, True, "always"),
                                        ("never", 0, False, "never"), ("never", 7, "static_items", "always"),
                                        ("never", 5, "static_experts", "never")]:
            api.set_pair_mma(pair)
            api.set_gemm_ctas(ctas)
            api.set_claim_order(mode)
            api.set_fused_combine(fused)
            outs.append(api.moe_forward_shared(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"],
                                               g["w_down"], *sw, cfg.top_k).clone())
    finally:
        api.set_pair_mma("auto")
        api.set_gemm_ctas(0)
        api.set_claim_order(False)
        api.set_fused_combine("auto")
    idx_ref, gate_ref = oracle.route(c["x"], c["router_w"], c["bias"], cfg.top_k)
    compare_out(outs[0], _oracle(c, idx_ref, gate_ref, sw), "sh_deep pairs")
    compare_out(outs[2], _oracle(c, idx_ref, gate_ref, sw), "sh_deep one-CTA")
    for o in outs[1:2]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    for o in outs[3:]:
        assert torch.equal(o.view(torch.int16), outs[2].view(torch.int16))


@pytest.mark.parametrize("T", [48, 640])
def test_shared_expert_schedule_independence(T):
    # T = 48 sums inside the down GEMM's epilogue, where the CTA that completes a
    # token's k + 2 rows depends on the schedule; the order of the sum does not.
    cfg = CONFIGS["tiny"].replace(name="sh_sched", T=T, H=512, E=16, top_k=4, I=384, seed=65)
    g, c = device_inputs(cfg)
    sw = [t.cuda() for t in make_shared_weights(cfg, 2 * cfg.I)]
    outs = []
    try:
        for ctas, mode in [(0, False), (1, False), (7, True), (0, "static_experts"), (3, "static_items")]:
            api.set_gemm_ctas(ctas)
            api.set_claim_order(mode)
            outs.append(api.moe_forward_shared(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"],
                                               g["w_down"], *sw, cfg.top_k).clone())
    finally:
        api.set_gemm_ctas(0)
        api.set_claim_order(False)
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    idx_ref, gate_ref = oracle.route(c["x"], c["router_w"], c["bias"], cfg.top_k)
    compare_out(outs[0], _oracle(c, idx_ref, gate_ref, sw), f"sh_sched T={T}")


def test_zero_width_shared_expert_is_moe_forward():
    cfg = CONFIGS["tiny"].replace(name="sh_zero", T=200, seed=66)
    g, _ = device_inputs(cfg)
    ref = api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], cfg.top_k)
    z = torch.empty(0, cfg.H, dtype=torch.bfloat16, device="cuda")
    out = api.moe_forward_shared(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], z, z,
                                 torch.empty(cfg.H, 0, dtype=torch.bfloat16, device="cuda"), cfg.top_k)
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_skewed_full_size_with_shared_expert_sampled():
    # The Skewed workload (pair tiles) with a shared expert of 2 x I, checked on 64
    # sampled tokens.
    cfg = CONFIGS["skewed"]
    g, c = device_inputs(cfg)
    sw = make_shared_weights(cfg, 2 * cfg.I, device="cuda")
    out = api.moe_forward_shared(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], *sw,
                                 cfg.top_k)
    idx_ref, gate_ref = oracle.route(c["x"], c["router_w"], c["bias"], cfg.top_k)
    tok = np.sort(np.random.default_rng(3).choice(cfg.T, 64, replace=False)).astype(np.int32)
    ref = oracle.combine_ffn(c["x"], idx_ref, gate_ref, c["w_gate"], c["w_up"], c["w_down"], tokens=tok)
    ref = ref + oracle.shared_ffn(c["x"], *[t.cpu() for t in sw], tokens=tok)
    compare_out(out[torch.as_tensor(tok, device="cuda").long()], ref, "skewed + shared")
