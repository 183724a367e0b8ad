"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Routing (expert indices), the permutation, the group offsets and the tile list
must match bit for bit; gates to a relative 1e-5; the layer output (bf16) to
max-abs <= 2e-2 and relative L2 <= 5e-3 against the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (compare_out, compare_permute, compare_routing, device_inputs,
                         hot_expert_tokens, sample_tokens)
from routed_grouped_gemm_softmax_b200 import api
from routed_grouped_gemm_softmax_b200.inputs import CONFIGS, make_shared_weights

pytestmark = pytest.mark.gpu

# Small-to-mid shapes that the oracle finishes in seconds, spanning several tiles
# and ragged tails in rows (groups not a multiple of 128) and columns (I = 64 mod 128).
SMALL = {
    "tiny": CONFIGS["tiny"],
    "ragged": CONFIGS["tiny"].replace(name="ragged", T=300, H=512, E=16, top_k=4, I=192, seed=11),
    "ragged_bias": CONFIGS["tiny"].replace(name="ragged_bias", T=517, H=320, E=12, top_k=3, I=320,
                                           seed=12, zipf_s=1.2),
    "one_token": CONFIGS["tiny"].replace(name="one_token", T=1, H=256, E=8, top_k=2, seed=13),
    "top1": CONFIGS["tiny"].replace(name="top1", T=200, top_k=1, seed=14),
    "topk_all": CONFIGS["tiny"].replace(name="topk_all", T=96, top_k=8, seed=15),
    "wide_e": CONFIGS["tiny"].replace(name="wide_e", T=40, H=256, E=300, top_k=5, I=128, seed=16),
}


@pytest.fixture(scope="module", autouse=True)
def _lib_and_defaults():
    api.lib()
    api.set_gemm_ctas(0)
    api.set_claim_order(False)
    yield
    api.set_gemm_ctas(0)
    api.set_claim_order(False)


def _full_layer_check(cfg, zero_router=False):
    g, c = device_inputs(cfg, zero_router)
    k = cfg.top_k
    idx_ref, gate_ref = oracle.route(c["x"], c["router_w"], c["bias"], k)
    idx, w = api.moe_route(g["x"], g["router_w"], g["bias"], k)
    compare_routing(idx, w, idx_ref, gate_ref, cfg.name)
    perm_ref = oracle.permute(idx_ref, cfg.E)
    compare_permute(api.moe_permute(idx, cfg.E), perm_ref, cfg.name)
    ws = api.workspace(cfg.T, cfg.H, cfg.I, cfg.E, k, "cuda")
    out = api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], k, ws=ws)
    assert api.moe_get_device_status(ws) == api.MOE_OK
    ref = oracle.combine_ffn(c["x"], idx_ref, gate_ref, c["w_gate"], c["w_up"], c["w_down"])
    return compare_out(out, ref, cfg.name)


@pytest.mark.parametrize("name", list(SMALL))
def test_layer_small(name):
    _full_layer_check(SMALL[name])


def test_uniform_router_all_to_first_experts():
    # router_w = 0: every logit ties, so every token picks experts 0..k-1 (lower index
    # wins) with gates 1/k -- k groups of T rows (several tiles each), the rest empty.
    cfg = CONFIGS["tiny"].replace(name="ties", T=300, top_k=3, seed=21)
    _full_layer_check(cfg, zero_router=True)


def test_one_hot_expert_takes_everything():
    # A huge bias on one expert routes every token's first choice there (one group of
    # T rows = many m-tiles on one expert; the claim queue spreads them over all SMs).
    cfg = CONFIGS["tiny"].replace(name="hot", T=700, top_k=2, seed=22)
    g, c = device_inputs(cfg)
    bias = torch.zeros(cfg.E, dtype=torch.float32)
    bias[3] = 1000.0
    g["bias"], c["bias"] = bias.cuda(), bias
    idx_ref, gate_ref = oracle.route(c["x"], c["router_w"], bias, 2)
    assert np.all(idx_ref[:, 0] == 3)
    out = api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], 2)
    ref = oracle.combine_ffn(c["x"], idx_ref, gate_ref, c["w_gate"], c["w_up"], c["w_down"])
    compare_out(out, ref, "hot")


def test_router_expert_slice_without_candidates():
    # The certified router (T > 32) splits the experts of a token block over a
    # cluster of CTAs; a bias that routes every token to experts 0..3 leaves the upper
    # slices without a single candidate.  Those CTAs still read and release every
    # staged chunk, and the routing is the oracle's.
    cfg = CONFIGS["tiny"].replace(name="slice", T=256, H=256, E=64, I=128, top_k=4, seed=28)
    g, c = device_inputs(cfg)
    bias = torch.zeros(cfg.E, dtype=torch.float32)
    bias[:4] = 1000.0
    g["bias"], c["bias"] = bias.cuda(), bias
    idx_ref, gate_ref = oracle.route(c["x"], c["router_w"], bias, cfg.top_k)
    assert np.all(np.sort(idx_ref, axis=1) == np.arange(4))
    ws = api.workspace(cfg.T, cfg.H, cfg.I, cfg.E, cfg.top_k, "cuda")
    out = api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], cfg.top_k, ws=ws)
    assert api.moe_get_device_status(ws) == api.MOE_OK
    ref = oracle.combine_ffn(c["x"], idx_ref, gate_ref, c["w_gate"], c["w_up"], c["w_down"])
    compare_out(out, ref, "slice")
    idx, w = api.moe_route(g["x"], g["router_w"], g["bias"], cfg.top_k)
    compare_routing(idx, w, idx_ref, gate_ref, "slice")


def test_group_sizes_at_tile_edges():
    # Groups of exactly 128 rows (one full tile), 129 rows (a full tile plus one row)
    # and 5 rows.  Router rows 0 and 1 give logit(e) = x0*e - x1*e^2, which with
    # x1 = 1 peaks exactly at e = x0/2, so x0 chooses each token's expert.
    cfg = CONFIGS["tiny"].replace(name="edges", T=128 + 129 + 5, top_k=1, seed=23)
    g, c = device_inputs(cfg)
    x = c["x"].clone()
    rw = torch.zeros_like(c["router_w"])
    e = torch.arange(8, dtype=torch.float32)
    rw[0, :] = e.to(torch.bfloat16)
    rw[1, :] = (-e * e).to(torch.bfloat16)
    x[:, 1] = 1.0
    x[:128, 0] = 0.0      # expert 0
    x[128:257, 0] = 14.0  # expert 7
    x[257:, 0] = 6.0      # expert 3
    g["x"], c["x"] = x.cuda(), x
    g["router_w"], c["router_w"] = rw.cuda(), rw
    idx_ref, gate_ref = oracle.route(x, rw, None, 1)
    counts = np.bincount(idx_ref[:, 0], minlength=8)
    assert counts[0] == 128 and counts[7] == 129 and counts[3] == 5
    perm_ref = oracle.permute(idx_ref, 8)
    idx, w = api.moe_route(g["x"], g["router_w"], None, 1)
    compare_routing(idx, w, idx_ref, gate_ref, "edges")
    compare_permute(api.moe_permute(idx, 8), perm_ref, "edges")
    out = api.moe_forward(g["x"], g["router_w"], None, g["w_gate"], g["w_up"], g["w_down"], 1)
    ref = oracle.combine_ffn(x, idx_ref, gate_ref, c["w_gate"], c["w_up"], c["w_down"])
    compare_out(out, ref, "edges")


@pytest.mark.parametrize("T", [640, 48])
def test_schedule_independence(T):
    # The result is bitwise the same whatever the number of persistent CTAs and the
    # order in which they claim items: sums are ordered by the tile, not the schedule.
    # T = 48 combines inside the down GEMM, where the CTA that completes a token's
    # rows (and so does its sum) depends on the schedule; the sum's order does not.
    cfg = CONFIGS["tiny"].replace(name="sched", T=T, H=512, E=16, top_k=4, I=384, seed=24)
    g, _ = device_inputs(cfg)
    outs = []
    api.set_fused_combine("always" if T <= 64 else "auto")
    try:
        for ctas, rev in [(0, False), (1, False), (7, True), (148, False), (0, True), (3, True),
                          (0, "static_items"), (0, "static_experts"), (5, "static_experts")]:
            api.set_gemm_ctas(ctas)
            api.set_claim_order(rev)
            outs.append(api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"],
                                        g["w_down"], cfg.top_k).clone())
    finally:
        api.set_gemm_ctas(0)
        api.set_claim_order(False)
        api.set_fused_combine("auto")
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    # and the common result against the oracle
    _, c = device_inputs(cfg)
    idx_ref, gate_ref = oracle.route(c["x"], c["router_w"], c["bias"], cfg.top_k)
    compare_out(outs[0], oracle.combine_ffn(c["x"], idx_ref, gate_ref, c["w_gate"], c["w_up"], c["w_down"]),
                f"sched T={T}")


PAIR_CASES = {
    "ragged": SMALL["ragged"],            # ~75 rows per expert: pair tiles with an empty second half
    "ragged_bias": SMALL["ragged_bias"],  # H = 320: a down n-tile whose second half lies past H
    "deep": CONFIGS["tiny"].replace(name="deep", T=2048, H=256, E=4, top_k=2, I=256, seed=25),  # full pairs
}


@pytest.mark.parametrize("name", list(PAIR_CASES))
def test_pair_cta_gemms(name):
    # The pair-of-CTA GEMMs (cta_group::2) against the oracle, and bitwise stable
    # across grid sizes and claim orders.
    cfg = PAIR_CASES[name]
    g, c = device_inputs(cfg)
    k = cfg.top_k
    outs = []
    try:
        api.set_pair_mma("always")
        for ctas, rev in [(0, False), (2, False), (0, True), (10, True)]:
            api.set_gemm_ctas(ctas)
            api.set_claim_order(rev)
            ws = api.workspace(cfg.T, cfg.H, cfg.I, cfg.E, k, "cuda")
            outs.append(api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], k,
                                        ws=ws).clone())
            assert api.moe_get_device_status(ws) == api.MOE_OK
    finally:
        api.set_pair_mma("auto")
        api.set_gemm_ctas(0)
        api.set_claim_order(False)
    # the combine inside the pair down GEMM's epilogue: the same sum in the same order
    try:
        api.set_pair_mma("always")
        api.set_fused_combine("always")
        for ctas in (0, 6):
            api.set_gemm_ctas(ctas)
            outs.append(api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"],
                                        k).clone())
    finally:
        api.set_pair_mma("auto")
        api.set_fused_combine("auto")
        api.set_gemm_ctas(0)
    idx_ref, gate_ref = oracle.route(c["x"], c["router_w"], c["bias"], k)
    ref = oracle.combine_ffn(c["x"], idx_ref, gate_ref, c["w_gate"], c["w_up"], c["w_down"])
    compare_out(outs[0], ref, f"{name} pair GEMMs")
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))


def test_repeat_calls_same_workspace():
    # Counters and status are reset by the calls themselves: back-to-back calls on one
    # workspace give identical results (graph-replay style reuse).
    cfg = SMALL["ragged"]
    g, _ = device_inputs(cfg)
    ws = api.workspace(cfg.T, cfg.H, cfg.I, cfg.E, cfg.top_k, "cuda")
    a = api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], cfg.top_k, ws=ws).clone()
    b = api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], cfg.top_k, ws=ws)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert api.moe_get_device_status(ws) == api.MOE_OK


ROUTING_CASES = {
    "decode": CONFIGS["decode"],
    "one_token": SMALL["one_token"],
    "small32": CONFIGS["decode"].replace(name="small32", T=29, E=64, top_k=6, seed=31),
    "odd_e_small": CONFIGS["tiny"].replace(name="odd_e_small", T=20, H=192, E=12, top_k=3, seed=32),
    "tiny": CONFIGS["tiny"],
    "ragged_bias": SMALL["ragged_bias"],
    "wide_e": SMALL["wide_e"],
}


@pytest.mark.parametrize("name", list(ROUTING_CASES))
def test_forward_routing_matches_oracle(name):
    # The forward's own routing and permutation (read back from its workspace) must be
    # bit-exact too -- for small batches they come from the fused router+permute kernel --
    # and so must the router's fp32 chain values: all of them for T <= 32, the chosen
    # experts' ones for the certified tensor-core router above.
    cfg = ROUTING_CASES[name]
    g, c = device_inputs(cfg)
    k = cfg.top_k
    ws = api.workspace(cfg.T, cfg.H, cfg.I, cfg.E, k, "cuda")
    idx_ref, gate_ref, l32, _ = oracle.get().route(c["x"], c["router_w"], c["bias"], k, want_logits=True)
    for _ in range(2):  # the second call checks the self-reset of the router's ticket
        api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], k, ws=ws)
        assert api.moe_get_device_status(ws) == api.MOE_OK
        r = api.forward_routing(ws, cfg.T, cfg.H, cfg.I, cfg.E, k)
        compare_routing(r["topk_idx"], r["topk_w"], idx_ref, gate_ref, name)
        compare_permute(r, oracle.permute(idx_ref, cfg.E), name)
        lg = r["logits"].cpu().numpy()
        if cfg.T <= 32:
            bad = np.argwhere(lg.view(np.uint32) != l32.view(np.uint32))
        else:
            rows = np.arange(cfg.T)[:, None]
            bad = np.argwhere(lg[rows, idx_ref].view(np.uint32) != l32[rows, idx_ref].view(np.uint32))
        assert bad.size == 0, f"{name}: chain values differ at {bad[:5].tolist()}"


def test_cuda_graph_replay():
    cfg = SMALL["ragged"]
    g, c = device_inputs(cfg)
    ws = api.workspace(cfg.T, cfg.H, cfg.I, cfg.E, cfg.top_k, "cuda")
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], cfg.top_k,
                        out=out, ws=ws)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], cfg.top_k,
                        out=out, ws=ws)
    out.zero_()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    idx_ref, gate_ref = oracle.route(c["x"], c["router_w"], c["bias"], cfg.top_k)
    ref = oracle.combine_ffn(c["x"], idx_ref, gate_ref, c["w_gate"], c["w_up"], c["w_down"])
    compare_out(out, ref, "graph")
    del graph


def test_pipeline_wait_timeout_is_reported_and_recoverable():
    # Test hook: every GEMM CTA's MMA thread first waits on a barrier that nothing
    # signals, with a 2 ms bound.  The wait runs out, the kernels record
    # MOE_ERR_TIMEOUT, drain their own copies and return; the next call with the
    # default settings must be correct on the same workspace.
    cfg = SMALL["ragged"]
    g, c = device_inputs(cfg)
    ws = api.workspace(cfg.T, cfg.H, cfg.I, cfg.E, cfg.top_k, "cuda")
    try:
        api.set_wait_limit_us(2000, stall_test=True)
        api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], cfg.top_k, ws=ws)
        assert api.moe_get_device_status(ws) == 5  # MOE_ERR_TIMEOUT
    finally:
        api.set_wait_limit_us(0, stall_test=False)
    out = api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], cfg.top_k, ws=ws)
    assert api.moe_get_device_status(ws) == api.MOE_OK
    idx_ref, gate_ref = oracle.route(c["x"], c["router_w"], c["bias"], cfg.top_k)
    compare_out(out, oracle.combine_ffn(c["x"], idx_ref, gate_ref, c["w_gate"], c["w_up"], c["w_down"]), "after timeout")


def test_bad_expert_index_flagged():
    idx = torch.tensor([[0, 1], [5, 9]], dtype=torch.int32, device="cuda")  # 9 >= E=8
    ws = api.workspace(2, 256, 64, 8, 2, "cuda")
    api.moe_permute(idx, 8, ws=ws)
    assert api.moe_get_device_status(ws) == 6  # MOE_ERR_BAD_INDEX
    assert api.moe_get_device_status(ws) == api.MOE_OK  # cleared by the read


def test_empty_batch_is_noop():
    x = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    rw = torch.zeros(256, 8, dtype=torch.bfloat16, device="cuda")
    wg = torch.zeros(8, 64, 256, dtype=torch.bfloat16, device="cuda")
    wd = torch.zeros(8, 256, 64, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    out = api.moe_forward(x, rw, None, wg, wg, wd, 2, ws=ws)
    assert out.shape == (0, 256)


# ------------------------------------------------------------- full-size configs

@pytest.mark.parametrize("name", ["decode", "prefill", "skewed"])
def test_full_size(name):
    """Full-size workloads: routing, permutation and offsets bit-exact for every token;
    the layer output checked on a sample of tokens the oracle evaluates one by one --
    at least 256 tokens (every token of Decode), 64 of them routed to the most popular
    expert, whose group spans the most tiles (on Skewed, pair-of-CTA tiles)."""
    cfg = CONFIGS[name]
    g, c = device_inputs(cfg)
    k = cfg.top_k
    idx_ref, gate_ref = oracle.route(c["x"], c["router_w"], c["bias"], k)
    idx, w = api.moe_route(g["x"], g["router_w"], g["bias"], k)
    compare_routing(idx, w, idx_ref, gate_ref, name)
    compare_permute(api.moe_permute(idx, cfg.E), oracle.permute(idx_ref, cfg.E), name)
    ws = api.workspace(cfg.T, cfg.H, cfg.I, cfg.E, k, "cuda")
    out = api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], k, ws=ws)
    assert api.moe_get_device_status(ws) == api.MOE_OK
    hot = hot_expert_tokens(idx_ref, 64, seed=cfg.seed)
    rest = np.setdiff1d(sample_tokens(cfg.T, cfg.T, seed=cfg.seed), hot)  # every other token, shuffled below
    rng = np.random.default_rng(cfg.seed)
    extra = rng.permutation(rest)[:max(0, min(cfg.T, 256) - hot.size)]
    tok = np.union1d(np.union1d(hot, extra), [0, cfg.T - 1]).astype(np.int32)
    assert tok.size >= min(cfg.T, 256) and np.intersect1d(tok, hot).size == hot.size
    ref = oracle.combine_ffn(c["x"], idx_ref, gate_ref, c["w_gate"], c["w_up"], c["w_down"], tokens=tok)
    max_abs, rel = compare_out(out[torch.as_tensor(tok, device="cuda").long()], ref, name)
    print(f"full size {name}: {tok.size} tokens, max_abs={max_abs:.3e} rel_l2={rel:.3e}")


LAYER_CASES = {
    "ragged": (SMALL["ragged"], "auto"),
    "ragged_bias": (SMALL["ragged_bias"], "auto"),
    "small_fused_combine": (CONFIGS["tiny"].replace(name="lay48", T=48, H=512, E=16, top_k=4, I=384, seed=26), "auto"),
    "deep_pairs": (PAIR_CASES["deep"], "always"),
    "decode": (CONFIGS["decode"], "auto"),
}


@pytest.mark.parametrize("name", list(LAYER_CASES))
def test_layer_gemm_matches_two_launches(name):
    # Both expert GEMMs in one persistent launch (down items wait on per-m-tile
    # readiness counts of the gate/up epilogues) give the two-launch result bit for
    # bit, over grid sizes (one CTA included: it runs every gate/up item first) and
    # both queue orders, and the oracle's within tolerance.
    cfg, pair = LAYER_CASES[name]
    g, c = device_inputs(cfg)
    k = cfg.top_k
    outs = []
    try:
        api.set_pair_mma(pair)
        for lg, ctas, rev in [("never", 0, False), ("always", 0, False), ("always", 2 if pair == "always" else 1, False),
                              ("always", 6, True), ("always", 148, False)]:
            api.set_layer_gemm(lg)
            api.set_gemm_ctas(ctas)
            api.set_claim_order(rev)
            ws = api.workspace(cfg.T, cfg.H, cfg.I, cfg.E, k, "cuda")
            outs.append(api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], k,
                                        ws=ws).clone())
            assert api.moe_get_device_status(ws) == api.MOE_OK
            plan = api.forward_plan(cfg.T, cfg.H, cfg.I, cfg.E, k)
            assert bool(plan & api.PLAN_LAYER_GEMM) == (lg == "always")
    finally:
        api.set_pair_mma("auto")
        api.set_layer_gemm("auto")
        api.set_gemm_ctas(0)
        api.set_claim_order(False)
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    idx_ref, gate_ref = oracle.route(c["x"], c["router_w"], c["bias"], k)
    tok = sample_tokens(cfg.T, 64, seed=cfg.seed)
    ref = oracle.combine_ffn(c["x"], idx_ref, gate_ref, c["w_gate"], c["w_up"], c["w_down"], tokens=tok)
    compare_out(outs[1][torch.as_tensor(tok, device="cuda").long()], ref, f"{name} layer GEMM")


DIRECT_A_CASES = {
    "ragged": (SMALL["ragged"], "auto", 0),            # ragged group tails
    "one_token": (SMALL["one_token"], "auto", 0),      # one-row tiles
    "wide_e": (SMALL["wide_e"], "auto", 0),            # 300 experts, mostly one-row groups
    "ragged_bias": (SMALL["ragged_bias"], "auto", 0),  # H = 320: five 64-column K blocks
    "decode": (CONFIGS["decode"], "auto", 0),
    "prefill_rows": (CONFIGS["tiny"].replace(name="da_pf", T=1024, H=512, E=8, top_k=2, I=256, seed=27), "auto", 0),
    "deep_pairs": (PAIR_CASES["deep"], "always", 0),
    "ragged_pairs": (PAIR_CASES["ragged"], "always", 0),  # pair tiles with an empty or short second half
    "ragged_shared": (SMALL["ragged"], "auto", 2),        # the shared expert's tiles read x with row boxes
    "pairs_shared": (PAIR_CASES["ragged_bias"], "always", 1),
}


@pytest.mark.parametrize("name", list(DIRECT_A_CASES))
def test_direct_a_rows_match_the_sorted_copy(name):
    # The gate/up GEMM gathering its A rows straight from x (four rows per TMA
    # tile::gather4, the tail's missing rows repeating the last) gives the result of
    # reading the expert-sorted copy of x bit for bit: one or two GEMM launches, one
    # CTA per SM or a few, both queue orders, with the router's one-launch form (the
    # tile list written by the kernel just before the GEMM) and its multi-kernel form.
    cfg, pair, mult = DIRECT_A_CASES[name]
    g, c = device_inputs(cfg)
    k = cfg.top_k
    sw = [t.cuda() for t in make_shared_weights(cfg, mult * cfg.I)] if mult else None
    outs = []
    try:
        api.set_pair_mma(pair)
        for da, lg, ctas, rev in [("never", "never", 0, False), ("always", "never", 0, False),
                                  ("always", "always", 0, False), ("never", "always", 0, False),
                                  ("always", "always", 4, True), ("always", "never", 6, True)]:
            api.set_direct_a(da)
            api.set_layer_gemm(lg)
            api.set_gemm_ctas(ctas)
            api.set_claim_order(rev)
            if sw:
                ws = torch.empty(api.moe_workspace_size_shared(cfg.T, cfg.H, cfg.I, cfg.E, k, mult * cfg.I),
                                 dtype=torch.uint8, device="cuda")
                o = api.moe_forward_shared(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"],
                                           *sw, k, ws=ws)
            else:
                ws = api.workspace(cfg.T, cfg.H, cfg.I, cfg.E, k, "cuda")
                o = api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], k, ws=ws)
            outs.append(o.clone())
            assert api.moe_get_device_status(ws) == api.MOE_OK
            plan = api.forward_plan(cfg.T, cfg.H, cfg.I, cfg.E, k)
            assert bool(plan & api.PLAN_DIRECT_A) == (da == "always")
    finally:
        api.set_pair_mma("auto")
        api.set_direct_a("auto")
        api.set_layer_gemm("auto")
        api.set_gemm_ctas(0)
        api.set_claim_order(False)
    for i, o in enumerate(outs[1:], 1):
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16)), (name, i)
    if sw is None:
        idx_ref, gate_ref = oracle.route(c["x"], c["router_w"], c["bias"], k)
        tok = sample_tokens(cfg.T, 64, seed=cfg.seed)
        ref = oracle.combine_ffn(c["x"], idx_ref, gate_ref, c["w_gate"], c["w_up"], c["w_down"], tokens=tok)
        compare_out(outs[1][torch.as_tensor(tok, device="cuda").long()], ref, f"{name} direct A rows")


def test_stage_events_outside_and_inside_capture():
    # The stage marks are recorded on the forward's stream both when the stream is
    # being captured into a CUDA graph (as graph nodes) and when it is not.
    cfg = SMALL["ragged"]
    g, _ = device_inputs(cfg)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(api.STAGES.__len__() + 1)]
    for e in ev:
        e.record()
    ws = api.workspace(cfg.T, cfg.H, cfg.I, cfg.E, cfg.top_k, "cuda")
    try:
        api.set_stage_events(ev)
        api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], cfg.top_k, ws=ws)
        torch.cuda.synchronize()
        direct = [ev[i].elapsed_time(ev[i + 1]) for i in range(len(ev) - 1)]
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(graph, stream=s):
                api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], cfg.top_k,
                                ws=ws, stream=s)
    finally:
        api.set_stage_events(None)
    torch.cuda.current_stream().wait_stream(s)
    graph.replay()
    torch.cuda.synchronize()
    replayed = [ev[i].elapsed_time(ev[i + 1]) for i in range(len(ev) - 1)]
    del graph
    assert all(t >= 0 for t in direct) and sum(direct) > 0
    assert all(t >= 0 for t in replayed) and sum(replayed) > 0
    assert api.moe_get_device_status(ws) == api.MOE_OK
