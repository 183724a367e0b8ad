"""FP8 block-scaled layer: CUDA path vs the CPU oracle through the C ABI.

The activation quantiser's codes and scales must match the oracle bit for bit (same
bf16 inputs, same fp32 decisions).  The layer output is compared with the fp8
oracle at relative L2 <= 3e-2; routing is the bf16 router and stays bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import compare_routing, sample_tokens
from routed_grouped_gemm_softmax_b200 import api
from routed_grouped_gemm_softmax_b200.inputs import CONFIGS, make_fp8_weights, make_inputs

pytestmark = pytest.mark.gpu

FP8_REL_L2 = 3e-2


def rel_l2(out_gpu, ref):
    o = out_gpu.float().cpu().double().numpy()
    return float(np.linalg.norm(o - ref) / np.linalg.norm(ref))


def test_quantizer_bit_exact():
    rng = np.random.default_rng(1)
    a = torch.as_tensor(rng.standard_normal((37, 1024)).astype(np.float32) * 3).to(torch.bfloat16)
    a[3, 128:256] = 0.0                    # all-zero group -> scale 1, codes 0
    a[5, :] *= 1e-30                       # tiny values (subnormal e4m3 codes)
    a[7, 0] = 1e4                          # one huge value per group
    a[7, 5] = -0.004                       # a negative value that rounds to zero: code -0 (0x80)
    q, s = api.moe_quantize_rows_fp8(a.cuda())
    qr, sr = oracle.quantize_rows(a)
    assert np.array_equal(s.cpu().numpy(), sr)
    assert np.array_equal(q.cpu().numpy(), qr)


def _fp8_case(cfg, device="cuda"):
    inp = make_inputs(cfg, device=device, weights=False)
    w = make_fp8_weights(cfg, device=device)
    return inp, w


def _run_fp8(cfg, inp, w):
    g = {k: v.cuda() for k, v in w.items()}
    ws = api.workspace(cfg.T, cfg.H, cfg.I, cfg.E, cfg.top_k, "cuda", api.DTYPE_FP8)
    bias = None if inp.bias is None else inp.bias.cuda()
    out = api.moe_forward_fp8(inp.x.cuda(), inp.router_w.cuda(), bias, g["w_gate_q"], g["w_gate_s"],
                              g["w_up_q"], g["w_up_s"], g["w_down_q"], g["w_down_s"], cfg.top_k, ws=ws)
    assert api.moe_get_device_status(ws) == api.MOE_OK
    return out


def _oracle_fp8(cfg, inp, w, tokens=None):
    x, rw = inp.x.cpu(), inp.router_w.cpu()
    bias = None if inp.bias is None else inp.bias.cpu()
    idx, gate = oracle.route(x, rw, bias, cfg.top_k)
    if tokens is None:
        wc = {k: v.cpu() for k, v in w.items()}
        return oracle.combine_ffn_fp8(x, idx, gate, wc["w_gate_q"], wc["w_gate_s"], wc["w_up_q"],
                                      wc["w_up_s"], wc["w_down_q"], wc["w_down_s"]), idx, gate
    # only the experts the sampled tokens use, re-indexed
    used = np.unique(idx[tokens].reshape(-1))
    remap = np.full(cfg.E, -1, np.int32)
    remap[used] = np.arange(used.size, dtype=np.int32)
    sel = torch.as_tensor(used, device=w["w_gate_q"].device).long()
    wc = {k: v.index_select(0, sel).cpu() for k, v in w.items()}
    idx_c = np.where(np.isin(np.arange(cfg.T)[:, None], tokens), remap[idx], 0).astype(np.int32)
    out = oracle.combine_ffn_fp8(x, idx_c, gate, wc["w_gate_q"], wc["w_gate_s"], wc["w_up_q"], wc["w_up_s"],
                                 wc["w_down_q"], wc["w_down_s"], tokens=tokens)
    return out, idx, gate


SMALL = {
    "fp8_small": CONFIGS["fp8"].replace(name="fp8_small", T=64, H=256, E=8, top_k=2, I=256),
    "fp8_ragged": CONFIGS["fp8"].replace(name="fp8_ragged", T=150, H=384, E=12, top_k=3, I=384, seed=7),
    "fp8_bias": CONFIGS["fp8"].replace(name="fp8_bias", T=130, H=512, E=16, top_k=4, I=256, seed=8,
                                       zipf_s=1.2),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_fp8_layer_small(name):
    cfg = SMALL[name]
    inp, w = _fp8_case(cfg)
    out = _run_fp8(cfg, inp, w)
    ref, idx, gate = _oracle_fp8(cfg, inp, w)
    bias = None if inp.bias is None else inp.bias.cuda()
    i_g, w_g = api.moe_route(inp.x.cuda(), inp.router_w.cuda(), bias, cfg.top_k)
    compare_routing(i_g, w_g, idx, gate, name)
    r = rel_l2(out, ref)
    assert r <= FP8_REL_L2, f"{name}: rel_l2={r:.3e}"


def test_fp8_zero_router_all_tokens_to_first_experts():
    cfg = SMALL["fp8_small"].replace(name="fp8_ties", T=300, top_k=3, seed=9)
    inp, w = _fp8_case(cfg)
    inp.router_w = torch.zeros_like(inp.router_w)
    out = _run_fp8(cfg, inp, w)
    ref, _, _ = _oracle_fp8(cfg, inp, w)
    assert rel_l2(out, ref) <= FP8_REL_L2


def test_fp8_full_size_sampled():
    cfg = CONFIGS["fp8"]
    inp, w = _fp8_case(cfg)
    out = _run_fp8(cfg, inp, w)
    tok = sample_tokens(cfg.T, 128, seed=cfg.seed)
    assert tok.size >= 128
    ref, idx, gate = _oracle_fp8(cfg, inp, w, tokens=tok)
    i_g, w_g = api.moe_route(inp.x, inp.router_w, None, cfg.top_k)
    compare_routing(i_g, w_g, idx, gate, "fp8")
    o = out[torch.as_tensor(tok, device="cuda").long()]
    r = rel_l2(o, ref)
    max_abs = float(np.abs(o.float().cpu().double().numpy() - ref).max())
    print(f"fp8 full size: {tok.size} tokens, rel_l2={r:.3e} max_abs={max_abs:.3e} (reported)")
    assert r <= FP8_REL_L2, f"fp8 full size: rel_l2={r:.3e}"


SWAP_CASES = {
    "ragged": SMALL["fp8_ragged"],   # ~38 rows per expert: 48-row MMAs, partial chunks
    "bias": SMALL["fp8_bias"],       # skewed groups: 16- to 128-row tiles in one launch
    "full_tiles": SMALL["fp8_small"].replace(name="fp8_full_tiles", T=300, top_k=3, seed=9),  # zero router below
    "k_chunks": CONFIGS["fp8"].replace(name="fp8_k_chunks", T=96, H=2304, E=8, top_k=2, I=256, seed=11),  # 18 K blocks
}


@pytest.mark.parametrize("name", list(SWAP_CASES))
def test_fp8_swapped_gate_up_gemm(name):
    # The gate/up GEMM with swapped MMA operands (weights on M, token rows on N)
    # against the oracle and against the one-CTA fp8 kernel, and bitwise stable
    # across grid sizes and claim orders.
    cfg = SWAP_CASES[name]
    inp, w = _fp8_case(cfg)
    if name == "full_tiles":
        inp.router_w = torch.zeros_like(inp.router_w)   # 300 rows on each of experts 0-2
    outs = []
    try:
        api.set_fp8_swap_ab("never")
        base = _run_fp8(cfg, inp, w).clone()
        api.set_fp8_swap_ab("always")
        for ctas, mode in [(0, False), (3, True), (0, "static_items"), (7, "static_experts")]:
            api.set_gemm_ctas(ctas)
            api.set_claim_order(mode)
            outs.append(_run_fp8(cfg, inp, w).clone())
    finally:
        api.set_fp8_swap_ab("auto")
        api.set_gemm_ctas(0)
        api.set_claim_order(False)
    ref, _, _ = _oracle_fp8(cfg, inp, w)
    assert rel_l2(outs[0], ref) <= FP8_REL_L2, f"{name} swapped: rel_l2={rel_l2(outs[0], ref):.3e}"
    assert rel_l2(base, ref) <= FP8_REL_L2, f"{name} one-CTA: rel_l2={rel_l2(base, ref):.3e}"
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    # same blockwise products and the same fp32 promotion, SwiGLU and quantiser
    assert torch.equal(outs[0].view(torch.int16), base.view(torch.int16))
