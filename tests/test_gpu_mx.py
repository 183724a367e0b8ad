"""MX (FP4 weights, FP8 activations, per-32 power-of-two scales) layer: CUDA path vs
the CPU oracle through the C ABI.

The activation quantiser's e4m3 codes and e8m0 scale codes must match the oracle bit
for bit (same bf16 inputs, same fp32 decisions).  The layer output is compared with
the oracle's MX layer (oracle_combine_ffn_mx: the same quantisation steps, exact
block sums in fp64) at relative L2 <= 3e-2 -- the tolerance of the other quantised
(fp8) layer: the GPU accumulates in fp32 and rounds y and out to bf16, and an h value
within rounding of an e4m3 boundary may take the neighbouring code.  Routing is the
bf16 router and stays bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import compare_routing, sample_tokens
from routed_grouped_gemm_softmax_b200 import api
from routed_grouped_gemm_softmax_b200.inputs import CONFIGS, make_inputs, make_mx_weights, pack_e2m1

pytestmark = pytest.mark.gpu

MX_REL_L2 = 3e-2
MX_E4M3 = 0


def rel_l2(out_gpu, ref):
    o = out_gpu.float().cpu().double().numpy()
    return float(np.linalg.norm(o - ref) / np.linalg.norm(ref))


def test_mx_quantizer_bit_exact():
    rng = np.random.default_rng(5)
    a = torch.as_tensor(rng.standard_normal((41, 1024)).astype(np.float32) * 3).to(torch.bfloat16)
    a[3, 64:96] = 0.0                      # an all-zero block: scale code 127, zero codes
    a[5, :] *= 1e-30                       # tiny values
    a[7, 0] = 1e4                          # one huge value in a block
    a[7, 21] = -0.018                      # a negative value that rounds to zero: code +0 (0x00)
    a[9, 32:64] = 2.0 ** torch.arange(32).float().to(torch.bfloat16).float() * 1e-6  # wide range in a block
    a[11, 128:160] = 448.0                 # exactly the largest e4m3 magnitude times a power of two
    q, x = api.moe_quantize_rows_mx(a.cuda())
    qr, xr = oracle.get().mx_quantize_rows(a.float().numpy(), MX_E4M3)
    assert np.array_equal(x.cpu().numpy(), xr)
    assert np.array_equal(q.cpu().numpy(), qr)


def _mx_case(cfg, device="cuda"):
    inp = make_inputs(cfg, device=device, weights=False)
    w = make_mx_weights(cfg, device=device)
    return inp, w


def _packed(w):
    return [pack_e2m1(w["w_gate_q"]).cuda(), w["w_gate_x"].cuda(), pack_e2m1(w["w_up_q"]).cuda(), w["w_up_x"].cuda(),
            pack_e2m1(w["w_down_q"]).cuda(), w["w_down_x"].cuda()]


def _run_mx(cfg, inp, w, ws=None):
    ws = api.workspace(cfg.T, cfg.H, cfg.I, cfg.E, cfg.top_k, "cuda", api.DTYPE_MX) if ws is None else ws
    bias = None if inp.bias is None else inp.bias.cuda()
    out = api.moe_forward_mx(inp.x.cuda(), inp.router_w.cuda(), bias, *_packed(w), cfg.top_k, ws=ws)
    assert api.moe_get_device_status(ws) == api.MOE_OK
    return out


def _oracle_mx(cfg, inp, w, tokens=None):
    x, rw = inp.x.cpu(), inp.router_w.cpu()
    bias = None if inp.bias is None else inp.bias.cpu()
    idx, gate = oracle.route(x, rw, bias, cfg.top_k)
    names = ("w_gate_q", "w_gate_x", "w_up_q", "w_up_x", "w_down_q", "w_down_x")
    if tokens is None:
        wc = [w[n].cpu() for n in names]
        return oracle.get().combine_ffn_mx(x, idx, gate, *wc), idx, gate
    # only the experts the sampled tokens use, re-indexed
    used = np.unique(idx[tokens].reshape(-1))
    remap = np.full(cfg.E, -1, np.int32)
    remap[used] = np.arange(used.size, dtype=np.int32)
    sel = torch.as_tensor(used, device=w["w_gate_q"].device).long()
    wc = [w[n].index_select(0, sel).cpu() for n in names]
    idx_c = np.where(np.isin(np.arange(cfg.T)[:, None], tokens), remap[idx], 0).astype(np.int32)
    return oracle.get().combine_ffn_mx(x, idx_c, gate, *wc, tokens=tokens), idx, gate


SMALL = {
    "mx_small": CONFIGS["fp8"].replace(name="mx_small", T=64, H=512, E=8, top_k=2, I=512, seed=70),
    "mx_ragged": CONFIGS["fp8"].replace(name="mx_ragged", T=300, H=1024, E=16, top_k=4, I=512, seed=71),
    "mx_bias": CONFIGS["fp8"].replace(name="mx_bias", T=130, H=512, E=16, top_k=4, I=1024, seed=72, zipf_s=1.2),
    "mx_decode": CONFIGS["decode"].replace(name="mx_decode", T=16, E=64, seed=73),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_mx_layer_small(name):
    cfg = SMALL[name]
    inp, w = _mx_case(cfg)
    out = _run_mx(cfg, inp, w)
    ref, idx, gate = _oracle_mx(cfg, inp, w)
    bias = None if inp.bias is None else inp.bias.cuda()
    i_g, w_g = api.moe_route(inp.x.cuda(), inp.router_w.cuda(), bias, cfg.top_k)
    compare_routing(i_g, w_g, idx, gate, name)
    r = rel_l2(out, ref)
    print(f"{name}: rel_l2={r:.3e}")
    assert r <= MX_REL_L2, f"{name}: rel_l2={r:.3e}"


def test_mx_zero_router_and_schedules():
    # router_w = 0: 300 rows on each of experts 0-2 (full 64-row halves and a partial
    # one); bitwise the same result over grid sizes and every claim order.
    cfg = SMALL["mx_small"].replace(name="mx_ties", T=300, top_k=3, seed=74)
    inp, w = _mx_case(cfg)
    inp.router_w = torch.zeros_like(inp.router_w)
    outs = []
    try:
        for ctas, mode in [(0, False), (3, True), (0, "static_items"), (7, "static_experts")]:
            api.set_gemm_ctas(ctas)
            api.set_claim_order(mode)
            outs.append(_run_mx(cfg, inp, w).clone())
    finally:
        api.set_gemm_ctas(0)
        api.set_claim_order(False)
    ref, _, _ = _oracle_mx(cfg, inp, w)
    assert rel_l2(outs[0], ref) <= MX_REL_L2
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))


def test_mx_fp8_shapes_sampled():
    # The FP8 workload's shapes (T=1024, H=7168, E=256, top-8, I=2048) with MX weights,
    # routing bit-exact, the output on 32 sampled tokens.
    cfg = CONFIGS["fp8"].replace(name="mx_full")
    inp, w = _mx_case(cfg)
    out = _run_mx(cfg, inp, w)
    tok = sample_tokens(cfg.T, 30, seed=cfg.seed)
    ref, idx, gate = _oracle_mx(cfg, inp, w, tokens=tok)
    i_g, w_g = api.moe_route(inp.x, inp.router_w, None, cfg.top_k)
    compare_routing(i_g, w_g, idx, gate, "mx_full")
    r = rel_l2(out[torch.as_tensor(tok, device="cuda").long()], ref)
    print(f"mx full shapes: {tok.size} tokens, rel_l2={r:.3e}")
    assert r <= MX_REL_L2, f"mx full shapes: rel_l2={r:.3e}"
