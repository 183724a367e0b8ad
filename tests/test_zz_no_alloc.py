"""The forward entry point for callers that cannot allocate device memory.

moe_forward_noalloc runs the layer with the library's fixed internal scratch
instead of a caller-provided workspace -- for code that has no access to an
allocator on its serving path.  Its results must match the regular
moe_forward (which takes a workspace) on the same inputs, call after call.
This file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import oracle
from gpu_helpers import compare_out, device_inputs
from routed_grouped_gemm_softmax_b200 import api
from routed_grouped_gemm_softmax_b200.inputs import CONFIGS

pytestmark = pytest.mark.gpu


def _call_noalloc(g, k, out):
    """Straight through the C ABI, with the device pointers only."""
    T, H = g["x"].shape
    E, I, _ = g["w_gate"].shape
    d = api.dims(T, H, I, E, k)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return api.lib().moe_forward_noalloc(ctypes.byref(d), p(g["x"]), p(g["router_w"]), p(g["bias"]),
                                         p(g["w_gate"]), p(g["w_up"]), p(g["w_down"]), p(out), st)


def test_noalloc_matches_workspace_forward_on_a_dirty_array():
    # Decode, then Tiny, then Decode again: every call after the first runs on the
    # contents the previous call left in the shared array (Decode takes the small
    # router path that clears its counters in-kernel, Tiny the path that clears them
    # with a memset).  The no-alloc call runs the same deterministic kernels as
    # moe_forward, so each result must equal moe_forward's bit for bit, twice in a row.
    cases = {}
    for name in ("decode", "tiny"):
        cfg = CONFIGS[name]
        g, c = device_inputs(cfg)
        ref = api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], cfg.top_k)
        torch.cuda.synchronize()
        cases[name] = (cfg, g, c, ref)
    for name in ("decode", "tiny", "decode"):
        cfg, g, c, ref = cases[name]
        for call in range(2):
            out = torch.full_like(ref, float("nan"))
            assert _call_noalloc(g, cfg.top_k, out) == api.MOE_OK
            torch.cuda.synchronize()
            assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"{name} no-alloc call {call}"
    # and against the oracle on a few tokens, within the layer's tolerance
    for name, (cfg, g, c, _) in cases.items():
        out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(g, cfg.top_k, out) == api.MOE_OK
        torch.cuda.synchronize()
        idx, gate = oracle.route(c["x"], c["router_w"], c["bias"], cfg.top_k)
        tok = [0, cfg.T // 2, cfg.T - 1]
        o = oracle.combine_ffn(c["x"], idx, gate, c["w_gate"], c["w_up"], c["w_down"], tokens=tok)
        compare_out(out[tok], o, f"{name} no-alloc vs oracle")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # the first batch size whose workspace exceeds the fixed scratch (183 tokens with
    # H=2048, I=512, E=256, k=8; 182 is the largest that fits) is rejected before any
    # device work
    H, I, E, k = 2048, 512, 256, 8
    T = next(t for t in range(1, 100000) if api.moe_workspace_size(t, H, I, E, k) > api.NOALLOC_SCRATCH_BYTES)
    assert T == 183
    d = api.dims(T, H, I, E, k)
    dummy = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    rc = api.lib().moe_forward_noalloc(ctypes.byref(d), p, p, None, p, p, p, p, None)
    assert rc == 7  # MOE_ERR_TOO_LARGE, before any device work
    bad = api.dims(16, 2048, 512, 256, 0)
    assert api.lib().moe_forward_noalloc(ctypes.byref(bad), p, p, None, p, p, p, p, None) == 1


def test_noalloc_status_reports_a_pipeline_timeout():
    # The stall hook: every GEMM CTA's MMA thread first waits, with a 2 ms bound, on a
    # barrier that nothing signals.  The timeout lands in the status word of the
    # library's scratch, which moe_noalloc_get_device_status reads (and clears); the next
    # call with the default settings is correct and reports MOE_OK.
    cfg = CONFIGS["tiny"]
    g, c = device_inputs(cfg)
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    try:
        api.set_wait_limit_us(2000, stall_test=True)
        assert _call_noalloc(g, cfg.top_k, out) == api.MOE_OK
        assert api.noalloc_device_status() == 5  # MOE_ERR_TIMEOUT
    finally:
        api.set_wait_limit_us(0, stall_test=False)
    assert api.noalloc_device_status() == api.MOE_OK  # cleared by the read
    ref = api.moe_forward(g["x"], g["router_w"], g["bias"], g["w_gate"], g["w_up"], g["w_down"], cfg.top_k)
    assert _call_noalloc(g, cfg.top_k, out) == api.MOE_OK
    assert api.noalloc_device_status() == api.MOE_OK
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
