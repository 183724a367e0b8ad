"""CPU oracle of the routed MoE layer forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  The CUDA library never loads it and shares no code
with it; both are handed the same seeded input buffers.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64; the router logit is the
fp32 fused-multiply-add chain both sides agree on).  This module only compiles
it with gcc and marshals numpy arrays through ctypes.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(brute force, closed forms, invariants, library routines) -- none is unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "moe_oracle.c")
LIB = os.path.join(_HERE, "libmoe_oracle.so")


def build(src: str = SRC, out: str = LIB, force: bool = False) -> str:
    """Compile the oracle with gcc (no fp contraction, so only the explicit fmaf
    calls fuse)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
               "-shared", "-o", tmp, src, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bf16_bits(t) -> np.ndarray:
    """bf16 tensor (torch) or uint16 array -> contiguous uint16 numpy array of its bits."""
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16
        return np.ascontiguousarray(t)
    import torch
    assert t.dtype == torch.bfloat16
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _f32(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t, dtype=np.float32)
    return np.ascontiguousarray(t.detach().cpu().float().numpy())


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


class Oracle:
    """ctypes view of one build of the oracle library."""

    def __init__(self, lib_path: str | None = None):
        lib = ctypes.CDLL(lib_path or build())
        P = ctypes.c_void_p
        i = ctypes.c_int
        lib.oracle_route.argtypes = [i, i, i, i, P, P, P, P, P, P, P, i]
        lib.oracle_route.restype = i
        lib.oracle_permute.argtypes = [i, i, P, P, P, P, i, P, P]
        lib.oracle_permute.restype = i
        lib.oracle_combine_ffn.argtypes = [i, i, i, P, P, P, P, P, P, i, P, P, i]
        lib.oracle_combine_ffn.restype = i
        lib.oracle_shared_ffn.argtypes = [i, i, P, P, P, P, i, P, P, i]
        lib.oracle_shared_ffn.restype = i
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_encode_array.argtypes = [i, P, P]
        lib.oracle_e4m3_encode_array.restype = None
        lib.oracle_quantize_rows.argtypes = [i, i, P, P, P]
        lib.oracle_quantize_rows.restype = i
        lib.oracle_combine_ffn_fp8.argtypes = [i, i, i, P, P, P, P, P, P, P, P, P, i, P, P, i]
        lib.oracle_combine_ffn_fp8.restype = i
        lib.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e2m1_decode.restype = ctypes.c_double
        lib.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        lib.oracle_e2m1_encode.restype = ctypes.c_uint8
        lib.oracle_mx_quantize_rows.argtypes = [i, i, P, i, P, P]
        lib.oracle_mx_quantize_rows.restype = i
        lib.oracle_combine_ffn_mx.argtypes = [i, i, i, P, P, P, P, P, P, P, P, P, i, P, P, i]
        lib.oracle_combine_ffn_mx.restype = i
        self.lib = lib

    def route(self, x, router_w, bias, top_k: int, want_logits: bool = False,
              nthreads: int | None = None):
        """Router + softmax over the top-k.  Returns (idx int32 [T,k], gate fp64 [T,k])
        and, with ``want_logits``, also (logits fp32 [T,E], logits fp64 [T,E])."""
        xb, wb, bb = _bf16_bits(x), _bf16_bits(router_w), _f32(bias)
        T, H = xb.shape
        H2, E = wb.shape
        assert H == H2
        idx = np.zeros((T, top_k), np.int32)
        gate = np.zeros((T, top_k), np.float64)
        l32 = np.zeros((T, E), np.float32) if want_logits else None
        l64 = np.zeros((T, E), np.float64) if want_logits else None
        rc = self.lib.oracle_route(T, H, E, top_k, _ptr(xb), _ptr(wb), _ptr(bb), _ptr(idx),
                                   _ptr(gate), _ptr(l32), _ptr(l64), nthreads or default_threads())
        if rc:
            raise ValueError(f"oracle_route rejected its arguments (code {rc})")
        return (idx, gate, l32, l64) if want_logits else (idx, gate)

    def permute(self, idx, E: int, bm: int = 128):
        """Stable counting sort of the flat assignments by expert.  Returns a dict with
        offsets [E+1], sorted_to_flat [A], flat_to_sorted [A], tile_list [n,3], num_tiles."""
        fl = np.ascontiguousarray(np.asarray(idx, dtype=np.int32).reshape(-1))
        A = fl.size
        off = np.zeros(E + 1, np.int32)
        s2f = np.zeros(max(A, 1), np.int32)
        f2s = np.zeros(max(A, 1), np.int32)
        nt = np.zeros(1, np.int32)
        rc = self.lib.oracle_permute(A, E, _ptr(fl), _ptr(off), _ptr(s2f), _ptr(f2s), bm, None,
                                     _ptr(nt))
        if rc:
            raise ValueError(f"oracle_permute rejected its arguments (code {rc})")
        tl = np.zeros((max(int(nt[0]), 1), 3), np.int32)
        self.lib.oracle_permute(A, E, _ptr(fl), _ptr(off), _ptr(s2f), _ptr(f2s), bm, _ptr(tl),
                                _ptr(nt))
        return {"offsets": off, "sorted_to_flat": s2f[:A], "flat_to_sorted": f2s[:A],
                "tile_list": tl[: int(nt[0])], "num_tiles": int(nt[0])}

    def combine_ffn(self, x, idx, gate, w_gate, w_up, w_down, tokens=None,
                    nthreads: int | None = None):
        """Gate-weighted sum of the selected experts' SwiGLU FFN outputs, fp64 [n,H]."""
        xb = _bf16_bits(x)
        T, H = xb.shape
        wg, wu, wd = _bf16_bits(w_gate), _bf16_bits(w_up), _bf16_bits(w_down)
        E, I, H2 = wg.shape
        assert H2 == H and wd.shape == (E, H, I) and wu.shape == wg.shape
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        gate = np.ascontiguousarray(gate, dtype=np.float64)
        k = idx.shape[1]
        tok = None if tokens is None else np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
        n = T if tok is None else tok.size
        out = np.zeros((n, H), np.float64)
        rc = self.lib.oracle_combine_ffn(H, I, k, _ptr(xb), _ptr(idx), _ptr(gate), _ptr(wg),
                                         _ptr(wu), _ptr(wd), n, _ptr(tok), _ptr(out),
                                         nthreads or default_threads())
        if rc:
            raise ValueError(f"oracle_combine_ffn rejected its arguments (code {rc})")
        return out

    def shared_ffn(self, x, w_gate, w_up, w_down, tokens=None, nthreads: int | None = None):
        """A shared expert's SwiGLU FFN output for every token (weight 1), fp64 [n,H]:
        w_gate, w_up [I,H], w_down [H,I] bf16.  The layer with a shared expert is
        combine_ffn(...) + shared_ffn(...)."""
        xb = _bf16_bits(x)
        T, H = xb.shape
        wg, wu, wd = _bf16_bits(w_gate), _bf16_bits(w_up), _bf16_bits(w_down)
        I, H2 = wg.shape
        assert H2 == H and wu.shape == wg.shape and wd.shape == (H, I)
        tok = None if tokens is None else np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
        n = T if tok is None else tok.size
        out = np.zeros((n, H), np.float64)
        rc = self.lib.oracle_shared_ffn(H, I, _ptr(xb), _ptr(wg), _ptr(wu), _ptr(wd), n, _ptr(tok),
                                        _ptr(out), nthreads or default_threads())
        if rc:
            raise ValueError(f"oracle_shared_ffn rejected its arguments (code {rc})")
        return out

    # ------------------------------------------------------------ FP8 variant

    def e4m3_decode(self, codes) -> np.ndarray:
        c = np.asarray(codes, dtype=np.uint8).reshape(-1)
        return np.array([self.lib.oracle_e4m3_decode(int(v)) for v in c]).reshape(np.shape(codes))

    def e4m3_encode(self, values) -> np.ndarray:
        v = np.ascontiguousarray(np.asarray(values, dtype=np.float32).reshape(-1))
        q = np.zeros(v.size, np.uint8)
        self.lib.oracle_e4m3_encode_array(v.size, _ptr(v), _ptr(q))
        return q.reshape(np.shape(values))

    def quantize_rows(self, a):
        """Per-row, per-128-column e4m3 quantisation of a bf16 [R,K] matrix:
        returns (codes uint8 [R,K], scales fp32 [R,K/128])."""
        ab = _bf16_bits(a)
        R, K = ab.shape
        q = np.zeros((R, K), np.uint8)
        s = np.zeros((R, K // 128), np.float32)
        rc = self.lib.oracle_quantize_rows(R, K, _ptr(ab), _ptr(q), _ptr(s))
        if rc:
            raise ValueError(f"oracle_quantize_rows rejected its arguments (code {rc})")
        return q, s

    def combine_ffn_fp8(self, x, idx, gate, wg_q, wg_s, wu_q, wu_s, wd_q, wd_s, tokens=None,
                        nthreads: int | None = None):
        """FP8 block-scaled expert FFN + gate-weighted combine, fp64 [n,H]."""
        xb = _bf16_bits(x)
        T, H = xb.shape
        def u8(t):
            return np.ascontiguousarray(t.cpu().view(__import__("torch").uint8).numpy()
                                        if hasattr(t, "cpu") else np.asarray(t, dtype=np.uint8))
        wg, wu, wd = u8(wg_q), u8(wu_q), u8(wd_q)
        sg, su, sd = _f32(wg_s), _f32(wu_s), _f32(wd_s)
        E, I, H2 = wg.shape
        assert H2 == H and wd.shape == (E, H, I)
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        gate = np.ascontiguousarray(gate, dtype=np.float64)
        k = idx.shape[1]
        tok = None if tokens is None else np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
        n = T if tok is None else tok.size
        out = np.zeros((n, H), np.float64)
        rc = self.lib.oracle_combine_ffn_fp8(H, I, k, _ptr(xb), _ptr(idx), _ptr(gate), _ptr(wg), _ptr(sg),
                                             _ptr(wu), _ptr(su), _ptr(wd), _ptr(sd), n, _ptr(tok),
                                             _ptr(out), nthreads or default_threads())
        if rc:
            raise ValueError(f"oracle_combine_ffn_fp8 rejected its arguments (code {rc})")
        return out

    # ---------------------------------------------- MX (FP4 weights, FP8 activations)

    MX_E4M3, MX_E2M1 = 0, 1

    def e2m1_decode(self, codes) -> np.ndarray:
        c = np.asarray(codes, dtype=np.uint8).reshape(-1)
        return np.array([self.lib.oracle_e2m1_decode(int(v)) for v in c]).reshape(np.shape(codes))

    def e2m1_encode(self, values) -> np.ndarray:
        v = np.asarray(values, dtype=np.float32).reshape(-1)
        return np.array([self.lib.oracle_e2m1_encode(float(a)) for a in v], np.uint8).reshape(np.shape(values))

    def mx_quantize_rows(self, a, fmt: int):
        """OCP MX quantisation of an fp32 matrix [R,K] (K % 32 == 0) per row and per 32
        columns: (codes uint8 [R,K], e8m0 scale codes uint8 [R,K/32])."""
        af = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
        R, K = af.shape
        q = np.zeros((R, K), np.uint8)
        x = np.zeros((R, K // 32), np.uint8)
        rc = self.lib.oracle_mx_quantize_rows(R, K, _ptr(af), int(fmt), _ptr(q), _ptr(x))
        if rc:
            raise ValueError(f"oracle_mx_quantize_rows rejected its arguments (code {rc})")
        return q, x

    def combine_ffn_mx(self, x, idx, gate, wg_q, wg_x, wu_q, wu_x, wd_q, wd_x, tokens=None,
                       nthreads: int | None = None):
        """The MX variant of combine_ffn: e2m1 weight codes [E,N,K] with e8m0 scale codes
        [E,N,K/32]; x and h quantised to MX e4m3 per 32 values.  fp64 [n,H]."""
        xb = _bf16_bits(x)
        T, H = xb.shape
        arrs = [np.ascontiguousarray(np.asarray(a, dtype=np.uint8)) for a in (wg_q, wg_x, wu_q, wu_x, wd_q, wd_x)]
        E, I, H2 = arrs[0].shape
        assert H2 == H and arrs[1].shape == (E, I, H // 32) and arrs[4].shape == (E, H, I)
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        gate = np.ascontiguousarray(gate, dtype=np.float64)
        tok = None if tokens is None else np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
        n = T if tok is None else tok.size
        out = np.zeros((n, H), np.float64)
        rc = self.lib.oracle_combine_ffn_mx(H, I, idx.shape[1], _ptr(xb), _ptr(idx), _ptr(gate),
                                            *[_ptr(a) for a in arrs], n, _ptr(tok), _ptr(out),
                                            nthreads or default_threads())
        if rc:
            raise ValueError(f"oracle_combine_ffn_mx rejected its arguments (code {rc})")
        return out

    def forward(self, x, router_w, bias, w_gate, w_up, w_down, top_k: int, tokens=None,
                nthreads: int | None = None):
        """The whole layer for the given tokens (all when None): (out fp64, idx, gate)."""
        idx, gate = self.route(x, router_w, bias, top_k, nthreads=nthreads)
        out = self.combine_ffn(x, idx, gate, w_gate, w_up, w_down, tokens, nthreads)
        return out, idx, gate


_default: Oracle | None = None


def get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def route(*a, **kw):
    return get().route(*a, **kw)


def permute(*a, **kw):
    return get().permute(*a, **kw)


def combine_ffn(*a, **kw):
    return get().combine_ffn(*a, **kw)


def forward(*a, **kw):
    return get().forward(*a, **kw)


def quantize_rows(*a, **kw):
    return get().quantize_rows(*a, **kw)


def shared_ffn(*a, **kw):
    return get().shared_ffn(*a, **kw)


def combine_ffn_fp8(*a, **kw):
    return get().combine_ffn_fp8(*a, **kw)
