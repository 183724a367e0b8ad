"""Seeded synthetic inputs for the MoE layer workloads.

This module is shared by the CUDA path's tests/benchmark and by the CPU oracle's
tests.  It holds none of the layer's arithmetic: it only draws numbers.

Generator (counter based, identical on CPU and CUDA up to last-ulp differences of
the fp64 ``log``/``cos`` between host libm and the device):

* splitmix64 (S. Vigna's published mixer): output ``i`` of the stream with key
  ``K`` is ``mix(K + (i + 1) * 0x9E3779B97F4A7C15)`` with
  ``mix(z) = z3`` where ``z1 = (z ^ z>>30) * 0xBF58476D1CE4E5B9``,
  ``z2 = (z1 ^ z1>>27) * 0x94D049BB133111EB``, ``z3 = z2 ^ z2>>31`` (mod 2**64,
  logical shifts).
* uniforms from the top 53 bits; Box-Muller from two consecutive draws
  ``n = sqrt(-2 ln u1) cos(2 pi u2)`` with ``u1`` in (0, 1] and ``u2`` in [0, 1).
* scaled by the tensor's standard deviation in fp64, rounded to fp32, then
  round-to-nearest-even to bf16.

Every tensor has its own stream key ``mix(seed * 0x9E3779B97F4A7C15 + tensor_id)``;
tensors are drawn as x (0), router_w (1), bias (2), w_gate (3), w_up (4),
w_down (5).

The five workloads are the configurations of the layer the pages describe
(vLLM fused-MoE page, section 02: a router picks top-k of E experts, each a
gate/up/down SwiGLU FFN; shapes and distributions as listed in ``CONFIGS``).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

_GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1

TENSOR_IDS = {"x": 0, "router_w": 1, "bias": 2, "w_gate": 3, "w_up": 4, "w_down": 5,
              "shared_gate": 6, "shared_up": 7, "shared_down": 8}


def _s64(v: int) -> int:
    v &= _MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    # logical right shift of an int64 tensor holding a uint64 bit pattern
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix_t(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _lsr(z, 30)) * _s64(_M1)
    z = (z ^ _lsr(z, 27)) * _s64(_M2)
    return z ^ _lsr(z, 31)


def _mix_int(z: int) -> int:
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _M1) & _MASK64
    z = ((z ^ (z >> 27)) * _M2) & _MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, tensor_id: int) -> int:
    return _mix_int(seed * _GOLDEN + tensor_id)


def splitmix64(key: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """Raw 64-bit outputs ``start .. start+count-1`` of the stream (int64 bit patterns)."""
    i = torch.arange(start + 1, start + 1 + count, dtype=torch.int64, device=device)
    z = i * _s64(_GOLDEN) + _s64(key)
    return _mix_t(z)


def normal(key: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """Standard normals ``start .. start+count-1`` of a stream, in fp64."""
    z = splitmix64(key, 2 * start, 2 * count, device).view(count, 2)
    two53 = 2.0 ** -53
    u1 = (_lsr(z[:, 0], 11).to(torch.float64) + 1.0) * two53
    u2 = _lsr(z[:, 1], 11).to(torch.float64) * two53
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


def gaussian_tensor(seed: int, name: str, shape, std: float, device="cpu",
                    out_dtype=torch.bfloat16, chunk: int = 1 << 24) -> torch.Tensor:
    """``std * N(0,1)`` drawn from the tensor's stream, fp64 -> fp32 -> ``out_dtype``."""
    key = stream_key(seed, TENSOR_IDS[name])
    n = 1
    for s in shape:
        n *= int(s)
    out = torch.empty(n, dtype=out_dtype, device=device)
    for s0 in range(0, n, chunk):
        c = min(chunk, n - s0)
        v = normal(key, s0, c, device) * std
        out[s0:s0 + c] = v.to(torch.float32).to(out_dtype)
    return out.view(*shape)


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    H: int
    E: int
    top_k: int
    I: int
    seed: int
    dtype: str = "bf16"          # "bf16", "fp8" or "mx" (e2m1 weights, e4m3 activations)
    zipf_s: float | None = None  # per-expert router bias making popularity ~ Zipf(s)
    router_std: float = 0.02
    shared_mult: int = 0         # a shared expert of shared_mult * I columns (0: none)

    @property
    def A(self) -> int:
        return self.T * self.top_k

    def replace(self, **kw) -> "MoEConfig":
        d = dict(self.__dict__)
        d.update(kw)
        return MoEConfig(**d)


CONFIGS = {
    "tiny": MoEConfig("tiny", T=64, H=256, E=8, top_k=2, I=512, seed=0),
    "decode": MoEConfig("decode", T=16, H=2048, E=256, top_k=8, I=512, seed=1),
    "prefill": MoEConfig("prefill", T=4096, H=2048, E=256, top_k=8, I=512, seed=2),
    "skewed": MoEConfig("skewed", T=8192, H=4096, E=64, top_k=6, I=1408, seed=3, zipf_s=1.2),
    "fp8": MoEConfig("fp8", T=1024, H=7168, E=256, top_k=8, I=2048, seed=4, dtype="fp8"),
}

# Further workloads of the layer's variants (not among the five configurations above):
# the MX (FP4 weight) layer on the FP8 workload's shapes and inputs, and the Prefill
# workload with a shared expert of 2 x I columns.
EXTRA_WORKLOADS = {
    "mx": CONFIGS["fp8"].replace(name="mx", dtype="mx"),
    "prefill_shared": CONFIGS["prefill"].replace(name="prefill_shared", shared_mult=2),
}


def zipf_bias(E: int, s: float) -> torch.Tensor:
    """Per-expert router bias ``ln p_e`` with ``p_e ~ (e+1)^-s`` normalised (expert 0 hottest).

    Under Gumbel-like logit noise of unit scale, top-1 choice frequencies then follow
    the Zipf law; this is an input recipe, not part of the layer.
    """
    r = torch.arange(1, E + 1, dtype=torch.float64)
    p = r.pow(-s)
    p = p / p.sum()
    return torch.log(p).to(torch.float32)


@dataclass
class MoEInputs:
    cfg: MoEConfig
    x: torch.Tensor            # [T, H] bf16
    router_w: torch.Tensor     # [H, E] bf16
    bias: torch.Tensor | None  # [E] fp32 or None
    w_gate: torch.Tensor       # [E, I, H] bf16 (fp32 master values for the fp8 config)
    w_up: torch.Tensor         # [E, I, H]
    w_down: torch.Tensor       # [E, H, I]
    extra: dict = field(default_factory=dict)


def quantize_blocks_e4m3(w: torch.Tensor):
    """Input recipe of the fp8 workload's weights (given to the layer pre-quantised):
    one fp32 scale per 128x128 block of each expert matrix [E, N, K],
    s = amax/448 (s = 1 for an all-zero block), codes = e4m3(clamp(w/s, +-448))
    via torch's float8_e4m3fn cast.  Returns (codes uint8 [E,N,K], scales fp32
    [E, N/128, K/128])."""
    E, N, K = w.shape
    b = w.view(E, N // 128, 128, K // 128, 128).float()
    amax = b.abs().amax(dim=(2, 4))
    s = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)
    q = (b / s[:, :, None, :, None]).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    return q.view(torch.uint8).reshape(E, N, K).contiguous(), s.contiguous()


def make_fp8_weights(cfg: MoEConfig, device="cpu", experts_per_chunk: int = 8):
    """The fp8 workload's expert weights: drawn like the bf16 ones (fp32 master values
    ~ N(0, 1/sqrt(fan_in)), same streams) and block-quantised, a few experts at a
    time so the fp32 values never exist in full.  Returns a dict of codes/scales."""
    E, I, H = cfg.E, cfg.I, cfg.H
    out = {}
    for name, (N, K) in (("w_gate", (I, H)), ("w_up", (I, H)), ("w_down", (H, I))):
        key = stream_key(cfg.seed, TENSOR_IDS[name])
        std = 1.0 / math.sqrt(K)
        q = torch.empty((E, N, K), dtype=torch.uint8, device=device)
        sc = torch.empty((E, N // 128, K // 128), dtype=torch.float32, device=device)
        per = N * K
        for e0 in range(0, E, experts_per_chunk):
            e1 = min(E, e0 + experts_per_chunk)
            v = torch.empty((e1 - e0) * per, dtype=torch.float32, device=device)
            step = 1 << 24
            for s0 in range(0, v.numel(), step):
                c = min(step, v.numel() - s0)
                v[s0:s0 + c] = (normal(key, e0 * per + s0, c, device) * std).to(torch.float32)
            qq, ss = quantize_blocks_e4m3(v.view(e1 - e0, N, K))
            q[e0:e1] = qq
            sc[e0:e1] = ss
        out[name + "_q"] = q
        out[name + "_s"] = sc
    return out


E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)  # codes 0..7 (OCP MX v1.0)


def quantize_blocks_mx_e2m1(w: torch.Tensor):
    """Input recipe of MX (FP4) expert weights: per row, per 32 values along K, a
    power-of-two scale 2^X with X = floor(log2(amax)) - 2 (clamped to [-127, 127];
    X = 0 for an all-zero block), stored as the e8m0 code X + 127, and e2m1 codes of
    w / 2^X clamped to +-6, rounded to the nearest magnitude with ties to the even
    code.  One code per byte (sign in bit 3).  Returns (codes uint8 [E,N,K], scale
    codes uint8 [E,N,K/32])."""
    E, N, K = w.shape
    b = w.reshape(E, N, K // 32, 32).double()
    amax = b.abs().amax(-1)
    X = (torch.frexp(amax).exponent - 3).clamp(-127, 127)
    X = torch.where(amax == 0, torch.zeros_like(X), X)
    r = torch.ldexp(b, -X[..., None]).clamp(-6.0, 6.0)
    mags = torch.tensor(E2M1_MAGNITUDES, dtype=torch.float64, device=w.device)
    d = (r.abs()[..., None] - mags).abs() + 1e-12 * (torch.arange(8, device=w.device) & 1)  # ties -> even code
    c = d.argmin(-1).to(torch.uint8)
    c = torch.where((r < 0) & (c != 0), c | 8, c)
    return c.reshape(E, N, K).contiguous(), (X + 127).to(torch.uint8).contiguous()


def make_mx_weights(cfg: MoEConfig, device="cpu", experts_per_chunk: int = 8):
    """MX (FP4) expert weights: drawn like the bf16 ones (fp32 master values ~
    N(0, 1/sqrt(fan_in)), same streams) and quantised by quantize_blocks_mx_e2m1, a
    few experts at a time.  Returns {name_q: codes [E,N,K], name_x: scale codes [E,N,K/32]}."""
    E, I, H = cfg.E, cfg.I, cfg.H
    out = {}
    for name, (N, K) in (("w_gate", (I, H)), ("w_up", (I, H)), ("w_down", (H, I))):
        key = stream_key(cfg.seed, TENSOR_IDS[name])
        std = 1.0 / math.sqrt(K)
        q = torch.empty((E, N, K), dtype=torch.uint8, device=device)
        sx = torch.empty((E, N, K // 32), dtype=torch.uint8, device=device)
        per = N * K
        for e0 in range(0, E, experts_per_chunk):
            e1 = min(E, e0 + experts_per_chunk)
            v = (normal(key, e0 * per, (e1 - e0) * per, device) * std).to(torch.float32)
            qq, xx = quantize_blocks_mx_e2m1(v.view(e1 - e0, N, K))
            q[e0:e1] = qq
            sx[e0:e1] = xx
        out[name + "_q"] = q
        out[name + "_x"] = sx
    return out


def make_shared_weights(cfg: MoEConfig, shared_I: int, device="cpu"):
    """A shared expert's bf16 weights, drawn like the routed experts' (N(0, 1/sqrt(fan_in)),
    streams 6-8 of the config's seed): (shared_gate [shared_I, H], shared_up [shared_I, H],
    shared_down [H, shared_I])."""
    H = cfg.H
    wg = gaussian_tensor(cfg.seed, "shared_gate", (shared_I, H), 1.0 / math.sqrt(H), device)
    wu = gaussian_tensor(cfg.seed, "shared_up", (shared_I, H), 1.0 / math.sqrt(H), device)
    wd = gaussian_tensor(cfg.seed, "shared_down", (H, shared_I), 1.0 / math.sqrt(shared_I), device)
    return wg, wu, wd


def pack_e2m1(codes: torch.Tensor) -> torch.Tensor:
    """e2m1 codes one per byte [..., K] -> two per byte [..., K/2]: the code of element
    2i in the low nibble of byte i, of element 2i+1 in the high nibble (the packed
    FP4 storage the MX layer reads)."""
    c = codes.to(torch.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def make_inputs(cfg: MoEConfig, device="cpu", weights: bool = True) -> MoEInputs:
    """Draw the workload's tensors in the fixed order x, router_w, [bias], w_gate, w_up, w_down.

    Expert weights ~ N(0, 1/sqrt(fan_in)) (fan_in = H for gate/up, I for down);
    x ~ N(0, 1); router_w ~ N(0, 0.02).  For the fp8 workload the expert weights
    are returned as fp32 underlying values; ``make_fp8_weights`` gives the quantised
    codes and block scales both sides consume.
    """
    T, H, E, I = cfg.T, cfg.H, cfg.E, cfg.I
    x = gaussian_tensor(cfg.seed, "x", (T, H), 1.0, device)
    rw = gaussian_tensor(cfg.seed, "router_w", (H, E), cfg.router_std, device)
    bias = zipf_bias(E, cfg.zipf_s).to(device) if cfg.zipf_s is not None else None
    wdt = torch.float32 if cfg.dtype == "fp8" else torch.bfloat16
    if weights:
        wg = gaussian_tensor(cfg.seed, "w_gate", (E, I, H), 1.0 / math.sqrt(H), device, wdt)
        wu = gaussian_tensor(cfg.seed, "w_up", (E, I, H), 1.0 / math.sqrt(H), device, wdt)
        wd = gaussian_tensor(cfg.seed, "w_down", (E, H, I), 1.0 / math.sqrt(I), device, wdt)
    else:
        wg = wu = wd = None
    return MoEInputs(cfg, x, rw, bias, wg, wu, wd)
