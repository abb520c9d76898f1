"""Seeded synthetic inputs for the routed-expert MoE layer.

This module only draws input data: it holds none of the layer's arithmetic and
is the one piece of code that both the CUDA path's tests / benchmark and the CPU
oracle consume.  Every tensor comes from a seeded ``torch.Generator`` on the
requested device, so a given (config, seed, device) always yields the same bytes;
the oracle receives host copies of exactly the tensors the GPU path receives.

Value distributions (the workloads of the source pages are GLM-5.2-shaped MoE
layers: 256 routed experts per layer plus a shared expert, ~19 MB int4 per
expert -- colibri (tantan.ink), "它的核心判断"):
  * int4 weights uniform on [-8, 7] (offset-binary nibbles uniform on [0, 15]);
  * per-group fp16 scales exp(N(ln 0.02, 0.3));
  * router weights fp32 N(0, 0.02);
  * hidden states fp32 N(0, 1).
Zipf routing (prefill and tiered workloads): hidden-state column 0 is the
constant 1.0 and router column 0 carries a per-expert bias
b_e = kappa * ln(p_rank(e) / p_1), p_r ~ r^-s over a seeded random ranking of
the experts, kappa = sigma * sqrt(6) / pi where sigma = 0.02 * sqrt(H - 1) is the
std of the rest of the logit (the Gumbel scale that matches that noise), so the
expert popularity falls off like Zipf(s).  Realised counts are reported by the
callers.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

GROUP = 64   # int4 weights: one fp16 scale per 64 consecutive inputs
BLOCK = 32   # Q8_0 activations: one fp32 scale per 32 consecutive values


def matrix_bytes(N: int, K: int) -> int:
    """Bytes of one [N][K] int4 gs64 matrix: packed nibbles then fp16 scales."""
    return N * (K // 2) + N * (K // GROUP) * 2


def expert_bytes(H: int, I: int) -> int:
    """gate [I][H] | up [I][H] | down [H][I]."""
    return 2 * matrix_bytes(I, H) + matrix_bytes(H, I)


@dataclass(frozen=True)
class Workload:
    name: str
    H: int
    I: int
    E: int
    k: int
    T: int
    layers: int = 1
    zipf_s: float | None = None
    rho: float | None = None          # token-to-token persistence of x
    cache_bytes: int | None = None    # HBM expert-cache capacity (tiered)
    seed: int = 1
    T_list: tuple = field(default=())

    @property
    def blob_bytes(self) -> int:
        return expert_bytes(self.H, self.I)


GLM = dict(H=6144, I=2048, E=256, k=8)
WORKLOADS = {
    # tiny layer: 16 experts x SwiGLU 128 + 1 shared, top-2, 4 tokens
    "tiny": Workload("tiny", H=256, I=128, E=16, k=2, T=4, seed=1),
    # one GLM-5.2-shaped layer, batch 1, all experts resident
    "decode": Workload("decode", **GLM, T=1, seed=2),
    # 8 stacked GLM-5.2-shaped layers, batch 1 / 4 / 16
    "stacked": Workload("stacked", **GLM, T=16, layers=8, seed=3, T_list=(1, 2, 3, 4, 16)),
    # prefill, 2048 tokens, Zipf(1.1) expert popularity
    "prefill": Workload("prefill", **GLM, T=2048, zipf_s=1.1, seed=4),
    # tiered decode: 16 layers in pinned host memory, 20 GiB HBM cache, 512 tokens
    "tiered": Workload("tiered", **GLM, T=512, layers=16, zipf_s=1.1, rho=0.9,
                       cache_bytes=20 << 30, seed=5),
}


def _gen(seed: int, device) -> torch.Generator:
    dev = torch.device(device)
    g = torch.Generator(device=dev.type if dev.type == "cuda" else "cpu")
    g.manual_seed(int(seed) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def sub_seed(seed: int, layer: int, role: int) -> int:
    return (seed * 1_000_003 + layer * 10_007 + role * 101) & 0x7FFF_FFFF


def fill_blob(out: torch.Tensor, H: int, I: int, seed: int) -> torch.Tensor:
    """Fill one expert blob (uint8 [expert_bytes]) in place from its own seed."""
    assert out.numel() == expert_bytes(H, I) and out.dtype == torch.uint8
    dev = out.device
    g = _gen(seed, dev)
    out.random_(0, 256, generator=g)
    mg = matrix_bytes(I, H)
    for base, N, K in ((0, I, H), (mg, I, H), (2 * mg, H, I)):
        s0 = base + N * (K // 2)
        cnt = N * (K // GROUP)
        z = torch.randn(cnt, generator=g, device=dev, dtype=torch.float32)
        s = torch.exp(z * 0.3 + math.log(0.02)).to(torch.float16)
        out[s0:s0 + 2 * cnt] = s.view(torch.uint8)
    return out


def fill_blob_mx(out: torch.Tensor, H: int, I: int, seed: int) -> torch.Tensor:
    """Fill one MXFP4 expert blob in place from its own seed: random bytes for the
    packed E2M1 codes (every 4-bit code is a valid value), and per 32-block an
    E8M0 exponent E = 127 + round(log2(8 s / 6)) with s drawn like the int4
    scales (exp(N(ln 0.02, 0.3))), so the largest weight 6 * 2^(E-127) is near
    the int4 workload's 8 s."""
    assert out.numel() == expert_bytes(H, I) and out.dtype == torch.uint8
    dev = out.device
    g = _gen(seed, dev)
    out.random_(0, 256, generator=g)
    mg = matrix_bytes(I, H)
    for base, N, K in ((0, I, H), (mg, I, H), (2 * mg, H, I)):
        e0 = base + N * (K // 2)
        cnt = N * (K // 32)
        z = torch.randn(cnt, generator=g, device=dev, dtype=torch.float32)
        s = torch.exp(z * 0.3 + math.log(0.02))
        e = 127 + torch.round(torch.log2(s * (8.0 / 6.0)))
        out[e0:e0 + cnt] = e.clamp(0, 254).to(torch.uint8)
    return out


def make_blobs_mx(H: int, I: int, n: int, seed: int, device="cpu") -> torch.Tensor:
    """MXFP4 expert blobs [n][expert_bytes], blob e from its own seed."""
    out = torch.zeros((n, expert_bytes(H, I)), dtype=torch.uint8, device=device)
    for e in range(n):
        fill_blob_mx(out[e], H, I, blob_seed(seed, e))
    return out


def blob_seed(seed: int, e: int) -> int:
    return (seed * 7919 + e * 104_729 + 13) & 0x7FFF_FFFF


def make_blobs(H: int, I: int, n: int, seed: int, device="cpu", only=None) -> torch.Tensor:
    """Expert blobs [n][expert_bytes]; blob e is drawn from its own seed, so any
    subset can be regenerated alone.  `only`: fill just these rows (others 0)."""
    out = torch.zeros((n, expert_bytes(H, I)), dtype=torch.uint8, device=device)
    for e in (range(n) if only is None else only):
        fill_blob(out[e], H, I, blob_seed(seed, e))
    return out


def zipf_bias(E: int, H: int, s: float, seed: int) -> torch.Tensor:
    g = _gen(seed, "cpu")
    rank = torch.randperm(E, generator=g) + 1          # rank of expert e (1 = most popular)
    logp = -s * torch.log(rank.to(torch.float64))       # ln(p_r / p_1)
    sigma = 0.02 * math.sqrt(H - 1)
    kappa = sigma * math.sqrt(6.0) / math.pi
    return (kappa * logp).to(torch.float32)


def make_router(E: int, H: int, seed: int, device="cpu", zipf_s: float | None = None) -> torch.Tensor:
    g = _gen(seed, device)
    wr = torch.randn((E, H), generator=g, device=device, dtype=torch.float32) * 0.02
    if zipf_s is not None:
        wr[:, 0] = zipf_bias(E, H, zipf_s, seed + 7).to(device)
    return wr


def make_x(T: int, H: int, seed: int, device="cpu", zipf: bool = False,
           rho: float | None = None) -> torch.Tensor:
    g = _gen(seed, device)
    eps = torch.randn((T, H), generator=g, device=device, dtype=torch.float32)
    if rho is not None and T > 1:
        x = torch.empty_like(eps)
        x[0] = eps[0]
        c = math.sqrt(1.0 - rho * rho)
        for t in range(1, T):
            x[t] = rho * x[t - 1] + c * eps[t]
        eps = x
    if zipf:
        eps[:, 0] = 1.0
    return eps.contiguous()


def make_layer(w: Workload, layer: int = 0, device="cpu", T: int | None = None):
    """(x [T][H] fp32, Wr [E][H] fp32, blobs uint8 [E+1][blob]) of one layer."""
    T = w.T if T is None else T
    x = make_x(T, w.H, sub_seed(w.seed, layer, 1), device, zipf=w.zipf_s is not None, rho=w.rho)
    wr = make_router(w.E, w.H, sub_seed(w.seed, layer, 2), device, zipf_s=w.zipf_s)
    blobs = make_blobs(w.H, w.I, w.E + 1, sub_seed(w.seed, layer, 3), device)
    return x, wr, blobs


def chain_next(x, out, gamma: float = 0.5, zipf: bool = False):
    """Input of the next stacked layer (workload glue between layers, not part
    of the MoE layer): v = x + gamma * out / rms(out); x_next = v / rms(v); the
    constant bias feature of the Zipf workloads is kept at 1.  NumPy float32 on
    the host, so every consumer of a stacked workload derives the same inputs."""
    import numpy as np
    x = np.asarray(x, np.float32)
    out = np.asarray(out, np.float32)
    ro = np.sqrt(np.mean(out.astype(np.float64) ** 2, axis=-1, keepdims=True)).astype(np.float32)
    ro = np.where(ro > 0, ro, np.float32(1.0))
    v = (x + np.float32(gamma) * out / ro).astype(np.float32)
    rv = np.sqrt(np.mean(v.astype(np.float64) ** 2, axis=-1, keepdims=True) + 1e-12).astype(np.float32)
    nx = (v / rv).astype(np.float32)
    if zipf:
        nx[..., 0] = 1.0
    return nx


def shrink(w: Workload, **kw) -> Workload:
    """Same workload with some fields replaced (smaller parity cases)."""
    d = {f: getattr(w, f) for f in w.__dataclass_fields__}
    d.update(kw)
    return Workload(**d)
