"""Seeded synthetic inputs for the low-bit MoE layer.

This module only makes input bytes: random tensors with the workload's
distributions and the encoder that turns N(0, 0.02) float weights into the
frozen 4-bit base (packed nibbles + group scales). It holds none of the
dequantize / GEMM / routing arithmetic; both the CUDA library and the CPU
oracle read what it writes.

Formats written (the library's weight formats):
  packed : uint8 [E, N, K/2]; byte i of a row holds element 2i in its low
           nibble and element 2i+1 in its high nibble.
  scales : [E, K/32, N] group-major; bfloat16 for INT4 (symmetric, codes
           -8..7, two's complement), uint8 E8M0 for MXFP4 (E2M1 elements).
"""

from __future__ import annotations

import torch

from .configs import MoEConfig


# --------------------------------------------------------------------------
# Encoders (run once, offline, to produce the frozen base)
# --------------------------------------------------------------------------

def _pack_codes(codes: torch.Tensor) -> torch.Tensor:
    """[..., K] uint8 codes 0..15 -> [..., K/2] bytes, even element in the low nibble."""
    return codes[..., 0::2] | (codes[..., 1::2] << 4)


def quantize_int4(w: torch.Tensor):
    """Symmetric INT4 with one BF16 scale per 32 elements along K.

    s = bf16(amax / 7) (1 when the group is all zero), q = clamp(round(w / s), -8, 7).
    Returns (packed uint8 [..., N, K/2], scales bfloat16 [..., K/32, N]).
    """
    *lead, N, K = w.shape
    g = w.float().reshape(*lead, N, K // 32, 32)
    amax = g.abs().amax(-1)
    s = (amax / 7.0).to(torch.bfloat16)
    s = torch.where(amax == 0, torch.ones_like(s), s)
    q = torch.round(g / s.float().unsqueeze(-1)).clamp_(-8, 7).to(torch.int16)
    codes = (q & 0xF).to(torch.uint8).reshape(*lead, N, K)
    return _pack_codes(codes), s.transpose(-1, -2).contiguous()


# E2M1 grid midpoints; a value exactly on a midpoint goes to the even code.
_E2M1_MID = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def quantize_mxfp4(w: torch.Tensor):
    """MXFP4: E2M1 elements, one E8M0 scale per 32 elements along K.

    The shared exponent puts the group's largest magnitude in [4, 8) before
    rounding (X = floor(log2 amax) - 2 + 127); elements round to the nearest
    E2M1 value (ties to even) and saturate at +-6.
    Returns (packed uint8 [..., N, K/2], scales uint8 [..., K/32, N]).
    """
    *lead, N, K = w.shape
    g = w.float().reshape(*lead, N, K // 32, 32)
    amax = g.abs().amax(-1)
    _, ex = torch.frexp(amax)                   # amax = m * 2**ex, m in [0.5, 1)
    X = (ex.to(torch.int32) - 1 - 2 + 127).clamp(0, 254)
    X = torch.where(amax == 0, torch.full_like(X, 127), X)
    scaled = g * torch.exp2(-(X.float() - 127.0)).unsqueeze(-1)
    a = scaled.abs()
    code = torch.zeros_like(a, dtype=torch.uint8)
    for i, m in enumerate(_E2M1_MID):
        up = (a > m) if i % 2 == 0 else (a >= m)
        code += up.to(torch.uint8)
    code |= (scaled < 0).to(torch.uint8) << 3
    return _pack_codes(code.reshape(*lead, N, K)), X.to(torch.uint8).transpose(-1, -2).contiguous()


def quantize(w: torch.Tensor, fmt: str):
    if fmt == "int4":
        return quantize_int4(w)
    if fmt == "mxfp4":
        return quantize_mxfp4(w)
    raise ValueError(f"unknown format {fmt!r}")


# --------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------

class QWeightT:
    """Torch-side 4-bit expert stack (packed, scales) with its format tag."""

    def __init__(self, fmt: str, packed: torch.Tensor, scales: torch.Tensor):
        self.fmt, self.packed, self.scales = fmt, packed, scales

    @property
    def E(self):
        return self.packed.shape[0]

    @property
    def N(self):
        return self.packed.shape[1]

    @property
    def K(self):
        return self.packed.shape[2] * 2

    def to(self, device) -> "QWeightT":
        return QWeightT(self.fmt, self.packed.to(device), self.scales.to(device))

    def nbytes(self) -> int:
        return self.packed.numel() + self.scales.numel() * self.scales.element_size()


def random_qweight(gen: torch.Generator, E: int, N: int, K: int, fmt: str, device,
                   std: float = 0.02) -> QWeightT:
    """E experts of N(0, std) [N, K] weights, quantized one expert at a time."""
    packed = torch.empty((E, N, K // 2), dtype=torch.uint8, device=device)
    sdt = torch.bfloat16 if fmt == "int4" else torch.uint8
    scales = torch.empty((E, K // 32, N), dtype=sdt, device=device)
    for e in range(E):
        w = torch.randn((N, K), generator=gen, device=device, dtype=torch.float32) * std
        packed[e], scales[e] = quantize(w, fmt)
    return QWeightT(fmt, packed, scales)


def router_logits(gen: torch.Generator, cfg: MoEConfig, T: int, device) -> torch.Tensor:
    if cfg.logits == "uniform":
        return torch.rand((T, cfg.E), generator=gen, device=device, dtype=torch.float32)
    lg = torch.randn((T, cfg.E), generator=gen, device=device, dtype=torch.float32)
    if cfg.logits == "zipf":
        # Popularity ranks 1..E in a seeded random order; the bias is the Zipf
        # log-probability -s * ln(rank) with s = 1.1 (constant dropped).
        rank = torch.randperm(cfg.E, generator=gen, device=device).float() + 1.0
        lg = lg + (-1.1 * torch.log(rank)).unsqueeze(0)
    return lg


def make_workload(cfg: MoEConfig, device="cpu", T: int | None = None) -> dict:
    """All inputs of one layer step, drawn in a fixed order from one seeded generator."""
    T = cfg.T if T is None else T
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg.seed)
    out = {"cfg": cfg, "T": T}
    out["logits"] = router_logits(gen, cfg, T, device)
    out["x"] = torch.randn((T, cfg.d), generator=gen, device=device).to(torch.bfloat16)
    if cfg.swiglu:
        out["w_gu"] = random_qweight(gen, cfg.E, 2 * cfg.f, cfg.d, cfg.fmt, device)
        out["w_d"] = random_qweight(gen, cfg.E, cfg.d, cfg.f, cfg.fmt, device)
    else:
        out["w_up"] = random_qweight(gen, cfg.E, cfg.f, cfg.d, cfg.fmt, device)
    if cfg.adapter:
        noise = torch.randn((cfg.E, cfg.d // 32, 32, 32), generator=gen, device=device) * 1e-3
        eye = torch.eye(32, device=device).expand_as(noise)
        out["adapter"] = (eye + noise).to(torch.bfloat16)
    if cfg.train:
        out["dy"] = torch.randn((T, cfg.d), generator=gen, device=device).to(torch.bfloat16)
    return out
