"""Byte and flop accounting of the grouped low-bit GEMMs (used for GB/s, TFLOP/s).

Storage per parameter of the two 4-bit bases: 4 bits of element plus the
group scale spread over its 32 elements -- INT4 with a BF16 scale costs
0.5 + 2/32 = 0.5625 bytes, MXFP4 with an 8-bit scale 0.5 + 1/32 = 0.53125.
The open-weight MoE explainer (section 三, "storage arithmetic") estimates a
quantized checkpoint the same way: 4-bit main weights, one 8-bit scale per
32-element group, and a small share of "sensitive" parameters kept in FP16.
"""

from __future__ import annotations

SCALE_BYTES = {"int4": 2, "mxfp4": 1}
GROUP = 32


def bytes_per_param(fmt: str) -> float:
    return 0.5 + SCALE_BYTES[fmt] / GROUP


def storage_estimate(total_params: float, bits: int = 4, group_size: int = 32,
                     scale_bits: int = 8, sensitive_ratio: float = 0.02) -> float:
    """Bytes of a group-quantized checkpoint: quantized body + one scale per
    group + the sensitive share kept at 2 bytes per parameter."""
    body_params = total_params * (1.0 - sensitive_ratio)
    body = body_params * bits / 8.0
    scales = body_params / group_size * scale_bits / 8.0
    sensitive = total_params * sensitive_ratio * 2.0
    return body + scales + sensitive


def expert_weight_bytes(N: int, K: int, fmt: str) -> int:
    """Packed nibbles + group scales of one [N, K] expert matrix."""
    return N * K // 2 + N * (K // GROUP) * SCALE_BYTES[fmt]


def gemm_flops(rows_per_expert, N: int, K: int) -> int:
    """Useful flops 2 * sum_e m_e * N * K (no padding)."""
    return 2 * int(sum(int(m) for m in rows_per_expert)) * N * K


def active_weight_bytes(rows_per_expert, N: int, K: int, fmt: str) -> int:
    """Weight bytes streamed by one grouped GEMM: only experts with rows are read."""
    n_active = sum(1 for m in rows_per_expert if int(m) > 0)
    return n_active * expert_weight_bytes(N, K, fmt)
