"""Shared helpers of the test suite: torch <-> oracle conversions and the
parity criteria."""

from __future__ import annotations

import numpy as np
import torch

import oracle as O

# BF16 outputs that end the computation (y, out, dx, d_adapter): the
# workload's tolerance against the oracle.
MAX_ABS = 2e-2
REL_L2 = 5e-3


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 values of a bf16/fp32 tensor."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_qweight(w) -> O.QWeight:
    if w.fmt == "int4":
        scales = bf16_bits(w.scales)
    else:
        scales = w.scales.detach().cpu().numpy()
    return O.QWeight(w.fmt, w.packed.detach().cpu().numpy(), scales)


def assert_close_final(got: np.ndarray, want: np.ndarray, what: str,
                       max_abs: float = MAX_ABS, rel_l2: float = REL_L2):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - want)
    mx = float(err.max()) if err.size else 0.0
    rl2 = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)) if err.size else 0.0
    assert mx <= max_abs and rl2 <= rel_l2, f"{what}: max-abs {mx:.3e} rel-L2 {rl2:.3e}"
    return mx, rl2


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return np.ldexp(1.0, np.frexp(ax)[1] - 8)


def assert_close_intermediate(got: np.ndarray, want: np.ndarray, what: str, abs_tol: float = 2e-2):
    """Per-slot intermediates: |err| <= abs_tol + one BF16 ulp of the oracle value."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    err = np.abs(got - want)
    lim = abs_tol + bf16_ulp(want)
    bad = err > lim
    assert not np.any(bad), f"{what}: {int(bad.sum())} elements out of tolerance, worst {float(err.max()):.3e}"


def adapter_grad_bound(x_rows: np.ndarray, dxa_rows: np.ndarray, row_expert: np.ndarray, E: int,
                       base: float = 2e-2) -> np.ndarray:
    """Element bound for the FP32 adapter gradient dR[e,b,i,j] = sum_p x[p,32b+i] dx'[p,32b+j].

    dx' is a BF16 intermediate: the library and the oracle may round each of
    its elements to neighbouring BF16 values (their FP32 sums differ in
    order), so dR may differ by up to sum_p |x[p,32b+i]| * ulp(dx'[p,32b+j]),
    plus the base absolute tolerance of the final outputs.
    """
    nb = x_rows.shape[1] // 32
    out = np.zeros((E, nb, 32, 32))
    ax = np.abs(x_rows).reshape(x_rows.shape[0], nb, 32)
    ul = bf16_ulp(dxa_rows).reshape(dxa_rows.shape[0], nb, 32)
    for e in range(E):
        sel = row_expert == e
        out[e] = np.einsum("mbi,mbj->bij", ax[sel], ul[sel])
    return base + out


def assert_close_bounded(got: np.ndarray, want: np.ndarray, bound: np.ndarray, what: str,
                         rel_l2: float = REL_L2):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape == bound.shape, (what, got.shape, want.shape, bound.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - want)
    bad = err > bound
    rl2 = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))
    assert not np.any(bad) and rl2 <= rel_l2, \
        f"{what}: {int(bad.sum())} elements above their bound, rel-L2 {rl2:.3e}"
