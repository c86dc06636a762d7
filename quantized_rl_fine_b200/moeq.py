"""ctypes binding of libmoeq (include/moeq.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. PyTorch supplies device memory (outputs, workspaces) and the current
stream. There is no CPU fallback: if the library is not built, or no CUDA
device is present, every call raises.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

from .synth import QWeightT

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libmoeq.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_MISALIGNED",
                3: "MOE_ERR_UNSUPPORTED", 4: "MOE_ERR_WORKSPACE", 5: "MOE_ERR_CUDA",
                6: "MOE_ERR_DEVICE"}
W_INT4 = 1
W_MXFP4 = 2
FMT = {"int4": W_INT4, "mxfp4": W_MXFP4}
EPI_NONE, EPI_SWIGLU, EPI_SWIGLU_BWD = 0, 1, 2
DEVERR_NONE, DEVERR_WAIT_TIMEOUT, DEVERR_BAD_OFFSETS = 0, 1, 2

EXPORTED = ("moe_route_permute", "moe_route_permute_noalloc", "moe_grouped_qgemm_fwd", "moe_grouped_qgemm_bwd_dx",
            "moe_unpermute_combine", "moe_get_device_error", "moe_status_string",
            "moe_abi_version", "moe_test_dequant", "moe_test_set_wait_budget",
            "moe_dequant_experts", "moe_ep_regroup", "moe_nvtx_enabled")


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


class QWeightC(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("E", ctypes.c_int32), ("N", ctypes.c_int32), ("K", ctypes.c_int32),
                ("fmt", ctypes.c_int32)]


class GroupsC(ctypes.Structure):
    _fields_ = [("expert_offsets", ctypes.c_void_p), ("active", ctypes.c_void_p),
                ("num_active", ctypes.c_void_p), ("chunk_offsets", ctypes.c_void_p),
                ("num_chunks", ctypes.c_void_p), ("E", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libmoeq.so is not built ({LIB_PATH}); run "
                           "`python -m quantized_rl_fine_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.POINTER(ctypes.c_size_t)
    L.moe_route_permute.argtypes = [vp, vp, i64, i32, i32, i64, i32, vp, vp, vp, vp, vp, vp, vp,
                                    vp, vp, vp, vp, sz, vp]
    L.moe_route_permute_noalloc.argtypes = [vp, vp, i64, i32, i32, i64, i32, vp, vp, vp, vp, vp,
                                            vp, vp, vp, vp, vp, vp]
    L.moe_grouped_qgemm_fwd.argtypes = [vp, vp, i64, ctypes.POINTER(QWeightC),
                                        ctypes.POINTER(GroupsC), vp, i32, vp, vp, vp, sz, vp]
    L.moe_grouped_qgemm_bwd_dx.argtypes = [vp, i64, ctypes.POINTER(QWeightC),
                                           ctypes.POINTER(GroupsC), i32, vp, vp, vp, vp, vp, vp,
                                           vp, sz, vp]
    L.moe_unpermute_combine.argtypes = [vp, vp, vp, i64, i32, i64, vp, i32, vp]
    L.moe_get_device_error.argtypes = [ctypes.POINTER(i32), vp]
    L.moe_status_string.argtypes = [i32]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_abi_version.argtypes = []
    L.moe_test_dequant.argtypes = [vp, vp, i64, i32, i32, vp, vp]
    L.moe_test_set_wait_budget.argtypes = [i64]
    L.moe_dequant_experts.argtypes = [ctypes.POINTER(QWeightC), vp, i32, vp, vp]
    L.moe_ep_regroup.argtypes = [vp, i32, i32, i64, vp, vp, i64, i32, i32, vp, vp, vp, vp, vp, vp]
    for name in EXPORTED:
        if name not in ("moe_status_string",):
            getattr(L, name).restype = ctypes.c_int32
    _lib = L
    return L


def _check(status: int, what: str):
    if status != MOE_OK:
        raise MoeError(status, what)


def _p(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libmoeq takes CUDA tensors only")


def _workspace(nbytes: int, device):
    """(tensor or None, pointer or None, size argument) for a queried workspace size."""
    if int(nbytes) == 0:
        return None, None, None
    ws = torch.empty(int(nbytes), dtype=torch.uint8, device=device)
    return ws, ws.data_ptr(), ctypes.byref(ctypes.c_size_t(ws.numel()))


# --------------------------------------------------------------------------
# Routing
# --------------------------------------------------------------------------

@dataclass
class Routing:
    topk_idx: torch.Tensor        # [T, k] int32
    gates: torch.Tensor           # [T, k] fp32
    expert_offsets: torch.Tensor  # [E+1] int32
    active: torch.Tensor          # [E] int32
    num_active: torch.Tensor      # [1] int32
    chunk_offsets: torch.Tensor   # [E+1] int32
    num_chunks: torch.Tensor      # [1] int32
    perm_token: torch.Tensor      # [T*k] int32
    inv_perm: torch.Tensor        # [T*k] int32
    x_perm: torch.Tensor | None   # [T*k, d] bf16
    E: int
    k: int

    def groups(self) -> GroupsC:
        return GroupsC(_p(self.expert_offsets), _p(self.active), _p(self.num_active),
                       _p(self.chunk_offsets), _p(self.num_chunks), self.E)


def moe_route_permute(logits: torch.Tensor, x: torch.Tensor | None, k: int, chunk_size: int,
                      stream=None, out: Routing | None = None) -> Routing:
    _require_cuda(logits, x)
    T, E = logits.shape
    dev = logits.device
    if out is None:
        i32 = dict(dtype=torch.int32, device=dev)
        out = Routing(
            topk_idx=torch.empty((T, k), **i32), gates=torch.empty((T, k), dtype=torch.float32, device=dev),
            expert_offsets=torch.empty(E + 1, **i32), active=torch.empty(E, **i32),
            num_active=torch.empty(1, **i32), chunk_offsets=torch.empty(E + 1, **i32),
            num_chunks=torch.empty(1, **i32), perm_token=torch.empty(T * k, **i32),
            inv_perm=torch.empty(T * k, **i32),
            x_perm=None if x is None else torch.empty((T * k, x.shape[1]), dtype=torch.bfloat16, device=dev),
            E=E, k=k)
    L = lib()
    d = 0 if x is None else x.shape[1]
    wsb = ctypes.c_size_t(0)
    args = lambda ws, wsz: (_p(logits), _p(x), T, E, k, d, chunk_size, _p(out.topk_idx),
                            _p(out.gates), _p(out.expert_offsets), _p(out.active),
                            _p(out.num_active), _p(out.chunk_offsets), _p(out.num_chunks),
                            _p(out.perm_token), _p(out.inv_perm), _p(out.x_perm), ws, wsz,
                            _stream(stream))
    _check(L.moe_route_permute(*args(None, ctypes.byref(wsb))), "moe_route_permute (workspace query)")
    ws, wsp, wsz = _workspace(wsb.value, dev)
    _check(L.moe_route_permute(*args(wsp, wsz)), "moe_route_permute")
    return out


# --------------------------------------------------------------------------
# Grouped GEMMs
# --------------------------------------------------------------------------

def qweight_c(w: QWeightT) -> QWeightC:
    _require_cuda(w.packed, w.scales)
    return QWeightC(_p(w.packed), _p(w.scales), w.E, w.N, w.K, FMT[w.fmt])


def moe_grouped_qgemm_fwd(a: torch.Tensor, w: QWeightT, routing: Routing, epi: int = EPI_NONE,
                          adapter: torch.Tensor | None = None, save_gu: bool = False,
                          stream=None, out: torch.Tensor | None = None,
                          saved: torch.Tensor | None = None, a_rows: torch.Tensor | None = None):
    """Returns out [M, N] (none) or (out [M, N/2], saved [M, N] or None) (swiglu).
    With a_rows (int32 [M], e.g. routing.perm_token), row p of the input is a[a_rows[p]]."""
    _require_cuda(a, adapter, a_rows)
    M = a_rows.shape[0] if a_rows is not None else a.shape[0]
    F = w.N // 2 if epi == EPI_SWIGLU else w.N
    if out is None:
        out = torch.empty((M, F), dtype=torch.bfloat16, device=a.device)
    if save_gu and saved is None:
        saved = torch.empty((M, w.N), dtype=torch.bfloat16, device=a.device)
    qw, g = qweight_c(w), routing.groups()
    wsb = ctypes.c_size_t(0)
    L = lib()
    args = lambda ws, wsz: (_p(a), _p(a_rows), M, ctypes.byref(qw), ctypes.byref(g), _p(adapter),
                            epi, _p(out), _p(saved) if save_gu else None, ws, wsz, _stream(stream))
    _check(L.moe_grouped_qgemm_fwd(*args(None, ctypes.byref(wsb))),
           "moe_grouped_qgemm_fwd (workspace query)")
    ws, wsp, wsz = _workspace(wsb.value, a.device)
    _check(L.moe_grouped_qgemm_fwd(*args(wsp, wsz)), "moe_grouped_qgemm_fwd")
    if epi == EPI_SWIGLU:
        return out, (saved if save_gu else None)
    return out


def moe_grouped_qgemm_bwd_dx(dout: torch.Tensor, w: QWeightT, routing: Routing,
                             epi: int = EPI_NONE, saved_gu: torch.Tensor | None = None,
                             adapter: torch.Tensor | None = None, a: torch.Tensor | None = None,
                             stream=None, out: torch.Tensor | None = None,
                             a_rows: torch.Tensor | None = None):
    """Returns din ([M, K], or [M, 2K] for swiglu_bwd), plus d_adapter when an adapter is given.
    With a_rows, row p of the adapter's input a is a[a_rows[p]]."""
    _require_cuda(dout, saved_gu, adapter, a, a_rows)
    M = dout.shape[0]
    width = 2 * w.K if epi == EPI_SWIGLU_BWD else w.K
    if out is None:
        out = torch.empty((M, width), dtype=torch.bfloat16, device=dout.device)
    d_adapter = None
    if adapter is not None:
        d_adapter = torch.empty((w.E, w.K // 32, 32, 32), dtype=torch.float32, device=dout.device)
    qw, g = qweight_c(w), routing.groups()
    wsb = ctypes.c_size_t(0)
    L = lib()
    args = lambda ws, wsz: (_p(dout), M, ctypes.byref(qw), ctypes.byref(g), epi, _p(saved_gu),
                            _p(adapter), _p(a), _p(a_rows), _p(out), _p(d_adapter), ws, wsz,
                            _stream(stream))
    _check(L.moe_grouped_qgemm_bwd_dx(*args(None, ctypes.byref(wsb))),
           "moe_grouped_qgemm_bwd_dx (workspace query)")
    ws, wsp, wsz = _workspace(wsb.value, dout.device)
    _check(L.moe_grouped_qgemm_bwd_dx(*args(wsp, wsz)), "moe_grouped_qgemm_bwd_dx")
    return (out, d_adapter) if adapter is not None else out


def moe_unpermute_combine(rows: torch.Tensor, routing: Routing, gates: torch.Tensor | None,
                          T: int, mode: int = 0, stream=None, out: torch.Tensor | None = None):
    """mode 0: [T*k, D] -> [T, D] gate-weighted sum; mode 1: [T, D] -> [T*k, D] gate-scaled scatter."""
    _require_cuda(rows, gates)
    k = routing.k
    D = rows.shape[1]
    if out is None:
        shape = (T, D) if mode == 0 else (T * k, D)
        out = torch.empty(shape, dtype=torch.bfloat16, device=rows.device)
    _check(lib().moe_unpermute_combine(_p(rows), _p(routing.inv_perm), _p(gates), T, k, D,
                                       _p(out), mode, _stream(stream)), "moe_unpermute_combine")
    return out


def moe_get_device_error(stream=None) -> int:
    code = ctypes.c_int32(0)
    _check(lib().moe_get_device_error(ctypes.byref(code), _stream(stream)), "moe_get_device_error")
    return code.value


def moe_test_dequant(packed: torch.Tensor, scales: torch.Tensor, fmt: str, stream=None) -> torch.Tensor:
    """packed [R, K/2] uint8, scales [K/32, R] -> bf16 [R, K] with the GEMM's dequant functions."""
    _require_cuda(packed, scales)
    R, half = packed.shape
    out = torch.empty((R, 2 * half), dtype=torch.bfloat16, device=packed.device)
    _check(lib().moe_test_dequant(_p(packed), _p(scales), R, 2 * half, FMT[fmt], _p(out),
                                  _stream(stream)), "moe_test_dequant")
    return out


def moe_dequant_experts(w: QWeightT, experts: torch.Tensor, stream=None,
                        out: torch.Tensor | None = None) -> torch.Tensor:
    """Whole experts dequantized to BF16: out [count, N, K] = W[experts]."""
    _require_cuda(experts)
    count = int(experts.numel())
    if out is None:
        out = torch.empty((count, w.N, w.K), dtype=torch.bfloat16, device=experts.device)
    qw = qweight_c(w)
    _check(lib().moe_dequant_experts(ctypes.byref(qw), _p(experts), count, _p(out), _stream(stream)),
           "moe_dequant_experts")
    return out


def moe_ep_regroup(counts: torch.Tensor, rows: torch.Tensor, direction: int, chunk_size: int = 8,
                   stream=None, out: torch.Tensor | None = None):
    """Expert parallelism: received rows [R, D] reordered source-major -> local
    expert-major (direction 0, returns (rows, local Routing tables)) or back
    (direction 1, returns rows). counts: device int32 [W, E_loc]."""
    _require_cuda(counts, rows)
    W, E_loc = counts.shape
    R, D = rows.shape
    if out is None:
        out = torch.empty_like(rows)
    dev = rows.device
    i32 = dict(dtype=torch.int32, device=dev)
    if direction == 0:
        t = dict(expert_offsets=torch.empty(E_loc + 1, **i32), active=torch.empty(E_loc, **i32),
                 num_active=torch.empty(1, **i32), chunk_offsets=torch.empty(E_loc + 1, **i32),
                 num_chunks=torch.empty(1, **i32))
    else:
        t = dict(expert_offsets=None, active=None, num_active=None, chunk_offsets=None, num_chunks=None)
    _check(lib().moe_ep_regroup(_p(counts), W, E_loc, R, _p(rows), _p(out), D, direction, chunk_size,
                                _p(t["expert_offsets"]), _p(t["active"]), _p(t["num_active"]),
                                _p(t["chunk_offsets"]), _p(t["num_chunks"]), _stream(stream)),
           "moe_ep_regroup")
    if direction == 1:
        return out
    groups = Routing(topk_idx=None, gates=None, perm_token=None, inv_perm=None, x_perm=out,
                     E=E_loc, k=1, **t)
    return out, groups


def moe_test_set_wait_budget(cycles: int):
    _check(lib().moe_test_set_wait_budget(int(cycles)), "moe_test_set_wait_budget")
