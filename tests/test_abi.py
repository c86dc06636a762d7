"""The C ABI on the host: the library loads, exports every entry point the
header declares, and rejects bad arguments before launching anything.
These run without a GPU (validation happens before any launch)."""

import ctypes
import os
import re

import pytest

from quantized_rl_fine_b200 import build, moeq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moeq.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return moeq.lib()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert "moe_route_permute" in names and "moe_grouped_qgemm_bwd_dx" in names
    for n in names:
        assert hasattr(L, n), n
    assert set(moeq.EXPORTED) == set(names)


def test_abi_version_and_status_strings(L):
    assert L.moe_abi_version() == 2


def test_default_build_has_nvtx_ranges(L):
    # every entry point that launches work opens an NVTX range (compile flag MOEQ_NVTX)
    assert L.moe_nvtx_enabled() == 1
    assert L.moe_status_string(0) == b"MOE_OK"
    assert L.moe_status_string(4) == b"MOE_ERR_WORKSPACE"


def _qw(packed=0x10000, scales=0x20000, E=4, N=256, K=512, fmt=moeq.W_INT4):
    return moeq.QWeightC(packed, scales, E, N, K, fmt)


def _groups(E=4):
    return moeq.GroupsC(0x30000, 0x40000, 0x50000, 0x60000, 0x70000, E)


def _fwd(L, a=0x80000, M=64, qw=None, g=None, adapter=None, epi=0, out=0x90000, saved=None,
         ws=None, wsb=None, rows=None):
    qw = qw or _qw()
    g = g or _groups(qw.E)
    wsb = wsb if wsb is not None else ctypes.c_size_t(0)
    return L.moe_grouped_qgemm_fwd(a, rows, M, ctypes.byref(qw), ctypes.byref(g), adapter, epi, out,
                                   saved, ws, ctypes.byref(wsb), None)


def test_fwd_workspace_query_and_validation(L):
    wsb = ctypes.c_size_t(123)
    assert _fwd(L, wsb=wsb) == moeq.MOE_OK
    assert wsb.value == 0                                            # no adapter: no workspace
    wsb2 = ctypes.c_size_t(0)
    assert _fwd(L, adapter=0xA0000, wsb=wsb2) == moeq.MOE_OK
    base = wsb2.value
    assert base >= 64 * 512 * 2 and base % 256 == 0                  # a' rows
    # Shape rules (a reading of the boundary): K % 64, N % 64, and N % 128
    # for the SwiGLU gate/up weight; a K with a 64-element tail is accepted.
    assert _fwd(L, qw=_qw(K=96)) == 3                                # K % 64
    assert _fwd(L, qw=_qw(K=32)) == 3
    assert _fwd(L, qw=_qw(N=100)) == 3                               # N % 64
    assert _fwd(L, qw=_qw(N=80)) == 3
    assert _fwd(L, qw=_qw(K=576)) == moeq.MOE_OK                     # K % 128 == 64
    assert _fwd(L, qw=_qw(N=320)) == moeq.MOE_OK                     # N % 128 == 64, no SwiGLU
    assert _fwd(L, qw=_qw(fmt=7)) == 1
    assert _fwd(L, qw=_qw(packed=0x10008)) == 2                      # misaligned
    assert _fwd(L, epi=2) == 1                                       # backward epilogue in fwd
    assert _fwd(L, qw=_qw(N=192), epi=1) == 3                        # SwiGLU needs N % 128
    assert _fwd(L, M=0) == 1
    small = ctypes.c_size_t(16)
    assert _fwd(L, adapter=0xA0000, ws=0x100000, wsb=small) == 4     # workspace too small
    ok = ctypes.c_size_t(base)
    assert _fwd(L, adapter=0xA0000, ws=0x100008, wsb=ok) == 2        # ws not 256-aligned
    assert _fwd(L, adapter=0xA0000, ws=0x100000, wsb=ok, a=0x80004) == 2
    # no workspace at all: fine without an adapter, an error with one
    qw, g = _qw(), _groups()
    assert L.moe_grouped_qgemm_fwd(0x80004, None, 64, ctypes.byref(qw), ctypes.byref(g), None, 0,
                                   0x90000, None, None, None, None) == 2
    assert L.moe_grouped_qgemm_fwd(0x80000, None, 64, ctypes.byref(qw), ctypes.byref(g), 0xA0000, 0,
                                   0x90000, None, None, None, None) == 4
    # a row index for gathered input rows: 16-byte aligned like every pointer
    assert L.moe_grouped_qgemm_fwd(0x80000, 0xB0004, 64, ctypes.byref(qw), ctypes.byref(g), None, 0,
                                   0x90000, None, None, None, None) == 2


def test_bwd_argument_rules(L):
    qw, g = _qw(), _groups()
    wsb = ctypes.c_size_t(0)

    def call(epi=0, saved=None, adapter=None, a=None, dad=None, rows=None):
        return L.moe_grouped_qgemm_bwd_dx(0x80000, 64, ctypes.byref(qw), ctypes.byref(g), epi,
                                          saved, adapter, a, rows, 0x90000, dad, None,
                                          ctypes.byref(wsb), None)
    assert call() == moeq.MOE_OK
    assert call(epi=2) == 1                      # SwiGLU backward needs saved g|u
    assert call(epi=2, saved=0xB0000) == moeq.MOE_OK
    assert call(adapter=0xA0000) == 1            # adapter needs a and d_adapter
    assert call(adapter=0xA0000, a=0xC0000, dad=0xD0000) == moeq.MOE_OK
    assert call(epi=2, saved=0xB0000, adapter=0xA0000, a=0xC0000, dad=0xD0000) == 1
    assert call(a=0xC0000) == 1
    assert call(rows=0xE0000) == 1               # a row index only with an adapter
    assert call(adapter=0xA0000, a=0xC0000, dad=0xD0000, rows=0xE0000) == moeq.MOE_OK
    assert call(epi=1) == 1


def test_route_and_combine_validation(L):
    wsb = ctypes.c_size_t(0)
    p = 0x10000

    def route(T=64, E=8, k=2, d=256, C=8, x=p, ws=None, wsb=wsb, logits=p):
        return L.moe_route_permute(logits, x, T, E, k, d, C, p, p, p, p, p, p, p, p, p, p, ws,
                                   ctypes.byref(wsb), None)
    # The single-pass tail (T <= 1024 and E * ceil(T/32) <= 8192) needs no
    # workspace; larger launches need ceil(T/64) * E int32 histogram entries.
    assert route() == moeq.MOE_OK and wsb.value == 0
    assert route(T=1024, E=256) == moeq.MOE_OK and wsb.value == 0
    assert route(T=1024, E=257) == moeq.MOE_OK and wsb.value >= 16 * 257 * 4
    assert route(T=4096, E=384) == moeq.MOE_OK and wsb.value >= 64 * 384 * 4
    assert wsb.value % 256 == 0
    # a single-pass launch runs without any workspace (ws and ws_bytes NULL)
    # as far as validation goes: here its misaligned logits are refused
    assert L.moe_route_permute(p + 4, p, 64, 8, 2, 256, 8, p, p, p, p, p, p, p, p, p, p, None,
                               None, None) == 2
    # a larger one without a workspace is a workspace error
    assert L.moe_route_permute(p, p, 4096, 384, 8, 256, 8, p, p, p, p, p, p, p, p, p, p, None,
                               None, None) == 4
    assert route(k=9) == 1 and route(k=0) == 1 and route(E=1025) == 1 and route(C=0) == 1
    assert route(k=33, E=64) == 1
    full = ctypes.c_size_t(wsb.value)
    assert route(ws=0x200000, wsb=full, d=12) == 1                  # d % 8
    assert route(ws=0x200000, wsb=full, logits=p + 4) == 2
    assert L.moe_unpermute_combine(p, p, None, 4, 2, 12, p, 0, None) == 1
    assert L.moe_unpermute_combine(p, p, None, 4, 2, 16, p, 2, None) == 1
    assert L.moe_unpermute_combine(p + 8, p, None, 4, 2, 16, p, 0, None) == 2
    assert L.moe_test_dequant(p, p, 4, 48, 1, p, None) == 1


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        moeq.moe_route_permute(torch.zeros((4, 4)), None, 2, 1)


def test_plain_c_host_compiles_links_and_calls(L, tmp_path):
    """The header is plain C99 (no CUDA or C++ headers needed), and a C program
    links against the library and calls the host-only entry points."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler on this host")
    src = tmp_path / "host.c"
    src.write_text(
        '#include <stdio.h>\n#include "moeq.h"\n'
        "int main(void) {\n"
        '  printf("%d %s\\n", (int)moe_abi_version(), moe_status_string(MOE_ERR_WORKSPACE));\n'
        "  return 0;\n}\n")
    exe = tmp_path / "host"
    libdir = os.path.dirname(moeq.LIB_PATH)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-lmoeq", "-Wl,-rpath," + libdir],
                   check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert out == [str(L.moe_abi_version()), "MOE_ERR_WORKSPACE"]
