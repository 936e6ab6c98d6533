"""The C ABI library on the CPU: it loads, exports every function include/kda.h
declares, and its host-side validation rejects bad calls before any launch
(no compute call is made: every accepted call here has zero sequences)."""
import ctypes
import os
import re

import pytest

import kimi_delta_attention_22_b200 as kda
from kimi_delta_attention_22_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load_library()


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(kda_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("kda_chunk_fwd", "kda_chunk_fwd_workspace_size", "kda_decode_step", "kda_status_str",
              "kda_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"libkda.so does not export {name}"


def test_status_strings(lib):
    assert kda.kda_status_str(0) == "ok"
    assert "aligned" in kda.kda_status_str(3)
    assert b"sm_100a" in lib.kda_version()


def _shape(B=1, T=8, H=2, dk=128, dv=128, N=None, dtype=kda.KDA_BF16, gate=kda.KDA_GATE_CHANNEL,
           chunk=64):
    return kda.Shape(B, T, H, dk, dv, B if N is None else N, dtype, gate, chunk, None)


P = ctypes.c_void_p
A = P(0x10000)  # a 16-byte aligned fake address: only ever seen by host-side checks


def _chunk(lib, sh, q=A, g=A, cu=None, S0=None, ws=None, ws_bytes=0):
    return lib.kda_chunk_fwd(None if sh is None else ctypes.byref(sh), q, A, A, g, A, S0, cu, A,
                             None, ws, ws_bytes, None)


def test_chunk_validation(lib):
    assert _chunk(lib, None) == 1
    # zero sequences: valid, nothing launched
    assert _chunk(lib, _shape(B=0, N=0)) == 0
    assert _chunk(lib, _shape(B=0, N=0, dtype=kda.KDA_F32, dk=16, dv=32, chunk=16)) == 0
    # num_seqs must equal B for a dense batch
    assert _chunk(lib, _shape(B=0, N=3)) == 1
    # varlen needs B == 1
    assert _chunk(lib, _shape(B=2, N=0), cu=A) == 1
    # gate NONE requires g == NULL and vice versa
    assert _chunk(lib, _shape(B=0, N=0, gate=kda.KDA_GATE_NONE)) == 1
    assert _chunk(lib, _shape(B=0, N=0, gate=kda.KDA_GATE_CHANNEL), g=None) == 1
    # bad enums
    assert _chunk(lib, _shape(B=0, N=0, dtype=7)) == 1
    assert _chunk(lib, _shape(B=0, N=0, gate=9)) == 1
    # negative sizes
    assert _chunk(lib, _shape(B=0, N=0, T=-1)) == 1
    assert _chunk(lib, _shape(B=0, N=0, H=0)) == 1
    # misaligned pointers
    assert _chunk(lib, _shape(B=0, N=0), q=P(0x10004)) == 3
    assert _chunk(lib, _shape(B=0, N=0), S0=P(0x10008)) == 3
    assert _chunk(lib, _shape(B=0, N=0), g=P(0x10004)) == 3                       # per-channel g
    assert _chunk(lib, _shape(B=0, N=0, gate=kda.KDA_GATE_SCALAR), g=P(0x10004)) == 0  # scalar g
    assert _chunk(lib, _shape(B=1, N=0), cu=P(0x10004)) == 0                      # cu_seqlens
    # unsupported head sizes / chunks
    assert _chunk(lib, _shape(B=0, N=0, dk=24, dv=24, dtype=kda.KDA_F32)) == 2
    assert _chunk(lib, _shape(B=0, N=0, dk=256, dv=128, dtype=kda.KDA_F32)) == 2
    assert _chunk(lib, _shape(B=0, N=0, chunk=48, dtype=kda.KDA_F32)) == 2
    # null tensors with tokens present
    assert _chunk(lib, _shape(B=1, T=4, N=1), q=None) == 1


def test_workspace_size_and_checks(lib):
    sh = _shape(B=4, T=2048, H=16, N=4)
    # one record of 74240 bytes per (chunk, head) plus the job list
    n = lib.kda_chunk_fwd_workspace_size(ctypes.byref(sh), 0)
    assert n >= 4 * 32 * 16 * 74240 and n < 4 * 32 * 16 * 74240 + 65536
    # packed batches reserve one extra partial chunk per sequence and the chunk offsets
    shv = _shape(B=1, T=2048, H=16, N=4)
    assert lib.kda_chunk_fwd_workspace_size(ctypes.byref(shv), 1) >= (32 + 4) * 16 * 74240
    # the CUDA-core path needs none
    sf = _shape(B=4, T=64, H=1, dk=16, dv=16, N=4, dtype=kda.KDA_F32, chunk=16)
    assert lib.kda_chunk_fwd_workspace_size(ctypes.byref(sf), 0) == 0
    assert lib.kda_chunk_fwd_workspace_size(None, 0) == 0
    # zero sequences with a workspace: too small, misaligned, enough
    z = _shape(B=0, N=0)
    need = lib.kda_chunk_fwd_workspace_size(ctypes.byref(z), 0)
    assert _chunk(lib, z, ws=A, ws_bytes=need) == 0
    assert _chunk(lib, _shape(B=1, T=64, N=1), ws=A, ws_bytes=16) == 1
    assert _chunk(lib, z, ws=P(0x10010), ws_bytes=need + 1024) == 3


def _decode(lib, sh, g=A, S=A):
    return lib.kda_decode_step(None if sh is None else ctypes.byref(sh), A, A, A, g, A, S, A, None)


def test_decode_validation(lib):
    assert _decode(lib, None) == 1
    assert _decode(lib, _shape(B=0, T=1, N=0)) == 0
    assert _decode(lib, _shape(B=0, T=2, N=0)) == 1          # one token per call
    assert _decode(lib, _shape(B=0, T=1, N=0, dk=64)) == 2   # d_k = 128 only
    assert _decode(lib, _shape(B=0, T=1, N=0, gate=kda.KDA_GATE_NONE)) == 1
    assert _decode(lib, _shape(B=0, T=1, N=0), S=P(0x10002)) == 3
    assert _decode(lib, _shape(B=2, T=1, N=2), S=None) == 1


def test_binding_refuses_host_tensors(lib):
    import torch

    q = torch.zeros(1, 4, 1, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd(q, q, q, None, torch.zeros(1, 4, 1), chunk=64)
