"""Failure detection without a GPU fault.  Every wait of the tensor-core
kernels is a bounded mbarrier wait that, when it runs out, ORs KDA_DEV_TIMEOUT
into the caller's status word and returns.  kda_selftest_bounded_wait takes
that wait on a barrier that never completes (nothing else is in flight), so the
expiry path runs for real: the status bit appears, the wait lasted its budget,
other status bits survive, and the context stays usable for a checked call.
The host-side checks of the entry run on the CPU."""
import ctypes

import pytest
import torch

import kimi_delta_attention_22_b200 as kda
from kimi_delta_attention_22_b200 import build as kbuild
from kimi_delta_attention_22_b200 import inputs
from parity import check, oracle_chunk, run_chunk


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load_library()


def test_selftest_validation(lib):
    """Rejected before any launch: no status word, misaligned word, budget out of range."""
    A = ctypes.c_void_p(0x10000)
    assert lib.kda_selftest_bounded_wait(None, 1000, 0, None) == 1
    assert lib.kda_selftest_bounded_wait(ctypes.c_void_p(0x10002), 1000, 0, None) == 1
    assert lib.kda_selftest_bounded_wait(A, 0, 0, None) == 1
    assert lib.kda_selftest_bounded_wait(A, 1000001, 0, None) == 1


@pytest.mark.gpu
def test_wait_runs_out_and_reports():
    st = torch.full((1,), kda.KDA_DEV_BAD_SEQLENS, dtype=torch.int32, device="cuda")
    budget_us = 2000
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    kda.kda_selftest_bounded_wait(st, budget_us)
    e1.record()
    torch.cuda.synchronize()
    assert int(st.item()) == kda.KDA_DEV_BAD_SEQLENS | kda.KDA_DEV_TIMEOUT
    assert e0.elapsed_time(e1) >= budget_us * 1e-3 * 0.95


@pytest.mark.gpu
def test_wait_that_completes_reports_nothing():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kda.kda_selftest_bounded_wait(st, 1000000, complete=True)
    torch.cuda.synchronize()
    assert int(st.item()) == 0


@pytest.mark.gpu
def test_context_usable_after_expiry():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kda.kda_selftest_bounded_wait(st, 500)
    torch.cuda.synchronize()
    assert int(st.item()) & kda.KDA_DEV_TIMEOUT
    d = inputs.draw(2, 130, 2, 128, 128, dtype=torch.bfloat16, gate="channel", s0_std=0.02, seed=77)
    out, ST = run_chunk(d, 64)
    ro, rs = oracle_chunk(d, "channel")
    check(out, ro, "bf16", "out after an expired wait")
    check(ST, rs, "bf16", "S_T after an expired wait")
