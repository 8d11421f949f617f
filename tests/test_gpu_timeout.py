"""Failure detection on the GPU without a fault: every wait in the kernels is
bounded, and a wait that runs out sets the TIMEOUT status bit, aborts the
CTA's pipeline (later waits return at once, copies in flight are drained with
the full budget, TMEM is released) and the kernel returns.  The tests shorten
the waits' budget through the library's internal test hook so that they run
out, read the status on the host, and check that the context and the
workspace are still usable afterwards."""
import numpy as np
import pytest
import torch

from rans_decode_gemm_b200 import ans
from rans_decode_gemm_b200 import workloads as WL

from _gpu_util import make_case, rel_fro, run_gemm, status_tensor

pytestmark = pytest.mark.gpu

TOL = 1e-3


@pytest.fixture
def wait_budget():
    yield ans._set_wait_budget
    ans._set_wait_budget(0)


def test_wait_on_a_barrier_nothing_arrives_on_times_out(cuda, wait_budget):
    wait_budget(200_000)            # about 0.1 ms
    st = status_tensor()
    ans._wait_probe(st)
    torch.cuda.synchronize()
    assert int(st.item()) & ans.STATUS_TIMEOUT


@pytest.mark.parametrize("schedule,M", [("local", 16), ("central", 64)])
def test_gemm_waits_run_out_then_the_next_call_is_exact(cuda, oracle, wait_budget, plan_limits,
                                                         schedule, M):
    plan_limits(schedule=schedule)
    cfg, d, lay, layer = make_case("bf16_4096", 512, 1024, state_bits=64)
    X = WL.make_x(cfg, M, 1024)
    wait_budget(2000)               # about a microsecond: the pipeline's waits run out
    Y, st, ws = run_gemm(cfg, d, lay, layer, X, compressed=True)
    assert st & ans.STATUS_TIMEOUT
    wait_budget(0)
    # every CTA still took part in split-K: the counters are back at zero, so
    # the same workspace serves the next call, which is exact
    nseg = lay.N // lay.tile_n
    assert int(ws[:4 * nseg].view(torch.int32).abs().sum().item()) == 0
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True, ws=ws)
    assert st == 0
    Yref = oracle.gemm(cfg.dtype, X, M, 1024, d["w"], 512)
    assert rel_fro(Y.cpu().numpy(), Yref) <= TOL


def test_decode_tiles_with_short_waits_is_exact_or_flagged(cuda, wait_budget):
    # the standalone decode waits only for its own bulk copies, which usually
    # land inside mbarrier.try_wait's own suspend window: with a short budget
    # the result is exact, or the status says the wait ran out -- never wrong
    # without a flag; with the default budget it is exact
    cfg, d, lay, layer = make_case("fp8_405b", 512, 2048, state_bits=64)
    out = torch.empty(512 * 2048, dtype=torch.uint8, device="cuda")
    st = status_tensor()
    wait_budget(1)
    ans.ans_decode_tiles(layer.tiles, out, st)
    torch.cuda.synchronize()
    flags = int(st.item())
    assert flags in (0, ans.STATUS_TIMEOUT) or flags & ans.STATUS_TIMEOUT
    if flags == 0:
        assert np.array_equal(out.cpu().numpy(), d["w"])
    wait_budget(0)
    st = status_tensor()
    ans.ans_decode_tiles(layer.tiles, out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(out.cpu().numpy(), d["w"])


def test_large_m_waits_run_out_then_the_next_call_is_exact(cuda, oracle, wait_budget):
    # the fused first pass and the dense GEMM of the remaining tokens both
    # return on a run-out wait with the flag set; the next call is exact
    cfg, d, lay, layer = make_case("bf16_4096", 512, 1024, state_bits=64)
    M = 700
    X = WL.make_x(cfg, M, 1024)
    wait_budget(2000)
    Y, st, ws = run_gemm(cfg, d, lay, layer, X, compressed=True)
    assert st & ans.STATUS_TIMEOUT
    wait_budget(0)
    nseg = lay.N // lay.tile_n
    assert int(ws[:4 * nseg].view(torch.int32).abs().sum().item()) == 0
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True, ws=ws)
    assert st == 0
    Yref = oracle.gemm(cfg.dtype, X, M, 1024, d["w"], 512)
    assert rel_fro(Y.cpu().numpy(), Yref) <= TOL
