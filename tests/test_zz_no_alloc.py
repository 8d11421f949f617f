"""ans_gemm_noalloc: the allocation-free variant of ans_gemm for callers that
cannot call cudaMalloc (graph-capture regions, plug-ins inside a framework
that owns device memory, paths that must not synchronise on an allocation).
Its scratch lives in a fixed device array inside the library, so the test
checks that two calls in a row give the same result as ans_gemm with a
caller-provided workspace, and that oversize shapes are refused cleanly.
This file is collected last so a failure here comes after every other test."""
import numpy as np
import pytest
import torch

from rans_decode_gemm_b200 import ans
from rans_decode_gemm_b200 import workloads as WL

from _gpu_util import make_case, rel_fro, run_gemm, status_tensor, x_dev

pytestmark = pytest.mark.gpu

TOL = 1e-3  # the relative Frobenius bar the GEMM parity tests use


def _scales(d):
    if d["scales"] is None:
        return None
    s = np.ascontiguousarray(d["scales"])
    return torch.from_numpy(s.view(np.int16) if s.dtype == np.uint16 else s).cuda()


@pytest.mark.parametrize("state_bits", [32, 64])
@pytest.mark.parametrize("name,N,K,M", [("bf16_4096", 1024, 4096, 16),
                                        ("fp8_405b", 256, 2048, 5),
                                        ("int4_70b", 512, 1024, 40)])
def test_noalloc_matches_workspace_entry_point(cuda, name, N, K, M, state_bits):
    cfg, d, lay, layer = make_case(name, N, K, state_bits=state_bits)
    X = WL.make_x(cfg, M, K)
    Y_ref, st_ref, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    assert st_ref == 0
    dX = x_dev(X)
    sc = _scales(d)
    for call in range(2):  # the shared scratch keeps the previous call's contents
        Y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        st = status_tensor()
        ans.ans_gemm_noalloc(dX, M, layer.tiles, cfg.scale_kind, sc, cfg.group_k, Y, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0, call
        err = rel_fro(Y.cpu().numpy(), Y_ref.cpu().numpy().astype(np.float64))
        assert err <= TOL, (call, err)
        assert torch.equal(Y, Y_ref), call   # same kernel and schedule: bit-identical


def test_noalloc_refuses_oversize_shape(cuda):
    cfg, d, lay, layer = make_case("bf16_4096", 4096, 4096)
    M = 2048        # the decoded copy of W for the dense GEMM alone is 32 MiB
    assert ans.ans_gemm_workspace(lay, M, 0) > 16 << 20
    X = torch.zeros(M, 4096, dtype=torch.int16, device="cuda")
    Y = torch.zeros(M, 4096, dtype=torch.float32, device="cuda")
    with pytest.raises(ans.AnsError) as e:
        ans.ans_gemm_noalloc(X, M, layer.tiles, 0, None, 0, Y, status_tensor())
    assert e.value.status == 4
    assert "scratch" in str(e.value)


def test_noalloc_after_a_flagged_call_and_beside_a_refused_one(cuda):
    # a call on a corrupt stream (its status says so) leaves nothing behind that
    # spoils the next call; a call refused for a bad argument while a valid one
    # is still running queues nothing, so the valid call's result stands
    cfg, d, lay, layer = make_case("bf16_4096", 1024, 4096)
    M = 16
    X = WL.make_x(cfg, M, 4096)
    Y_ref, st_ref, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    assert st_ref == 0
    dX = x_dev(X)
    bad = layer.h_stream.copy()
    bad[200] ^= 0x10
    broken = ans.CompressedLayer(lay, layer.codebook, bad, layer.h_offsets, layer.h_raw)
    Y = torch.zeros(M, 1024, dtype=torch.float32, device="cuda")
    st = status_tensor()
    ans.ans_gemm_noalloc(dX, M, broken.tiles, 0, None, 0, Y, st)
    torch.cuda.synchronize()
    assert int(st.item()) & ans.STATUS_CORRUPT
    Y = torch.full((M, 1024), float("nan"), dtype=torch.float32, device="cuda")
    st = status_tensor()
    ans.ans_gemm_noalloc(dX, M, layer.tiles, 0, None, 0, Y, st)
    with pytest.raises(ans.AnsError) as e:            # no status word: refused
        ans.ans_gemm_noalloc(dX, M, layer.tiles, 0, None, 0, Y, None)
    assert e.value.status == 1
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(Y, Y_ref)


def test_noalloc_large_m_within_the_scratch(cuda):
    # a call above one token pass whose workspace (the decoded copy of W
    # included) fits the fixed scratch runs there, same result as ans_gemm
    cfg, d, lay, layer = make_case("bf16_4096", 1024, 4096)
    M = 700
    assert ans.ans_gemm_workspace(lay, M, 0) <= 16 << 20
    X = WL.make_x(cfg, M, 4096)
    Y_ref, st_ref, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    assert st_ref == 0
    Y = torch.full((M, 1024), float("nan"), dtype=torch.float32, device="cuda")
    st = status_tensor()
    ans.ans_gemm_noalloc(x_dev(X), M, layer.tiles, 0, None, 0, Y, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(Y, Y_ref)
