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


@pytest.mark.parametrize("name,N,K,M", [("bf16_4096", 1024, 4096, 16),
                                        ("fp8_405b", 256, 2048, 5),
                                        ("int4_70b", 512, 1024, 40)])
def test_noalloc_matches_workspace_entry_point(cuda, name, N, K, M):
    cfg, d, lay, layer = make_case(name, N, K)
    X = WL.make_x(cfg, M, K)
    Y_ref, st_ref, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    assert st_ref == 0
    dX = x_dev(X)
    sc = None
    if d["scales"] is not None:
        s = np.ascontiguousarray(d["scales"])
        sc = torch.from_numpy(s.view(np.int16) if s.dtype == np.uint16 else s).cuda()
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
    cfg, d, lay, layer = make_case("bf16_4096", 1024, 4096)
    M = 2048                                  # needs far more than the 16 MiB scratch
    assert ans.ans_gemm_workspace(lay, M, 0) > 16 << 20
    X = torch.zeros(M, 4096, dtype=torch.int16, device="cuda")
    Y = torch.zeros(M, 1024, dtype=torch.float32, device="cuda")
    with pytest.raises(ans.AnsError) as e:
        ans.ans_gemm_noalloc(X, M, layer.tiles, 0, None, 0, Y, status_tensor())
    assert e.value.status == 4
    assert "scratch" in str(e.value)
