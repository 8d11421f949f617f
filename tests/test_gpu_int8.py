"""GPU parity of int8 weights (symbol q + 128, per-row fp32 scale, MMA in f16):
GPU histogram equal to the oracle's, standalone decode bit-exact and equal to
the oracle's decode of the same stream, fused GEMM bit-identical to the
uncompressed variant and within 1e-3 relative Frobenius error of the fp64
oracle, in both schedules and both stream formats.  The batched launch of int8
layers is tested in test_gpu_batched.py."""
import numpy as np
import pytest
import torch

from rans_decode_gemm_b200 import ans
from rans_decode_gemm_b200 import workloads as WL

from _gpu_util import make_case, rel_fro, run_gemm, status_tensor, to_dev

pytestmark = pytest.mark.gpu

TOL = 1e-3
SMALL = [(512, 1024), (256, 4096), (1024, 512)]


@pytest.fixture(scope="module")
def cases():
    return {}


def _case(cases, N, K, state_bits):
    key = (N, K, state_bits)
    if key not in cases:
        cases[key] = make_case("int8_8b", N, K, state_bits=state_bits)
    return cases[key]


def _decode(layer, lay):
    out = torch.full((lay.N * lay.K,), 0xA5, dtype=torch.uint8, device="cuda")
    st = status_tensor()
    ans.ans_decode_tiles(layer.tiles, out, st)
    torch.cuda.synchronize()
    return out.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("N,K", [(512, 1024), (3, 37), (1, 16)])
def test_int8_histogram_gpu(cuda, oracle, N, K):
    w = np.random.default_rng(N + K).integers(0, 256, size=N * K).astype(np.uint8)
    lay = ans.make_layout(ans.INT8, N, K, 128, 64)
    h = torch.zeros(256, dtype=torch.int64, device="cuda")
    ans.ans_histogram(to_dev(w), lay, h)
    torch.cuda.synchronize()
    assert np.array_equal(h.cpu().numpy().astype(np.uint64), oracle.histogram(WL.INT8, w, N * K))


@pytest.mark.parametrize("state_bits", [32, 64])
@pytest.mark.parametrize("N,K", SMALL)
def test_int8_decode_bit_exact(cuda, oracle, cases, N, K, state_bits):
    cfg, d, lay, layer = _case(cases, N, K, state_bits)
    out, st = _decode(layer, lay)
    assert st == 0 and np.array_equal(out, d["w"])
    sto, ref = oracle.decode(WL.INT8, layer.h_stream, layer.h_offsets, None, N, K, cfg.tile_n,
                             cfg.tile_k, layer.codebook.freq_array(), state_bits=state_bits)
    assert sto == 0 and np.array_equal(out, ref)


@pytest.mark.parametrize("state_bits", [32, 64])
@pytest.mark.parametrize("N,K", SMALL)
@pytest.mark.parametrize("M", [1, 16, 17, 64, 128, 300])
def test_int8_gemm_parity(cuda, oracle, cases, N, K, M, state_bits):
    cfg, d, lay, layer = _case(cases, N, K, state_bits)
    X = WL.make_x(cfg, M, K)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0
    assert torch.equal(Y, Yu), "ans_gemm must be bit-identical to ans_gemm_uncompressed"
    Yref = oracle.gemm(WL.INT8, X, M, K, d["w"], N, cfg.scale_kind, d["scales"])
    assert rel_fro(Y.cpu().numpy(), Yref) <= TOL


@pytest.mark.parametrize("schedule", ["local", "central"])
@pytest.mark.parametrize("ctas,producers", [(8, 16), (3, 7)])
def test_int8_gemm_schedules(cuda, oracle, cases, plan_limits, schedule, ctas, producers):
    plan_limits(schedule=schedule, max_ctas=ctas, max_producers=producers)
    for state_bits in (32, 64):
        cfg, d, lay, layer = _case(cases, 512, 1024, state_bits)
        X = WL.make_x(cfg, 16, 1024)
        Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
        Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
        assert st == 0 and stu == 0 and torch.equal(Y, Yu)
        Yref = oracle.gemm(WL.INT8, X, 16, 1024, d["w"], 512, cfg.scale_kind, d["scales"])
        assert rel_fro(Y.cpu().numpy(), Yref) <= TOL


def test_int8_extreme_codes_exact(cuda, oracle):
    # every code including -128 and 127, unit scales, small-integer X: exact
    N, K = 128, 256
    q = (np.arange(N * K) % 256).astype(np.uint8)
    lay = ans.make_layout(ans.INT8, N, K, 128, 64, 64)
    layer = ans.CompressedLayer.from_weights(q, lay, device="cuda")
    xi = np.random.default_rng(3).integers(-4, 5, size=(16, K)).astype(np.float32)
    X = WL.to_bf16_bits(xi)
    cfg = type("Cfg", (), {"scale_kind": 0, "group_k": 0, "dtype": ans.INT8})()
    Y, st, _ = run_gemm(cfg, {"w": q, "scales": None}, lay, layer, X, compressed=True)
    assert st == 0
    Yref = oracle.gemm(WL.INT8, X, 16, K, q, N)
    assert np.array_equal(Y.cpu().numpy().astype(np.float64), Yref)


@pytest.mark.parametrize("M", [1, 16])
def test_int8_gemm_full_size(cuda, oracle, cases, M):
    cfg, d, lay, layer = _case(cases, None, None, 64)
    X = WL.make_x(cfg, M)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0 and torch.equal(Y, Yu)
    rows = np.random.default_rng(M).choice(lay.N, size=256, replace=False).astype(np.uint32)
    Yref = oracle.gemm(WL.INT8, X, M, lay.K, d["w"], lay.N, cfg.scale_kind, d["scales"], rows=rows)
    assert rel_fro(Y.cpu().numpy()[:, rows], Yref) <= TOL
    out, st = _decode(layer, lay)
    assert st == 0 and np.array_equal(out, d["w"])
