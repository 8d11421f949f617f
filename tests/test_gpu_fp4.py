"""GPU parity of fp4 e2m1 weights (per-row fp32 scale, MMA in bf16), coded one
symbol per code or one per packed byte (pair symbols): GPU histogram equal to
the oracle's, standalone decode bit-exact and equal to the oracle's decode of
the same stream, fused GEMM bit-identical to the uncompressed variant (and,
for pair symbols, to the per-code coding) and within 1e-3 relative Frobenius
error of the fp64 oracle, in both schedules and both stream formats.  The
batched launch of fp4 layers is tested in test_gpu_batched.py."""
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


def _case(cases, N, K, state_bits, dtype=ans.FP4_E2M1):
    key = (N, K, state_bits, dtype)
    if key not in cases:
        cases[key] = make_case("fp4_8b", N, K, state_bits=state_bits, dtype=dtype)
    return cases[key]


def _decode(layer, lay):
    out = torch.full((lay.N * lay.K // 2,), 0xA5, dtype=torch.uint8, device="cuda")
    st = status_tensor()
    ans.ans_decode_tiles(layer.tiles, out, st)
    torch.cuda.synchronize()
    return out.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("dtype", [ans.FP4_E2M1, ans.FP4_PAIRS])
@pytest.mark.parametrize("N,K", [(512, 1024), (3, 38), (1, 16)])
def test_fp4_histogram_gpu(cuda, oracle, N, K, dtype):
    w = np.random.default_rng(N + K).integers(0, 256, size=N * K // 2).astype(np.uint8)
    lay = ans.make_layout(dtype, N, K, 128, 64)
    h = torch.zeros(ans.ALPHABET[dtype], dtype=torch.int64, device="cuda")
    ans.ans_histogram(to_dev(w), lay, h)
    torch.cuda.synchronize()
    assert np.array_equal(h.cpu().numpy().astype(np.uint64), oracle.histogram(dtype, w, N * K))


@pytest.mark.parametrize("dtype", [ans.FP4_E2M1, ans.FP4_PAIRS])
@pytest.mark.parametrize("state_bits", [32, 64])
@pytest.mark.parametrize("N,K", SMALL)
def test_fp4_decode_bit_exact(cuda, oracle, cases, N, K, state_bits, dtype):
    cfg, d, lay, layer = _case(cases, N, K, state_bits, dtype)
    out, st = _decode(layer, lay)
    assert st == 0 and np.array_equal(out, d["w"])
    sto, ref = oracle.decode(dtype, layer.h_stream, layer.h_offsets, None, N, K, cfg.tile_n,
                             cfg.tile_k, layer.codebook.freq_array(), state_bits=state_bits)
    assert sto == 0 and np.array_equal(out, ref)


@pytest.mark.parametrize("dtype", [ans.FP4_E2M1, ans.FP4_PAIRS])
@pytest.mark.parametrize("state_bits", [32, 64])
@pytest.mark.parametrize("N,K", SMALL)
@pytest.mark.parametrize("M", [1, 16, 17, 64, 128, 300])
def test_fp4_gemm_parity(cuda, oracle, cases, N, K, M, state_bits, dtype):
    cfg, d, lay, layer = _case(cases, N, K, state_bits, dtype)
    X = WL.make_x(cfg, M, K)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0
    assert torch.equal(Y, Yu), "ans_gemm must be bit-identical to ans_gemm_uncompressed"
    if dtype == ans.FP4_PAIRS:   # the per-code coding fills the same slabs
        _, _, lay1, layer1 = _case(cases, N, K, state_bits)
        Y1, st1, _ = run_gemm(cfg, d, lay1, layer1, X, compressed=True)
        assert st1 == 0 and torch.equal(Y, Y1)
    Yref = oracle.gemm(WL.FP4_E2M1, X, M, K, d["w"], N, cfg.scale_kind, d["scales"])
    assert rel_fro(Y.cpu().numpy(), Yref) <= TOL


@pytest.mark.parametrize("schedule", ["local", "central"])
@pytest.mark.parametrize("ctas,producers", [(8, 16), (3, 7)])
def test_fp4_gemm_schedules(cuda, oracle, cases, plan_limits, schedule, ctas, producers):
    plan_limits(schedule=schedule, max_ctas=ctas, max_producers=producers)
    for state_bits, dtype in ((32, ans.FP4_E2M1), (64, ans.FP4_E2M1), (64, ans.FP4_PAIRS)):
        cfg, d, lay, layer = _case(cases, 512, 1024, state_bits, dtype)
        X = WL.make_x(cfg, 16, 1024)
        Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
        Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
        assert st == 0 and stu == 0 and torch.equal(Y, Yu)
        Yref = oracle.gemm(WL.FP4_E2M1, X, 16, 1024, d["w"], 512, cfg.scale_kind, d["scales"])
        assert rel_fro(Y.cpu().numpy(), Yref) <= TOL


def test_fp4_every_code_exact(cuda, oracle):
    # every code (including -0), unit scales, small-integer X: exact
    N, K = 128, 256
    codes = (np.arange(N * K) % 16).astype(np.uint8)
    w = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)
    lay = ans.make_layout(ans.FP4_E2M1, N, K, 128, 64, 64)
    layer = ans.CompressedLayer.from_weights(w, lay, device="cuda")
    xi = np.random.default_rng(3).integers(-4, 5, size=(16, K)).astype(np.float32)
    X = WL.to_bf16_bits(xi)
    cfg = type("Cfg", (), {"scale_kind": 0, "group_k": 0, "dtype": ans.FP4_E2M1})()
    Y, st, _ = run_gemm(cfg, {"w": w, "scales": None}, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, {"w": w, "scales": None}, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0 and torch.equal(Y, Yu)
    Yref = oracle.gemm(WL.FP4_E2M1, X, 16, K, w, N)
    assert np.array_equal(Y.cpu().numpy().astype(np.float64), Yref)


@pytest.mark.parametrize("M", [1, 16])
def test_fp4_gemm_full_size(cuda, oracle, cases, M):
    cfg, d, lay, layer = _case(cases, None, None, 64)
    X = WL.make_x(cfg, M)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0 and torch.equal(Y, Yu)
    rows = np.random.default_rng(M).choice(lay.N, size=256, replace=False).astype(np.uint32)
    Yref = oracle.gemm(WL.FP4_E2M1, X, M, lay.K, d["w"], lay.N, cfg.scale_kind, d["scales"], rows=rows)
    assert rel_fro(Y.cpu().numpy()[:, rows], Yref) <= TOL
    out, st = _decode(layer, lay)
    assert st == 0 and np.array_equal(out, d["w"])
