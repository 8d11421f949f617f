"""GPU parity of the wide-state stream variant (64-bit lane states, 32-bit
words, one renormalisation test per pair of symbols): the standalone decode is
bit-exact and agrees with the oracle's decode of the same stream, and the
fused GEMM is bit-identical to the uncompressed variant (hence to the default
format's result) and within 1e-3 relative Frobenius error of the fp64 oracle,
in both schedules."""
import numpy as np
import pytest
import torch

from rans_decode_gemm_b200 import ans
from rans_decode_gemm_b200 import workloads as WL

from _gpu_util import make_case, rel_fro, run_gemm, status_tensor

pytestmark = pytest.mark.gpu

TOL = 1e-3
SMALL = [("tiny_int4", 512, 512), ("bf16_4096", 512, 1024), ("bf16_4096", 1024, 4096),
         ("llama8b_mlp", 384, 2048), ("int4_70b", 512, 1024), ("fp8_405b", 256, 2048)]


@pytest.fixture(scope="module")
def cases():
    return {}


def _case(cases, name, N, K):
    key = (name, N, K)
    if key not in cases:
        cases[key] = make_case(name, N, K, state_bits=64)
    return cases[key]


def _decode(layer, lay):
    nbytes = lay.N * lay.K // 2 if lay.dtype == ans.INT4 else lay.N * lay.K * (2 if lay.dtype == ans.BF16_SPLIT else 1)
    out = torch.full((nbytes,), 0xA5, dtype=torch.uint8, device="cuda")
    st = status_tensor()
    ans.ans_decode_tiles(layer.tiles, out, st)
    torch.cuda.synchronize()
    return out.cpu().numpy(), int(st.item())


def _bytes(w):
    return np.ascontiguousarray(w).view(np.uint8).reshape(-1)


@pytest.mark.parametrize("name,N,K", SMALL)
def test_wide_decode_bit_exact(cuda, oracle, cases, name, N, K):
    cfg, d, lay, layer = _case(cases, name, N, K)
    assert lay.state_bits == 64
    out, st = _decode(layer, lay)
    assert st == 0
    assert np.array_equal(out, _bytes(d["w"]))
    sto, ref = oracle.decode(cfg.dtype, layer.h_stream, layer.h_offsets, layer.h_raw, N, K,
                             cfg.tile_n, cfg.tile_k, layer.codebook.freq_array(), state_bits=64)
    assert sto == 0 and np.array_equal(out, _bytes(ref))


@pytest.mark.parametrize("name", ["bf16_4096", "int4_70b"])
def test_wide_decode_full_size(cuda, cases, name):
    cfg, d, lay, layer = _case(cases, name, None, None)
    out, st = _decode(layer, lay)
    assert st == 0 and np.array_equal(out, _bytes(d["w"]))


def test_wide_single_symbol_layer(cuda, oracle):
    N, K = 256, 128
    w = np.full(N * K, 0x41, np.uint8)
    lay = ans.make_layout(ans.FP8_E4M3, N, K, 128, 64, 64)
    layer = ans.CompressedLayer.from_weights(w, lay, device="cuda")
    # each tile is its state block: a zero length table (8 bytes), 32 states
    # 2^32 in 5 bytes each, 8 bytes of padding
    assert list(layer.h_offsets) == [0, 176, 352, 528, 704]
    out, st = _decode(layer, lay)
    assert st == 0 and np.array_equal(out, w)
    X = WL.make_x(WL.CONFIGS["bf16_4096"], 16, K)
    cfg = type("Cfg", (), {"scale_kind": 0, "group_k": 0, "dtype": ans.FP8_E4M3})()
    dd = {"w": w, "scales": None}
    Y, st, _ = run_gemm(cfg, dd, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, dd, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0 and torch.equal(Y, Yu)


def test_wide_corrupt_stream_is_flagged(cuda, cases):
    cfg, d, lay, layer = _case(cases, "bf16_4096", 512, 1024)
    rng = np.random.default_rng(19)
    flagged = 0
    for trial in range(8):
        bad = layer.h_stream.copy()
        for _ in range(4):
            pos = int(rng.integers(0, bad.size))
            bad[pos] ^= np.uint8(1 << int(rng.integers(0, 8)))
        broken = ans.CompressedLayer(lay, layer.codebook, bad, layer.h_offsets, layer.h_raw)
        out, st = _decode(broken, lay)
        assert st & ~ans.STATUS_CORRUPT == 0
        if st & ans.STATUS_CORRUPT:
            flagged += 1
        else:
            assert not np.array_equal(out, _bytes(d["w"]))
        X = WL.make_x(cfg, 16, 1024)
        Y, stg, _ = run_gemm(cfg, d, lay, broken, X, compressed=True)
        assert stg & ~ans.STATUS_CORRUPT == 0
    assert flagged >= 6


@pytest.mark.parametrize("name,N,K", SMALL)
@pytest.mark.parametrize("M", [1, 16, 17, 64, 128, 300])
def test_wide_gemm_parity(cuda, oracle, cases, name, N, K, M):
    cfg, d, lay, layer = _case(cases, name, N, K)
    X = WL.make_x(cfg, M, K)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0
    assert torch.equal(Y, Yu), "ans_gemm must be bit-identical to ans_gemm_uncompressed"
    Yref = oracle.gemm(cfg.dtype, X, M, K, d["w"], N, cfg.scale_kind, d["scales"], cfg.group_k)
    assert rel_fro(Y.cpu().numpy(), Yref) <= TOL


@pytest.mark.parametrize("schedule", ["local", "central"])
@pytest.mark.parametrize("ctas,producers", [(8, 16), (3, 7)])
@pytest.mark.parametrize("name,N,K,M", [("bf16_4096", 1024, 2048, 16), ("int4_70b", 512, 2048, 16),
                                        ("fp8_405b", 512, 1024, 32), ("tiny_int4", 512, 512, 1),
                                        ("llama8b_mlp", 384, 2048, 130)])
def test_wide_gemm_schedules_and_long_runs(cuda, oracle, cases, plan_limits, schedule, ctas,
                                           producers, name, N, K, M):
    plan_limits(schedule=schedule, max_ctas=ctas, max_producers=producers)
    cfg, d, lay, layer = _case(cases, name, N, K)
    X = WL.make_x(cfg, M, K)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0 and torch.equal(Y, Yu)
    Yref = oracle.gemm(cfg.dtype, X, M, K, d["w"], N, cfg.scale_kind, d["scales"], cfg.group_k)
    assert rel_fro(Y.cpu().numpy(), Yref) <= TOL


@pytest.mark.parametrize("name,N,K,M", [("bf16_4096", 128, 64, 1), ("int4_70b", 256, 128, 3),
                                        ("fp8_405b", 128, 16384, 5), ("bf16_4096", 4096, 64, 16)])
def test_wide_gemm_minimal_and_extreme_shapes(cuda, oracle, cases, name, N, K, M):
    cfg, d, lay, layer = _case(cases, name, N, K)
    X = WL.make_x(cfg, M, K)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0 and torch.equal(Y, Yu)
    Yref = oracle.gemm(cfg.dtype, X, M, K, d["w"], N, cfg.scale_kind, d["scales"], cfg.group_k)
    assert rel_fro(Y.cpu().numpy(), Yref) <= TOL


@pytest.mark.parametrize("M", [1, 16, 128])
def test_wide_gemm_full_size_bf16_4096(cuda, oracle, cases, M):
    # the benchmarked workload at full size; fp64 check on 256 sampled W rows
    cfg, d, lay, layer = _case(cases, "bf16_4096", None, None)
    X = WL.make_x(cfg, M)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0 and torch.equal(Y, Yu)
    rows = np.random.default_rng(M).choice(lay.N, size=256, replace=False).astype(np.uint32)
    Yref = oracle.gemm(cfg.dtype, X, M, lay.K, d["w"], lay.N, rows=rows)
    assert rel_fro(Y.cpu().numpy()[:, rows], Yref) <= TOL
