"""GPU parity of int4 weights coded as pair symbols (one symbol per packed
byte, two consecutive K elements; half as many decode steps per tile): the GPU
histogram equals the oracle's, the standalone decode is bit-exact and agrees
with the oracle's decode of the same stream, and the fused GEMM is
bit-identical to the uncompressed variant and to the per-element coding of the
same weights, and within 1e-3 relative Frobenius error of the fp64 oracle, in
both schedules and both stream formats."""
import numpy as np
import pytest
import torch

from rans_decode_gemm_b200 import ans
from rans_decode_gemm_b200 import workloads as WL

from _gpu_util import make_case, rel_fro, run_gemm, status_tensor, to_dev

pytestmark = pytest.mark.gpu

TOL = 1e-3
SMALL = [("tiny_int4", 512, 512), ("int4_70b", 512, 1024), ("int4_70b", 1024, 2048)]


@pytest.fixture(scope="module")
def cases():
    return {}


def _case(cases, name, N, K, state_bits, dtype=ans.INT4_PAIRS):
    key = (name, N, K, state_bits, dtype)
    if key not in cases:
        cases[key] = make_case(name, N, K, state_bits=state_bits, dtype=dtype)
    return cases[key]


def _decode(layer, lay):
    out = torch.full((lay.N * lay.K // 2,), 0xA5, dtype=torch.uint8, device="cuda")
    st = status_tensor()
    ans.ans_decode_tiles(layer.tiles, out, st)
    torch.cuda.synchronize()
    return out.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("N,K", [(512, 512), (3, 22), (1, 2), (7, 4096)])
def test_pairs_histogram_gpu(cuda, oracle, N, K):
    # includes byte counts that leave a ragged tail after the 16-byte body
    cfg = WL.CONFIGS["int4_70b"]
    rng = np.random.default_rng(N * 7 + K)
    codes = np.clip(np.rint(rng.laplace(0, 0.9, size=(N, K))), -8, 7).astype(np.int8)
    w = WL.pack_int4(codes)
    lay = ans.make_layout(ans.INT4_PAIRS, N, K, cfg.tile_n, cfg.tile_k)
    h = torch.zeros(256, dtype=torch.int64, device="cuda")
    ans.ans_histogram(to_dev(w), lay, h)
    torch.cuda.synchronize()
    ref = oracle.histogram(WL.INT4_PAIRS, w, N * K)
    assert np.array_equal(h.cpu().numpy().astype(np.uint64), ref)


@pytest.mark.parametrize("state_bits", [32, 64])
@pytest.mark.parametrize("name,N,K", SMALL)
def test_pairs_decode_bit_exact(cuda, oracle, cases, name, N, K, state_bits):
    cfg, d, lay, layer = _case(cases, name, N, K, state_bits)
    out, st = _decode(layer, lay)
    assert st == 0
    assert np.array_equal(out, d["w"])
    sto, ref = oracle.decode(WL.INT4_PAIRS, layer.h_stream, layer.h_offsets, None, N, K,
                             cfg.tile_n, cfg.tile_k, layer.codebook.freq_array(),
                             state_bits=state_bits)
    assert sto == 0 and np.array_equal(out, ref)


def test_pairs_stream_matches_oracle_encoder(cuda, oracle, cases):
    # the library's host encoder and the oracle's write the same bytes
    for state_bits in (32, 64):
        cfg, d, lay, layer = _case(cases, "int4_70b", 512, 1024, state_bits)
        st, stream, offsets, _ = oracle.encode(WL.INT4_PAIRS, d["w"], 512, 1024, cfg.tile_n,
                                               cfg.tile_k, layer.codebook.freq_array(),
                                               state_bits=state_bits)
        assert st == 0
        assert np.array_equal(stream, layer.h_stream) and np.array_equal(offsets, layer.h_offsets)


def test_pairs_decode_full_size(cuda, cases):
    cfg, d, lay, layer = _case(cases, "int4_70b", None, None, 64)
    out, st = _decode(layer, lay)
    assert st == 0 and np.array_equal(out, d["w"])


def test_pairs_single_symbol_layer(cuda):
    # every packed byte 0x88 (codes -8, -8): one pair symbol with f = 4096
    N, K = 256, 128
    w = np.full(N * K // 2, 0x88, np.uint8)
    for state_bits in (32, 64):
        lay = ans.make_layout(ans.INT4_PAIRS, N, K, 128, 64, state_bits)
        layer = ans.CompressedLayer.from_weights(w, lay, device="cuda")
        out, st = _decode(layer, lay)
        assert st == 0 and np.array_equal(out, w)
        X = WL.make_x(WL.CONFIGS["int4_70b"], 16, K)
        cfg = type("Cfg", (), {"scale_kind": 0, "group_k": 0, "dtype": ans.INT4})()
        dd = {"w": w, "scales": None}
        Y, st, _ = run_gemm(cfg, dd, lay, layer, X, compressed=True)
        Yu, stu, _ = run_gemm(cfg, dd, lay, layer, X, compressed=False)
        assert st == 0 and stu == 0 and torch.equal(Y, Yu)
        xs = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).double().sum(dim=1)
        assert torch.allclose(Y.double().cpu(), (-8.0 * xs)[:, None].expand(16, N), rtol=1e-5, atol=1e-3)


def test_pairs_corrupt_stream_is_flagged(cuda, cases):
    cfg, d, lay, layer = _case(cases, "int4_70b", 512, 1024, 32)
    rng = np.random.default_rng(23)
    flagged = 0
    for trial in range(8):
        bad = layer.h_stream.copy()
        for _ in range(4):
            pos = int(rng.integers(0, bad.size))
            bad[pos] ^= np.uint8(1 << int(rng.integers(0, 8)))
        broken = ans.CompressedLayer(lay, layer.codebook, bad, layer.h_offsets, None)
        out, st = _decode(broken, lay)
        assert st & ~ans.STATUS_CORRUPT == 0
        if st & ans.STATUS_CORRUPT:
            flagged += 1
        else:
            assert not np.array_equal(out, d["w"])
        X = WL.make_x(cfg, 16, 1024)
        Y, stg, _ = run_gemm(cfg, d, lay, broken, X, compressed=True)
        assert stg & ~ans.STATUS_CORRUPT == 0
    assert flagged >= 6


@pytest.mark.parametrize("state_bits", [32, 64])
@pytest.mark.parametrize("name,N,K", SMALL)
@pytest.mark.parametrize("M", [1, 16, 17, 24, 32, 64, 128, 300])
def test_pairs_gemm_parity(cuda, oracle, cases, name, N, K, M, state_bits):
    cfg, d, lay, layer = _case(cases, name, N, K, state_bits)
    X = WL.make_x(cfg, M, K)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0
    assert torch.equal(Y, Yu), "ans_gemm must be bit-identical to ans_gemm_uncompressed"
    # the per-element coding of the same weights fills the same slabs: the
    # same result, bit for bit where both codings get the same schedule (on
    # 256-row tiles at 17-32 tokens pair symbols take the small-M schedule,
    # whose order of additions differs)
    _, _, lay1, layer1 = _case(cases, name, N, K, state_bits, dtype=ans.INT4)
    Y1, st1, _ = run_gemm(cfg, d, lay1, layer1, X, compressed=True)
    assert st1 == 0
    if lay.tile_n == 256 and 17 <= M <= 32:
        assert rel_fro(Y.cpu().numpy(), Y1.cpu().numpy().astype(np.float64)) <= 1e-5
    else:
        assert torch.equal(Y, Y1)
    Yref = oracle.gemm(WL.INT4, X, M, K, d["w"], N, cfg.scale_kind, d["scales"], cfg.group_k)
    assert rel_fro(Y.cpu().numpy(), Yref) <= TOL


@pytest.mark.parametrize("schedule", ["local", "central"])
@pytest.mark.parametrize("ctas,producers", [(8, 16), (3, 7)])
@pytest.mark.parametrize("name,N,K,M", [("int4_70b", 512, 2048, 16), ("tiny_int4", 512, 512, 1),
                                        ("int4_70b", 1024, 1024, 130), ("int4_70b", 512, 2048, 32),
                                        ("int4_70b", 512, 2048, 21)])
def test_pairs_gemm_schedules_and_long_runs(cuda, oracle, cases, plan_limits, schedule, ctas,
                                            producers, name, N, K, M):
    plan_limits(schedule=schedule, max_ctas=ctas, max_producers=producers)
    for state_bits in (32, 64):
        cfg, d, lay, layer = _case(cases, name, N, K, state_bits)
        X = WL.make_x(cfg, M, K)
        Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
        Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
        assert st == 0 and stu == 0 and torch.equal(Y, Yu)
        Yref = oracle.gemm(WL.INT4, X, M, K, d["w"], N, cfg.scale_kind, d["scales"], cfg.group_k)
        assert rel_fro(Y.cpu().numpy(), Yref) <= TOL


@pytest.mark.parametrize("name,N,K,M", [("int4_70b", 256, 128, 3), ("tiny_int4", 128, 16384, 5),
                                        ("tiny_int4", 4096, 32, 16)])
def test_pairs_gemm_minimal_and_extreme_shapes(cuda, oracle, cases, name, N, K, M):
    cfg, d, lay, layer = _case(cases, name, N, K, 64)
    X = WL.make_x(cfg, M, K)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0 and torch.equal(Y, Yu)
    Yref = oracle.gemm(WL.INT4, X, M, K, d["w"], N, cfg.scale_kind, d["scales"], cfg.group_k)
    assert rel_fro(Y.cpu().numpy(), Yref) <= TOL


@pytest.mark.parametrize("M", [1, 16])
def test_pairs_gemm_full_size_int4_70b(cuda, oracle, cases, M):
    # the 70B MLP up-projection at full size; fp64 check on 256 sampled W rows
    cfg, d, lay, layer = _case(cases, "int4_70b", None, None, 64)
    X = WL.make_x(cfg, M)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0 and torch.equal(Y, Yu)
    rows = np.random.default_rng(M).choice(lay.N, size=256, replace=False).astype(np.uint32)
    Yref = oracle.gemm(WL.INT4, X, M, lay.K, d["w"], lay.N, cfg.scale_kind, d["scales"],
                       cfg.group_k, rows=rows)
    assert rel_fro(Y.cpu().numpy()[:, rows], Yref) <= TOL
