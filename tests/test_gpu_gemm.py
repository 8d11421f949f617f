"""GPU parity of the fused decode + GEMM (ans_gemm) through the C ABI:
bit-exact against the same kernel fed the uncompressed weights
(ans_gemm_uncompressed), and within a relative Frobenius error of 1e-3 of the
oracle's fp64 GEMM (the bar the method's statement sets; fp32 accumulation
over K <= 16384 lands near 1e-6)."""
import numpy as np
import pytest
import torch

from rans_decode_gemm_b200 import ans
from rans_decode_gemm_b200 import workloads as WL

from _gpu_util import make_case, rel_fro, run_gemm, status_tensor, x_dev

pytestmark = pytest.mark.gpu

TOL = 1e-3

# (config, N, K): small shapes spanning several tiles, split-K over CTAs and
# rounds that cross W row blocks
SMALL = [("tiny_int4", 512, 512), ("bf16_4096", 512, 1024), ("bf16_4096", 1024, 4096),
         ("llama8b_mlp", 384, 2048), ("int4_70b", 512, 1024), ("fp8_405b", 256, 2048)]
MS = [1, 5, 16, 17, 64, 128, 200, 300, 600]


@pytest.fixture(scope="module")
def cases():
    return {}


def _case(cases, name, N, K):
    key = (name, N, K)
    if key not in cases:
        cases[key] = make_case(name, N, K)
    return cases[key]


@pytest.mark.parametrize("name,N,K", SMALL)
@pytest.mark.parametrize("M", MS)
def test_gemm_parity_small(cuda, oracle, cases, name, N, K, M):
    cfg, d, lay, layer = _case(cases, name, N, K)
    X = WL.make_x(cfg, M, K)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0
    assert torch.equal(Y, Yu), "ans_gemm must be bit-identical to ans_gemm_uncompressed"
    Yref = oracle.gemm(cfg.dtype, X, M, K, d["w"], N, cfg.scale_kind, d["scales"], cfg.group_k)
    err = rel_fro(Y.cpu().numpy(), Yref)
    assert err <= TOL, err


@pytest.mark.parametrize("M", [1, 16, 128])
def test_gemm_full_size_bf16_4096(cuda, oracle, cases, M):
    # the benchmarked workload, at full size, in the launch configuration the
    # benchmark times; the fp64 check runs on 256 sampled W rows
    cfg, d, lay, layer = _case(cases, "bf16_4096", None, None)
    X = WL.make_x(cfg, M)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0 and torch.equal(Y, Yu)
    rows = np.random.default_rng(M).choice(lay.N, size=256, replace=False).astype(np.uint32)
    Yref = oracle.gemm(cfg.dtype, X, M, lay.K, d["w"], lay.N, rows=rows)
    assert rel_fro(Y.cpu().numpy()[:, rows], Yref) <= TOL


def test_workspace_reuse_and_determinism(cuda, cases):
    cfg, d, lay, layer = _case(cases, "bf16_4096", 1024, 4096)
    X = WL.make_x(cfg, 16, 4096)
    Y1, st1, ws = run_gemm(cfg, d, lay, layer, X)
    Y2, st2, _ = run_gemm(cfg, d, lay, layer, X, ws=ws)
    Y3, st3, _ = run_gemm(cfg, d, lay, layer, X, ws=ws)
    assert st1 == st2 == st3 == 0
    assert torch.equal(Y1, Y2) and torch.equal(Y1, Y3)
    # split-K counters are back at zero
    nseg = (lay.N // lay.tile_n)
    assert int(ws[:4 * nseg].view(torch.int32).abs().sum().item()) == 0


def test_gemm_argument_errors(cuda, cases):
    cfg, d, lay, layer = _case(cases, "bf16_4096", 512, 1024)
    X = x_dev(WL.make_x(cfg, 4, 1024))
    Y = torch.zeros(4, 512, dtype=torch.float32, device="cuda")
    st = status_tensor()
    need = ans.ans_gemm_workspace(lay, 4, 0)
    small = torch.zeros(max(1, need // 2), dtype=torch.uint8, device="cuda")
    with pytest.raises(ans.AnsError) as e:
        ans.ans_gemm(X, 4, layer.tiles, 0, None, 0, Y, small, small.numel(), st)
    assert e.value.status == 4
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    Xflat = torch.zeros(4 * 1024 + 1, dtype=torch.int16, device="cuda")
    with pytest.raises(ans.AnsError) as e:   # misaligned X
        ans.ans_gemm(Xflat[1:], 4, layer.tiles, 0, None, 0, Y, ws, ws.numel(), st)
    assert e.value.status == 1
    # the raw side stream is fetched with 16-byte bulk copies
    shifted = ans.AnsTiles.from_buffer_copy(layer.tiles)
    shifted.raw = layer.tiles.raw + 8
    with pytest.raises(ans.AnsError) as e:
        ans.ans_gemm(X, 4, shifted, 0, None, 0, Y, ws, ws.numel(), st)
    assert e.value.status == 1
    # M == 0 is a no-op
    ans.ans_gemm(X, 0, layer.tiles, 0, None, 0, Y, ws, ws.numel(), st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0


def test_gemm_corrupt_stream_flags_status(cuda, cases):
    cfg, d, lay, layer = _case(cases, "bf16_4096", 512, 1024)
    bad = layer.h_stream.copy()
    bad[200] ^= 0x10
    bad[5000] ^= 0x01
    broken = ans.CompressedLayer(lay, layer.codebook, bad, layer.h_offsets, layer.h_raw)
    X = WL.make_x(cfg, 16, 1024)
    Y, st, _ = run_gemm(cfg, d, lay, broken, X)
    assert st & ans.STATUS_CORRUPT
    assert not st & ans.STATUS_TIMEOUT


@pytest.mark.parametrize("schedule", ["local", "central"])
@pytest.mark.parametrize("ctas,producers", [(8, 16), (5, 3), (3, 7)])
@pytest.mark.parametrize("name,N,K,M", [("bf16_4096", 1024, 2048, 16), ("int4_70b", 512, 2048, 40),
                                        ("fp8_405b", 512, 1024, 300), ("tiny_int4", 512, 512, 130),
                                        ("int4_70b", 512, 2048, 16), ("fp8_405b", 512, 1024, 32),
                                        ("tiny_int4", 512, 512, 1)])
def test_gemm_multi_round_schedules(cuda, oracle, cases, plan_limits, schedule, ctas, producers,
                                    name, N, K, M):
    # few CTAs and few producer warps: many rounds (shared-accumulator
    # schedule) or long per-warp runs crossing W row blocks (local schedule,
    # M <= 32 only; larger M always takes the shared-accumulator schedule),
    # slab, chunk and X rings wrapping many times
    plan_limits(schedule=schedule, max_ctas=ctas, max_producers=producers)
    cfg, d, lay, layer = _case(cases, name, N, K)
    X = WL.make_x(cfg, M, K)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0 and torch.equal(Y, Yu)
    Yref = oracle.gemm(cfg.dtype, X, M, K, d["w"], N, cfg.scale_kind, d["scales"], cfg.group_k)
    assert rel_fro(Y.cpu().numpy(), Yref) <= TOL


@pytest.mark.parametrize("name,N,K,M", [("bf16_4096", 1024, 4096, 16), ("int4_70b", 512, 2048, 8),
                                        ("fp8_405b", 256, 2048, 32), ("tiny_int4", 512, 512, 1)])
def test_gemm_both_schedules_small_m(cuda, oracle, cases, plan_limits, name, N, K, M):
    # at M <= 32 the local schedule is the default; the shared-accumulator one
    # must agree with the fp64 oracle too (the two add in different orders, so
    # they agree to rounding, not bit for bit)
    cfg, d, lay, layer = _case(cases, name, N, K)
    X = WL.make_x(cfg, M, K)
    Yref = oracle.gemm(cfg.dtype, X, M, K, d["w"], N, cfg.scale_kind, d["scales"], cfg.group_k)
    out = {}
    for schedule in ["local", "central"]:
        plan_limits(schedule=schedule)
        Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
        Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
        assert st == 0 and stu == 0 and torch.equal(Y, Yu), schedule
        assert rel_fro(Y.cpu().numpy(), Yref) <= TOL, schedule
        out[schedule] = Y
    assert rel_fro(out["local"].cpu().numpy(), out["central"].cpu().numpy().astype(np.float64)) <= 1e-5


@pytest.mark.parametrize("schedule", ["local", "central"])
def test_gemm_bad_offsets_flag_status(cuda, cases, plan_limits, schedule):
    # an offset table that points past the stream: the affected tiles are
    # skipped (treated as zero), the status says why, nothing reads outside
    plan_limits(schedule=schedule)
    cfg, d, lay, layer = _case(cases, "bf16_4096", 512, 1024)
    off = layer.h_offsets.copy()
    off[7] = off[-1] + 4096
    broken = ans.CompressedLayer(lay, layer.codebook, layer.h_stream, off, layer.h_raw)
    X = WL.make_x(cfg, 16, 1024)
    Y, st, _ = run_gemm(cfg, d, lay, broken, X)
    assert st & ans.STATUS_BAD_OFFSETS
    assert not st & ans.STATUS_TIMEOUT


@pytest.mark.parametrize("ctas", [3, 7])
@pytest.mark.parametrize("name,N,K,M", [("bf16_4096", 1024, 2048, 16), ("int4_70b", 512, 2048, 16),
                                        ("fp8_405b", 512, 1024, 32), ("tiny_int4", 512, 512, 1),
                                        ("llama8b_mlp", 384, 2048, 5)])
def test_gemm_local_long_producer_runs(cuda, oracle, cases, plan_limits, ctas, name, N, K, M):
    # few CTAs: every producer warp of the local schedule owns a long run of
    # tiles crossing W row blocks (chunk rings wrap many times, several
    # accumulators per producer); bit-identical to the uncompressed variant
    # and within the bar of the fp64 oracle
    plan_limits(max_ctas=ctas)
    cfg, d, lay, layer = _case(cases, name, N, K)
    X = WL.make_x(cfg, M, K)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0 and torch.equal(Y, Yu)
    Yref = oracle.gemm(cfg.dtype, X, M, K, d["w"], N, cfg.scale_kind, d["scales"], cfg.group_k)
    assert rel_fro(Y.cpu().numpy(), Yref) <= TOL


def test_gemm_long_runs_corrupt_and_bad_offsets(cuda, cases, plan_limits):
    # a corrupt or badly indexed tile in the middle of a producer's run
    plan_limits(max_ctas=4)
    cfg, d, lay, layer = _case(cases, "bf16_4096", 512, 1024)
    X = WL.make_x(cfg, 16, 1024)
    bad = layer.h_stream.copy()
    bad[200] ^= 0x10
    broken = ans.CompressedLayer(lay, layer.codebook, bad, layer.h_offsets, layer.h_raw)
    Y, st, _ = run_gemm(cfg, d, lay, broken, X)
    assert st & ans.STATUS_CORRUPT and not st & ans.STATUS_TIMEOUT
    off = layer.h_offsets.copy()
    off[9] = off[-1] + 4096
    broken = ans.CompressedLayer(lay, layer.codebook, layer.h_stream, off, layer.h_raw)
    Y, st, _ = run_gemm(cfg, d, lay, broken, X)
    assert st & ans.STATUS_BAD_OFFSETS and not st & ans.STATUS_TIMEOUT


def _single_symbol_weights(dtype, N, K, rng):
    """Weights whose coded symbol takes one value (a one-symbol codebook):
    int4 all code 3, fp8 all 0x38, bf16 one exponent with random sign and
    mantissa bytes."""
    if dtype == ans.INT4:
        return np.full(N * K // 2, 0x33, np.uint8), WL.to_bf16_bits(rng.uniform(0.005, 0.02, N))
    if dtype == ans.FP8_E4M3:
        return np.full(N * K, 0x38, np.uint8), rng.uniform(0.5, 2.0, N).astype(np.float32)
    raw = rng.integers(0, 256, N * K).astype(np.uint16)
    bits = ((raw & 0x80) << 8) | (np.uint16(0x7A) << 7) | (raw & 0x7F)
    return bits.astype(np.uint16), None


@pytest.mark.parametrize("dtype", [ans.INT4, ans.FP8_E4M3, ans.BF16_SPLIT])
@pytest.mark.parametrize("M", [1, 40])
def test_gemm_single_symbol_codebook(cuda, oracle, dtype, M):
    # every tile is a run of one symbol: the producers take their constant
    # path (no stream reads past the lane states) in both schedules
    rng = np.random.default_rng(11)
    N, K = 256, 512
    tile_n, tile_k = (128, 64)
    w, scales = _single_symbol_weights(dtype, N, K, rng)
    lay = ans.make_layout(dtype, N, K, tile_n, tile_k)
    layer = ans.CompressedLayer.from_weights(w, lay, device="cuda")
    assert (layer.codebook.freq_array() == 4096).sum() == 1
    scale_kind = {ans.INT4: ans.SCALE_ROW_BF16, ans.FP8_E4M3: ans.SCALE_ROW_F32, ans.BF16_SPLIT: 0}[dtype]
    cfg = type("Cfg", (), {"scale_kind": scale_kind, "group_k": 0, "dtype": dtype})()
    d = {"w": w, "scales": scales}
    X = WL.make_x(WL.CONFIGS["bf16_4096"], M, K)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0 and torch.equal(Y, Yu)
    Yref = oracle.gemm(dtype, X, M, K, w, N, scale_kind, scales, 0)
    assert rel_fro(Y.cpu().numpy(), Yref) <= TOL


@pytest.mark.parametrize("name,N,K,M", [("bf16_4096", 128, 64, 1), ("int4_70b", 256, 128, 3),
                                        ("fp8_405b", 128, 128, 17), ("tiny_int4", 128, 32, 1),
                                        ("bf16_4096", 4096, 64, 16), ("fp8_405b", 128, 16384, 5)])
def test_gemm_minimal_and_extreme_shapes(cuda, oracle, cases, name, N, K, M):
    # one tile; one K tile with many row blocks (every segment one unit);
    # one row block with many K tiles (one segment split over every CTA)
    cfg, d, lay, layer = _case(cases, name, N, K)
    X = WL.make_x(cfg, M, K)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0 and torch.equal(Y, Yu)
    Yref = oracle.gemm(cfg.dtype, X, M, K, d["w"], N, cfg.scale_kind, d["scales"], cfg.group_k)
    assert rel_fro(Y.cpu().numpy(), Yref) <= TOL


@pytest.mark.parametrize("name,M", [("int4_70b", 16), ("fp8_405b", 16)])
def test_gemm_full_size_large_layers_sampled(cuda, oracle, cases, name, M):
    # the largest workloads at full size in the launch configuration the
    # sweep times; the fp64 check runs on 256 sampled W rows, bit-identity
    # with the uncompressed variant on all of Y
    cfg, d, lay, layer = _case(cases, name, None, None)
    X = WL.make_x(cfg, M)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0 and torch.equal(Y, Yu)
    rows = np.random.default_rng(M).choice(lay.N, size=256, replace=False).astype(np.uint32)
    Yref = oracle.gemm(cfg.dtype, X, M, lay.K, d["w"], lay.N, cfg.scale_kind, d["scales"],
                       cfg.group_k, rows=rows)
    assert rel_fro(Y.cpu().numpy()[:, rows], Yref) <= TOL


@pytest.mark.parametrize("name,M,dtype", [("fp8_405b", 2048, None), ("fp8_405b", 256, None),
                                          ("int4_70b", 1024, ans.INT4_PAIRS),
                                          ("int4_70b", 1024, None), ("llama8b_mlp", 512, None)])
def test_gemm_full_size_large_m_sampled(cuda, oracle, name, M, dtype):
    # large token counts at full size, in the launch configuration the sweep
    # times (several token passes of the shared-accumulator schedule for the
    # 405B-shaped layer at M = 2048 and the 70B-shaped one at M = 1024):
    # bit-identical to the uncompressed variant on all of Y, and within the
    # bar of the fp64 oracle on 256 sampled W rows
    cfg, d, lay, layer = make_case(name, state_bits=64, dtype=dtype)
    X = WL.make_x(cfg, M)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0 and torch.equal(Y, Yu)
    rows = np.random.default_rng(M + 7).choice(lay.N, size=256, replace=False).astype(np.uint32)
    Yref = oracle.gemm(cfg.dtype, X, M, lay.K, d["w"], lay.N, cfg.scale_kind, d["scales"],
                       cfg.group_k, rows=rows)
    assert rel_fro(Y.cpu().numpy()[:, rows], Yref) <= TOL


@pytest.mark.parametrize("name,N,K,M", [("bf16_4096", 512, 1024, 513), ("bf16_4096", 512, 1024, 812),
                                        ("fp8_405b", 256, 2048, 1100), ("int4_70b", 512, 1024, 257),
                                        ("int8_8b", 384, 1024, 700), ("fp4_8b", 384, 1024, 530),
                                        ("tiny_int4", 512, 512, 600), ("tiny_int4", 128, 96, 600)])
def test_gemm_large_m_dense_path_edges(cuda, oracle, cases, name, N, K, M):
    # more tokens than one pass: the first pass fused, the rest through the
    # dense GEMM on the decoded weights -- a single token left over (one row
    # of X in the dense kernel's box), two token blocks with a ragged second,
    # every coded format and scale kind (row bf16: the tiny int4 layer); K not
    # a multiple of 64 keeps every pass fused
    cfg, d, lay, layer = _case(cases, name, N, K)
    X = WL.make_x(cfg, M, K)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0
    assert torch.equal(Y, Yu), "ans_gemm must be bit-identical to ans_gemm_uncompressed"
    Yref = oracle.gemm(cfg.dtype, X, M, K, d["w"], N, cfg.scale_kind, d["scales"], cfg.group_k)
    assert rel_fro(Y.cpu().numpy(), Yref) <= TOL


@pytest.mark.parametrize("dtype", [ans.INT4_PAIRS, ans.FP4_PAIRS])
def test_gemm_large_m_pair_symbols(cuda, oracle, dtype):
    # pair-symbol layouts store the same decoded weights as per-element ones
    name = "int4_70b" if dtype == ans.INT4_PAIRS else "fp4_8b"
    cfg, d, lay, layer = make_case(name, 512, 1024, state_bits=64, dtype=dtype)
    M = 700
    X = WL.make_x(cfg, M, 1024)
    Y, st, _ = run_gemm(cfg, d, lay, layer, X, compressed=True)
    Yu, stu, _ = run_gemm(cfg, d, lay, layer, X, compressed=False)
    assert st == 0 and stu == 0 and torch.equal(Y, Yu)
    Yref = oracle.gemm(cfg.dtype, X, M, 1024, d["w"], 512, cfg.scale_kind, d["scales"], cfg.group_k)
    assert rel_fro(Y.cpu().numpy(), Yref) <= TOL
