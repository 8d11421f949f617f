"""CPU tests of the launch planner (host code of the fused GEMM): for every
workload, state width, token count and SM count the plan fits the B200's
limits (TMEM columns, shared memory, accumulator slots, CTAs), covers all
tokens, and does not depend on whether the weights arrive compressed (the
condition for ans_gemm and ans_gemm_uncompressed to add in the same order)."""
import ctypes as C

import pytest

from rans_decode_gemm_b200 import ans
from rans_decode_gemm_b200 import workloads as WL

FIELDS = ["local", "grid", "D", "n_slots", "tmem_cols", "smem_bytes", "T", "T_pass", "n_pass",
          "NT", "n_bufs", "fmt", "ab_f16", "H", "C", "x_stages", "n_units", "n_segments",
          "ws_lo", "ws_hi", "dense"]
SMEM_MAX = 232448          # sm_100 per-block dynamic shared memory
FMT = {"bf16": 0, "int4_bf16": 1, "int4_group": 2, "fp8": 3, "int4_pair": 4,
       "int4_pair_group": 5, "int8": 6, "fp4": 7, "fp4_pair": 8}


def _plan(lay, M, kind, decode, sms):
    lib = ans.load()
    fn = lib.ansdev_gemm_plan
    fn.argtypes = [C.c_void_p, C.c_uint32, C.c_uint32, C.c_int, C.c_int, C.c_void_p]
    fn.restype = C.c_int
    out = (C.c_uint32 * 21)()
    r = fn(C.addressof(lay), M, kind, decode, sms, out)
    return r, dict(zip(FIELDS, list(out)))


def _expected_fmt(dtype, kind, decode):
    if dtype == WL.BF16_SPLIT:
        return FMT["bf16"]
    if dtype == WL.FP8_E4M3:
        return FMT["fp8"]
    if dtype == WL.INT8:
        return FMT["int8"]
    if dtype == WL.FP4_E2M1 or (dtype == WL.FP4_PAIRS and not decode):
        return FMT["fp4"]
    if dtype == WL.FP4_PAIRS:
        return FMT["fp4_pair"]
    group = kind == WL.SCALE_GROUP_BF16
    if dtype == WL.INT4_PAIRS and decode:
        return FMT["int4_pair_group"] if group else FMT["int4_pair"]
    return FMT["int4_group"] if group else FMT["int4_bf16"]


CODINGS = [(name, dt) for name, cfg in WL.CONFIGS.items()
           for dt in ([cfg.dtype] + ([WL.INT4_PAIRS] if cfg.dtype == WL.INT4 else [])
                      + ([WL.FP4_PAIRS] if cfg.dtype == WL.FP4_E2M1 else []))]


@pytest.mark.parametrize("name,dtype", CODINGS)
@pytest.mark.parametrize("state_bits", [32, 64])
def test_plans_fit_and_cover(ans_lib, name, dtype, state_bits):
    cfg = WL.CONFIGS[name]
    N, K = cfg.matrices[0][1] or cfg.N, cfg.matrices[0][2] or cfg.K
    lay = ans.make_layout(dtype, N, K, cfg.tile_n, cfg.tile_k, state_bits)
    n_tiles = (N // cfg.tile_n) * (K // cfg.tile_k)
    H = cfg.tile_n // 128
    for M in sorted(set(cfg.Ms + [1, 15, 17, 32, 33, 300, 1024])):
        for sms in (148, 74, 18, 1):
            r, p = _plan(lay, M, cfg.scale_kind, 1, sms)
            assert r == 1, (M, sms)
            ru, pu = _plan(lay, M, cfg.scale_kind, 0, sms)
            assert ru == 1
            # the schedule does not depend on whether the weights are compressed;
            # the shared-accumulator schedule's copy variant lays out shared
            # memory without the slot table and chunk rings (a deeper X ring),
            # which does not change the order of the additions
            layout = {"fmt"} | (set() if p["local"] else {"smem_bytes", "x_stages"})
            # more tokens than one pass: a fused first pass of 16 tokens on
            # the small-M schedule, then the dense GEMM; the workspace holds
            # the decoded (or formatted) weights for both variants
            # (unless the first pass does not fit the small-M schedule, on a
            # device of very few SMs)
            assert p["dense"] == 0 or (M > 512 // H and K % 64 == 0)
            if sms >= 18:
                assert p["dense"] == (1 if M > 512 // H and K % 64 == 0 else 0)
            assert {k: v for k, v in p.items() if k not in layout} == \
                   {k: v for k, v in pu.items() if k not in layout}, (M, sms)
            assert p["fmt"] == _expected_fmt(dtype, cfg.scale_kind, True)
            assert pu["fmt"] == _expected_fmt(dtype, cfg.scale_kind, False)
            assert p["ab_f16"] == (1 if p["fmt"] in (2, 3, 5, 6) else 0)
            assert p["H"] == H and p["C"] == cfg.tile_k // 16
            assert 1 <= p["grid"] <= sms
            assert p["smem_bytes"] <= SMEM_MAX
            tc = p["tmem_cols"]
            assert 32 <= tc <= 512 and tc & (tc - 1) == 0
            assert p["T_pass"] * p["n_pass"] >= M
            if p["dense"]:
                assert p["local"] == 1 and p["T"] == 16 and p["T_pass"] == 512 // H
                assert p["n_units"] == n_tiles and p["n_segments"] == N // cfg.tile_n
                assert p["D"] <= 15 and p["n_slots"] * H * 16 <= tc
                assert p["ws_lo"] + (p["ws_hi"] << 32) >= 2 * N * K   # W16
            elif p["local"]:
                T = (M + 15) // 16 * 16
                pair = dtype in (WL.INT4_PAIRS, WL.FP4_PAIRS)
                assert p["T"] == T and p["n_pass"] == 1
                assert H * T <= 32 or (pair and T <= 32 and H * T <= 64)
                assert 1 <= p["D"] <= 15 and 1 <= p["n_slots"] <= 32
                assert p["n_slots"] * H * T <= tc
                assert p["n_units"] == n_tiles and p["n_segments"] == N // cfg.tile_n
            else:
                assert 1 <= p["D"] <= 14 and p["n_bufs"] in (1, 2)
                # X stages: enough to cover the TMA latency of the X slabs
                assert p["x_stages"] >= 3 and pu["x_stages"] >= p["x_stages"]
                assert pu["smem_bytes"] <= SMEM_MAX
                assert p["n_bufs"] * H * p["T_pass"] <= tc <= 512
                assert p["n_units"] == n_tiles * p["n_pass"]
                assert p["n_segments"] == (N // cfg.tile_n) * p["n_pass"]
            assert p["ws_lo"] + (p["ws_hi"] << 32) > 0


def test_small_m_takes_the_local_schedule(ans_lib):
    lay = ans.make_layout(WL.BF16_SPLIT, 4096, 4096, 128, 64, 64)
    for M, local in ((1, 1), (16, 1), (32, 1), (33, 0), (128, 0)):
        r, p = _plan(lay, M, 0, 1, 148)
        assert r == 1 and p["local"] == local, M
    r, p = _plan(lay, 16, 0, 1, 148)
    # every SM; a decoder warp per tile of the CTA's share (2048 / 148 -> 14), at most 15
    assert p["grid"] == 148 and p["D"] == 14
    r, p = _plan(ans.make_layout(WL.BF16_SPLIT, 14336, 4096, 128, 64, 64), 16, 0, 1, 148)
    assert p["grid"] == 148 and p["D"] == 15


def test_plan_rejects_bad_layouts(ans_lib):
    r, _ = _plan(ans.make_layout(WL.BF16_SPLIT, 4000, 4096, 128, 64), 16, 0, 1, 148)
    assert r == -1
