"""GPU parity of ans_gemm_batched (several layers in one call, of one layout or
of different shapes): each layer's Y is bit-identical to ans_gemm and to
ans_gemm_uncompressed on the same layer confined to the same number of SMs
(one launch, small M) or on the whole GPU (consecutive launches, larger M),
and within 1e-3 relative Frobenius error of the fp64 oracle."""
import numpy as np
import pytest
import torch

from rans_decode_gemm_b200 import ans
from rans_decode_gemm_b200 import workloads as WL

from _gpu_util import rel_fro, run_gemm, scales_dev, status_tensor, x_dev

pytestmark = pytest.mark.gpu

TOL = 1e-3


def _layers(name, N, K, n, state_bits=64, dtype=None):
    """n layers of one layout with different weights (seeds), compressed."""
    base = WL.CONFIGS[name]
    out = []
    for j in range(n):
        cfg = WL.Config(**{**base.__dict__, "seed": base.seed + 1000 * (j + 1)})
        d = WL.make_weights(cfg, 0, N=N, K=K)
        lay = ans.make_layout(cfg.dtype if dtype is None else dtype, N, K, cfg.tile_n, cfg.tile_k,
                              state_bits)
        out.append((cfg, d, lay, ans.CompressedLayer.from_weights(d["w"], lay, device="cuda")))
    return out


def _run_batched(layers, M, ws=None):
    cfg0 = layers[0][0]
    Xs, Ys, scs, jobs = [], [], [], []
    for j, (cfg, d, lay, layer) in enumerate(layers):
        X = WL.make_x(cfg, M, lay.K, stream=j)
        Xs.append(X)
        dX = x_dev(X)
        Y = torch.full((M, lay.N), float("nan"), dtype=torch.float32, device="cuda")
        sc = scales_dev(cfg, d)
        Ys.append(Y)
        scs.append((dX, sc))
        jobs.append((dX, layer.tiles, sc, Y))
    nb = ans.ans_gemm_batched_workspace(jobs, M, cfg0.scale_kind)
    if ws is None:
        ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device="cuda")
    st = status_tensor()
    ans.ans_gemm_batched(jobs, M, cfg0.scale_kind, cfg0.group_k, ws, ws.numel(), st)
    torch.cuda.synchronize()
    return Xs, Ys, int(st.item())


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _shares(layers, sms):
    """The SM share of each layer in one launch, as include/ans.h states it:
    proportional to the weight count, at least one, the largest giving back
    while the sum is too large, the rest one each to the first layers."""
    w = [lay.N * lay.K for (_, _, lay, _) in layers]
    G = [max(1, int(sms * wj / sum(w))) for wj in w]
    while sum(G) > sms and max(G) > 1:
        G[G.index(max(G))] -= 1
    for j in range(len(G)):
        if sum(G) >= sms:
            break
        G[j] += 1
    return G


CASES = [("bf16_4096", 1024, 2048, 64, None), ("int4_70b", 512, 1024, 64, ans.INT4_PAIRS),
         ("int8_8b", 512, 1024, 64, None), ("fp4_8b", 512, 1024, 32, None),
         ("fp4_8b", 512, 1024, 64, ans.FP4_PAIRS),
         ("int4_70b", 512, 1024, 32, None), ("fp8_405b", 256, 2048, 64, None),
         ("tiny_int4", 512, 512, 32, None), ("llama8b_mlp", 512, 1024, 64, None)]


@pytest.mark.parametrize("name,N,K,state_bits,dtype", CASES)
@pytest.mark.parametrize("n", [1, 2, 3, 8])
@pytest.mark.parametrize("M", [1, 16])
def test_batched_one_launch_parity(cuda, oracle, plan_limits, name, N, K, state_bits, dtype, n, M):
    layers = _layers(name, N, K, n, state_bits, dtype)
    Xs, Ys, st = _run_batched(layers, M)
    assert st == 0
    # the single-layer calls on the same share of the SMs add in the same order
    G = _shares(layers, _sms())
    for j, (cfg, d, lay, layer) in enumerate(layers):
        plan_limits(max_ctas=G[j])
        Y1, st1, _ = run_gemm(cfg, d, lay, layer, Xs[j], compressed=True)
        Yu, stu, _ = run_gemm(cfg, d, lay, layer, Xs[j], compressed=False)
        assert st1 == 0 and stu == 0
        assert torch.equal(Ys[j], Y1) and torch.equal(Ys[j], Yu), j
        Yref = oracle.gemm(cfg.dtype, Xs[j], M, K, d["w"], N, cfg.scale_kind, d["scales"],
                           cfg.group_k)
        assert rel_fro(Ys[j].cpu().numpy(), Yref) <= TOL


@pytest.mark.parametrize("name,N,K,M", [("bf16_4096", 512, 1024, 64), ("int4_70b", 512, 1024, 48),
                                        ("fp8_405b", 256, 1024, 300), ("bf16_4096", 512, 1024, 600),
                                        ("int4_70b", 512, 1024, 300)])
def test_batched_consecutive_launches_parity(cuda, oracle, name, N, K, M):
    # shapes past the small-M schedule run one full-GPU launch per layer --
    # above one token pass (the last two cases) the fused first pass and the
    # dense GEMM of each layer
    layers = _layers(name, N, K, 3)
    Xs, Ys, st = _run_batched(layers, M)
    assert st == 0
    for j, (cfg, d, lay, layer) in enumerate(layers):
        Y1, st1, _ = run_gemm(cfg, d, lay, layer, Xs[j], compressed=True)
        assert st1 == 0 and torch.equal(Ys[j], Y1), j
        Yref = oracle.gemm(cfg.dtype, Xs[j], M, K, d["w"], N, cfg.scale_kind, d["scales"],
                           cfg.group_k)
        assert rel_fro(Ys[j].cpu().numpy(), Yref) <= TOL


def test_batched_llama_gate_up_full_size(cuda, oracle):
    # the MLP's gate and up projections (14336 x 4096 each) in one call, M = 16;
    # fp64 check on 128 sampled W rows of each
    base = WL.CONFIGS["llama8b_mlp"]
    layers = []
    for mi in (0, 1):
        d = WL.make_weights(base, mi)
        lay = ans.make_layout(base.dtype, d["N"], d["K"], base.tile_n, base.tile_k, 64)
        layers.append((base, d, lay, ans.CompressedLayer.from_weights(d["w"], lay, device="cuda")))
    Xs, Ys, st = _run_batched(layers, 16)
    assert st == 0
    for j, (cfg, d, lay, layer) in enumerate(layers):
        rows = np.random.default_rng(j).choice(lay.N, size=128, replace=False).astype(np.uint32)
        Yref = oracle.gemm(cfg.dtype, Xs[j], 16, lay.K, d["w"], lay.N, rows=rows)
        assert rel_fro(Ys[j].cpu().numpy()[:, rows], Yref) <= TOL


def test_batched_workspace_and_status(cuda):
    layers = _layers("bf16_4096", 256, 512, 2)
    cfg = layers[0][0]
    jobs = [(x_dev(WL.make_x(cfg, 16, 512)), l[3].tiles, None,
             torch.empty(16, 256, dtype=torch.float32, device="cuda")) for l in layers]
    nb = ans.ans_gemm_batched_workspace(jobs, 16, 0)
    assert nb >= 2 * 256
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    st = status_tensor()
    with pytest.raises(ans.AnsError) as e:
        ans.ans_gemm_batched(jobs, 16, 0, 0, ws, nb - 256, st)
    assert e.value.status == 4   # ANS_ERR_BUFFER_TOO_SMALL
    # M = 0 is a no-op
    ans.ans_gemm_batched(jobs, 0, 0, 0, ws, nb, st)
    # the workspace is left reusable: two calls in a row give the same result
    ans.ans_gemm_batched(jobs, 16, 0, 0, ws, nb, st)
    torch.cuda.synchronize()
    Y0 = [j[3].clone() for j in jobs]
    ans.ans_gemm_batched(jobs, 16, 0, 0, ws, nb, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert all(torch.equal(a, j[3]) for a, j in zip(Y0, jobs))


def _layer(name, N, K, tile_n=None, tile_k=None, state_bits=64, dtype=None, seed_off=0, matrix=0):
    base = WL.CONFIGS[name]
    cfg = WL.Config(**{**base.__dict__, "seed": base.seed + seed_off})
    d = WL.make_weights(cfg, matrix, N=N, K=K)
    lay = ans.make_layout(cfg.dtype if dtype is None else dtype, d["N"], d["K"],
                          tile_n or cfg.tile_n, tile_k or cfg.tile_k, state_bits)
    return cfg, d, lay, ans.CompressedLayer.from_weights(d["w"], lay, device="cuda")


MIXED = [
    # an MLP in miniature: gate and up (N x K) with down (K x N)
    [("llama8b_mlp", 768, 512, None, None), ("llama8b_mlp", 768, 512, None, None),
     ("llama8b_mlp", 512, 768, None, None)],
    # different tile widths and shapes of one dtype
    [("bf16_4096", 1024, 512, 128, 64), ("bf16_4096", 256, 2048, 128, 128),
     ("bf16_4096", 512, 256, 128, 32)],
    # 256-row tiles next to 128-row tiles, int4 pair symbols with group scales
    [("int4_70b", 512, 1024, 256, 64), ("int4_70b", 384, 512, 128, 64)],
    # very unequal weight counts: the small layer still gets one SM
    [("fp8_405b", 2048, 2048, None, None), ("fp8_405b", 128, 128, None, None)],
]


@pytest.mark.parametrize("case", range(len(MIXED)))
@pytest.mark.parametrize("state_bits", [32, 64])
@pytest.mark.parametrize("M", [1, 16])
def test_batched_mixed_layouts_one_launch(cuda, oracle, plan_limits, case, state_bits, M):
    spec = MIXED[case]
    dtype = ans.INT4_PAIRS if spec[0][0] == "int4_70b" else None
    layers = [_layer(nm, N, K, tn, tk, state_bits, dtype, seed_off=100 * j)
              for j, (nm, N, K, tn, tk) in enumerate(spec)]
    Xs, Ys, st = _run_batched(layers, M)
    assert st == 0
    G = _shares(layers, _sms())
    assert sum(G) <= _sms() and min(G) >= 1
    for j, (cfg, d, lay, layer) in enumerate(layers):
        plan_limits(max_ctas=G[j])
        Y1, st1, _ = run_gemm(cfg, d, lay, layer, Xs[j], compressed=True)
        Yu, stu, _ = run_gemm(cfg, d, lay, layer, Xs[j], compressed=False)
        assert st1 == 0 and stu == 0
        assert torch.equal(Ys[j], Y1) and torch.equal(Ys[j], Yu), j
        Yref = oracle.gemm(cfg.dtype, Xs[j], M, lay.K, d["w"], lay.N, cfg.scale_kind, d["scales"],
                           cfg.group_k)
        assert rel_fro(Ys[j].cpu().numpy(), Yref) <= TOL


def test_batched_mixed_layouts_consecutive_launches(cuda, oracle):
    # past the small-M schedule the layers of different shapes run one after
    # the other on the whole GPU: bit-identical to ans_gemm
    layers = [_layer("llama8b_mlp", 768, 512), _layer("llama8b_mlp", 512, 768, seed_off=7)]
    Xs, Ys, st = _run_batched(layers, 96)
    assert st == 0
    for j, (cfg, d, lay, layer) in enumerate(layers):
        Y1, st1, _ = run_gemm(cfg, d, lay, layer, Xs[j], compressed=True)
        assert st1 == 0 and torch.equal(Ys[j], Y1), j
        Yref = oracle.gemm(cfg.dtype, Xs[j], 96, lay.K, d["w"], lay.N)
        assert rel_fro(Ys[j].cpu().numpy(), Yref) <= TOL


def test_batched_whole_llama_mlp_full_size(cuda, oracle, plan_limits):
    # gate and up (14336 x 4096) and down (4096 x 14336) of the Llama-8B-shaped
    # MLP in one launch at M = 16; each bit-identical to ans_gemm on its share
    # of the SMs, fp64 check on 128 sampled W rows of each
    base = WL.CONFIGS["llama8b_mlp"]
    layers = []
    for mi in (0, 1, 2):
        d = WL.make_weights(base, mi)
        lay = ans.make_layout(base.dtype, d["N"], d["K"], base.tile_n, base.tile_k, 64)
        layers.append((base, d, lay, ans.CompressedLayer.from_weights(d["w"], lay, device="cuda")))
    Xs, Ys, st = _run_batched(layers, 16)
    assert st == 0
    G = _shares(layers, _sms())
    for j, (cfg, d, lay, layer) in enumerate(layers):
        plan_limits(max_ctas=G[j])
        Y1, st1, _ = run_gemm(cfg, d, lay, layer, Xs[j], compressed=True)
        assert st1 == 0 and torch.equal(Ys[j], Y1), j
        rows = np.random.default_rng(j).choice(lay.N, size=128, replace=False).astype(np.uint32)
        Yref = oracle.gemm(cfg.dtype, Xs[j], 16, lay.K, d["w"], lay.N, rows=rows)
        assert rel_fro(Ys[j].cpu().numpy()[:, rows], Yref) <= TOL
