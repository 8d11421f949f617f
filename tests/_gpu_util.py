"""Shared helpers for the GPU tests: upload a compressed layer through the
C-ABI binding and run the kernels on torch tensors."""
import numpy as np
import torch

from rans_decode_gemm_b200 import ans
from rans_decode_gemm_b200 import workloads as WL


def make_case(name, N=None, K=None, matrix=0, state_bits=32, dtype=None):
    """dtype: the coded symbol kind when it differs from the workload's storage
    dtype (int4 weights coded as pair symbols)."""
    cfg = WL.CONFIGS[name]
    d = WL.make_weights(cfg, matrix, N=N, K=K)
    lay = ans.make_layout(cfg.dtype if dtype is None else dtype, d["N"], d["K"], cfg.tile_n,
                          cfg.tile_k, state_bits)
    layer = ans.CompressedLayer.from_weights(d["w"], lay, device="cuda")
    return cfg, d, lay, layer


def status_tensor():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def to_dev(a: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def scales_dev(cfg, d):
    if d["scales"] is None:
        return None
    s = np.ascontiguousarray(d["scales"])
    if s.dtype == np.uint16:
        return to_dev(s.view(np.int16))
    return to_dev(s)


def x_dev(X_bits: np.ndarray):
    return to_dev(X_bits.view(np.int16))


def run_gemm(cfg, d, lay, layer, X_bits, compressed=True, ws=None):
    M = X_bits.shape[0]
    dX = x_dev(X_bits)
    Y = torch.full((M, lay.N), float("nan"), dtype=torch.float32, device="cuda")
    nbytes = ans.ans_gemm_workspace(lay, M, cfg.scale_kind)
    if ws is None:
        ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device="cuda")
    st = status_tensor()
    sc = scales_dev(cfg, d)
    if compressed:
        ans.ans_gemm(dX, M, layer.tiles, cfg.scale_kind, sc, cfg.group_k, Y, ws, ws.numel(), st)
    else:
        dW = to_dev(d["w"].view(np.int16) if d["w"].dtype == np.uint16 else d["w"])
        ans.ans_gemm_uncompressed(dX, M, dW, lay, cfg.scale_kind, sc, cfg.group_k, Y, ws,
                                  ws.numel(), st)
    torch.cuda.synchronize()
    return Y, int(st.item()), ws


def rel_fro(Y, Yref):
    Y = np.asarray(Y, np.float64)
    return float(np.linalg.norm(Y - Yref) / max(np.linalg.norm(Yref), 1e-300))
