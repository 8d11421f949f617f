"""GPU parity of the standalone decode (ans_decode_tiles) and the GPU
histogram (ans_histogram), through the C ABI.  Decoding is lossless, so the
decoded weights must equal the originals bit for bit."""
import numpy as np
import pytest
import torch

from rans_decode_gemm_b200 import ans
from rans_decode_gemm_b200 import workloads as WL

from _gpu_util import make_case, status_tensor, to_dev

pytestmark = pytest.mark.gpu

SMALL = [("tiny_int4", 512, 512), ("bf16_4096", 512, 1024), ("llama8b_mlp", 384, 1024),
         ("int4_70b", 512, 1024), ("fp8_405b", 256, 1024)]


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
def test_decode_bit_exact_small(cuda, oracle, name, N, K):
    cfg, d, lay, layer = make_case(name, N, K)
    out, st = _decode(layer, lay)
    assert st == 0
    assert np.array_equal(out, _bytes(d["w"]))
    # the oracle's decode of the same stream agrees too
    sto, ref = oracle.decode(cfg.dtype, layer.h_stream, layer.h_offsets, layer.h_raw, N, K,
                             cfg.tile_n, cfg.tile_k, layer.codebook.freq_array())
    assert sto == 0 and np.array_equal(out, _bytes(ref))


@pytest.mark.parametrize("name", ["bf16_4096", "int4_70b"])
def test_decode_bit_exact_full_size(cuda, name):
    cfg, d, lay, layer = make_case(name)
    out, st = _decode(layer, lay)
    assert st == 0
    assert np.array_equal(out, _bytes(d["w"]))


@pytest.mark.parametrize("name,N,K", SMALL)
def test_gpu_histogram_matches_oracle(cuda, oracle, name, N, K):
    cfg = WL.CONFIGS[name]
    d = WL.make_weights(cfg, 0, N=N, K=K)
    lay = ans.make_layout(cfg.dtype, N, K, cfg.tile_n, cfg.tile_k)
    w = d["w"]
    dw = to_dev(w.view(np.int16) if w.dtype == np.uint16 else w)
    hist = torch.full((ans.ALPHABET[cfg.dtype],), 7, dtype=torch.int64, device="cuda")
    ans.ans_histogram(dw, lay, hist)
    torch.cuda.synchronize()
    assert np.array_equal(hist.cpu().numpy().astype(np.uint64), oracle.histogram(cfg.dtype, w, N * K))


def test_single_symbol_layer_decodes(cuda):
    N, K = 256, 128
    w = np.full(N * K, 0x41, np.uint8)
    lay = ans.make_layout(ans.FP8_E4M3, N, K, 128, 64)
    layer = ans.CompressedLayer.from_weights(w, lay, device="cuda")
    out, st = _decode(layer, lay)
    assert st == 0 and np.array_equal(out, w)


def test_corrupt_stream_is_flagged_not_faulting(cuda):
    cfg, d, lay, layer = make_case("bf16_4096", 256, 512)
    rng = np.random.default_rng(9)
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
    assert flagged >= 6


def test_bad_offsets_are_flagged(cuda):
    # 256 x 512 fp8 with 128 x 128 tiles: tiles 0..3 form row block 0.
    cfg, d, lay, layer = make_case("fp8_405b", 256, 512)
    off = layer.h_offsets.copy()
    off[1] += 8                    # tiles 0 and 1 lose their 16-byte alignment
    off[3] = off[-1] + 4096        # tile 2 ends and tile 3 starts past the stream
    broken = ans.CompressedLayer(lay, layer.codebook, layer.h_stream, off, None)
    out, st = _decode(broken, lay)
    assert st & ans.STATUS_BAD_OFFSETS
    o = out.reshape(256, 512)
    w = d["w"].reshape(256, 512)
    assert (o[:128] == 0xA5).all()             # rejected tiles are not written
    assert np.array_equal(o[128:], w[128:])    # the other row block decodes exactly
