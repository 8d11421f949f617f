"""GPU decode of bf16 coded as whole 16-bit symbols (ans_decode_tiles16,
"Approaching Shannon Bound", s4.1) through the C ABI: bit-exact against the
original weights for both state widths, on small layers and at full size;
a corrupt stream and bad offsets are flagged, a single-symbol layer decodes."""
import numpy as np
import pytest
import torch

from rans_decode_gemm_b200 import ans
from rans_decode_gemm_b200 import workloads as WL

from _gpu_util import status_tensor, to_dev

pytestmark = pytest.mark.gpu


def _coded(w, N, K, tile_n, tile_k, state_bits, prob_bits=16):
    freq = ans.ans_build_codebook16(ans.ans_histogram16_host(w), prob_bits)
    lay = ans.make_layout(ans.BF16_WHOLE, N, K, tile_n, tile_k, state_bits)
    stream, offsets = ans.ans_encode_tiles16(w, lay, freq, prob_bits)
    table = ans.ans_decode_table16(freq, prob_bits)
    return lay, freq, stream, offsets, table


def _decode(lay, stream, offsets, table):
    d_stream = to_dev(np.concatenate([stream, np.zeros(16, np.uint8)]))
    d_off = to_dev(offsets.view(np.int64))
    d_table = to_dev(table)
    out = torch.zeros(lay.N * lay.K, dtype=torch.int16, device="cuda")
    st = status_tensor()
    ans.ans_decode_tiles16(lay, d_table, d_stream, stream.size, d_off, out, st)
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint16), int(st.item())


@pytest.mark.parametrize("state_bits", [32, 64])
@pytest.mark.parametrize("name,N,K,tile_n,tile_k", [("bf16_4096", 1024, 1024, 128, 64),
                                                     ("bf16_4096", 512, 2048, 256, 64),
                                                     ("llama8b_mlp", 384, 2048, 128, 64),
                                                     ("bf16_4096", 128, 64, 128, 64)])
def test_decode16_bit_exact(cuda, name, N, K, tile_n, tile_k, state_bits):
    w = WL.make_weights(WL.CONFIGS[name], 0, N=N, K=K)["w"]
    lay, freq, stream, offsets, table = _coded(w, N, K, tile_n, tile_k, state_bits)
    out, st = _decode(lay, stream, offsets, table)
    assert st == 0
    assert np.array_equal(out, w)


@pytest.mark.parametrize("state_bits,prob_bits", [(32, 14), (32, 13), (64, 12)])
def test_decode16_lower_precision(cuda, state_bits, prob_bits):
    # 2^14, 2^13 or 2^12 slots: buckets of 4, 2 or 1 slot in the first-level
    # table (the wide-state format is defined at 12 and 16 bits)
    w = WL.make_weights(WL.CONFIGS["bf16_4096"], 0, N=512, K=1024)["w"]
    lay, freq, stream, offsets, table = _coded(w, 512, 1024, 128, 64, state_bits, prob_bits)
    assert int(freq.sum()) == 1 << prob_bits
    out, st = _decode(lay, stream, offsets, table)
    assert st == 0 and np.array_equal(out, w)


@pytest.mark.parametrize("state_bits", [32, 64])
def test_decode16_full_size_4096(cuda, state_bits):
    cfg = WL.CONFIGS["bf16_4096"]
    w = WL.make_weights(cfg, 0)["w"]
    lay, freq, stream, offsets, table = _coded(w, cfg.N, cfg.K, 128, 64, state_bits)
    out, st = _decode(lay, stream, offsets, table)
    assert st == 0 and np.array_equal(out, w)


def test_decode16_corrupt_stream_and_bad_offsets_are_flagged(cuda):
    w = WL.make_weights(WL.CONFIGS["bf16_4096"], 0, N=512, K=512)["w"]
    lay, freq, stream, offsets, table = _coded(w, 512, 512, 128, 64, 64)
    flagged = 0
    for pos in (300, 5000, 20000):
        bad = stream.copy()
        bad[pos] ^= 0x21
        out, st = _decode(lay, bad, offsets, table)
        assert st & ~ans.STATUS_CORRUPT == 0
        flagged += bool(st & ans.STATUS_CORRUPT)
        # an unflagged run decodes exactly (a flip inside tile padding)
        if not st & ans.STATUS_CORRUPT:
            assert np.array_equal(out, w)
    assert flagged >= 2
    off = offsets.copy()
    off[3] += 8                                   # no longer 16-byte aligned
    _, st = _decode(lay, stream, off, table)
    assert st & ans.STATUS_BAD_OFFSETS


@pytest.mark.parametrize("state_bits", [32, 64])
def test_decode16_single_symbol_layer(cuda, state_bits):
    w = np.full(256 * 128, 0x3F80, np.uint16)     # bf16 1.0 everywhere
    lay, freq, stream, offsets, table = _coded(w, 256, 128, 128, 64, state_bits)
    assert freq[0x3F80] == 65536
    out, st = _decode(lay, stream, offsets, table)
    assert st == 0 and np.array_equal(out, w)
