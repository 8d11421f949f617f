"""CPU tests of bf16 coded as whole 16-bit symbols (the library's host side,
"Approaching Shannon Bound", s4.1): the histogram, the normalisation to 2^16
and the tile encoder give what the oracle gives (bytes of the stream
included, both state widths), and the decoder's lookup-table image maps every
slot to the symbol whose frequency range holds it."""
import numpy as np
import pytest

from rans_decode_gemm_b200 import ans
from rans_decode_gemm_b200 import workloads as WL


def _weights(N=256, K=512, seed=0):
    return WL.make_weights(WL.CONFIGS["bf16_4096"], 0, N=N, K=K)["w"]


def test_histogram16_matches_oracle(ans_lib, oracle):
    w = _weights()
    hist = ans.ans_histogram16_host(w)
    assert np.array_equal(hist, oracle.histogram(ans.BF16_WHOLE, w, w.size))
    assert int(hist.sum()) == w.size


@pytest.mark.parametrize("prob_bits", [16, 14])
def test_codebook16_matches_oracle_normalisation(ans_lib, oracle, prob_bits):
    w = _weights()
    hist = ans.ans_histogram16_host(w)
    freq = ans.ans_build_codebook16(hist, prob_bits)
    st, ref = oracle.normalize(hist, prob_bits)
    assert st == 0
    assert np.array_equal(freq, ref)
    assert int(freq.sum()) == 1 << prob_bits
    assert np.array_equal(freq > 0, hist > 0)


def test_codebook16_errors(ans_lib):
    hist = np.zeros(65536, np.uint64)
    with pytest.raises(ans.AnsError):
        ans.ans_build_codebook16(hist, 16)            # empty histogram
    hist[:300] = 1
    with pytest.raises(ans.AnsError) as e:
        ans.ans_build_codebook16(hist, 8)             # 300 present symbols > 2^8 slots
    assert e.value.status == 3


@pytest.mark.parametrize("state_bits,prob_bits", [(32, 16), (64, 16), (32, 14), (64, 12)])
def test_encode16_bytes_match_oracle(ans_lib, oracle, state_bits, prob_bits):
    N, K = 256, 512
    w = _weights(N, K)
    freq = ans.ans_build_codebook16(ans.ans_histogram16_host(w), prob_bits)
    lay = ans.make_layout(ans.BF16_WHOLE, N, K, 128, 64, state_bits)
    stream, offsets = ans.ans_encode_tiles16(w, lay, freq, prob_bits)
    st, ref_stream, ref_offsets, _ = oracle.encode(ans.BF16_WHOLE, w, N, K, 128, 64, freq,
                                                   prob_bits=prob_bits, state_bits=state_bits)
    assert st == 0
    assert np.array_equal(offsets, ref_offsets)
    assert np.array_equal(stream, ref_stream)
    st, back = oracle.decode(ans.BF16_WHOLE, stream, offsets, None, N, K, 128, 64, freq,
                             prob_bits=prob_bits, state_bits=state_bits)
    assert st == 0 and np.array_equal(back, w)


def test_encode16_rejects_bad_arguments(ans_lib):
    w = _weights(256, 256)
    freq = ans.ans_build_codebook16(ans.ans_histogram16_host(w), 16)
    bad = freq.copy()
    bad[np.flatnonzero(bad)[0]] += 1                  # no longer sums to 2^16
    lay = ans.make_layout(ans.BF16_WHOLE, 256, 256, 128, 64, 64)
    with pytest.raises(ans.AnsError) as e:
        ans.ans_encode_tiles16(w, lay, bad, 16)
    assert e.value.status == 3
    absent = freq.copy()
    s0 = int(w[0])
    k = int(np.flatnonzero(absent)[-1] if np.flatnonzero(absent)[-1] != s0 else np.flatnonzero(absent)[-2])
    absent[k] += absent[s0]
    absent[s0] = 0                                    # a symbol of the layer given no slot
    with pytest.raises(ans.AnsError) as e:
        ans.ans_encode_tiles16(w, lay, absent, 16)
    assert e.value.status == 3
    split = ans.make_layout(ans.BF16_SPLIT, 256, 256, 128, 64, 64)
    with pytest.raises(ans.AnsError) as e:
        ans.ans_encode_tiles16(w, split, freq, 16)    # not a 16-bit-symbol layout
    assert e.value.status == 1
    f14 = ans.ans_build_codebook16(ans.ans_histogram16_host(w), 14)
    with pytest.raises(ans.AnsError) as e:
        ans.ans_encode_tiles16(w, lay, f14, 14)       # wide states: 12 or 16 bits only
    assert e.value.status == 1


@pytest.mark.parametrize("prob_bits", [16, 13])
def test_decode_table16_maps_every_slot(ans_lib, prob_bits):
    w = _weights()
    freq = ans.ans_build_codebook16(ans.ans_histogram16_host(w), prob_bits)
    table = ans.ans_decode_table16(freq, prob_bits)
    assert table.size % 16 == 0
    n_present, n = table[:8].view(np.uint32)
    assert n == prob_bits and n_present == int((freq > 0).sum())
    first = table[8:8 + 8192].view(np.uint16)
    ent = table[8 + 8192:8 + 8192 + 4 * n_present].view(np.uint32)
    sym = table[8 + 8192 + 4 * n_present:8 + 8192 + 6 * n_present].view(np.uint16)
    present = np.flatnonzero(freq)
    cdf = np.concatenate([[0], np.cumsum(freq[present].astype(np.int64))])
    assert np.array_equal(sym, present)
    assert np.array_equal(ent & 0xFFFF, cdf[:-1])
    assert np.array_equal((ent >> 16) + 1, freq[present])
    # every slot: the bucket's first symbol, then forward while past the range
    slots = np.arange(1 << prob_bits)
    k = first[slots >> (prob_bits - 12)].astype(np.int64)
    while True:
        past = (slots - (ent[k] & 0xFFFF)) > (ent[k] >> 16)
        if not past.any():
            break
        k = k + past
    owner = np.searchsorted(cdf, slots, side="right") - 1
    assert np.array_equal(k, owner)


def test_decode_table16_limits(ans_lib):
    freq = np.zeros(65536, np.uint32)
    freq[:16385] = 1
    freq[0] += 65536 - 16385                          # 16,385 present symbols
    with pytest.raises(ans.AnsError) as e:
        ans.ans_decode_table16(freq, 16)
    assert e.value.status == 8
    small = np.zeros(65536, np.uint32)
    small[0] = 1 << 11
    with pytest.raises(ans.AnsError) as e:
        ans.ans_decode_table16(small, 11)             # the decoder needs n >= 12
    assert e.value.status == 8
