"""CPU tests of the C-ABI library: it loads, exports every entry point that
include/ans.h declares, and its host codec (histogram, entropy, codebook,
tile encoder) agrees with the CPU oracle byte for byte."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from rans_decode_gemm_b200 import ans
from rans_decode_gemm_b200 import workloads as WL

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(ans_\w+)\s*\(", text, re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol(ans_lib):
    names = declared_functions()
    assert len(names) >= 14
    lib = ans_lib.load()
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert sorted(ans.EXPORTS) == names


def test_status_strings_and_layout_checks(ans_lib):
    assert ans.ans_status_string(0) == "ok"
    assert ans.ans_layout_check(ans.make_layout(0, 512, 512, 128, 32)) == 0
    assert ans.ans_layout_check(ans.make_layout(0, 500, 512, 128, 32)) == 2    # N % tile_n
    assert ans.ans_layout_check(ans.make_layout(0, 512, 520, 128, 40)) == 2    # tile_k % 16
    assert ans.ans_layout_check(ans.make_layout(0, 512, 512, 64, 32)) == 2     # tile_n
    assert ans.ans_layout_check(ans.make_layout(8, 512, 512, 128, 32)) == 1    # dtype
    assert ans.ans_layout_check(ans.make_layout(7, 512, 512, 128, 32)) == 0    # 16-bit symbols
    assert ans.ans_num_tiles(ans.make_layout(7, 512, 512, 128, 32)) == 64
    # the one-byte-symbol entry points refuse the 16-bit-symbol layout
    whole = ans.make_layout(7, 512, 512, 128, 32)
    ws = C.c_size_t(0)
    assert ans.load().ans_gemm_workspace(C.byref(whole), 16, 0, C.byref(ws)) == 1
    assert ans.ans_layout_check(ans.make_layout(6, 512, 512, 128, 32)) == 0    # fp4 pairs
    assert ans.ans_layout_check(ans.make_layout(5, 512, 512, 128, 32)) == 0    # fp4
    assert ans.ans_layout_check(ans.make_layout(4, 512, 512, 128, 32)) == 0    # int8
    assert ans.ans_layout_check(ans.make_layout(3, 512, 512, 128, 32)) == 0    # int4 pairs
    assert ans.ans_layout_check(ans.make_layout(1, 0, 512, 128, 32)) == 2      # empty
    assert ans.ans_num_tiles(ans.make_layout(2, 53248, 16384, 128, 128)) == 53248
    assert ans.ans_layout_check(ans.make_layout(0, 512, 512, 128, 32, 64)) == 0
    assert ans.ans_layout_check(ans.make_layout(0, 512, 512, 128, 32, 0)) == 0    # 0 means 32
    assert ans.ans_layout_check(ans.make_layout(0, 512, 512, 128, 32, 48)) == 1   # state width


CASES = [("tiny_int4", 512, 512), ("bf16_4096", 512, 512), ("llama8b_mlp", 256, 1024),
         ("int4_70b", 512, 512), ("fp8_405b", 256, 1024), ("int8_8b", 256, 1024),
         ("fp4_8b", 256, 1024)]


@pytest.mark.parametrize("pairs", [False, True])
@pytest.mark.parametrize("state_bits", [32, 64])
@pytest.mark.parametrize("name,N,K", CASES)
def test_host_codec_matches_oracle(oracle, ans_lib, name, N, K, state_bits, pairs):
    cfg = WL.CONFIGS[name]
    if pairs:
        if cfg.dtype not in (WL.INT4, WL.FP4_E2M1):
            pytest.skip("pair symbols are a coding of packed nibbles")
        cfg = WL.Config(**{**cfg.__dict__,
                           "dtype": WL.INT4_PAIRS if cfg.dtype == WL.INT4 else WL.FP4_PAIRS})
    d = WL.make_weights(WL.CONFIGS[name], 0, N=N, K=K)
    lay = ans.make_layout(cfg.dtype, N, K, cfg.tile_n, cfg.tile_k, state_bits)
    hist = ans.ans_histogram_host(d["w"], lay)
    assert np.array_equal(hist, oracle.histogram(cfg.dtype, d["w"], N * K))
    assert abs(ans.ans_entropy(hist) - oracle.entropy(hist)) < 1e-12
    cb = ans.ans_build_codebook(hist, ans.ALPHABET[cfg.dtype], 12)
    st, f_or = oracle.normalize(hist, 12)
    assert st == 0 and np.array_equal(cb.freq_array(), f_or)
    cdf = np.concatenate([[0], np.cumsum(f_or)])
    assert np.array_equal(np.ctypeslib.as_array(cb.cdf)[:ans.ALPHABET[cfg.dtype] + 1], cdf)
    stream, offsets, raw = ans.ans_encode_tiles(d["w"], lay, cb)
    st, s_or, off_or, raw_or = oracle.encode(cfg.dtype, d["w"], N, K, cfg.tile_n, cfg.tile_k, f_or,
                                             state_bits=state_bits)
    assert st == 0
    assert np.array_equal(offsets, off_or)
    assert np.array_equal(stream, s_or)
    if raw is not None:
        assert np.array_equal(raw, raw_or)
    # and the oracle decodes the library's stream back to the weights
    st, out = oracle.decode(cfg.dtype, stream, offsets, raw, N, K, cfg.tile_n, cfg.tile_k, f_or,
                            state_bits=state_bits)
    assert st == 0 and np.array_equal(out, d["w"])


def test_codebook_matches_oracle_on_fuzzed_histograms(oracle, ans_lib):
    rng = np.random.default_rng(21)
    for trial in range(200):
        A = 16 if trial % 2 else 256
        k = int(rng.integers(1, A + 1))
        h = np.zeros(A, np.uint64)
        idx = rng.choice(A, size=k, replace=False)
        h[idx] = rng.integers(1, 10 ** int(rng.integers(1, 9)), size=k).astype(np.uint64)
        pb = int(rng.choice([8, 10, 12]))
        st, f = oracle.normalize(h, pb)
        if st != 0:
            with pytest.raises(ans.AnsError):
                ans.ans_build_codebook(h, A, pb)
            continue
        cb = ans.ans_build_codebook(h, A, pb)
        assert np.array_equal(cb.freq_array(), f), trial


def test_host_error_paths(ans_lib):
    lay = ans.make_layout(ans.FP8_E4M3, 128, 32, 128, 32)
    w = np.zeros(128 * 32, np.uint8)
    w[3] = 9
    h = np.zeros(256, np.uint64)
    h[0] = 1
    cb = ans.ans_build_codebook(h, 256)       # only symbol 0 present
    with pytest.raises(ans.AnsError) as e:
        ans.ans_encode_tiles(w, lay, cb)
    assert e.value.status == 3
    with pytest.raises(ans.AnsError) as e:
        ans.ans_build_codebook(np.zeros(16, np.uint64), 16)
    assert e.value.status == 1
    with pytest.raises(ans.AnsError) as e:
        ans.ans_build_codebook(np.ones(16, np.uint64), 16, prob_bits=3)
    assert e.value.status == 3
    bad = ans.ans_build_codebook(np.ones(256, np.uint64), 256)
    bad.freq[0] += 1                          # freq no longer sums to 4096
    with pytest.raises(ans.AnsError) as e:
        ans.ans_encode_tiles(np.zeros(128 * 32, np.uint8), lay, bad)
    assert e.value.status == 3
    with pytest.raises(ans.AnsError) as e:
        ans.ans_encode_tiles(w, ans.make_layout(ans.FP8_E4M3, 100, 32, 128, 32), cb)
    assert e.value.status == 2


def test_single_symbol_layer(oracle, ans_lib):
    # a constant layer codes to 112 bytes per tile and decodes: a zero length
    # table (every state at L = 2^16 takes the least 3 bytes), 32 states 00 00 01,
    # 12 bytes of padding
    N, K = 256, 64
    w = np.full(N * K, 0x3C, np.uint8)
    lay = ans.make_layout(ans.FP8_E4M3, N, K, 128, 64)
    cb = ans.ans_build_codebook(ans.ans_histogram_host(w, lay), 256)
    assert cb.freq[0x3C] == 4096
    stream, offsets, _ = ans.ans_encode_tiles(w, lay, cb)
    assert list(offsets) == [0, 112, 224]
    tile = bytes(4) + bytes([0, 0, 1]) * 32 + bytes(12)
    assert stream.tobytes() == tile * 2
    st, out = oracle.decode(ans.FP8_E4M3, stream, offsets, None, N, K, 128, 64, cb.freq_array())
    assert st == 0 and np.array_equal(out, w)


def test_batched_argument_checks(ans_lib):
    # argument and layout errors are reported before any device is touched
    a = ans.make_layout(ans.BF16_SPLIT, 256, 128, 128, 64)
    b = ans.make_layout(ans.FP8_E4M3, 128, 128, 128, 64)   # shapes may differ, dtypes may not
    cb = ans.AnsCodebook()
    ta, tb = ans.AnsTiles(a, cb, None, 0, None, None), ans.AnsTiles(b, cb, None, 0, None, None)
    with pytest.raises(ans.AnsError) as e:
        ans.ans_gemm_batched_workspace([], 16, 0)
    assert e.value.status == 1
    with pytest.raises(ans.AnsError) as e:
        ans.ans_gemm_batched_workspace([(None, ta, None, None)] * (ans.MAX_BATCH + 1), 16, 0)
    assert e.value.status == 1
    with pytest.raises(ans.AnsError) as e:
        ans.ans_gemm_batched_workspace([(None, ta, None, None), (None, tb, None, None)], 16, 0)
    assert e.value.status == 2
    wide = ans.AnsTiles(ans.make_layout(ans.BF16_SPLIT, 256, 128, 128, 64, 64), cb, None, 0, None,
                        None)
    lib = ans.load()
    arr = ans._jobs([(None, ta, None, None), (None, wide, None, None)])
    assert lib.ans_gemm_batched(arr, 2, 16, 0, 0, None, 0, None, None) == 2   # state widths differ


def test_host_codec_matches_oracle_fuzzed(oracle, ans_lib):
    # random shapes, tile shapes, state widths and skews for every coded dtype:
    # the library's encoder writes the oracle's bytes and its histogram is the oracle's
    rng = np.random.default_rng(77)
    for trial in range(24):
        dtype = int(rng.choice([WL.INT4, WL.BF16_SPLIT, WL.FP8_E4M3, WL.INT4_PAIRS, WL.INT8,
                                WL.FP4_E2M1, WL.FP4_PAIRS]))
        tile_n = int(rng.choice([128, 256]))
        tile_k = int(rng.choice([16, 32, 64, 128]))
        N, K = tile_n * int(rng.integers(1, 3)), tile_k * int(rng.integers(1, 4))
        state_bits = int(rng.choice([32, 64]))
        scale = float(rng.choice([0.3, 1.0, 3.0]))
        if dtype in (WL.INT4, WL.INT4_PAIRS, WL.FP4_E2M1, WL.FP4_PAIRS):
            nib = np.clip(np.rint(rng.laplace(0, scale, size=N * K)), -8, 7).astype(np.int8) & 0xF
            w = (nib[0::2] | (nib[1::2] << 4)).astype(np.uint8)
        elif dtype == WL.BF16_SPLIT:
            w = WL.to_bf16_bits(rng.standard_normal(N * K) * 0.02 * scale)
        else:
            w = np.clip(np.rint(rng.laplace(0, 8 * scale, size=N * K)), -128, 127).astype(np.int8).view(np.uint8)
        lay = ans.make_layout(dtype, N, K, tile_n, tile_k, state_bits)
        hist = ans.ans_histogram_host(w, lay)
        assert np.array_equal(hist, oracle.histogram(dtype, w, N * K)), trial
        cb = ans.ans_build_codebook(hist, ans.ALPHABET[dtype], 12)
        stream, offsets, raw = ans.ans_encode_tiles(w, lay, cb)
        st, s_or, off_or, raw_or = oracle.encode(dtype, w, N, K, tile_n, tile_k, cb.freq_array(),
                                                 state_bits=state_bits)
        assert st == 0, trial
        assert np.array_equal(stream, s_or) and np.array_equal(offsets, off_or), trial
        if raw is not None:
            assert np.array_equal(raw, raw_or), trial
        st, out = oracle.decode(dtype, stream, offsets, raw, N, K, tile_n, tile_k,
                                cb.freq_array(), state_bits=state_bits)
        assert st == 0 and np.array_equal(out, w), trial


def test_dtype_constants_agree_with_the_header():
    # the binding's dtype, scale and status constants are the header's values
    text = open(os.path.join(ROOT, "include", "ans.h")).read()
    enum = dict((k, int(v)) for k, v in re.findall(r"\b(ANS_[A-Z0-9_]+)\s*=\s*(\d+)", text))
    assert enum["ANS_INT4"] == ans.INT4 and enum["ANS_BF16_SPLIT"] == ans.BF16_SPLIT
    assert enum["ANS_FP8_E4M3"] == ans.FP8_E4M3 and enum["ANS_INT4_PAIRS"] == ans.INT4_PAIRS
    assert enum["ANS_INT8"] == ans.INT8 and enum["ANS_FP4_E2M1"] == ans.FP4_E2M1
    assert enum["ANS_FP4_PAIRS"] == ans.FP4_PAIRS and enum["ANS_BF16_WHOLE"] == ans.BF16_WHOLE
    assert enum["ANS_SCALE_GROUP_BF16"] == ans.SCALE_GROUP_BF16
    assert enum["ANS_SCALE_ROW_F32"] == ans.SCALE_ROW_F32
    flags = dict((k, int(v, 16)) for k, v in re.findall(r"#define\s+(ANS_STATUS_[A-Z_]+)\s+0x([0-9a-fA-F]+)u", text))
    assert flags["ANS_STATUS_CORRUPT"] == ans.STATUS_CORRUPT
    assert flags["ANS_STATUS_TIMEOUT"] == ans.STATUS_TIMEOUT
    assert flags["ANS_STATUS_BAD_OFFSETS"] == ans.STATUS_BAD_OFFSETS
    assert flags["ANS_STATUS_SMEM_ALIGN"] == ans.STATUS_SMEM_ALIGN
    assert int(re.search(r"#define\s+ANS_MAX_BATCH\s+(\d+)", text).group(1)) == ans.MAX_BATCH
    # the workload generators use the same dtype numbers
    assert (WL.INT4, WL.BF16_SPLIT, WL.FP8_E4M3, WL.INT4_PAIRS, WL.INT8, WL.FP4_E2M1,
            WL.FP4_PAIRS) == (0, 1, 2, 3, 4, 5, 6)


@pytest.mark.parametrize("state_bits", [32, 64])
def test_encode_bound_holds_for_the_costliest_layer(oracle, ans_lib, state_bits):
    # every symbol of the layer has f = 1 (12 bits each, the most a symbol can
    # cost): the stream comes close to the bound (2 bytes a symbol, plus the
    # full-width state block, the word boundary and the padding of every tile)
    # and stays under it; host bytes equal the oracle's
    N, K = 256, 128
    freq = np.zeros(256, np.uint64)
    freq[0] = 4096 - 255
    freq[1:] = 1
    rng = np.random.default_rng(41)
    w = rng.integers(1, 256, size=N * K).astype(np.uint8)
    lay = ans.make_layout(ans.FP8_E4M3, N, K, 128, 64, state_bits)
    cb = ans.AnsCodebook()
    cb.alphabet, cb.prob_bits = 256, 12
    run = 0
    for s in range(256):
        cb.freq[s], cb.cdf[s] = int(freq[s]), run
        run += int(freq[s])
    cb.cdf[256] = run
    stream, offsets, _ = ans.ans_encode_tiles(w, lay, cb)
    bound = ans.ans_encode_bound(lay)
    assert stream.size <= bound
    assert stream.size > 0.7 * bound
    st, ref, ref_off, _ = oracle.encode(ans.FP8_E4M3, w, N, K, 128, 64, freq.astype(np.uint32),
                                        state_bits=state_bits)
    assert st == 0 and np.array_equal(stream, ref) and np.array_equal(offsets, ref_off)
    assert bound == oracle.encode_bound(N, K, 128, 64, state_bits)
