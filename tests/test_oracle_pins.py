"""Pins of the CPU oracle against facts fixed outside the oracle itself:
closed-form entropies, hand-derived rANS state sequences (tests/golden),
brute force over every frequency composition, the bit-packing special case of
rANS, the e4m3 format as implemented by torch's float8_e4m3fn, and exact
integer / library matmuls."""
import json
import math
import os

import numpy as np
import pytest
import torch

from rans_decode_gemm_b200 import workloads as WL

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---- entropy ------------------------------------------------------------------
def test_entropy_closed_forms(oracle):
    # uniform over 16 symbols: exactly 4 bits
    assert oracle.entropy([7] * 16) == 4.0
    # uniform ternary: log2 3 = 1.585 bits ("突破1.58比特极限", 三元大模型的量化前沿)
    assert abs(oracle.entropy([5, 5, 5] + [0] * 13) - math.log2(3)) < 1e-15
    assert abs(oracle.entropy([5, 5, 5]) - 1.584962500721156) < 1e-15
    # a single present symbol carries nothing
    assert oracle.entropy([0, 0, 123, 0]) == 0.0
    # Bernoulli(1/4): 2 - (3/4) log2 3
    assert abs(oracle.entropy([1, 3]) - 0.8112781244591328) < 1e-15
    # scaling all counts leaves H unchanged; absent symbols add nothing
    assert abs(oracle.entropy([3, 9, 0, 12]) - oracle.entropy([1, 3, 4])) < 1e-15


# ---- normalisation -------------------------------------------------------------
def _cost(c, f, M):
    return sum(ci * math.log2(M / fi) for ci, fi in zip(c, f) if ci > 0)


def _brute_min(counts, M):
    """Minimum cost over every composition of M into the present symbols
    (each >= 1), enumerated exhaustively (vectorised over a grid)."""
    c = np.array([v for v in counts if v > 0], np.float64)
    k = c.size
    if k == 1:
        return 0.0
    grids = np.meshgrid(*([np.arange(1, M + 1)] * (k - 1)), indexing="ij")
    f = np.stack([g.reshape(-1) for g in grids], axis=1).astype(np.float64)
    last = M - f.sum(axis=1)
    ok = last >= 1
    f = np.concatenate([f[ok], last[ok, None]], axis=1)
    cost = (c[None, :] * np.log2(M / f)).sum(axis=1)
    return float(cost.min())


@pytest.mark.parametrize("prob_bits", [4, 6])
def test_normalize_is_optimal_by_brute_force(oracle, prob_bits):
    M = 1 << prob_bits
    rng = np.random.default_rng(7)
    cases = [[5, 1], [1, 1, 1], [100, 1, 1, 1], [3, 0, 9, 27], [1, 0, 0, 1000]]
    for _ in range(60):
        A = int(rng.integers(2, 5))
        c = rng.integers(0, 500, size=A)
        c[rng.integers(0, A)] = max(1, c[0])
        cases.append([int(v) for v in c])
    for c in cases:
        if sum(1 for v in c if v > 0) > M:
            continue
        st, f = oracle.normalize(c, prob_bits)
        assert st == 0
        assert int(f.sum()) == M
        assert all((fi > 0) == (ci > 0) for fi, ci in zip(f, c)), (c, f)
        assert _cost(c, f, M) <= _brute_min(c, M) + 1e-9, (c, list(f))


def test_normalize_exact_fractions_and_edges(oracle):
    st, f = oracle.normalize([2, 1, 1] + [0] * 13)
    assert st == 0 and list(f[:3]) == [2048, 1024, 1024] and f[3:].sum() == 0
    st, f = oracle.normalize([0] * 5 + [77] + [0] * 10)
    assert st == 0 and f[5] == 4096 and f.sum() == 4096
    # more present symbols than slots
    st, _ = oracle.normalize([1] * 17, prob_bits=4)
    assert st == 3
    st, _ = oracle.normalize([0] * 16)
    assert st == 1
    # every present symbol keeps at least one slot even when hugely outnumbered
    c = np.zeros(256, np.uint64)
    c[0] = 10 ** 9
    c[1:200] = 1
    st, f = oracle.normalize(c)
    assert st == 0 and f.sum() == 4096 and (f[1:200] == 1).all() and f[0] == 4096 - 199


# ---- hand-derived rANS examples ------------------------------------------------------
def test_rans_hand_examples(oracle):
    with open(os.path.join(GOLDEN, "rans_hand_examples.json")) as fh:
        ex = json.load(fh)["examples"]
    for e in ex:
        st, states, words = oracle.encode_message(e["message"], e["freq"], e["prob_bits"])
        assert st == 0, e["name"]
        assert [int(s) for s in states] == e["states"], e["name"]
        assert [int(w) for w in words] == e["words"], e["name"]
        st, msg, dstates = oracle.decode_message(states[0], words, e["freq"], len(e["message"]),
                                                 e["prob_bits"])
        assert st == 0, e["name"]
        assert [int(m) for m in msg] == e["message"]
        # the decoder visits the encoder's states in reverse and ends at L
        assert [int(s) for s in dstates[:-1]] == e["states"]
        assert int(dstates[-1]) == 65536
        # stream length agrees with the information content (+ the 16 bits that
        # the final state carries beyond L)
        n = e["prob_bits"]
        info = sum(math.log2((1 << n) / e["freq"][s]) for s in e["message"])
        assert abs(info - e["information_bits"]) < 1e-3
        coded = 16 * len(e["words"]) + math.log2(int(states[0])) - 16
        assert abs(coded - info) < 0.05, e["name"]


# ---- bit-packing special case --------------------------------------------------
def test_equiprobable_16_is_bit_packing(oracle):
    # f = 256 for all 16 symbols: every step appends exactly 4 bits, so a lane
    # with T symbols (T % 4 == 0) emits exactly T/4 words and ends at 17 bits,
    # so a tile is a zero length table (4 bytes), 32 states of 3 bytes and
    # 32 * (T/4) * 2 bytes of words before padding.
    freq = np.full(16, 256, np.uint32)
    rng = np.random.default_rng(3)
    msg = rng.integers(0, 16, size=64).astype(np.uint8)
    st, states, words = oracle.encode_message(msg, freq)
    assert st == 0 and words.size == 16
    # the encode step is x -> (x >> 8) << 12 | s << 8 | (x & 255) on its own
    x = 65536
    for s in msg[::-1]:
        if x >= (1 << 28):
            x >>= 16
        x = ((x >> 8) << 12) | (int(s) << 8) | (x & 255)
    assert x == int(states[0])
    # tile form: int4 codes uniform over 16 values with f = 256 each
    N, K = 128, 64
    codes = rng.integers(-8, 8, size=(N, K)).astype(np.int8)
    w = WL.pack_int4(codes)
    st, stream, offsets, _ = oracle.encode(WL.INT4, w, N, K, 128, 64, freq)
    assert st == 0
    T = N * K // 32
    expect = 4 + 32 * 3 + 32 * (T // 4) * 2
    assert int(offsets[1]) == expect + (-expect) % 16
    # final states carry 4 + 12k bits beyond 2^16: they lie in [2^16, 2^17)
    assert stream[:4].tobytes() == bytes(4)
    states, first_word = _final_states(stream, False)
    assert first_word == 100
    assert all(65536 <= x < 131072 for x in states)


# ---- wide-state variant (64-bit state, 32-bit words, one test per pair) ----------
def test_rans64_hand_examples(oracle):
    with open(os.path.join(GOLDEN, "rans64_hand_examples.json")) as fh:
        ex = json.load(fh)["examples"]
    for e in ex:
        st, states, words = oracle.encode_message64(e["message"], e["freq"])
        assert st == 0, e["name"]
        assert [int(states[i]) for i in range(0, len(e["message"]), 2)] == e["pair_states"], e["name"]
        assert [int(w) for w in words] == e["words"], e["name"]
        st, msg, dstates = oracle.decode_message64(int(states[0]), words, e["freq"],
                                                   len(e["message"]))
        assert st == 0, e["name"]
        assert [int(m) for m in msg] == e["message"]
        assert [int(v) for v in dstates] == e["decode_states"], e["name"]


def test_rans64_equiprobable_16_closed_form(oracle):
    # f = 256 for all 16 symbols: coding s is x -> (x >> 8) << 12 | s << 8 |
    # (x & 255), which lengthens x by exactly 4 bits; a pair adds 8 bits and a
    # word leaves when x >= 2^40 * 256 * 256 = 2^56.  From x = 2^32 (33 bits)
    # the state is 41, 49, 57 bits after pairs 1-3; pair 4 finds 57 bits, pushes
    # 32 and ends at 33 bits again: one word every 4 pairs, floor(P / 4) words
    # for P pairs, and the final state lies in [2^32, 2^33) when 4 divides P.
    freq = np.full(16, 256, np.uint32)
    rng = np.random.default_rng(8)
    msg = rng.integers(0, 16, size=64).astype(np.uint8)
    st, states, words = oracle.encode_message64(msg, freq)
    assert st == 0 and words.size == 64 // 2 // 4
    assert (1 << 32) <= int(states[0]) < (1 << 33)
    x = 1 << 32
    for i in range(len(msg) - 2, -1, -2):
        if x >= (1 << 56):
            x >>= 32
        for s in (int(msg[i + 1]), int(msg[i])):
            x = ((x >> 8) << 12) | (s << 8) | (x & 255)
    assert x == int(states[0])
    # tile form: 128 x 32 int4 tile (T = 128 symbols per lane, P = 64 pairs):
    # a zero length table (8 bytes), 32 states of 5 bytes, 32 lanes * 16 words
    # * 4 bytes
    N, K = 128, 32
    codes = rng.integers(-8, 8, size=(N, K)).astype(np.int8)
    w = WL.pack_int4(codes)
    st, stream, offsets, _ = oracle.encode(WL.INT4, w, N, K, 128, 32, freq, state_bits=64)
    assert st == 0
    T = N * K // 32
    expect = 8 + 32 * 5 + 32 * ((T // 2) // 4) * 4
    assert int(offsets[1]) == expect + (-expect) % 16
    assert stream[:8].tobytes() == bytes(8)
    states, first_word = _final_states(stream, True)
    assert first_word == 168
    assert all((1 << 32) <= x < (1 << 33) for x in states)
    st, out = oracle.decode(WL.INT4, stream, offsets, None, N, K, 128, 32, freq, state_bits=64)
    assert st == 0 and np.array_equal(out, w)


def test_rans64_single_symbol_never_moves(oracle):
    # f = 4096: the pair bound 2^40 * 2^24 = 2^64 is above every state, and
    # coding leaves x unchanged, so a tile is its final-state block alone: a
    # zero length table, 32 states 2^32 in 5 bytes each, 8 bytes of padding.
    freq = np.zeros(256, np.uint32)
    freq[7] = 4096
    w = np.full(128 * 64, 7, np.uint8)
    st, stream, offsets, _ = oracle.encode(WL.FP8_E4M3, w, 128, 64, 128, 64, freq, state_bits=64)
    assert st == 0 and int(offsets[1]) == 176
    assert stream.tobytes() == bytes(8) + bytes([0, 0, 0, 0, 1]) * 32 + bytes(8)


# ---- final-state flush: byte counts from a bit-length recurrence ---------------
def _pow2_codebook():
    """f_s = 2^(12 - k_s) for s = 0..12 with k = 1..12, 12: coding s keeps the
    bits of x below f_s, shifts the rest up by 12 and adds c_s below them, so x
    grows by exactly k_s bits."""
    k = np.array(list(range(1, 13)) + [12])
    freq = np.zeros(256, np.uint32)
    freq[:13] = 1 << (12 - k)
    assert freq.sum() == 4096
    return k, freq


@pytest.mark.parametrize("state_bits", [32, 64])
def test_flush_byte_counts_follow_bit_lengths(oracle, state_bits):
    # A narrow lane gives up 16 bits before coding s when x >= f_s 2^20, i.e.
    # when x has at least 33 - k_s bits: its bit length stays in [17, 33) and
    # ends at 17 + (sum of k mod 16) after sum // 16 words, whatever the order.
    # A wide lane gives up 32 bits before a pair (a, b) when x has at least
    # 65 - k_a - k_b bits: it ends at 33 + (sum mod 32) after sum // 32 words.
    # Lane l holds rows l, l + 32, ... of the tile, so the length table, the
    # state block and the tile size follow from this bit arithmetic alone.
    k, freq = _pow2_codebook()
    N, K = 128, 64
    w2 = np.random.default_rng(5).integers(0, 13, size=(N, K)).astype(np.uint8)
    w = w2.reshape(-1)
    wide = state_bits == 64
    st, stream, offsets, _ = oracle.encode(WL.FP8_E4M3, w, N, K, 128, 64, freq,
                                           state_bits=state_bits)
    assert st == 0
    span = 32 if wide else 16
    bits, words = [], 0
    for l in range(32):
        total = int(k[w2[l::32, :]].sum())
        bits.append((33 if wide else 17) + total % span)
        words += total // span
    counts = [(b + 7) // 8 for b in bits]
    least, table, word = (5, 8, 4) if wide else (3, 4, 2)
    assert len(set(counts)) > 1                # lanes of several byte counts
    block = table + sum(counts)
    block += -block % word
    size = block + words * word
    assert int(offsets[1]) == size + (-size) % 16
    planes = [int.from_bytes(stream[4 * p:4 * p + 4].tobytes(), "little") for p in range(table // 4)]
    for l in range(32):
        assert sum(((pl >> l) & 1) << p for p, pl in enumerate(planes)) == counts[l] - least
    states, first_word = _final_states(stream, wide)
    assert first_word == block
    assert [x.bit_length() for x in states] == bits
    st, out = oracle.decode(WL.FP8_E4M3, stream, offsets, None, N, K, 128, 64, freq,
                            state_bits=state_bits)
    assert st == 0 and np.array_equal(out, w)


@pytest.mark.parametrize("state_bits", [32, 64])
def test_flush_table_and_boundary_are_checked(oracle, state_bits):
    # a flipped bit of the length table moves every later lane's state (the
    # decode then ends away from L); a non-zero byte before the word boundary
    # is rejected outright
    wide = state_bits == 64
    rng = np.random.default_rng(31)
    _, freq = _pow2_codebook()
    for trial in range(64):
        w = rng.integers(0, 13, size=128 * 64).astype(np.uint8)
        st, stream, offsets, _ = oracle.encode(WL.FP8_E4M3, w, 128, 64, 128, 64, freq,
                                               state_bits=state_bits)
        assert st == 0
        states, first_word = _final_states(stream, wide)
        block = (8 if wide else 4) + sum((x.bit_length() + 7) // 8 for x in states)
        if block != first_word:
            break
    assert block != first_word, "no tile with a word-boundary byte"
    st, out = oracle.decode(WL.FP8_E4M3, stream, offsets, None, 128, 64, 128, 64, freq,
                            state_bits=state_bits)
    assert st == 0 and np.array_equal(out, w)
    for lane in (0, 13, 30):
        bad = stream.copy()
        bad[lane // 8] ^= 1 << (lane % 8)
        st, _ = oracle.decode(WL.FP8_E4M3, bad, offsets, None, 128, 64, 128, 64, freq,
                              state_bits=state_bits)
        assert st == oracle.ERR_CORRUPT
    bad = stream.copy()
    bad[block] = 1
    st, _ = oracle.decode(WL.FP8_E4M3, bad, offsets, None, 128, 64, 128, 64, freq,
                          state_bits=state_bits)
    assert st == oracle.ERR_CORRUPT


@pytest.mark.parametrize("name,N,K", [("tiny_int4", 512, 512), ("bf16_4096", 256, 512),
                                      ("llama8b_mlp", 256, 512), ("int4_70b", 512, 256),
                                      ("fp8_405b", 256, 512)])
def test_rans64_encode_decode_identity(oracle, name, N, K):
    cfg, d = _small(name, N, K)
    counts = oracle.histogram(cfg.dtype, d["w"], N * K)
    _, freq = oracle.normalize(counts)
    st, stream, offsets, raw = oracle.encode(cfg.dtype, d["w"], N, K, cfg.tile_n, cfg.tile_k,
                                             freq, state_bits=64)
    assert st == 0
    assert (offsets % 16 == 0).all() and (np.diff(offsets.astype(np.int64)) > 0).all()
    st, out = oracle.decode(cfg.dtype, stream, offsets, raw, N, K, cfg.tile_n, cfg.tile_k, freq,
                            state_bits=64)
    assert st == 0 and np.array_equal(out, d["w"])
    # the other variant's decoder does not accept the stream
    st, _ = oracle.decode(cfg.dtype, stream, offsets, raw, N, K, cfg.tile_n, cfg.tile_k, freq)
    assert st == 6


def test_rans64_fuzz_identity_and_corruption(oracle):
    rng = np.random.default_rng(12)
    for trial in range(9):
        dtype = [WL.INT4, WL.BF16_SPLIT, WL.FP8_E4M3][trial % 3]
        tile_n = [128, 256][trial % 2]
        tile_k = [16, 32, 64][trial % 3]
        N, K = tile_n * int(rng.integers(1, 3)), tile_k * int(rng.integers(1, 4))
        A = 16 if dtype == WL.INT4 else 256
        k = int(rng.integers(1, A + 1))
        support = rng.choice(A, size=k, replace=False)
        p = rng.dirichlet(np.full(k, float(rng.choice([0.05, 0.5, 5.0]))))
        syms = support[rng.choice(k, size=N * K, p=p)]
        if dtype == WL.INT4:
            w = WL.pack_int4((syms - 8).astype(np.int8))
        elif dtype == WL.BF16_SPLIT:
            w = ((rng.integers(0, 256, N * K) & 0x80) << 8 | (syms << 7) |
                 rng.integers(0, 128, N * K)).astype(np.uint16)
        else:
            w = syms.astype(np.uint8)
        counts = oracle.histogram(dtype, w, N * K)
        _, freq = oracle.normalize(counts)
        st, stream, offsets, raw = oracle.encode(dtype, w, N, K, tile_n, tile_k, freq,
                                                 state_bits=64)
        assert st == 0
        st, out = oracle.decode(dtype, stream, offsets, raw, N, K, tile_n, tile_k, freq,
                                state_bits=64)
        assert st == 0 and np.array_equal(out, w), trial
        # a flipped bit in a state or a word is flagged or changes the output
        if stream.size > 256:
            bad = stream.copy()
            pos = int(rng.integers(0, int(offsets[1])))
            bad[pos] ^= np.uint8(1 << int(rng.integers(0, 8)))
            st, out = oracle.decode(dtype, bad, offsets, raw, N, K, tile_n, tile_k, freq,
                                    state_bits=64)
            assert st == 6 or not np.array_equal(out, w)


@pytest.mark.parametrize("name,N,K,band", [("tiny_int4", 512, 512, 0.33),
                                           ("bf16_4096", 512, 1024, 0.17),
                                           ("int4_70b", 512, 1024, 0.09),
                                           ("fp8_405b", 256, 1024, 0.10)])
def test_rans64_size_within_band_of_entropy(oracle, name, N, K, band):
    # The wide state interval starts at 2^32, not 2^16: a lane's initial state
    # costs 32 bits instead of 16, so the gap to the entropy grows by about 16
    # bits per lane and tile (the flushed final state costs about the same in
    # both widths: its information plus the rounding to whole bytes): +0.125
    # bit/weight for 4096-symbol tiles, +0.0625 for 8192, +0.03 for 16384.  The
    # 4096-symbol tiles stay outside the pages' 0.2-bit band.
    cfg, d = _small(name, N, K)
    counts = oracle.histogram(cfg.dtype, d["w"], N * K)
    H = oracle.entropy(counts)
    _, freq = oracle.normalize(counts)
    st, s32, _, _ = oracle.encode(cfg.dtype, d["w"], N, K, cfg.tile_n, cfg.tile_k, freq)
    st64, s64, _, _ = oracle.encode(cfg.dtype, d["w"], N, K, cfg.tile_n, cfg.tile_k, freq,
                                    state_bits=64)
    assert st == 0 and st64 == 0
    gap = 8.0 * s64.size / (N * K) - H
    assert -0.01 < gap < band, (name, gap)
    tiles = (N // cfg.tile_n) * (K // cfg.tile_k)
    extra = 8.0 * (s64.size - s32.size) / (tiles * 32)   # bits per lane and tile
    assert 6 < extra < 26, (name, extra)


# ---- e4m3 ------------------------------------------------------------------------
def test_e4m3_matches_torch_float8(oracle):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = oracle.e4m3_value(c)
        if math.isnan(ref[c]):
            assert math.isnan(v), c
        else:
            assert v == ref[c], (c, v, ref[c])


# ---- symbols, encode/decode identity, size bound ---------------------------------------
def _small(name, N, K, seed_matrix=0):
    cfg = WL.CONFIGS[name]
    return cfg, WL.make_weights(cfg, seed_matrix, N=N, K=K)


@pytest.mark.parametrize("name,N,K", [("tiny_int4", 512, 512), ("bf16_4096", 256, 512),
                                      ("llama8b_mlp", 256, 512), ("int4_70b", 512, 256),
                                      ("fp8_405b", 256, 512)])
def test_encode_decode_identity(oracle, name, N, K):
    cfg, d = _small(name, N, K)
    counts = oracle.histogram(cfg.dtype, d["w"], N * K)
    st, freq = oracle.normalize(counts)
    assert st == 0
    st, stream, offsets, raw = oracle.encode(cfg.dtype, d["w"], N, K, cfg.tile_n, cfg.tile_k, freq)
    assert st == 0
    assert (offsets % 16 == 0).all() and (np.diff(offsets.astype(np.int64)) > 0).all()
    st, out = oracle.decode(cfg.dtype, stream, offsets, raw, N, K, cfg.tile_n, cfg.tile_k, freq)
    assert st == 0
    assert np.array_equal(out, d["w"])
    # the thread count changes nothing
    st1, stream1, off1, raw1 = oracle.encode(cfg.dtype, d["w"], N, K, cfg.tile_n, cfg.tile_k,
                                             freq, threads=1)
    assert st1 == 0 and np.array_equal(stream1, stream) and np.array_equal(off1, offsets)


def test_bf16_symbol_split_reconstructs_bits(oracle):
    cfg, d = _small("llama8b_mlp", 128, 64)
    w = d["w"]
    counts_e = oracle.histogram(WL.BF16_SPLIT, w, w.size)
    # exponent histogram equals numpy's view of bits 7..14
    ref = np.bincount(((w >> 7) & 0xFF).astype(np.int64), minlength=256)
    assert np.array_equal(counts_e, ref)
    counts_r = oracle.histogram_bf16_raw(w)
    ref_r = np.bincount((((w >> 8) & 0x80) | (w & 0x7F)).astype(np.int64), minlength=256)
    assert np.array_equal(counts_r, ref_r)
    # int4 symbol = q + 8 against numpy's signed view of the nibbles
    cfg4, d4 = _small("tiny_int4", 128, 64)
    q = np.empty(128 * 64, np.int64)
    q[0::2] = (d4["w"] & 0xF).astype(np.int64)
    q[1::2] = (d4["w"] >> 4).astype(np.int64)
    q = np.where(q >= 8, q - 16, q)
    assert np.array_equal(oracle.histogram(WL.INT4, d4["w"], q.size),
                          np.bincount(q + 8, minlength=16))


def test_fuzz_identity_skews_and_shapes(oracle):
    rng = np.random.default_rng(11)
    for trial in range(12):
        dtype = [WL.INT4, WL.BF16_SPLIT, WL.FP8_E4M3][trial % 3]
        tile_n = [128, 256][trial % 2]
        tile_k = [16, 32, 48, 64, 128][trial % 5]
        N, K = tile_n * int(rng.integers(1, 3)), tile_k * int(rng.integers(1, 4))
        A = 16 if dtype == WL.INT4 else 256
        # a random skewed distribution over a random subset of the alphabet
        k = int(rng.integers(1, A + 1))
        support = rng.choice(A, size=k, replace=False)
        p = rng.dirichlet(np.full(k, float(rng.choice([0.05, 0.5, 5.0]))))
        syms = support[rng.choice(k, size=N * K, p=p)]
        if dtype == WL.INT4:
            w = WL.pack_int4((syms - 8).astype(np.int8))
        elif dtype == WL.BF16_SPLIT:
            w = ((rng.integers(0, 256, N * K) & 0x80) << 8 | (syms << 7) |
                 rng.integers(0, 128, N * K)).astype(np.uint16)
        else:
            w = syms.astype(np.uint8)
        counts = oracle.histogram(dtype, w, N * K)
        st, freq = oracle.normalize(counts)
        assert st == 0
        st, stream, offsets, raw = oracle.encode(dtype, w, N, K, tile_n, tile_k, freq)
        assert st == 0
        st, out = oracle.decode(dtype, stream, offsets, raw, N, K, tile_n, tile_k, freq)
        assert st == 0 and np.array_equal(out, w), trial


def test_absent_symbol_and_bad_shapes_rejected(oracle):
    w = np.zeros(128 * 32, np.uint8)
    w[5] = 7
    freq = np.zeros(256, np.uint32)
    freq[0] = 4096
    st, *_ = oracle.encode(WL.FP8_E4M3, w, 128, 32, 128, 32, freq)
    assert st == 3
    freq2 = np.zeros(256, np.uint32)
    freq2[0] = 4096
    assert oracle.encode(WL.FP8_E4M3, np.zeros(100 * 32, np.uint8), 100, 32, 128, 32, freq2)[0] == 2
    assert oracle.encode(WL.FP8_E4M3, np.zeros(128 * 24, np.uint8), 128, 24, 128, 24, freq2)[0] == 2


def test_corruption_is_flagged(oracle):
    cfg, d = _small("bf16_4096", 128, 128)
    N, K = 128, 128
    counts = oracle.histogram(cfg.dtype, d["w"], N * K)
    _, freq = oracle.normalize(counts)
    st, stream, offsets, raw = oracle.encode(cfg.dtype, d["w"], N, K, 128, 64, freq)
    rng = np.random.default_rng(5)
    flagged = 0
    for _ in range(40):
        bad = stream.copy()
        pos = int(rng.integers(0, int(offsets[-1])))
        bad[pos] ^= np.uint8(1 << int(rng.integers(0, 8)))
        st, out = oracle.decode(cfg.dtype, bad, offsets, raw, N, K, 128, 64, freq)
        # a flipped bit is either flagged or (if it hit padding-free slack that
        # rANS cannot see) changes the output; it never goes unnoticed silently
        # while reproducing the original
        flagged += st == 6
        if st == 0:
            assert not np.array_equal(out, d["w"])
    assert flagged >= 30


@pytest.mark.parametrize("name,N,K,band", [("tiny_int4", 512, 512, 0.20),
                                           ("bf16_4096", 512, 1024, 0.12),
                                           ("int4_70b", 512, 1024, 0.055),
                                           ("fp8_405b", 256, 1024, 0.075)])
def test_size_within_band_of_entropy(oracle, name, N, K, band):
    # "Approaching Shannon Bound", s4.1: tile-level ANS lands 0.01-0.1 bit/weight
    # above the empirical entropy for low-bit formats, 0.1-0.2 for bf16.  Per
    # lane and tile the gap is the initial state (16 bits), the final state's
    # rounding to whole bytes and its share of the length table (about 4.5
    # bits), the tile's padding and the normalisation loss, so small tiles sit
    # near the top of the band.
    cfg, d = _small(name, N, K)
    counts = oracle.histogram(cfg.dtype, d["w"], N * K)
    H = oracle.entropy(counts)
    _, freq = oracle.normalize(counts)
    st, stream, offsets, raw = oracle.encode(cfg.dtype, d["w"], N, K, cfg.tile_n, cfg.tile_k, freq)
    assert st == 0
    coded_bits = 8.0 * stream.size / (N * K)
    gap = coded_bits - H
    assert -0.01 < gap < band, (name, coded_bits, H)


# ---- int4 pair symbols (one symbol per packed byte) ---------------------------------
def test_pair_symbol_is_packed_byte_xor_0x88(oracle):
    # every packed byte once: the pair histogram is one count at byte ^ 0x88
    # (low nibble: code of the even element + 8; high nibble: odd element + 8)
    w = np.arange(256, dtype=np.uint8)
    counts = oracle.histogram(WL.INT4_PAIRS, w, 512)
    assert counts.size == 256 and (counts == 1).all()
    # hand example: byte 0x7F holds codes -1 (even) and 7 (odd): symbol 7 | 15 << 4
    counts = oracle.histogram(WL.INT4_PAIRS, np.array([0x7F], np.uint8), 2)
    assert int(np.argmax(counts)) == 0xF7 and counts.sum() == 1
    # marginals of the pair histogram are the int4 histograms of even / odd elements
    rng = np.random.default_rng(5)
    codes = np.clip(np.rint(rng.laplace(0, 1.2, size=(64, 128))), -8, 7).astype(np.int8)
    w = WL.pack_int4(codes)
    pc = oracle.histogram(WL.INT4_PAIRS, w, codes.size).reshape(16, 16)   # [hi][lo]
    even = np.bincount(codes[:, 0::2].reshape(-1) + 8, minlength=16)
    odd = np.bincount(codes[:, 1::2].reshape(-1) + 8, minlength=16)
    assert np.array_equal(pc.sum(axis=0), even) and np.array_equal(pc.sum(axis=1), odd)


def _final_states(tile, wide):
    """(the 32 final states, offset of the first word) of a tile: a table of
    byte counts (one little-endian u32 bit plane, two for 64-bit states; a
    lane's count is the least, 3 or 5, plus bit l of plane p times 2^p), the
    states in lane order, little-endian in their counts, zero bytes up to the
    word size."""
    b = bytes(tile)
    planes = [int.from_bytes(b[4 * p:4 * p + 4], "little") for p in range(2 if wide else 1)]
    least, pos, word = (5, 8, 4) if wide else (3, 4, 2)
    xs = []
    for l in range(32):
        n = least + sum(((pl >> l) & 1) << p for p, pl in enumerate(planes))
        xs.append(int.from_bytes(b[pos:pos + n], "little"))
        pos += n
    assert b[pos:pos + (-pos % word)] == bytes(-pos % word)
    return xs, pos + (-pos % word)


def _decode_equiprobable_256(stream, steps, wide):
    """Symbols (lane, step) of one tile coded with f = 16 for all 256 symbols.
    Then a decode step is plain bit surgery: the symbol is bits 4..11 of x and
    x -> (x >> 12) << 4 | (x & 15); narrow states take a 16-bit word when
    x < 2^16 after each step, wide ones a 32-bit word when x < 2^32 after each
    odd step.  Words are shared by the 32 lanes in increasing lane order."""
    wb = 4 if wide else 2
    x, pos = _final_states(stream, wide)
    out = np.zeros((32, steps), np.int64)
    for j in range(steps):
        for l in range(32):
            out[l, j] = (x[l] >> 4) & 255
            x[l] = ((x[l] >> 12) << 4) | (x[l] & 15)
            if (not wide or j % 2 == 1) and x[l] < (1 << (8 * wb)):
                x[l] = (x[l] << (8 * wb)) | int.from_bytes(stream[pos:pos + wb].tobytes(), "little")
                pos += wb
    return out


@pytest.mark.parametrize("tile_n,tile_k", [(128, 64), (256, 32)])
@pytest.mark.parametrize("state_bits", [32, 64])
def test_pair_lane_map_properties(oracle, tile_n, tile_k, state_bits):
    # Weights whose packed byte spells its own row (then its pair column) expose
    # the (lane, step) -> (row, column pair) map of one tile; check that it is a
    # bijection, that every 8 steps of a lane are 16 consecutive K elements of
    # one row, and that every 32 steps complete a 128-row x 16-column slab,
    # 128-row blocks first, then 16-column blocks.
    freq = np.full(256, 16, np.uint32)
    steps = tile_n * tile_k // 2 // 32
    maps = []
    for spell in ("row", "col"):
        r = np.arange(tile_n)[:, None] * np.ones((1, tile_k // 2), np.int64)
        c = np.ones((tile_n, 1), np.int64) * np.arange(tile_k // 2)[None, :]
        byte = (r if spell == "row" else c) % 256
        w = byte.astype(np.uint8).reshape(-1)   # packed bytes, row-major
        st, stream, offsets, _ = oracle.encode(WL.INT4_PAIRS, w, tile_n, tile_k, tile_n, tile_k,
                                               freq, state_bits=state_bits)
        assert st == 0 and offsets.size == 2
        sym = _decode_equiprobable_256(stream, steps, state_bits == 64)
        maps.append(sym ^ 0x88)            # symbol = byte ^ 0x88
    rows, cpairs = maps
    seen = np.zeros((tile_n, tile_k // 2), np.int64)
    np.add.at(seen, (rows.reshape(-1), cpairs.reshape(-1)), 1)
    assert (seen == 1).all()
    H = tile_n // 128
    for j0 in range(0, steps, 8):
        assert (rows[:, j0:j0 + 8] == rows[:, j0:j0 + 1]).all()
        assert (cpairs[:, j0:j0 + 8] == cpairs[:, j0:j0 + 1] + np.arange(8)).all()
    for q in range(steps // 32):
        h, s = q % H, q // H
        blk_r, blk_c = rows[:, 32 * q:32 * q + 32], cpairs[:, 32 * q:32 * q + 32]
        assert set(blk_r.reshape(-1)) == set(range(128 * h, 128 * h + 128))
        assert set(blk_c.reshape(-1)) == set(range(8 * s, 8 * s + 8))


@pytest.mark.parametrize("name,N,K", [("tiny_int4", 512, 512), ("int4_70b", 512, 256)])
@pytest.mark.parametrize("state_bits", [32, 64])
def test_pair_encode_decode_identity_and_size(oracle, name, N, K, state_bits):
    cfg, d = _small(name, N, K)
    counts = oracle.histogram(WL.INT4_PAIRS, d["w"], N * K)
    assert counts.sum() == N * K // 2
    H2 = oracle.entropy(counts)                     # bits per pair
    _, freq = oracle.normalize(counts)
    st, stream, offsets, raw = oracle.encode(WL.INT4_PAIRS, d["w"], N, K, cfg.tile_n, cfg.tile_k,
                                             freq, state_bits=state_bits)
    assert st == 0 and raw is None
    st, out = oracle.decode(WL.INT4_PAIRS, stream, offsets, None, N, K, cfg.tile_n, cfg.tile_k,
                            freq, state_bits=state_bits)
    assert st == 0 and np.array_equal(out, d["w"])
    # half as many symbols as the per-element coding, each carrying two codes:
    # the size stays within the per-element bands of the pair entropy (per
    # weight); the wide states' extra slack per lane costs more on small tiles
    gap = 8.0 * stream.size / (N * K) - H2 / 2
    band = {32: 0.21, 64: 0.34}[state_bits] if name == "tiny_int4" else 0.095
    assert -0.01 < gap < band, (name, gap)
    # the same GEMM as the per-element reading of the same bytes
    rng = np.random.default_rng(1)
    X = WL.to_bf16_bits(rng.standard_normal((2, K)))
    rows = np.arange(0, N, 37, dtype=np.uint32)
    Yp = oracle.gemm(WL.INT4_PAIRS, X, 2, K, d["w"], N, cfg.scale_kind, d["scales"], cfg.group_k,
                     rows=rows)
    Y1 = oracle.gemm(WL.INT4, X, 2, K, d["w"], N, cfg.scale_kind, d["scales"], cfg.group_k,
                     rows=rows)
    assert np.array_equal(Yp, Y1)


# ---- int8 symbols -------------------------------------------------------------------
def test_int8_symbol_is_code_plus_128(oracle):
    # every byte once: one count at byte ^ 0x80 = q + 128 for the two's complement q
    counts = oracle.histogram(WL.INT8, np.arange(256, dtype=np.uint8), 256)
    assert counts.size == 256 and (counts == 1).all()
    for byte, sym in ((0xFF, 127), (0x80, 0), (0x7F, 255), (0x00, 128)):
        c = oracle.histogram(WL.INT8, np.array([byte], np.uint8), 1)
        assert int(np.argmax(c)) == sym and c.sum() == 1


@pytest.mark.parametrize("state_bits,band", [(32, 0.11), (64, 0.18)])
def test_int8_encode_decode_identity_and_size(oracle, state_bits, band):
    cfg, d = _small("int8_8b", 512, 1024)
    counts = oracle.histogram(WL.INT8, d["w"], 512 * 1024)
    H = oracle.entropy(counts)
    _, freq = oracle.normalize(counts)
    st, stream, offsets, raw = oracle.encode(WL.INT8, d["w"], 512, 1024, cfg.tile_n, cfg.tile_k,
                                             freq, state_bits=state_bits)
    assert st == 0 and raw is None
    st, out = oracle.decode(WL.INT8, stream, offsets, None, 512, 1024, cfg.tile_n, cfg.tile_k,
                            freq, state_bits=state_bits)
    assert st == 0 and np.array_equal(out, d["w"])
    gap = 8.0 * stream.size / (512 * 1024) - H
    assert -0.01 < gap < band, gap
    # absmax-per-row int8 of Gaussian weights: entropy near log2(sigma / s * sqrt(2 pi e))
    # with sigma / s = 127 / E[max |z| of 1024 normals] (about 3.2): 7.0-7.4 bits
    assert 6.9 < H < 7.5


def test_gemm_int8_exact_integers(oracle):
    rng = np.random.default_rng(12)
    M, N, K = 4, 40, 96
    q = rng.integers(-128, 128, size=(N, K)).astype(np.int64)
    xi = rng.integers(-20, 21, size=(M, K)).astype(np.int64)
    Xb = WL.to_bf16_bits(xi.astype(np.float32))
    W = q.astype(np.int8).view(np.uint8).reshape(-1)
    Y = oracle.gemm(WL.INT8, Xb.reshape(M, K), M, K, W, N)
    assert np.array_equal(Y, (xi @ q.T).astype(np.float64))
    # row scales 2^-r (fp32) keep it exact
    s = np.array([2.0 ** -(n % 5) for n in range(N)], np.float32)
    Ys = oracle.gemm(WL.INT8, Xb, M, K, W, N, WL.SCALE_ROW_F32, s)
    assert np.array_equal(Ys, (xi @ q.T).astype(np.float64) * s.astype(np.float64)[None, :])


# ---- fp4 e2m1 ----------------------------------------------------------------------
# The e2m1 value table of the OCP Microscaling (MX) format specification: codes
# 0-7 are 0, 0.5, 1, 1.5, 2, 3, 4, 6; bit 3 is the sign.
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_values_match_the_mx_table(oracle):
    for c in range(16):
        v = oracle.e2m1_value(c)
        ref = E2M1_TABLE[c & 7]
        assert v == (-ref if c & 8 else ref), c
        assert math.copysign(1.0, v) == (-1.0 if c & 8 else 1.0)   # code 8 is -0


def test_fp4_symbol_is_the_code_low_nibble_first(oracle):
    c = oracle.histogram(WL.FP4_E2M1, np.array([0x21, 0xF7], np.uint8), 4)
    assert c.size == 16 and list(np.nonzero(c)[0]) == [1, 2, 7, 15] and c.sum() == 4


@pytest.mark.parametrize("state_bits,band", [(32, 0.11), (64, 0.18)])
def test_fp4_encode_decode_identity_and_size(oracle, state_bits, band):
    cfg, d = _small("fp4_8b", 512, 1024)
    counts = oracle.histogram(WL.FP4_E2M1, d["w"], 512 * 1024)
    H = oracle.entropy(counts)
    _, freq = oracle.normalize(counts)
    st, stream, offsets, raw = oracle.encode(WL.FP4_E2M1, d["w"], 512, 1024, cfg.tile_n,
                                             cfg.tile_k, freq, state_bits=state_bits)
    assert st == 0 and raw is None
    st, out = oracle.decode(WL.FP4_E2M1, stream, offsets, None, 512, 1024, cfg.tile_n,
                            cfg.tile_k, freq, state_bits=state_bits)
    assert st == 0 and np.array_equal(out, d["w"])
    gap = 8.0 * stream.size / (512 * 1024) - H
    assert -0.01 < gap < band, gap


def test_gemm_fp4_exact(oracle):
    rng = np.random.default_rng(13)
    M, N, K = 3, 32, 64
    codes = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    vals = np.array([(-1 if c & 8 else 1) * E2M1_TABLE[c & 7] for c in codes.reshape(-1)]).reshape(N, K)
    xi = rng.integers(-9, 10, size=(M, K)).astype(np.int64)
    Xb = WL.to_bf16_bits(xi.astype(np.float32))
    c = codes.reshape(-1)
    W = (c[0::2] | (c[1::2] << 4)).astype(np.uint8)
    Y = oracle.gemm(WL.FP4_E2M1, Xb.reshape(M, K), M, K, W, N)
    assert np.array_equal(Y, xi @ vals.T)
    s = np.array([2.0 ** -(n % 3) for n in range(N)], np.float32)
    Ys = oracle.gemm(WL.FP4_E2M1, Xb, M, K, W, N, WL.SCALE_ROW_F32, s)
    assert np.array_equal(Ys, (xi @ vals.T) * s.astype(np.float64)[None, :])


@pytest.mark.parametrize("state_bits", [32, 64])
def test_fp4_pairs_identity_marginals_and_gemm(oracle, state_bits):
    cfg, d = _small("fp4_8b", 512, 1024)
    pc = oracle.histogram(WL.FP4_PAIRS, d["w"], 512 * 1024)
    assert pc.size == 256 and pc.sum() == 512 * 1024 // 2
    # the packed byte is the symbol: the marginals are the per-code histograms
    # of the even and the odd elements
    b = d["w"]
    assert np.array_equal(pc.reshape(16, 16).sum(axis=0), np.bincount(b & 0xF, minlength=16))
    assert np.array_equal(pc.reshape(16, 16).sum(axis=1), np.bincount(b >> 4, minlength=16))
    _, freq = oracle.normalize(pc)
    st, stream, offsets, _ = oracle.encode(WL.FP4_PAIRS, b, 512, 1024, cfg.tile_n, cfg.tile_k,
                                           freq, state_bits=state_bits)
    assert st == 0
    st, out = oracle.decode(WL.FP4_PAIRS, stream, offsets, None, 512, 1024, cfg.tile_n,
                            cfg.tile_k, freq, state_bits=state_bits)
    assert st == 0 and np.array_equal(out, b)
    # the same lane map as int4 pairs: the int4-pair symbol of the byte b ^ 0x88
    # is b, so coding the bytes XOR 0x88 as int4 pairs gives the same stream
    st, s_i4, o_i4, _ = oracle.encode(WL.INT4_PAIRS, b ^ 0x88, 512, 1024, cfg.tile_n, cfg.tile_k,
                                      freq, state_bits=state_bits)
    assert st == 0 and np.array_equal(s_i4, stream) and np.array_equal(o_i4, offsets)
    rng = np.random.default_rng(2)
    X = WL.to_bf16_bits(rng.standard_normal((2, 1024)))
    rows = np.arange(0, 512, 41, dtype=np.uint32)
    Yp = oracle.gemm(WL.FP4_PAIRS, X, 2, 1024, b, 512, cfg.scale_kind, d["scales"], rows=rows)
    Y1 = oracle.gemm(WL.FP4_E2M1, X, 2, 1024, b, 512, cfg.scale_kind, d["scales"], rows=rows)
    assert np.array_equal(Yp, Y1)


# ---- bf16 as whole 16-bit symbols (probability precision 2^16) ---------------------
def test_bf16_whole_symbol_is_the_pattern(oracle):
    counts = oracle.histogram(WL.BF16_WHOLE, np.arange(65536, dtype=np.uint16), 65536)
    assert counts.size == 65536 and (counts == 1).all()


@pytest.mark.parametrize("state_bits", [32, 64])
def test_bf16_whole_equiprobable_closed_form(oracle, state_bits):
    # f = 1 for all 65536 symbols at n = 16: coding s is x -> x * 2^16 + s.
    # Narrow states start at 2^16, always give up their low 16 bits first and
    # end at 2^16 + s_0; wide states start at 2^32, give up their low 32 bits
    # before each pair and end at 2^32 + s_1 * 2^16 + s_0: one word per symbol
    # or per pair, 2 bytes per symbol either way.
    N, K = 128, 64
    rng = np.random.default_rng(21)
    w = rng.integers(0, 65536, size=N * K).astype(np.uint16)
    freq = np.ones(65536, np.uint32)
    st, stream, offsets, _ = oracle.encode(WL.BF16_WHOLE, w, N, K, 128, 64, freq, prob_bits=16,
                                           state_bits=state_bits)
    assert st == 0
    wide = state_bits == 64
    # final states of 17 or 33 bits: 3 or 5 bytes each, a zero length table
    block = 4 + 32 * 3 if not wide else 8 + 32 * 5
    size = block + 2 * N * K
    assert int(offsets[1]) == size + (-size) % 16
    states, first_word = _final_states(stream, wide)
    assert first_word == block
    w2 = w.reshape(N, K).astype(np.uint64)
    # lane l's first two symbols are row l, columns 0 and 1
    expect = (1 << 16) + w2[:32, 0] if not wide else (1 << 32) + (w2[:32, 1] << 16) + w2[:32, 0]
    assert np.array_equal(np.array(states, np.uint64), expect)
    st, out = oracle.decode(WL.BF16_WHOLE, stream, offsets, None, N, K, 128, 64, freq,
                            prob_bits=16, state_bits=state_bits)
    assert st == 0 and np.array_equal(out, w)


@pytest.mark.parametrize("state_bits,band", [(32, 0.12), (64, 0.19)])
def test_bf16_whole_identity_size_and_gemm(oracle, state_bits, band):
    cfg, d = _small("bf16_4096", 512, 1024)
    w = d["w"]
    counts = oracle.histogram(WL.BF16_WHOLE, w, w.size)
    H16 = oracle.entropy(counts)
    st, freq = oracle.normalize(counts, 16)
    assert st == 0 and freq.sum() == 65536 and ((freq > 0) == (counts > 0)).all()
    st, stream, offsets, raw = oracle.encode(WL.BF16_WHOLE, w, 512, 1024, 128, 64, freq,
                                             prob_bits=16, state_bits=state_bits)
    assert st == 0 and raw is None
    st, out = oracle.decode(WL.BF16_WHOLE, stream, offsets, None, 512, 1024, 128, 64, freq,
                            prob_bits=16, state_bits=state_bits)
    assert st == 0 and np.array_equal(out, w)
    gap = 8.0 * stream.size / w.size - H16
    assert -0.01 < gap < band, gap
    # the whole-value entropy is at most the split bound H(exponent) + 8
    He = oracle.entropy(oracle.histogram(WL.BF16_SPLIT, w, w.size))
    assert H16 <= He + 8 + 1e-9
    X = WL.to_bf16_bits(np.random.default_rng(3).standard_normal((2, 1024)))
    rows = np.arange(0, 512, 53, dtype=np.uint32)
    assert np.array_equal(oracle.gemm(WL.BF16_WHOLE, X, 2, 1024, w, 512, rows=rows),
                          oracle.gemm(WL.BF16_SPLIT, X, 2, 1024, w, 512, rows=rows))


# ---- fp64 GEMM ------------------------------------------------------------------
def test_gemm_int4_exact_integers(oracle):
    rng = np.random.default_rng(2)
    M, N, K = 5, 64, 96
    q = rng.integers(-8, 8, size=(N, K)).astype(np.int64)
    xi = rng.integers(-20, 21, size=(M, K)).astype(np.int64)
    Xb = WL.to_bf16_bits(xi.astype(np.float32))
    Y = oracle.gemm(WL.INT4, Xb.reshape(M, K), M, K, WL.pack_int4(q.astype(np.int8)), N)
    assert np.array_equal(Y, (xi @ q.T).astype(np.float64))
    # row scale 1.0 (bf16 0x3F80) and group scale 1.0 leave it exact
    Yr = oracle.gemm(WL.INT4, Xb, M, K, WL.pack_int4(q.astype(np.int8)), N, WL.SCALE_ROW_BF16,
                     np.full(N, 0x3F80, np.uint16))
    assert np.array_equal(Yr, Y)
    # group scale 2^g on group g of 32 columns: still exact
    sg = np.array([[0x3F80 + (g << 7) for g in range(K // 32)]] * N, np.uint16)
    Yg = oracle.gemm(WL.INT4, Xb, M, K, WL.pack_int4(q.astype(np.int8)), N, WL.SCALE_GROUP_BF16,
                     sg, group_k=32)
    ref = sum((xi[:, g * 32:(g + 1) * 32] @ q[:, g * 32:(g + 1) * 32].T) * 2 ** g
              for g in range(K // 32))
    assert np.array_equal(Yg, ref.astype(np.float64))


def test_gemm_matches_library_matmul(oracle):
    rng = np.random.default_rng(4)
    M, N, K = 3, 48, 80
    X = WL.to_bf16_bits(rng.standard_normal((M, K)))
    Xf = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).to(torch.float64)
    # bf16 weights
    W = WL.to_bf16_bits(rng.standard_normal((N, K)) * 0.02)
    Wf = torch.from_numpy(W.view(np.int16)).view(torch.bfloat16).to(torch.float64)
    Y = oracle.gemm(WL.BF16_SPLIT, X, M, K, W.reshape(-1), N)
    assert np.allclose(Y, (Xf @ Wf.T).numpy(), rtol=1e-12, atol=1e-12)
    # fp8 weights with fp32 row scales, on a sampled subset of rows
    codes = rng.integers(0, 256, size=(N, K)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0   # no NaN codes
    s = rng.uniform(0.5, 2.0, size=N).astype(np.float32)
    Wq = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64) * \
        torch.from_numpy(s).to(torch.float64)[:, None]
    rows = np.array([0, 7, 47, 13], np.uint32)
    Y8 = oracle.gemm(WL.FP8_E4M3, X, M, K, codes.reshape(-1), N, WL.SCALE_ROW_F32, s, rows=rows)
    assert np.allclose(Y8, (Xf @ Wq.T).numpy()[:, rows], rtol=1e-12, atol=1e-12)
