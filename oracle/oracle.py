"""ctypes front-end of the CPU oracle (``ans_oracle.cpp``).

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may use this module; the product path never
does.  Arrays are numpy; the oracle itself is plain C++ compiled with g++.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ans_oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")

INT4, BF16_SPLIT, FP8_E4M3, INT4_PAIRS, INT8, FP4_E2M1, FP4_PAIRS, BF16_WHOLE = 0, 1, 2, 3, 4, 5, 6, 7
SCALE_NONE, SCALE_ROW_BF16, SCALE_ROW_F32, SCALE_GROUP_BF16 = 0, 1, 2, 3
OK, ERR_ARG, ERR_SHAPE, ERR_ALPHABET, ERR_BUFFER_TOO_SMALL, ERR_CORRUPT = 0, 1, 2, 3, 4, 6

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so with g++ if it is missing or older than its source."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread",
                               SRC, "-o", tmp])
        os.replace(tmp, LIB)
    return LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = C.CDLL(LIB)
            P = C.c_void_p
            u32, u64, i32 = C.c_uint32, C.c_uint64, C.c_int
            L.oracle_alphabet_size.argtypes = [i32]
            L.oracle_e4m3_value.argtypes = [C.c_uint8]
            L.oracle_e4m3_value.restype = C.c_double
            L.oracle_e2m1_value.argtypes = [C.c_uint8]
            L.oracle_e2m1_value.restype = C.c_double
            L.oracle_histogram.argtypes = [i32, P, u64, P]
            L.oracle_histogram_bf16_raw.argtypes = [P, u64, P]
            L.oracle_entropy.argtypes = [P, i32]
            L.oracle_entropy.restype = C.c_double
            L.oracle_normalize.argtypes = [P, i32, i32, P]
            L.oracle_code_cost.argtypes = [P, P, i32, i32]
            L.oracle_code_cost.restype = C.c_double
            L.oracle_rans_encode_message.argtypes = [P, i32, P, i32, i32, P, P, i32, P]
            L.oracle_rans_decode_message.argtypes = [u32, P, i32, P, i32, i32, i32, P, P]
            L.oracle_rans64_encode_message.argtypes = [P, i32, P, i32, P, P, i32, P]
            L.oracle_rans64_decode_message.argtypes = [u64, P, i32, P, i32, i32, P, P]
            L.oracle_encode_bound.argtypes = [u32, u32, u32, u32, i32]
            L.oracle_encode_bound.restype = u64
            L.oracle_encode.argtypes = [i32, P, u32, u32, u32, u32, P, i32, P, u64, P, P, P, i32,
                                        i32]
            L.oracle_decode.argtypes = [i32, P, u64, P, P, u32, u32, u32, u32, P, i32, P,
                                        u64, u64, i32, i32]
            L.oracle_gemm.argtypes = [i32, P, u32, u32, P, u32, i32, P, u32, P, u32, P, i32]
            _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def alphabet_size(dtype: int) -> int:
    return lib().oracle_alphabet_size(dtype)


def e4m3_value(code: int) -> float:
    return lib().oracle_e4m3_value(code)


def e2m1_value(code: int) -> float:
    return lib().oracle_e2m1_value(code)


def histogram(dtype: int, w: np.ndarray, n_weights: int) -> np.ndarray:
    w = np.ascontiguousarray(w)
    counts = np.zeros(alphabet_size(dtype), np.uint64)
    lib().oracle_histogram(dtype, _p(w), n_weights, _p(counts))
    return counts


def histogram_bf16_raw(w: np.ndarray) -> np.ndarray:
    w = np.ascontiguousarray(w, dtype=np.uint16)
    counts = np.zeros(256, np.uint64)
    lib().oracle_histogram_bf16_raw(_p(w), w.size, _p(counts))
    return counts


def entropy(counts) -> float:
    c = np.ascontiguousarray(counts, dtype=np.uint64)
    return lib().oracle_entropy(_p(c), c.size)


def normalize(counts, prob_bits: int = 12):
    """Returns (status, freq uint32[A])."""
    c = np.ascontiguousarray(counts, dtype=np.uint64)
    f = np.zeros(c.size, np.uint32)
    st = lib().oracle_normalize(_p(c), c.size, prob_bits, _p(f))
    return st, f


def code_cost(counts, freq, prob_bits: int = 12) -> float:
    c = np.ascontiguousarray(counts, dtype=np.uint64)
    f = np.ascontiguousarray(freq, dtype=np.uint32)
    return lib().oracle_code_cost(_p(c), _p(f), c.size, prob_bits)


def encode_message(msg, freq, prob_bits: int = 12):
    """Single-lane coder. Returns (status, states[len], words[])."""
    m = np.ascontiguousarray(msg, dtype=np.uint8)
    f = np.ascontiguousarray(freq, dtype=np.uint32)
    states = np.zeros(max(1, m.size), np.uint32)
    words = np.zeros(max(1, m.size), np.uint16)
    nw = C.c_int(0)
    st = lib().oracle_rans_encode_message(_p(m), m.size, _p(f), f.size, prob_bits, _p(states),
                                          _p(words), words.size, C.byref(nw))
    return st, states[:m.size], words[:nw.value]


def decode_message(state: int, words, freq, length: int, prob_bits: int = 12):
    """Single-lane decoder. Returns (status, msg[length], states[length+1])."""
    w = np.ascontiguousarray(words, dtype=np.uint16)
    if w.size == 0:
        w = np.zeros(1, np.uint16)[:0]
    f = np.ascontiguousarray(freq, dtype=np.uint32)
    msg = np.zeros(max(1, length), np.uint8)
    states = np.zeros(length + 1, np.uint32)
    st = lib().oracle_rans_decode_message(int(state), _p(w) if w.size else None, w.size, _p(f),
                                          f.size, prob_bits, length, _p(msg), _p(states))
    return st, msg[:length], states


def encode_message64(msg, freq):
    """Single-lane wide-state coder (64-bit state, 32-bit words, one test per
    pair; 12-bit frequencies).  Returns (status, states[len] (even entries:
    state after each pair), words[] (uint32, decoder order))."""
    m = np.ascontiguousarray(msg, dtype=np.uint8)
    f = np.ascontiguousarray(freq, dtype=np.uint32)
    states = np.zeros(max(1, m.size), np.uint64)
    words = np.zeros(max(1, m.size), np.uint32)
    nw = C.c_int(0)
    st = lib().oracle_rans64_encode_message(_p(m), m.size, _p(f), f.size, _p(states), _p(words),
                                            words.size, C.byref(nw))
    return st, states[:m.size], words[:nw.value]


def decode_message64(state: int, words, freq, length: int):
    """Single-lane wide-state decoder. Returns (status, msg[length], states[length+1])."""
    w = np.ascontiguousarray(words, dtype=np.uint32)
    f = np.ascontiguousarray(freq, dtype=np.uint32)
    msg = np.zeros(max(1, length), np.uint8)
    states = np.zeros(length + 1, np.uint64)
    st = lib().oracle_rans64_decode_message(int(state), _p(w) if w.size else None, w.size, _p(f),
                                            f.size, length, _p(msg), _p(states))
    return st, msg[:length], states


def encode_bound(N, K, tile_n, tile_k, state_bits=32) -> int:
    return lib().oracle_encode_bound(N, K, tile_n, tile_k, state_bits)


def encode(dtype, w, N, K, tile_n, tile_k, freq, prob_bits=12, threads=0, state_bits=32):
    """Returns (status, stream uint8[], offsets uint64[n_tiles+1], raw uint8[] or None).
    state_bits 64 selects the wide-state variant (64-bit states, 32-bit words,
    one renormalisation test per pair of symbols)."""
    w = np.ascontiguousarray(w)
    f = np.ascontiguousarray(freq, dtype=np.uint32)
    cap = encode_bound(N, K, tile_n, tile_k, state_bits)
    n_tiles = (N // tile_n) * (K // tile_k) if cap else 0
    stream = np.zeros(max(cap, 16), np.uint8)
    offsets = np.zeros(n_tiles + 1, np.uint64)
    raw = np.zeros(N * K, np.uint8) if dtype == BF16_SPLIT else None
    nbytes = C.c_uint64(0)
    st = lib().oracle_encode(dtype, _p(w), N, K, tile_n, tile_k, _p(f), prob_bits, _p(stream),
                             cap, C.byref(nbytes), _p(offsets), _p(raw), threads, state_bits)
    return st, stream[:nbytes.value].copy(), offsets, raw


def decode(dtype, stream, offsets, raw, N, K, tile_n, tile_k, freq, prob_bits=12,
           tile_begin=0, tile_end=None, out=None, threads=0, state_bits=32):
    """Returns (status, decoded weights in the original packed format)."""
    stream = np.ascontiguousarray(stream, dtype=np.uint8)
    offsets = np.ascontiguousarray(offsets, dtype=np.uint64)
    f = np.ascontiguousarray(freq, dtype=np.uint32)
    if out is None:
        if dtype in (INT4, INT4_PAIRS, FP4_E2M1, FP4_PAIRS):
            out = np.zeros(N * K // 2, np.uint8)
        elif dtype in (BF16_SPLIT, BF16_WHOLE):
            out = np.zeros(N * K, np.uint16)
        else:
            out = np.zeros(N * K, np.uint8)
    if tile_end is None:
        tile_end = offsets.size - 1
    st = lib().oracle_decode(dtype, _p(stream) if stream.size else None, stream.size, _p(offsets),
                             _p(raw), N, K, tile_n, tile_k, _p(f), prob_bits, _p(out),
                             tile_begin, tile_end, threads, state_bits)
    return st, out


def gemm(dtype, X_bits, M, K, W, N, scale_kind=SCALE_NONE, scales=None, group_k=0, rows=None,
         threads=0):
    """fp64 Y (M x len(rows)) of X (bf16 bits, M x K) times dequant(W)^T."""
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    W = np.ascontiguousarray(W)
    sc = None if scales is None else np.ascontiguousarray(scales)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.uint32)
    n_rows = N if r is None else r.size
    Y = np.zeros((M, n_rows), np.float64)
    st = lib().oracle_gemm(dtype, _p(X_bits), M, K, _p(W), N, scale_kind, _p(sc), group_k,
                           _p(r), n_rows, _p(Y), threads)
    if st != OK:
        raise RuntimeError(f"oracle_gemm status {st}")
    return Y
