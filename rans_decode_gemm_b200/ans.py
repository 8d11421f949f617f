"""Python binding of the C ABI in ``include/ans.h`` (ctypes; argument
marshalling only -- every step of the codec runs in ``libans.so``).

Function names follow the C ABI.  Device buffers are torch CUDA tensors
(passed by ``data_ptr()``), host buffers are numpy arrays, streams are
``torch.cuda.Stream`` objects (default: the current stream).  A non-OK status
raises :class:`AnsError`.  There is no fallback: if the library cannot be
loaded, every call fails.
"""
from __future__ import annotations

import ctypes as C
import os
import threading

import numpy as np

from . import build as _build

INT4, BF16_SPLIT, FP8_E4M3, INT4_PAIRS, INT8, FP4_E2M1, FP4_PAIRS = 0, 1, 2, 3, 4, 5, 6
BF16_WHOLE = 7   # bf16 as whole 16-bit symbols: the ans_*16 entry points only
SCALE_NONE, SCALE_ROW_BF16, SCALE_ROW_F32, SCALE_GROUP_BF16 = 0, 1, 2, 3
STATUS_CORRUPT, STATUS_TIMEOUT, STATUS_BAD_OFFSETS, STATUS_SMEM_ALIGN = 0x1, 0x2, 0x4, 0x8
ALPHABET = {INT4: 16, BF16_SPLIT: 256, FP8_E4M3: 256, INT4_PAIRS: 256, INT8: 256, FP4_E2M1: 16,
            FP4_PAIRS: 256}

# every symbol include/ans.h declares
EXPORTS = ["ans_status_string", "ans_last_error", "ans_num_tiles", "ans_layout_check",
           "ans_histogram", "ans_histogram_host", "ans_entropy", "ans_build_codebook", "ans_encode_bound",
           "ans_encode_tiles", "ans_decode_tiles", "ans_histogram16_host", "ans_build_codebook16",
           "ans_encode_tiles16", "ans_decode_table16", "ans_decode_tiles16", "ans_gemm_workspace", "ans_gemm",
           "ans_gemm_noalloc", "ans_gemm_uncompressed", "ans_gemm_batched_workspace",
           "ans_gemm_batched", "ans_container_write", "ans_container_read"]
MAX_BATCH = 8


class AnsError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__(f"{where}: status {status} ({_status_text(status)})"
                         + (f": {detail}" if detail else ""))


class AnsCodebook(C.Structure):
    _fields_ = [("alphabet", C.c_uint32), ("prob_bits", C.c_uint32),
                ("freq", C.c_uint16 * 256), ("cdf", C.c_uint16 * 257), ("reserved", C.c_uint16)]

    def freq_array(self) -> np.ndarray:
        return np.ctypeslib.as_array(self.freq)[:self.alphabet].astype(np.uint32)


class AnsLayout(C.Structure):
    _fields_ = [("dtype", C.c_uint32), ("N", C.c_uint32), ("K", C.c_uint32),
                ("tile_n", C.c_uint32), ("tile_k", C.c_uint32), ("state_bits", C.c_uint32)]


class AnsTiles(C.Structure):
    _fields_ = [("layout", AnsLayout), ("codebook", AnsCodebook), ("stream", C.c_void_p),
                ("stream_bytes", C.c_uint64), ("offsets", C.c_void_p), ("raw", C.c_void_p)]


class AnsContainer(C.Structure):
    _fields_ = [("layout", AnsLayout), ("prob_bits", C.c_uint32), ("alphabet", C.c_uint32),
                ("stream_bytes", C.c_uint64), ("raw_bytes", C.c_uint64), ("freq", C.c_void_p),
                ("offsets", C.c_void_p), ("stream", C.c_void_p), ("raw", C.c_void_p),
                ("codebook", AnsCodebook)]


class AnsGemmJob(C.Structure):
    _fields_ = [("d_X", C.c_void_p), ("W", C.c_void_p), ("d_scales", C.c_void_p),
                ("d_Y", C.c_void_p)]


_lib = None
_lock = threading.Lock()


def load():
    """Loads (building in-tree first if missing or stale) libans.so."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            L = C.CDLL(path)
            P, u32, u64, i32, sz = C.c_void_p, C.c_uint32, C.c_uint64, C.c_int, C.c_size_t
            L.ans_status_string.argtypes = [i32]
            L.ans_status_string.restype = C.c_char_p
            L.ans_last_error.argtypes = []
            L.ans_last_error.restype = C.c_char_p
            L.ans_num_tiles.argtypes = [P]
            L.ans_num_tiles.restype = u64
            L.ans_layout_check.argtypes = [P]
            L.ans_histogram.argtypes = [P, P, P, P]
            L.ans_histogram_host.argtypes = [P, P, P]
            L.ans_entropy.argtypes = [P, u32, P]
            L.ans_build_codebook.argtypes = [P, u32, u32, P]
            L.ans_encode_bound.argtypes = [P, P]
            L.ans_encode_tiles.argtypes = [P, P, P, P, u64, P, P, P]
            L.ans_decode_tiles.argtypes = [P, P, P, P]
            L.ans_histogram16_host.argtypes = [P, u64, P]
            L.ans_build_codebook16.argtypes = [P, u32, P]
            L.ans_encode_tiles16.argtypes = [P, P, P, u32, P, u64, P, P]
            L.ans_decode_table16.argtypes = [P, u32, P, u64, P]
            L.ans_decode_tiles16.argtypes = [P, P, u64, P, u64, P, P, P, P]
            L.ans_gemm_workspace.argtypes = [P, u32, i32, P]
            L.ans_gemm.argtypes = [P, u32, P, i32, P, u32, P, P, sz, P, P]
            L.ans_gemm_noalloc.argtypes = [P, u32, P, i32, P, u32, P, P, P]
            L.ans_gemm_uncompressed.argtypes = [P, u32, P, P, i32, P, u32, P, P, sz, P, P]
            L.ans_gemm_batched_workspace.argtypes = [P, u32, u32, i32, P]
            L.ans_gemm_batched.argtypes = [P, u32, u32, i32, u32, P, sz, P, P]
            L.ans_container_write.argtypes = [P, P, u64, P]
            L.ans_container_read.argtypes = [P, u64, P]
            for name in EXPORTS:
                if name not in ("ans_status_string", "ans_last_error", "ans_num_tiles"):
                    getattr(L, name).restype = i32
            _lib = L
    return _lib


def _status_text(st: int) -> str:
    try:
        return load().ans_status_string(st).decode()
    except Exception:  # noqa: BLE001 - only used to decorate an error message
        return "?"


def _check(st: int, where: str):
    if st != 0:
        raise AnsError(st, where, load().ans_last_error().decode())


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data_as(C.c_void_p)
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def make_layout(dtype: int, N: int, K: int, tile_n: int, tile_k: int,
                state_bits: int = 32) -> AnsLayout:
    """state_bits 64 selects the wide-state stream variant (64-bit lane states,
    32-bit words, one renormalisation test per pair of symbols)."""
    return AnsLayout(dtype, N, K, tile_n, tile_k, state_bits)


# ---- the C ABI, one Python function per entry point -----------------------------
def ans_status_string(st: int) -> str:
    return load().ans_status_string(st).decode()


def ans_last_error() -> str:
    return load().ans_last_error().decode()


def ans_num_tiles(layout: AnsLayout) -> int:
    return load().ans_num_tiles(C.byref(layout))


def ans_layout_check(layout: AnsLayout) -> int:
    return load().ans_layout_check(C.byref(layout))


def ans_histogram(d_w, layout: AnsLayout, d_hist, stream=None):
    _check(load().ans_histogram(_ptr(d_w), C.byref(layout), _ptr(d_hist), _stream(stream)),
           "ans_histogram")


def ans_histogram_host(h_w: np.ndarray, layout: AnsLayout) -> np.ndarray:
    h_w = np.ascontiguousarray(h_w)
    hist = np.zeros(ALPHABET[layout.dtype], np.uint64)
    _check(load().ans_histogram_host(_ptr(h_w), C.byref(layout), _ptr(hist)),
           "ans_histogram_host")
    return hist


def ans_entropy(hist) -> float:
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    out = C.c_double(0)
    _check(load().ans_entropy(_ptr(h), h.size, C.byref(out)), "ans_entropy")
    return out.value


def ans_build_codebook(hist, alphabet: int | None = None, prob_bits: int = 12) -> AnsCodebook:
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    cb = AnsCodebook()
    _check(load().ans_build_codebook(_ptr(h), alphabet or h.size, prob_bits, C.byref(cb)),
           "ans_build_codebook")
    return cb


def ans_encode_bound(layout: AnsLayout) -> int:
    out = C.c_uint64(0)
    _check(load().ans_encode_bound(C.byref(layout), C.byref(out)), "ans_encode_bound")
    return out.value


def ans_encode_tiles(h_w: np.ndarray, layout: AnsLayout, codebook: AnsCodebook):
    """Returns (stream uint8[], offsets uint64[n_tiles + 1], raw uint8[] or None)."""
    h_w = np.ascontiguousarray(h_w)
    cap = ans_encode_bound(layout)
    stream = np.empty(max(cap, 16), np.uint8)
    offsets = np.empty(ans_num_tiles(layout) + 1, np.uint64)
    raw = np.empty(layout.N * layout.K, np.uint8) if layout.dtype == BF16_SPLIT else None
    nbytes = C.c_uint64(0)
    _check(load().ans_encode_tiles(_ptr(h_w), C.byref(layout), C.byref(codebook), _ptr(stream),
                                   cap, C.byref(nbytes), _ptr(offsets), _ptr(raw)),
           "ans_encode_tiles")
    return stream[:nbytes.value], offsets, raw


def ans_decode_tiles(tiles: AnsTiles, d_out, d_status, stream=None):
    _check(load().ans_decode_tiles(C.byref(tiles), _ptr(d_out), _ptr(d_status), _stream(stream)),
           "ans_decode_tiles")


def ans_histogram16_host(h_w: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> uint64[65536] histogram of the whole 16-bit symbols."""
    h_w = np.ascontiguousarray(h_w, dtype=np.uint16)
    hist = np.zeros(65536, np.uint64)
    _check(load().ans_histogram16_host(_ptr(h_w), h_w.size, _ptr(hist)), "ans_histogram16_host")
    return hist


def ans_build_codebook16(hist, prob_bits: int = 16) -> np.ndarray:
    """uint32[65536] frequencies summing to 2^prob_bits."""
    hist = np.ascontiguousarray(hist, dtype=np.uint64)
    freq = np.zeros(65536, np.uint32)
    _check(load().ans_build_codebook16(_ptr(hist), prob_bits, _ptr(freq)), "ans_build_codebook16")
    return freq


def ans_encode_tiles16(h_w: np.ndarray, layout: AnsLayout, freq, prob_bits: int = 16):
    """Returns (stream uint8[], offsets uint64[n_tiles + 1])."""
    h_w = np.ascontiguousarray(h_w, dtype=np.uint16)
    freq = np.ascontiguousarray(freq, dtype=np.uint32)
    cap = ans_encode_bound(layout)
    stream = np.empty(max(cap, 16), np.uint8)
    offsets = np.empty(ans_num_tiles(layout) + 1, np.uint64)
    nbytes = C.c_uint64(0)
    _check(load().ans_encode_tiles16(_ptr(h_w), C.byref(layout), _ptr(freq), prob_bits,
                                     _ptr(stream), cap, C.byref(nbytes), _ptr(offsets)),
           "ans_encode_tiles16")
    return stream[:nbytes.value], offsets


def ans_decode_table16(freq, prob_bits: int = 16) -> np.ndarray:
    """The decoder's lookup-table image (uint8[], a multiple of 16 bytes)."""
    freq = np.ascontiguousarray(freq, dtype=np.uint32)
    nbytes = C.c_uint64(0)
    L = load()
    _check(L.ans_decode_table16(_ptr(freq), prob_bits, None, 0, C.byref(nbytes)),
           "ans_decode_table16")
    table = np.zeros(nbytes.value, np.uint8)
    _check(L.ans_decode_table16(_ptr(freq), prob_bits, _ptr(table), table.size, C.byref(nbytes)),
           "ans_decode_table16")
    return table


def ans_decode_tiles16(layout: AnsLayout, d_table, d_stream, stream_bytes: int, d_offsets, d_out,
                       d_status, stream=None):
    _check(load().ans_decode_tiles16(C.byref(layout), _ptr(d_table), d_table.numel(),
                                     _ptr(d_stream), stream_bytes, _ptr(d_offsets), _ptr(d_out),
                                     _ptr(d_status), _stream(stream)),
           "ans_decode_tiles16")


def ans_gemm_workspace(layout: AnsLayout, M: int, scale_kind: int = SCALE_NONE) -> int:
    out = C.c_size_t(0)
    _check(load().ans_gemm_workspace(C.byref(layout), M, scale_kind, C.byref(out)),
           "ans_gemm_workspace")
    return out.value


def ans_gemm(d_X, M: int, tiles: AnsTiles, scale_kind: int, d_scales, group_k: int, d_Y, d_ws,
             ws_bytes: int, d_status, stream=None):
    _check(load().ans_gemm(_ptr(d_X), M, C.byref(tiles), scale_kind, _ptr(d_scales), group_k,
                           _ptr(d_Y), _ptr(d_ws), ws_bytes, _ptr(d_status), _stream(stream)),
           "ans_gemm")


def ans_gemm_noalloc(d_X, M: int, tiles: AnsTiles, scale_kind: int, d_scales, group_k: int, d_Y,
                     d_status, stream=None):
    """ans_gemm without a caller workspace (scratch inside the library)."""
    _check(load().ans_gemm_noalloc(_ptr(d_X), M, C.byref(tiles), scale_kind, _ptr(d_scales),
                                   group_k, _ptr(d_Y), _ptr(d_status), _stream(stream)),
           "ans_gemm_noalloc")


def ans_gemm_uncompressed(d_X, M: int, d_W, layout: AnsLayout, scale_kind: int, d_scales,
                          group_k: int, d_Y, d_ws, ws_bytes: int, d_status, stream=None):
    _check(load().ans_gemm_uncompressed(_ptr(d_X), M, _ptr(d_W), C.byref(layout), scale_kind,
                                        _ptr(d_scales), group_k, _ptr(d_Y), _ptr(d_ws),
                                        ws_bytes, _ptr(d_status), _stream(stream)),
           "ans_gemm_uncompressed")


def _jobs(jobs):
    """jobs: sequence of (d_X, tiles, d_scales, d_Y) -> a ctypes array (the
    AnsTiles structs must stay alive for the call)."""
    def addr(t):
        return None if t is None else _ptr(t).value
    arr = (AnsGemmJob * len(jobs))()
    for j, (x, tiles, sc, y) in enumerate(jobs):
        arr[j].d_X = addr(x)
        arr[j].W = C.addressof(tiles)
        arr[j].d_scales = addr(sc)
        arr[j].d_Y = addr(y)
    return arr


def ans_gemm_batched_workspace(jobs, M: int, scale_kind: int) -> int:
    out = C.c_size_t(0)
    arr = _jobs(jobs)
    _check(load().ans_gemm_batched_workspace(arr, len(jobs), M, scale_kind, C.byref(out)),
           "ans_gemm_batched_workspace")
    return out.value


def ans_gemm_batched(jobs, M: int, scale_kind: int, group_k: int, d_ws, ws_bytes: int, d_status,
                     stream=None):
    """Several layers of one layout in one call: jobs = [(d_X, tiles, d_scales, d_Y), ...]."""
    arr = _jobs(jobs)
    _check(load().ans_gemm_batched(arr, len(jobs), M, scale_kind, group_k, _ptr(d_ws), ws_bytes,
                                   _ptr(d_status), _stream(stream)),
           "ans_gemm_batched")


def ans_container_write(layout: AnsLayout, prob_bits: int, freq, stream: np.ndarray,
                        offsets: np.ndarray, raw: np.ndarray | None = None) -> np.ndarray:
    """The versioned container of a compressed layer (host arrays) as uint8[]."""
    freq = np.ascontiguousarray(freq, dtype=np.uint32)
    stream = np.ascontiguousarray(stream, dtype=np.uint8)
    offsets = np.ascontiguousarray(offsets, dtype=np.uint64)
    raw = None if raw is None else np.ascontiguousarray(raw, dtype=np.uint8)
    c = AnsContainer(layout, prob_bits, freq.size, stream.size, 0 if raw is None else raw.size,
                     _ptr(freq).value, _ptr(offsets).value, _ptr(stream).value,
                     None if raw is None else _ptr(raw).value, AnsCodebook())
    L = load()
    nbytes = C.c_uint64(0)
    _check(L.ans_container_write(C.byref(c), None, 0, C.byref(nbytes)), "ans_container_write")
    out = np.empty(nbytes.value, np.uint8)
    _check(L.ans_container_write(C.byref(c), _ptr(out), out.size, C.byref(nbytes)),
           "ans_container_write")
    return out


def _aligned_bytes(n: int) -> np.ndarray:
    """uint8[n] starting on a 16-byte boundary (ans_container_read's rule)."""
    block = np.empty(n + 16, np.uint8)
    skip = (-block.ctypes.data) % 16
    return block[skip:skip + n]


def ans_container_read(buf) -> dict:
    """A container's layer: layout, prob_bits, freq, offsets, stream, raw (views
    into the container's bytes) and, for the one-byte formats, the codebook."""
    buf = np.asarray(buf, dtype=np.uint8)
    if buf.ctypes.data % 16 != 0 or not buf.flags["C_CONTIGUOUS"]:
        aligned = _aligned_bytes(buf.size)
        aligned[:] = buf
        buf = aligned
    c = AnsContainer()
    _check(load().ans_container_read(_ptr(buf), buf.size, C.byref(c)), "ans_container_read")
    base = buf.ctypes.data

    def view(addr, nbytes):
        return buf[addr - base:addr - base + nbytes]
    n_tiles = ans_num_tiles(c.layout)
    return {"layout": c.layout, "prob_bits": c.prob_bits,
            "freq": view(c.freq, 4 * c.alphabet).view(np.uint32),
            "offsets": view(c.offsets, 8 * (n_tiles + 1)).view(np.uint64),
            "stream": view(c.stream, c.stream_bytes),
            "raw": view(c.raw, c.raw_bytes) if c.raw_bytes else None,
            "codebook": c.codebook if c.alphabet <= 256 else None}


def save_layer(path: str, layout: AnsLayout, prob_bits: int, freq, stream, offsets, raw=None):
    """Writes a compressed layer's container to a file."""
    ans_container_write(layout, prob_bits, freq, stream, offsets, raw).tofile(path)


def load_layer(path: str) -> dict:
    """Reads a container file (into 16-byte aligned memory) -> ans_container_read."""
    size = os.path.getsize(path)
    buf = _aligned_bytes(size)
    with open(path, "rb") as fh:
        if fh.readinto(memoryview(buf)) != size:
            raise AnsError(6, "load_layer", f"{path}: short read")
    return ans_container_read(buf)


def _set_plan_limits(max_ctas: int = 0, max_producers: int = 0, force_shared: bool = False):
    """Internal test hook of libans.so (not part of include/ans.h): caps on the
    CTAs and producer warps of every later fused-GEMM plan in this process,
    and a switch that sends every token count to the shared-accumulator
    schedule.  (0, 0, False) restores the defaults."""
    fn = load().ansdev_set_plan_limits
    fn.argtypes = [C.c_uint32, C.c_uint32, C.c_uint32]
    fn.restype = None
    fn(int(max_ctas), int(max_producers), 1 if force_shared else 0)


def _set_wait_budget(cycles: int = 0):
    """Internal test hook of libans.so: the budget (clock64 cycles) of every
    wait in the kernels that the pipeline's own progress ends, on the current
    device; 0 restores the default (about 1.5 s).  A wait that runs out sets
    the TIMEOUT status bit and the kernel returns."""
    fn = load().ansdev_set_wait_budget
    fn.argtypes = [C.c_longlong]
    fn.restype = C.c_int
    _check(fn(int(cycles)), "ansdev_set_wait_budget")


def _wait_probe(d_status, stream=None):
    """Internal test hook: one bounded wait on a barrier nothing arrives on
    (leaves the TIMEOUT bit in d_status)."""
    fn = load().ansdev_wait_probe
    fn.argtypes = [C.c_void_p, C.c_void_p]
    fn.restype = C.c_int
    _check(fn(_ptr(d_status), _stream(stream)), "ansdev_wait_probe")


# ---- marshalling helper: a compressed layer resident on a device -----------------
class CompressedLayer:
    """Host encode result uploaded to device tensors, plus the ans_tiles struct
    pointing at them.  Holds references so the device buffers stay alive."""

    def __init__(self, layout: AnsLayout, codebook: AnsCodebook, stream: np.ndarray,
                 offsets: np.ndarray, raw: np.ndarray | None, device="cuda"):
        import torch
        self.layout = layout
        self.codebook = codebook
        self.h_stream, self.h_offsets, self.h_raw = stream, offsets, raw
        n = max(16, (stream.size + 15) // 16 * 16)
        self.d_stream = torch.zeros(n, dtype=torch.uint8, device=device)
        if stream.size:
            self.d_stream[:stream.size].copy_(torch.from_numpy(stream))
        self.d_offsets = torch.from_numpy(offsets.view(np.int64)).to(device)
        self.d_raw = torch.from_numpy(raw).to(device) if raw is not None else None
        self.tiles = AnsTiles(layout, codebook, self.d_stream.data_ptr(), stream.size,
                              self.d_offsets.data_ptr(),
                              self.d_raw.data_ptr() if self.d_raw is not None else None)

    @property
    def compressed_bytes(self) -> int:
        """Stream + offset index + codebook + raw side stream."""
        cb = 2 * self.codebook.alphabet
        return int(self.h_stream.size + self.h_offsets.size * 8 + cb +
                   (self.h_raw.size if self.h_raw is not None else 0))

    def save(self, path: str):
        """Writes the layer's container file (ans_container_write)."""
        save_layer(path, self.layout, self.codebook.prob_bits, self.codebook.freq_array(),
                   self.h_stream, self.h_offsets, self.h_raw)

    @classmethod
    def load(cls, path: str, device="cuda"):
        """A layer from its container file (ans_container_read), uploaded to `device`."""
        d = load_layer(path)
        if d["codebook"] is None:
            raise AnsError(1, "CompressedLayer.load", "a 16-bit-symbol layer has no ans_tiles form")
        return cls(d["layout"], d["codebook"], d["stream"], d["offsets"], d["raw"], device)

    @classmethod
    def from_weights(cls, h_w: np.ndarray, layout: AnsLayout, hist=None, device="cuda"):
        """Offline path through the library: histogram (ans_histogram_host
        unless given) -> ans_build_codebook -> ans_encode_tiles -> upload."""
        if hist is None:
            hist = ans_histogram_host(h_w, layout)
        cb = ans_build_codebook(hist, ALPHABET[layout.dtype], 12)
        stream, offsets, raw = ans_encode_tiles(h_w, layout, cb)
        return cls(layout, cb, stream, offsets, raw, device)
