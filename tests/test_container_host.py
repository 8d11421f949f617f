"""CPU tests of the versioned on-disk container of a compressed layer
(ans_container_write / ans_container_read, "Approaching Shannon Bound", s3.1:
codebook, offset index and tile stream kept per layer): every format round
trips byte for byte, a loaded layer decodes through the oracle to the
original weights, the header sits where the format says, and damaged or
foreign bytes are refused."""
import struct

import numpy as np
import pytest

from rans_decode_gemm_b200 import ans
from rans_decode_gemm_b200 import workloads as WL


def _layer(name, N, K, state_bits, dtype=None):
    cfg = WL.CONFIGS[name]
    d = WL.make_weights(cfg, 0, N=N, K=K)
    dt = cfg.dtype if dtype is None else dtype
    lay = ans.make_layout(dt, N, K, cfg.tile_n, cfg.tile_k, state_bits)
    cb = ans.ans_build_codebook(ans.ans_histogram_host(d["w"], lay), ans.ALPHABET[dt], 12)
    stream, offsets, raw = ans.ans_encode_tiles(d["w"], lay, cb)
    return d["w"], lay, cb, stream, offsets, raw


def _header(buf):
    """The 96-byte header as the format defines it, read with struct."""
    magic, version, hbytes = struct.unpack_from("<8sII", buf, 0)
    fields = struct.unpack_from("<8I", buf, 16)
    sizes = struct.unpack_from("<6Q", buf, 48)
    return magic, version, hbytes, fields, sizes


def _fnv1a64(data: bytes) -> int:
    h = 14695981039346656037
    for b in data:
        h = ((h ^ b) * 1099511628211) & 0xFFFFFFFFFFFFFFFF
    return h


@pytest.mark.parametrize("state_bits", [32, 64])
@pytest.mark.parametrize("name,dtype", [("tiny_int4", None), ("tiny_int4", ans.INT4_PAIRS),
                                        ("bf16_4096", None), ("fp8_405b", None),
                                        ("int8_8b", None), ("fp4_8b", None),
                                        ("fp4_8b", ans.FP4_PAIRS)])
def test_round_trip_every_format(ans_lib, oracle, name, dtype, state_bits):
    w, lay, cb, stream, offsets, raw = _layer(name, 256, 512, state_bits, dtype)
    buf = ans.ans_container_write(lay, 12, cb.freq_array(), stream, offsets, raw)
    d = ans.ans_container_read(buf)
    got = d["layout"]
    assert (got.dtype, got.N, got.K, got.tile_n, got.tile_k, got.state_bits) == \
        (lay.dtype, lay.N, lay.K, lay.tile_n, lay.tile_k, state_bits)
    assert d["prob_bits"] == 12
    assert np.array_equal(d["freq"], cb.freq_array())
    assert np.array_equal(d["offsets"], offsets)
    assert d["stream"].tobytes() == stream.tobytes()
    assert (d["raw"] is None) == (raw is None)
    if raw is not None:
        assert d["raw"].tobytes() == raw.tobytes()
    # the codebook read back equals the one that coded the layer
    A = cb.alphabet
    assert d["codebook"].alphabet == A and d["codebook"].prob_bits == 12
    assert list(d["codebook"].freq[:A]) == list(cb.freq[:A])
    assert list(d["codebook"].cdf[:A + 1]) == list(cb.cdf[:A + 1])
    # stream and raw are served in place, 16-byte aligned
    assert d["stream"].ctypes.data % 16 == 0
    # the loaded layer decodes to the original weights
    st, out = oracle.decode(lay.dtype, d["stream"], d["offsets"], d["raw"], 256, 512,
                            lay.tile_n, lay.tile_k, d["freq"], state_bits=state_bits)
    assert st == 0 and np.array_equal(out, w)


def test_header_layout_and_checksum(ans_lib):
    w, lay, cb, stream, offsets, raw = _layer("bf16_4096", 256, 128, 64)
    buf = ans.ans_container_write(lay, 12, cb.freq_array(), stream, offsets, raw)
    magic, version, hbytes, fields, sizes = _header(buf)
    assert magic == b"RANSTILE" and version == 1 and hbytes == 96
    assert fields == (ans.BF16_SPLIT, 256, 128, 128, 64, 64, 12, 256)
    n_tiles, stream_bytes, raw_bytes, payload, checksum, reserved = sizes
    assert n_tiles == 4 and stream_bytes == stream.size and raw_bytes == 256 * 128
    assert reserved == 0
    r16 = lambda v: (v + 15) // 16 * 16
    assert payload == r16(4 * 256) + r16(8 * 5) + r16(stream.size) + r16(256 * 128)
    assert buf.size == 96 + payload
    # sections at their 16-byte boundaries
    f0 = 96
    o0 = f0 + r16(4 * 256)
    s0 = o0 + r16(8 * 5)
    q0 = s0 + r16(stream.size)
    assert np.array_equal(buf[f0:f0 + 1024].view(np.uint32), cb.freq_array())
    assert np.array_equal(buf[o0:o0 + 40].view(np.uint64), offsets)
    assert buf[s0:s0 + stream.size].tobytes() == stream.tobytes()
    assert buf[q0:q0 + raw.size].tobytes() == raw.tobytes()
    # FNV-1a over the header with the checksum field zero, then the payload
    head = bytearray(buf[:96].tobytes())
    head[80:88] = bytes(8)
    assert checksum == _fnv1a64(bytes(head) + buf[96:].tobytes())


def test_bf16_whole_layer_round_trips(ans_lib, oracle):
    cfg = WL.CONFIGS["bf16_4096"]
    w = WL.make_weights(cfg, 0, N=256, K=256)["w"]
    freq = ans.ans_build_codebook16(ans.ans_histogram16_host(w), 16)
    lay = ans.make_layout(ans.BF16_WHOLE, 256, 256, 128, 64, 64)
    stream, offsets = ans.ans_encode_tiles16(w, lay, freq, 16)
    d = ans.ans_container_read(ans.ans_container_write(lay, 16, freq, stream, offsets))
    assert d["prob_bits"] == 16 and d["codebook"] is None and d["raw"] is None
    assert np.array_equal(d["freq"], freq) and d["freq"].size == 65536
    st, out = oracle.decode(ans.BF16_WHOLE, d["stream"], d["offsets"], None, 256, 256, 128, 64,
                            d["freq"], prob_bits=16, state_bits=64)
    assert st == 0 and np.array_equal(out, w)


def test_file_round_trip(ans_lib, tmp_path):
    w, lay, cb, stream, offsets, raw = _layer("fp8_405b", 256, 256, 64)
    path = str(tmp_path / "layer.rans")
    ans.save_layer(path, lay, 12, cb.freq_array(), stream, offsets, raw)
    d = ans.load_layer(path)
    assert d["stream"].tobytes() == stream.tobytes()
    assert np.array_equal(d["offsets"], offsets)


def test_damage_is_refused(ans_lib):
    w, lay, cb, stream, offsets, raw = _layer("bf16_4096", 256, 128, 32)
    buf = ans.ans_container_write(lay, 12, cb.freq_array(), stream, offsets, raw)
    r16 = lambda v: (v + 15) // 16 * 16
    # one flipped bit in the header, the freq, the offsets, the stream, the raw bytes
    o0 = 96 + 1024
    s0 = o0 + r16(8 * 5)
    q0 = s0 + r16(stream.size)
    for pos in (20, 96 + 40, o0 + 9, s0 + 300, q0 + 1000, buf.size - 1):
        bad = buf.copy()
        bad[pos] ^= 0x08
        with pytest.raises(ans.AnsError) as e:
            ans.ans_container_read(bad)
        assert e.value.status == 6, pos
    with pytest.raises(ans.AnsError) as e:          # truncated
        ans.ans_container_read(buf[:-16])
    assert e.value.status == 6
    with pytest.raises(ans.AnsError) as e:          # trailing bytes
        ans.ans_container_read(np.concatenate([buf, np.zeros(16, np.uint8)]))
    assert e.value.status == 6
    with pytest.raises(ans.AnsError) as e:          # not a container
        ans.ans_container_read(np.zeros(256, np.uint8))
    assert e.value.status == 6
    newer = buf.copy()
    newer[8:12] = np.frombuffer(struct.pack("<I", 2), np.uint8)
    with pytest.raises(ans.AnsError) as e:          # another version
        ans.ans_container_read(newer)
    assert e.value.status == 8


def _reseal(buf):
    """The checksum of a buffer whose header was edited on purpose."""
    head = bytearray(buf[:96].tobytes())
    head[80:88] = bytes(8)
    buf[80:88] = np.frombuffer(struct.pack("<Q", _fnv1a64(bytes(head) + buf[96:].tobytes())),
                               np.uint8)
    return buf


def test_consistent_checksum_but_impossible_layer_is_refused(ans_lib):
    # a header edited and re-sealed: the checksum holds, the layer does not
    w, lay, cb, stream, offsets, raw = _layer("fp8_405b", 256, 256, 32)
    buf = ans.ans_container_write(lay, 12, cb.freq_array(), stream, offsets, raw)
    for off, value in ((20, 255),        # N not a multiple of tile_n
                       (36, 48),         # state_bits 48
                       (40, 11),         # prob_bits 11: freq no longer sum to 2^prob_bits
                       (16, 0)):         # dtype int4: alphabet 256 no longer matches
        bad = buf.copy()
        bad[off:off + 4] = np.frombuffer(struct.pack("<I", value), np.uint8)
        with pytest.raises(ans.AnsError) as e:
            ans.ans_container_read(_reseal(bad))
        assert e.value.status == 6, off
    bad = buf.copy()                     # offsets out of order
    o0 = 96 + 1024
    bad[o0 + 8:o0 + 16] = np.frombuffer(struct.pack("<Q", 16 * 10**6), np.uint8)
    with pytest.raises(ans.AnsError) as e:
        ans.ans_container_read(_reseal(bad))
    assert e.value.status == 6


def test_write_argument_errors(ans_lib):
    w, lay, cb, stream, offsets, raw = _layer("bf16_4096", 256, 128, 32)
    freq = cb.freq_array()
    with pytest.raises(ans.AnsError) as e:          # bf16 split without its raw bytes
        ans.ans_container_write(lay, 12, freq, stream, offsets, None)
    assert e.value.status == 1
    bad = freq.copy()
    bad[np.flatnonzero(bad)[0]] += 1
    with pytest.raises(ans.AnsError) as e:          # freq not summing to 4096
        ans.ans_container_write(lay, 12, bad, stream, offsets, raw)
    assert e.value.status == 3
    with pytest.raises(ans.AnsError) as e:          # precision of the one-byte formats
        ans.ans_container_write(lay, 14, freq, stream, offsets, raw)
    assert e.value.status == 3
    off = offsets.copy()
    off[2] += 8
    with pytest.raises(ans.AnsError) as e:          # a tile start off its 16-byte boundary
        ans.ans_container_write(lay, 12, freq, stream, off, raw)
    assert e.value.status == 1
    small = ans.make_layout(ans.BF16_SPLIT, 256, 100, 128, 64)
    with pytest.raises(ans.AnsError) as e:          # a layout the coder does not take
        ans.ans_container_write(small, 12, freq, stream, offsets, raw)
    assert e.value.status == 2
