// codec_host.h -- internal interface of the host-side codec (no CUDA).
#pragma once
#include <cstdint>
#include <vector>

namespace anshost {

enum : uint32_t { kInt4 = 0, kBf16Split = 1, kFp8 = 2, kInt4Pairs = 3, kInt8 = 4, kFp4 = 5, kFp4Pairs = 6 };

bool layout_valid(uint32_t N, uint32_t K, uint32_t tile_n, uint32_t tile_k);
void histogram(uint32_t dtype, const void* w, uint64_t n_weights, uint64_t* hist);
double entropy_bits(const uint64_t* hist, uint32_t alphabet);
// 0 ok, 1 bad argument, 3 too many present symbols.
int normalize(const uint64_t* hist, uint32_t alphabet, uint32_t prob_bits, uint32_t* freq);
// wide: the wide-state variant (64-bit states, 32-bit words, one renormalisation
// test per pair of symbols).
uint64_t encode_bound(uint32_t N, uint32_t K, uint32_t tile_n, uint32_t tile_k, bool wide);
// 0 ok, 3 symbol with zero frequency, 4 capacity too small (size still reported).
int encode(uint32_t dtype, const void* w, uint32_t N, uint32_t K, uint32_t tile_n,
           uint32_t tile_k, const uint32_t* freq, uint8_t* stream, uint64_t cap,
           uint64_t* stream_bytes, uint64_t* offsets, uint8_t* raw, bool wide);

// Appends one tile's bytes to `out`: the final-state block (the byte count of
// every lane's state as a table of bit planes, the 32 states in the fewest
// whole bytes that hold each, zero bytes up to the word boundary), then the
// pushed words in decoder order (the reverse of `pushed`), then zero bytes up
// to a 16-byte boundary.  The u16 form is the 32-bit-state format, the u32
// form the wide-state one.
void append_tile(std::vector<uint8_t>& out, const uint64_t* x, const std::vector<uint16_t>& pushed);
void append_tile(std::vector<uint8_t>& out, const uint64_t* x, const std::vector<uint32_t>& pushed);

// bf16 as whole 16-bit symbols (alphabet 65,536; codec16_host.cpp).
void histogram16(const uint16_t* w, uint64_t n_weights, uint64_t* hist);
// 0 ok, 1 bad argument, 3 too many present symbols.
int normalize16(const uint64_t* hist, uint32_t prob_bits, uint32_t* freq);
// 0 ok, 1 bad argument, 3 symbol with zero frequency or frequencies not
// summing to 2^prob_bits, 4 capacity too small (size still reported).
int encode16(const uint16_t* w, uint32_t N, uint32_t K, uint32_t tile_n, uint32_t tile_k,
             const uint32_t* freq, uint32_t prob_bits, uint8_t* stream, uint64_t cap,
             uint64_t* stream_bytes, uint64_t* offsets, bool wide);
// Size and contents of the decoder's lookup-table image.
uint64_t table16_bytes(const uint32_t* freq);
int table16(const uint32_t* freq, uint32_t prob_bits, uint8_t* out, uint64_t bytes);

// A compressed layer as the on-disk container holds it (container_host.cpp).
// Pointers are host memory; after container_read they point into the buffer.
struct ContainerLayer {
  uint32_t dtype, N, K, tile_n, tile_k, state_bits, prob_bits, alphabet;
  uint64_t n_tiles, stream_bytes, raw_bytes;
  const uint32_t* freq;
  const uint64_t* offsets;
  const uint8_t* stream;
  const uint8_t* raw;
};
// Arrays of a layer to be written: 0 ok, 1 missing array, 3 freq not summing
// to 2^prob_bits, 6 offsets not 0, 16-byte aligned, non-decreasing, ending at
// the stream size.
int container_check(const ContainerLayer& c);
// Size of the container of a layer (0 when a size is out of range).
uint64_t container_bytes(const ContainerLayer& c);
// 0 ok (*written = size; out may be NULL to query it), 1 size out of range,
// 4 capacity too small.
int container_write(const ContainerLayer& c, uint8_t* out, uint64_t cap, uint64_t* written);
// 0 ok, 6 not a container or damaged (magic, sizes, checksum), 8 another
// version.  Fills c with the header's fields and views into buf.
int container_read(const uint8_t* buf, uint64_t bytes, ContainerLayer* c);

}  // namespace anshost
