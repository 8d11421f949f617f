// container_host.cpp -- the versioned on-disk container of a compressed layer.
//
// "Approaching Shannon Bound with Lossless LLM Weight Compression", s3.1: the
// offline stage produces, per layer, the shared codebook, the tile offset
// index and the tile stream (plus, for the bf16 split, the raw sign/mantissa
// bytes); the container keeps those together with the layout they were coded
// for, so a layer is compressed once and loaded many times.
//
// Bytes (all little-endian):
//   [0, 96)  header: magic "RANSTILE", version (1), header size (96), dtype,
//            N, K, tile_n, tile_k, state_bits, prob_bits, alphabet (u32 each),
//            n_tiles, stream bytes, raw bytes, payload bytes, checksum,
//            reserved (u64 each)
//   payload: freq (alphabet x u32), offsets ((n_tiles + 1) x u64), stream,
//            raw; each section starts on a 16-byte boundary of the container
//            (zero bytes between them), so a container read into 16-byte
//            aligned memory serves its stream and raw bytes in place.
// The checksum is 64-bit FNV-1a over the header (checksum field zero) and
// the payload.
#include <cstring>

#include "codec_host.h"

namespace anshost {

namespace {

constexpr char kMagic[8] = {'R', 'A', 'N', 'S', 'T', 'I', 'L', 'E'};
constexpr uint32_t kVersion = 1;

struct Header {
  char magic[8];
  uint32_t version, header_bytes;
  uint32_t dtype, N, K, tile_n, tile_k, state_bits;
  uint32_t prob_bits, alphabet;
  uint64_t n_tiles, stream_bytes, raw_bytes, payload_bytes, checksum, reserved;
};
static_assert(sizeof(Header) == 96, "container header is 96 bytes");

uint64_t round16(uint64_t v) { return (v + 15) & ~uint64_t(15); }

// Fowler-Noll-Vo 1a, 64-bit (offset basis and prime of the published definition).
struct Fnv {
  uint64_t h = 14695981039346656037ull;
  void add(const uint8_t* p, uint64_t n) {
    for (uint64_t i = 0; i < n; ++i) {
      h ^= p[i];
      h *= 1099511628211ull;
    }
  }
};

// Section sizes of a payload; false when a size is out of range.
struct Sections {
  uint64_t freq, offsets, stream, raw, total;
};

bool sections(uint32_t alphabet, uint64_t n_tiles, uint64_t stream_bytes, uint64_t raw_bytes,
              Sections* s) {
  // far above any layer the 32-bit layout fields allow, and far below overflow
  const uint64_t kLimit = 1ull << 50;
  if (n_tiles >= kLimit / 8 || stream_bytes >= kLimit || raw_bytes >= kLimit) return false;
  s->freq = round16(4ull * alphabet);
  s->offsets = round16(8 * (n_tiles + 1));
  s->stream = round16(stream_bytes);
  s->raw = round16(raw_bytes);
  s->total = sizeof(Header) + s->freq + s->offsets + s->stream + s->raw;
  return true;
}

}  // namespace

int container_check(const ContainerLayer& c) {
  if (c.n_tiles == 0 || !c.freq || !c.offsets || (c.stream_bytes && !c.stream)) return 1;
  if ((c.raw_bytes != 0) != (c.raw != nullptr)) return 1;
  uint64_t run = 0;
  for (uint32_t s = 0; s < c.alphabet; ++s) run += c.freq[s];
  if (c.prob_bits > 16 || run != (1ull << c.prob_bits)) return 3;
  if (c.offsets[0] != 0 || c.offsets[c.n_tiles] != c.stream_bytes) return 6;
  for (uint64_t t = 0; t < c.n_tiles; ++t)
    if (c.offsets[t + 1] < c.offsets[t] || c.offsets[t] % 16 != 0) return 6;
  return 0;
}

uint64_t container_bytes(const ContainerLayer& c) {
  Sections s;
  return sections(c.alphabet, c.n_tiles, c.stream_bytes, c.raw_bytes, &s) ? s.total : 0;
}

int container_write(const ContainerLayer& c, uint8_t* out, uint64_t cap, uint64_t* written) {
  Sections s;
  if (!sections(c.alphabet, c.n_tiles, c.stream_bytes, c.raw_bytes, &s)) return 1;
  *written = s.total;
  if (!out) return 0;
  if (cap < s.total) return 4;
  Header h;
  std::memset(&h, 0, sizeof(h));
  std::memcpy(h.magic, kMagic, sizeof(kMagic));
  h.version = kVersion;
  h.header_bytes = sizeof(Header);
  h.dtype = c.dtype;
  h.N = c.N;
  h.K = c.K;
  h.tile_n = c.tile_n;
  h.tile_k = c.tile_k;
  h.state_bits = c.state_bits;
  h.prob_bits = c.prob_bits;
  h.alphabet = c.alphabet;
  h.n_tiles = c.n_tiles;
  h.stream_bytes = c.stream_bytes;
  h.raw_bytes = c.raw_bytes;
  h.payload_bytes = s.total - sizeof(Header);
  std::memset(out, 0, s.total);
  uint8_t* p = out + sizeof(Header);
  std::memcpy(p, c.freq, 4ull * c.alphabet);  // little-endian host
  p += s.freq;
  std::memcpy(p, c.offsets, 8 * (c.n_tiles + 1));
  p += s.offsets;
  if (c.stream_bytes) std::memcpy(p, c.stream, c.stream_bytes);
  p += s.stream;
  if (c.raw_bytes) std::memcpy(p, c.raw, c.raw_bytes);
  Fnv f;
  f.add(reinterpret_cast<const uint8_t*>(&h), sizeof(h));
  f.add(out + sizeof(Header), h.payload_bytes);
  h.checksum = f.h;
  std::memcpy(out, &h, sizeof(h));
  return 0;
}

int container_read(const uint8_t* buf, uint64_t bytes, ContainerLayer* c) {
  if (!buf || bytes < sizeof(Header)) return 6;
  Header h;
  std::memcpy(&h, buf, sizeof(h));
  if (std::memcmp(h.magic, kMagic, sizeof(kMagic)) != 0) return 6;
  if (h.version != kVersion || h.header_bytes != sizeof(Header)) return 8;
  Sections s;
  if (!sections(h.alphabet, h.n_tiles, h.stream_bytes, h.raw_bytes, &s)) return 6;
  if (s.total != bytes || h.payload_bytes != s.total - sizeof(Header)) return 6;
  const uint64_t sum = h.checksum;
  h.checksum = 0;
  Fnv f;
  f.add(reinterpret_cast<const uint8_t*>(&h), sizeof(h));
  f.add(buf + sizeof(Header), h.payload_bytes);
  if (f.h != sum) return 6;
  c->dtype = h.dtype;
  c->N = h.N;
  c->K = h.K;
  c->tile_n = h.tile_n;
  c->tile_k = h.tile_k;
  c->state_bits = h.state_bits;
  c->prob_bits = h.prob_bits;
  c->alphabet = h.alphabet;
  c->n_tiles = h.n_tiles;
  c->stream_bytes = h.stream_bytes;
  c->raw_bytes = h.raw_bytes;
  const uint8_t* p = buf + sizeof(Header);
  c->freq = reinterpret_cast<const uint32_t*>(p);
  p += s.freq;
  c->offsets = reinterpret_cast<const uint64_t*>(p);
  p += s.offsets;
  c->stream = p;
  p += s.stream;
  c->raw = h.raw_bytes ? p : nullptr;
  return 0;
}

}  // namespace anshost
