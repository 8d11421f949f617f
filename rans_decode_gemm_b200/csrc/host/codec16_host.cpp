// codec16_host.cpp -- host side of bf16 coded as whole 16-bit symbols: the
// 65,536-bin histogram, normalisation to 2^n (n <= 16), the tile encoder and
// the decoder's lookup-table image.
//
// "Approaching Shannon Bound with Lossless LLM Weight Compression", s4.1
// ("压缩率"): bf16's symbol table is large, so the finite precision of the
// normalised frequencies costs more there than for low-bit formats.  The
// symbol is the whole 16-bit pattern; everything else (tiles, 32 lanes, lane
// map, state widths, word sizes, tile bytes) is the stream format of
// include/ans.h, with 2^n slots instead of 2^12.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <thread>
#include <vector>

#include "codec_host.h"

namespace anshost {

namespace {

constexpr uint32_t kLanes = 32;
constexpr uint32_t kA16 = 65536;

unsigned workers(uint64_t jobs) {
  unsigned n = std::thread::hardware_concurrency();
  if (n == 0) n = 1;
  if (n > jobs) n = static_cast<unsigned>(jobs == 0 ? 1 : jobs);
  return n;
}

// Element offset (from the tile origin) of every (step j, lane l) symbol, at
// j * 32 + l: the lane map of the one-symbol-per-element formats.
std::vector<uint64_t> lanes16(uint32_t tile_n, uint32_t tile_k, uint64_t K) {
  const uint32_t halves = tile_n / 128;
  const uint32_t steps = tile_n * tile_k / kLanes;
  std::vector<uint64_t> off(static_cast<size_t>(steps) * kLanes);
  for (uint32_t j = 0; j < steps; ++j) {
    const uint32_t g = j >> 3, kk = j & 7;
    const uint32_t i = g & 3, c = (g >> 2) & 1, h = (g >> 3) % halves, s = g / (8 * halves);
    for (uint32_t l = 0; l < kLanes; ++l)
      off[static_cast<size_t>(j) * kLanes + l] = (l + 32ull * (4 * h + i)) * K + 16 * s + 8 * c + kk;
  }
  return off;
}

// One tile, 32-bit lane states in [2^16, 2^32), 16-bit words: a lane pushes
// its low word before coding s if x >= f_s * 2^(32 - n).
bool tile16_narrow(const std::vector<uint16_t>& sym, const uint32_t* freq, const uint32_t* cdf,
                   uint32_t n, std::vector<uint16_t>& words, std::vector<uint8_t>& out) {
  uint32_t x[kLanes];
  for (uint32_t l = 0; l < kLanes; ++l) x[l] = 1u << 16;
  words.clear();
  for (size_t q = sym.size(); q-- > 0;) {
    const uint32_t l = static_cast<uint32_t>(q & 31), s = sym[q], f = freq[s];
    if (f == 0) return false;
    uint32_t v = x[l];
    if (static_cast<uint64_t>(v) >= (static_cast<uint64_t>(f) << (32 - n))) {
      words.push_back(static_cast<uint16_t>(v));
      v >>= 16;
    }
    x[l] = static_cast<uint32_t>((static_cast<uint64_t>(v / f) << n) + v % f + cdf[s]);
  }
  uint64_t x64[kLanes];
  for (uint32_t l = 0; l < kLanes; ++l) x64[l] = x[l];
  append_tile(out, x64, words);
  return true;
}

// One tile, wide states: 64-bit lane states in [2^32, 2^64), 32-bit words,
// pairs of steps (2p, 2p + 1) coded last pair first; a lane pushes its low
// word before a pair (a, b) if x >= f_a f_b 2^(64 - 2n).
bool tile16_wide(const std::vector<uint16_t>& sym, const uint32_t* freq, const uint32_t* cdf,
                 uint32_t n, std::vector<uint32_t>& words, std::vector<uint8_t>& out) {
  uint64_t x[kLanes];
  for (uint32_t l = 0; l < kLanes; ++l) x[l] = 1ull << 32;
  words.clear();
  const size_t pairs = sym.size() / kLanes / 2;
  for (size_t p = pairs; p-- > 0;) {
    const uint16_t* sa = &sym[(2 * p) * kLanes];
    const uint16_t* sb = sa + kLanes;
    for (uint32_t l = kLanes; l-- > 0;) {
      const uint32_t fa = freq[sa[l]], fb = freq[sb[l]];
      if (fa == 0 || fb == 0) return false;
      uint64_t v = x[l];
      // f_a f_b <= 2^32, and the bound is a multiple of 2^(64 - 2n)
      if ((v >> (64 - 2 * n)) >= static_cast<uint64_t>(fa) * fb) {
        words.push_back(static_cast<uint32_t>(v));
        v >>= 32;
      }
      v = ((v / fb) << n) + v % fb + cdf[sb[l]];
      v = ((v / fa) << n) + v % fa + cdf[sa[l]];
      x[l] = v;
    }
  }
  append_tile(out, x, words);
  return true;
}

}  // namespace

void histogram16(const uint16_t* w, uint64_t n_weights, uint64_t* hist) {
  const unsigned nw = workers(n_weights / 65536 + 1);
  std::vector<std::vector<uint64_t>> part(nw, std::vector<uint64_t>(kA16, 0));
  std::vector<std::thread> pool;
  for (unsigned k = 0; k < nw; ++k)
    pool.emplace_back([&, k]() {
      const uint64_t a = n_weights * k / nw, b = n_weights * (k + 1) / nw;
      uint64_t* h = part[k].data();
      for (uint64_t i = a; i < b; ++i) h[w[i]]++;
    });
  for (auto& th : pool) th.join();
  for (uint32_t s = 0; s < kA16; ++s) {
    hist[s] = 0;
    for (unsigned k = 0; k < nw; ++k) hist[s] += part[k][s];
  }
}

// The normalisation of normalize() (same objective, same greedy moves, ties
// towards the lower symbol), over the present symbols of a 65,536-symbol
// alphabet, with each symbol's gain and loss cached.
int normalize16(const uint64_t* hist, uint32_t prob_bits, uint32_t* freq) {
  if (prob_bits < 1 || prob_bits > 16) return 1;
  const uint64_t target = 1ull << prob_bits;
  std::vector<uint32_t> sym;
  uint64_t total = 0;
  for (uint32_t s = 0; s < kA16; ++s)
    if (hist[s]) {
      sym.push_back(s);
      total += hist[s];
    }
  if (total == 0) return 1;
  if (sym.size() > target) return 3;
  const size_t P = sym.size();
  std::vector<uint64_t> f(P);
  uint64_t sum = 0;
  for (size_t i = 0; i < P; ++i) {
    const uint64_t share =
        static_cast<uint64_t>(static_cast<unsigned __int128>(hist[sym[i]]) * target / total);
    f[i] = share > 0 ? share : 1;
    sum += f[i];
  }
  std::vector<long double> up(P), down(P);
  auto refresh = [&](size_t i) {
    const long double c = static_cast<long double>(hist[sym[i]]), fi = static_cast<long double>(f[i]);
    up[i] = c * log2l((fi + 1.0L) / fi);
    down[i] = f[i] > 1 ? c * log2l(fi / (fi - 1.0L)) : 0.0L;
  };
  for (size_t i = 0; i < P; ++i) refresh(i);
  auto best_up = [&]() {
    long best = -1;
    for (size_t i = 0; i < P; ++i)
      if (best < 0 || up[i] > up[best]) best = static_cast<long>(i);
    return best;
  };
  auto best_down = [&](long skip) {
    long best = -1;
    for (size_t i = 0; i < P; ++i) {
      if (f[i] <= 1 || static_cast<long>(i) == skip) continue;
      if (best < 0 || down[i] < down[best]) best = static_cast<long>(i);
    }
    return best;
  };
  while (sum < target) {
    const long a = best_up();
    f[a]++;
    refresh(a);
    sum++;
  }
  while (sum > target) {
    const long b = best_down(-1);
    f[b]--;
    refresh(b);
    sum--;
  }
  for (;;) {
    const long a = best_up();
    const long b = best_down(a);
    if (a < 0 || b < 0 || !(up[a] > down[b])) break;
    f[a]++;
    f[b]--;
    refresh(a);
    refresh(b);
  }
  std::memset(freq, 0, kA16 * sizeof(uint32_t));
  for (size_t i = 0; i < P; ++i) freq[sym[i]] = static_cast<uint32_t>(f[i]);
  return 0;
}

int encode16(const uint16_t* w, uint32_t N, uint32_t K, uint32_t tile_n, uint32_t tile_k,
             const uint32_t* freq, uint32_t prob_bits, uint8_t* stream, uint64_t cap,
             uint64_t* stream_bytes, uint64_t* offsets, bool wide) {
  if (prob_bits < 1 || prob_bits > 16) return 1;
  // the wide-state format is defined at 12 and 16 bits of precision only
  if (wide && prob_bits != 12 && prob_bits != 16) return 1;
  std::vector<uint32_t> cdf(kA16 + 1, 0);
  uint64_t run = 0;
  for (uint32_t s = 0; s < kA16; ++s) {
    cdf[s] = static_cast<uint32_t>(run);
    run += freq[s];
  }
  if (run != (1ull << prob_bits)) return 3;
  cdf[kA16] = static_cast<uint32_t>(run);
  const uint32_t n_kt = K / tile_k;
  const uint64_t tiles = static_cast<uint64_t>(N / tile_n) * n_kt;
  const std::vector<uint64_t> order = lanes16(tile_n, tile_k, K);
  const size_t S = static_cast<size_t>(tile_n) * tile_k;
  const unsigned nw = workers(tiles);
  std::vector<std::vector<uint8_t>> bufs(nw);
  std::vector<std::vector<uint64_t>> sizes(nw);
  std::vector<int> ok(nw, 1);
  std::vector<std::thread> pool;
  for (unsigned k = 0; k < nw; ++k)
    pool.emplace_back([&, k]() {
      const uint64_t a = tiles * k / nw, b = tiles * (k + 1) / nw;
      std::vector<uint16_t> sym(S), words16;
      std::vector<uint32_t> words32;
      for (uint64_t t = a; t < b; ++t) {
        const uint64_t origin = (t / n_kt) * tile_n * static_cast<uint64_t>(K) + (t % n_kt) * tile_k;
        for (size_t q = 0; q < S; ++q) sym[q] = w[origin + order[q]];
        const size_t before = bufs[k].size();
        const bool good = wide ? tile16_wide(sym, freq, cdf.data(), prob_bits, words32, bufs[k])
                               : tile16_narrow(sym, freq, cdf.data(), prob_bits, words16, bufs[k]);
        if (!good) {
          ok[k] = 0;
          return;
        }
        sizes[k].push_back(bufs[k].size() - before);
      }
    });
  for (auto& th : pool) th.join();
  for (unsigned k = 0; k < nw; ++k)
    if (!ok[k]) return 3;
  uint64_t pos = 0, t = 0;
  for (unsigned k = 0; k < nw; ++k)
    for (uint64_t sz : sizes[k]) {
      offsets[t++] = pos;
      pos += sz;
    }
  offsets[tiles] = pos;
  *stream_bytes = pos;
  if (pos > cap) return 4;
  pos = 0;
  for (unsigned k = 0; k < nw; ++k) {
    if (!bufs[k].empty()) std::memcpy(stream + pos, bufs[k].data(), bufs[k].size());
    pos += bufs[k].size();
  }
  return 0;
}

// Decoder table image: [u32 n_present][u32 prob_bits][u16 first[4096]]
// [u32 entry[n_present]][u16 symbol[n_present]], zero-padded to 16 bytes.
// The present symbols in increasing order; entry = cdf | (f - 1) << 16;
// first[b] = the first present symbol whose slot range reaches slot
// b << (n - 12).  The decoder finds the symbol of slot x from first[x >> (n -
// 12)], stepping forward while x lies past the entry's range.
uint64_t table16_bytes(const uint32_t* freq) {
  uint64_t present = 0;
  for (uint32_t s = 0; s < kA16; ++s) present += freq[s] ? 1 : 0;
  return (8 + 2 * 4096 + 6 * present + 15) & ~uint64_t(15);
}

int table16(const uint32_t* freq, uint32_t prob_bits, uint8_t* out, uint64_t bytes) {
  if (prob_bits < 12 || prob_bits > 16) return 1;
  const uint64_t need = table16_bytes(freq);
  if (bytes < need) return 4;
  std::memset(out, 0, need);
  std::vector<uint32_t> ent;
  std::vector<uint16_t> syms;
  uint64_t run = 0;
  for (uint32_t s = 0; s < kA16; ++s) {
    if (!freq[s]) continue;
    if (freq[s] > 65536 || run > 65535) return 3;
    ent.push_back(static_cast<uint32_t>(run) | ((freq[s] - 1) << 16));
    syms.push_back(static_cast<uint16_t>(s));
    run += freq[s];
  }
  if (run != (1ull << prob_bits)) return 3;
  const uint32_t n_present = static_cast<uint32_t>(ent.size());
  std::memcpy(out, &n_present, 4);
  std::memcpy(out + 4, &prob_bits, 4);
  uint16_t* first = reinterpret_cast<uint16_t*>(out + 8);
  const uint32_t shift = prob_bits - 12;
  uint32_t k = 0;
  for (uint32_t b = 0; b < 4096; ++b) {
    const uint32_t slot = b << shift;
    while ((ent[k] & 0xFFFFu) + (ent[k] >> 16) < slot) ++k;  // last slot of k = cdf + f - 1
    first[b] = static_cast<uint16_t>(k);
  }
  std::memcpy(out + 8 + 2 * 4096, ent.data(), 4ull * n_present);
  std::memcpy(out + 8 + 2 * 4096 + 4ull * n_present, syms.data(), 2ull * n_present);
  return 0;
}

}  // namespace anshost
