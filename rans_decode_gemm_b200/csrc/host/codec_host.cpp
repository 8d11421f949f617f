// codec_host.cpp -- offline host side of the tile rANS codec: entropy,
// frequency normalisation and the multithreaded tile encoder.
//
// "Approaching Shannon Bound with Lossless LLM Weight Compression":
//   s2.1 per-layer histogram and Shannon entropy;
//   s3.1 offline stage: W is cut into GEMM-shaped tiles, every tile coded on
//        its own against one shared per-layer codebook, tile starts recorded
//        in an offset index, each tile split into 32 per-lane substreams;
//   s4.1 finite-precision frequency normalisation.
// The stream format is described in include/ans.h.
#include "codec_host.h"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <thread>
#include <vector>

namespace anshost {

namespace {

constexpr uint32_t kLanes = 32;
constexpr uint32_t kStateLow = 1u << 16;

// Element offset (relative to the tile origin, row-major in W) of every
// (step j, lane l) symbol, stored at j * 32 + l.
std::vector<uint64_t> lane_order(uint32_t tile_n, uint32_t tile_k, uint64_t K) {
  const uint32_t halves = tile_n / 128;
  const uint32_t steps = tile_n * tile_k / kLanes;
  std::vector<uint64_t> off(static_cast<size_t>(steps) * kLanes);
  for (uint32_t j = 0; j < steps; ++j) {
    const uint32_t g = j >> 3, kk = j & 7;
    const uint32_t i = g & 3, c = (g >> 2) & 1, h = (g >> 3) % halves, s = g / (8 * halves);
    for (uint32_t l = 0; l < kLanes; ++l) {
      const uint64_t row = l + 32 * (4 * h + i);
      const uint64_t col = 16 * s + 8 * c + kk;
      off[static_cast<size_t>(j) * kLanes + l] = row * K + col;
    }
  }
  return off;
}

// int4 pairs: element offset of the even element of every (step j, lane l)
// pair symbol, stored at j * 32 + l.  Eight steps of a lane cover 16
// consecutive columns of one row.
std::vector<uint64_t> lane_order_pairs(uint32_t tile_n, uint32_t tile_k, uint64_t K) {
  const uint32_t halves = tile_n / 128;
  const uint32_t steps = tile_n * tile_k / 2 / kLanes;
  std::vector<uint64_t> off(static_cast<size_t>(steps) * kLanes);
  for (uint32_t j = 0; j < steps; ++j) {
    const uint32_t g = j >> 3, kk = j & 7;
    const uint32_t i = g & 3, h = (g >> 2) % halves, s = g / (4 * halves);
    for (uint32_t l = 0; l < kLanes; ++l) {
      const uint64_t row = l + 32 * (4 * h + i);
      const uint64_t col = 16 * s + 2 * kk;
      off[static_cast<size_t>(j) * kLanes + l] = row * K + col;
    }
  }
  return off;
}

struct TileJob {
  bool wide;  // wide-state variant: 64-bit states, 32-bit words, one test per symbol pair
  uint32_t dtype;
  const uint8_t* w;
  uint64_t K;
  uint32_t tile_n, tile_k, n_kt;
  const std::vector<uint64_t>* order;
  uint32_t freq[256];
  uint32_t cdf[257];
};

// Codes one tile; appends its padded bytes to `out`.  Returns false if a
// symbol has zero frequency.
bool code_tile_wide(const TileJob& job, const std::vector<uint8_t>& sym, size_t S,
                    std::vector<uint8_t>& out, std::vector<uint32_t>& words);

bool code_tile(const TileJob& job, uint64_t t, std::vector<uint8_t>& out,
               std::vector<uint8_t>& sym, std::vector<uint16_t>& words,
               std::vector<uint32_t>& words32, uint8_t* raw_tile) {
  const uint64_t origin = (t / job.n_kt) * job.tile_n * job.K + (t % job.n_kt) * job.tile_k;
  const bool pairs = job.dtype == kInt4Pairs || job.dtype == kFp4Pairs;
  const size_t S = static_cast<size_t>(job.tile_n) * job.tile_k / (pairs ? 2 : 1);
  const std::vector<uint64_t>& order = *job.order;
  sym.resize(S);
  if (pairs) {
    const uint8_t flip = job.dtype == kInt4Pairs ? 0x88 : 0;  // fp4 pairs: the byte itself
    for (size_t q = 0; q < S; ++q) sym[q] = static_cast<uint8_t>(job.w[(origin + order[q]) >> 1] ^ flip);
  } else if (job.dtype == kInt4 || job.dtype == kFp4) {
    const uint8_t flip = job.dtype == kInt4 ? 8 : 0;  // int4: q + 8; fp4: the code
    for (size_t q = 0; q < S; ++q) {
      const uint64_t e = origin + order[q];
      const uint8_t b = job.w[e >> 1];
      sym[q] = static_cast<uint8_t>(((e & 1) ? (b >> 4) : (b & 15)) ^ flip);
    }
  } else if (job.dtype == kBf16Split) {
    const uint16_t* w16 = reinterpret_cast<const uint16_t*>(job.w);
    for (size_t q = 0; q < S; ++q) {
      const uint16_t b = w16[origin + order[q]];
      sym[q] = static_cast<uint8_t>(b >> 7);
      // raw byte of (j = q / 32, l = q % 32) at (j / 8) * 256 + l * 8 + j % 8
      const size_t j = q >> 5, l = q & 31;
      raw_tile[(j >> 3) * 256 + l * 8 + (j & 7)] =
          static_cast<uint8_t>(((b >> 8) & 0x80) | (b & 0x7F));
    }
  } else if (job.dtype == kInt8) {
    for (size_t q = 0; q < S; ++q) sym[q] = static_cast<uint8_t>(job.w[origin + order[q]] ^ 0x80);
  } else {
    for (size_t q = 0; q < S; ++q) sym[q] = job.w[origin + order[q]];
  }

  if (job.wide) return code_tile_wide(job, sym, S, out, words32);
  uint32_t x[kLanes];
  for (uint32_t l = 0; l < kLanes; ++l) x[l] = kStateLow;
  words.clear();
  for (size_t q = S; q-- > 0;) {  // last step first, highest lane first
    const uint32_t l = static_cast<uint32_t>(q & 31);
    const uint32_t s = sym[q];
    const uint32_t f = job.freq[s];
    if (f == 0) return false;
    uint32_t v = x[l];
    if (static_cast<uint64_t>(v) >= (static_cast<uint64_t>(f) << 20)) {
      words.push_back(static_cast<uint16_t>(v));
      v >>= 16;
    }
    x[l] = (v / f) * 4096u + (v % f) + job.cdf[s];
  }
  uint64_t x64[kLanes];
  for (uint32_t l = 0; l < kLanes; ++l) x64[l] = x[l];
  append_tile(out, x64, words);
  return true;
}

// Wide-state variant of one tile.  sym holds the tile's symbols in (step,
// lane) order.  Pairs of steps (2p, 2p + 1) are coded last pair first and,
// inside a pair step, highest lane first; a lane's state first gives up its low
// 32 bits if x >= 2^40 f_a f_b (tested as x >> 40 >= f_a f_b, exact because the
// bound is a multiple of 2^40), then takes b = step 2p + 1, then a = step 2p.
bool code_tile_wide(const TileJob& job, const std::vector<uint8_t>& sym, size_t S,
                    std::vector<uint8_t>& out, std::vector<uint32_t>& words) {
  uint64_t x[kLanes];
  for (uint32_t l = 0; l < kLanes; ++l) x[l] = 1ull << 32;
  words.clear();
  const size_t pairs = S / kLanes / 2;
  for (size_t p = pairs; p-- > 0;) {
    const uint8_t* sa = &sym[(2 * p) * kLanes];
    const uint8_t* sb = sa + kLanes;
    for (uint32_t l = kLanes; l-- > 0;) {
      const uint32_t fa = job.freq[sa[l]], fb = job.freq[sb[l]];
      if (fa == 0 || fb == 0) return false;
      uint64_t v = x[l];
      if ((v >> 40) >= static_cast<uint64_t>(fa) * fb) {
        words.push_back(static_cast<uint32_t>(v));
        v >>= 32;
      }
      v = (v / fb) * 4096u + (v % fb) + job.cdf[sb[l]];
      v = (v / fa) * 4096u + (v % fa) + job.cdf[sa[l]];
      x[l] = v;
    }
  }
  append_tile(out, x, words);
  return true;
}

// Tile bytes for either state width (Word = the renormalisation word).  A
// state x >= L needs (bit length + 7) / 8 bytes: 3..4 for 32-bit states
// (x >= 2^16), 5..8 for wide ones (x >= 2^32); the table stores that count
// minus the least, bit b of it in plane b.
template <typename Word>
void append_tile_impl(std::vector<uint8_t>& out, const uint64_t* x, const std::vector<Word>& pushed) {
  constexpr bool kWide = sizeof(Word) == 4;
  constexpr uint32_t kLeast = kWide ? 5 : 3, kTable = kWide ? 8 : 4;
  uint32_t len[kLanes], planes[2] = {0, 0};
  size_t states = 0;
  for (uint32_t l = 0; l < kLanes; ++l) {
    len[l] = (64u - static_cast<uint32_t>(__builtin_clzll(x[l])) + 7u) / 8u;
    const uint32_t extra = len[l] - kLeast;
    planes[0] |= (extra & 1u) << l;
    planes[1] |= (extra >> 1) << l;
    states += len[l];
  }
  const size_t head = (kTable + states + sizeof(Word) - 1) & ~(sizeof(Word) - 1);
  const size_t body = head + sizeof(Word) * pushed.size();
  const size_t base = out.size();
  out.resize(base + ((body + 15) & ~static_cast<size_t>(15)), 0);
  uint8_t* p = out.data() + base;
  std::memcpy(p, planes, kTable);  // little-endian host
  size_t at = kTable;
  for (uint32_t l = 0; l < kLanes; ++l) {
    std::memcpy(p + at, &x[l], len[l]);
    at += len[l];
  }
  for (size_t k = 0; k < pushed.size(); ++k) {
    const Word wv = pushed[pushed.size() - 1 - k];
    std::memcpy(p + head + sizeof(Word) * k, &wv, sizeof(Word));
  }
}

unsigned worker_count(uint64_t jobs) {
  unsigned n = std::thread::hardware_concurrency();
  if (n == 0) n = 1;
  if (n > jobs) n = static_cast<unsigned>(jobs == 0 ? 1 : jobs);
  return n;
}

}  // namespace

void append_tile(std::vector<uint8_t>& out, const uint64_t* x, const std::vector<uint16_t>& pushed) {
  append_tile_impl(out, x, pushed);
}

void append_tile(std::vector<uint8_t>& out, const uint64_t* x, const std::vector<uint32_t>& pushed) {
  append_tile_impl(out, x, pushed);
}

bool layout_valid(uint32_t N, uint32_t K, uint32_t tile_n, uint32_t tile_k) {
  return N > 0 && K > 0 && (tile_n == 128 || tile_n == 256) && tile_k > 0 && tile_k % 16 == 0 &&
         tile_k <= 256 && N % tile_n == 0 && K % tile_k == 0;
}

void histogram(uint32_t dtype, const void* w, uint64_t n_weights, uint64_t* hist) {
  const uint32_t A = (dtype == kInt4 || dtype == kFp4) ? 16 : 256;
  const uint64_t units = (dtype == kInt4 || dtype == kInt4Pairs || dtype == kFp4 || dtype == kFp4Pairs)
                             ? n_weights / 2 : n_weights;  // bytes or u16 words
  const unsigned nw = worker_count(units / 65536 + 1);
  std::vector<std::vector<uint64_t>> part(nw, std::vector<uint64_t>(256, 0));
  std::vector<std::thread> pool;
  for (unsigned k = 0; k < nw; ++k) {
    pool.emplace_back([&, k]() {
      const uint64_t a = units * k / nw, b = units * (k + 1) / nw;
      uint64_t* h = part[k].data();
      if (dtype == kInt4 || dtype == kFp4) {
        const uint8_t* p = static_cast<const uint8_t*>(w);
        const uint8_t flip = dtype == kInt4 ? 8 : 0;
        for (uint64_t i = a; i < b; ++i) { h[(p[i] & 15) ^ flip]++; h[(p[i] >> 4) ^ flip]++; }
      } else if (dtype == kInt4Pairs || dtype == kFp4Pairs) {
        const uint8_t* p = static_cast<const uint8_t*>(w);
        const uint8_t flip = dtype == kInt4Pairs ? 0x88 : 0;
        for (uint64_t i = a; i < b; ++i) h[p[i] ^ flip]++;
      } else if (dtype == kInt8) {
        const uint8_t* p = static_cast<const uint8_t*>(w);
        for (uint64_t i = a; i < b; ++i) h[p[i] ^ 0x80]++;
      } else if (dtype == kBf16Split) {
        const uint16_t* p = static_cast<const uint16_t*>(w);
        for (uint64_t i = a; i < b; ++i) h[(p[i] >> 7) & 0xFF]++;
      } else {
        const uint8_t* p = static_cast<const uint8_t*>(w);
        for (uint64_t i = a; i < b; ++i) h[p[i]]++;
      }
    });
  }
  for (auto& th : pool) th.join();
  for (uint32_t s = 0; s < A; ++s) {
    hist[s] = 0;
    for (unsigned k = 0; k < nw; ++k) hist[s] += part[k][s];
  }
}

double entropy_bits(const uint64_t* hist, uint32_t alphabet) {
  long double total = 0;
  for (uint32_t s = 0; s < alphabet; ++s) total += static_cast<long double>(hist[s]);
  if (total == 0) return 0.0;
  long double h = 0;
  for (uint32_t s = 0; s < alphabet; ++s) {
    if (!hist[s]) continue;
    const long double p = static_cast<long double>(hist[s]) / total;
    h -= p * log2l(p);
  }
  return static_cast<double>(h);
}

int normalize(const uint64_t* hist, uint32_t alphabet, uint32_t prob_bits, uint32_t* freq) {
  if (alphabet == 0 || alphabet > 256 || prob_bits < 1 || prob_bits > 15) return 1;
  const uint64_t target = 1ull << prob_bits;
  uint64_t total = 0, present = 0;
  for (uint32_t s = 0; s < alphabet; ++s) {
    total += hist[s];
    present += hist[s] ? 1 : 0;
  }
  if (total == 0) return 1;
  if (present > target) return 3;
  std::vector<uint64_t> f(alphabet, 0);
  uint64_t sum = 0;
  for (uint32_t s = 0; s < alphabet; ++s) {
    if (!hist[s]) continue;
    const uint64_t share = static_cast<uint64_t>(
        static_cast<unsigned __int128>(hist[s]) * target / total);
    f[s] = share > 0 ? share : 1;
    sum += f[s];
  }
  // saving of one more slot / cost of one slot fewer, c * log2((f+1)/f) and
  // c * log2(f/(f-1)), in long double.
  auto up = [&](uint32_t s) {
    return static_cast<long double>(hist[s]) *
           log2l((static_cast<long double>(f[s]) + 1.0L) / static_cast<long double>(f[s]));
  };
  auto down = [&](uint32_t s) {
    return static_cast<long double>(hist[s]) *
           log2l(static_cast<long double>(f[s]) / (static_cast<long double>(f[s]) - 1.0L));
  };
  auto best_up = [&]() {
    int b = -1;
    long double bv = 0;
    for (uint32_t s = 0; s < alphabet; ++s) {
      if (!hist[s]) continue;
      const long double v = up(s);
      if (b < 0 || v > bv) { b = static_cast<int>(s); bv = v; }
    }
    return b;
  };
  auto best_down = [&](int skip) {
    int b = -1;
    long double bv = 0;
    for (uint32_t s = 0; s < alphabet; ++s) {
      if (!hist[s] || f[s] <= 1 || static_cast<int>(s) == skip) continue;
      const long double v = down(s);
      if (b < 0 || v < bv) { b = static_cast<int>(s); bv = v; }
    }
    return b;
  };
  while (sum < target) { f[best_up()]++; sum++; }
  while (sum > target) { f[best_down(-1)]--; sum--; }
  for (;;) {
    const int a = best_up();
    const int b = best_down(a);
    if (a < 0 || b < 0 || !(up(a) > down(b))) break;
    f[a]++;
    f[b]--;
  }
  for (uint32_t s = 0; s < alphabet; ++s) freq[s] = static_cast<uint32_t>(f[s]);
  return 0;
}

uint64_t encode_bound(uint32_t N, uint32_t K, uint32_t tile_n, uint32_t tile_k, bool wide) {
  if (!layout_valid(N, K, tile_n, tile_k)) return 0;
  const uint64_t tiles = static_cast<uint64_t>(N / tile_n) * (K / tile_k);
  // length table, full-width states, word boundary; at most one word per
  // symbol (2 bytes) or per pair (4 bytes): 2 bytes a symbol; padding
  return tiles * ((wide ? 8ull : 4ull) * (kLanes + 1) + 4ull + 2ull * tile_n * tile_k + 16ull);
}

int encode(uint32_t dtype, const void* w, uint32_t N, uint32_t K, uint32_t tile_n,
           uint32_t tile_k, const uint32_t* freq, uint8_t* stream, uint64_t cap,
           uint64_t* stream_bytes, uint64_t* offsets, uint8_t* raw, bool wide) {
  const uint32_t n_kt = K / tile_k;
  const uint64_t tiles = static_cast<uint64_t>(N / tile_n) * n_kt;
  const std::vector<uint64_t> order =
      (dtype == kInt4Pairs || dtype == kFp4Pairs) ? lane_order_pairs(tile_n, tile_k, K)
                                                  : lane_order(tile_n, tile_k, K);
  TileJob job;
  job.wide = wide;
  job.dtype = dtype;
  job.w = static_cast<const uint8_t*>(w);
  job.K = K;
  job.tile_n = tile_n;
  job.tile_k = tile_k;
  job.n_kt = n_kt;
  job.order = &order;
  const uint32_t A = (dtype == kInt4 || dtype == kFp4) ? 16 : 256;
  uint32_t run = 0;
  for (uint32_t s = 0; s < 256; ++s) {
    job.freq[s] = s < A ? freq[s] : 0;
    job.cdf[s] = run;
    run += job.freq[s];
  }
  job.cdf[256] = run;
  const size_t S = static_cast<size_t>(tile_n) * tile_k;  // raw bytes per tile (bf16)

  const unsigned nw = worker_count(tiles);
  std::vector<std::vector<uint8_t>> bufs(nw);
  std::vector<std::vector<uint64_t>> sizes(nw);
  std::vector<int> ok(nw, 1);
  std::vector<std::thread> pool;
  for (unsigned w_i = 0; w_i < nw; ++w_i) {
    pool.emplace_back([&, w_i]() {
      const uint64_t a = tiles * w_i / nw, b = tiles * (w_i + 1) / nw;
      std::vector<uint8_t> sym;
      std::vector<uint16_t> words;
      std::vector<uint32_t> words32;
      words.reserve(S);
      for (uint64_t t = a; t < b; ++t) {
        const size_t before = bufs[w_i].size();
        uint8_t* raw_tile = (dtype == kBf16Split) ? raw + t * S : nullptr;
        if (!code_tile(job, t, bufs[w_i], sym, words, words32, raw_tile)) { ok[w_i] = 0; return; }
        sizes[w_i].push_back(bufs[w_i].size() - before);
      }
    });
  }
  for (auto& th : pool) th.join();
  for (unsigned w_i = 0; w_i < nw; ++w_i)
    if (!ok[w_i]) return 3;
  uint64_t pos = 0, t = 0;
  std::vector<uint64_t> starts(nw);
  for (unsigned w_i = 0; w_i < nw; ++w_i) {
    starts[w_i] = pos;
    for (uint64_t sz : sizes[w_i]) { offsets[t++] = pos; pos += sz; }
  }
  offsets[tiles] = pos;
  *stream_bytes = pos;
  if (pos > cap) return 4;
  std::vector<std::thread> copy;
  for (unsigned w_i = 0; w_i < nw; ++w_i)
    copy.emplace_back([&, w_i]() {
      if (!bufs[w_i].empty()) std::memcpy(stream + starts[w_i], bufs[w_i].data(), bufs[w_i].size());
    });
  for (auto& th : copy) th.join();
  return 0;
}

}  // namespace anshost
