// ans_oracle.cpp -- plain, slow, obviously-correct CPU oracle for tile-granular
// rANS weight coding and the dequantised GEMM that consumes the weights.
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the C-ABI library,
// its Python binding, the CUDA kernels) may include, link, import or call this
// file.  Only the test-suite, the smoke check and the CPU-baseline leg of the
// benchmark use it.  It shares no code, header, table or constant generator
// with the product; the two meet only through the seeded input generators and
// through the byte format, which both implement from its written definition.
//
// Sources (page title, section):
//   [SB]   "Approaching Shannon Bound with Lossless LLM Weight Compression"
//          (blog summary, marsggbo.github.io, 2026-07-22):
//          s2.1 "熵分析：逐层算直方图" (per-layer histogram + Shannon entropy),
//          s2.2 "为什么大家不用无损压缩？" (rANS chosen: >99% entropy efficiency,
//               byte-level streaming decode; tile-granular random access),
//          s3.1 "整体执行模型" (GEMM-shaped tiles, one shared codebook per
//               layer, tile offset index, R interleaved substreams with one
//               rANS state per warp lane),
//          s4.1 "压缩率" (finite-precision frequency normalisation).
//   [DF11] "70%大小，100%准确！完美压缩LLM性能0损失..." (aizws.net summary of
//          DFloat11): "实验方法" (Shannon entropy H of a discrete variable;
//          bf16 exponent carries ~2.6 bits, sign+mantissa near full width),
//          "无损LLM压缩框架，实现高效GPU推理" (exponent entropy-coded; sign and
//          mantissa kept raw in a separate PackedSignMantissa byte array).
//   [TERN] "突破1.58比特极限：三元LLM如何逼近信息论边界" (kongchang.com),
//          "三元大模型的量化前沿" (uniform ternary entropy = log2 3).
//
// The pages print no rANS formula (their formulas were lost in extraction), so
// the coder below is the textbook range-variant ANS with the constants that the
// pages leave open fixed as follows (the "readings"):
//   probability precision n = 12 (M = 2^n = 4096 frequency slots),
//   32-bit state x kept in [L, L*b) with L = 2^16 and renormalisation base
//   b = 2^16 (16-bit words), 32 lanes per tile, one state per lane, all lanes
//   sharing one interleaved word stream consumed in increasing lane order.
// Byte format of one tile (the final-state flush is left open by the pages;
// the reading taken is a variable-length one): a length table, then each
// lane's final encoder state in lane order, little-endian, in the fewest whole
// bytes that hold it (x >= L = 2^16, so 3 or 4 bytes), then zero bytes up to a
// word boundary (2 bytes), then the u16 words in decoder consumption order,
// then zero bytes up to a 16-byte boundary.  The length table is one
// little-endian u32 whose bit l is set when lane l's state takes 4 bytes.
//
// Wide-state variant (state_bits = 64; the same pages leave the state width
// open): 64-bit state x in [L, L*b) with L = 2^32 and b = 2^32 (32-bit words),
// and the renormalisation test made once per PAIR of consecutive symbols of a
// lane (steps 2i and 2i+1) instead of once per symbol.  Decoding two symbols
// from x >= 2^32 leaves x >= 2^8 (each step divides by at most 2^12), so one
// 32-bit word always restores x >= L.  Encoder side, for a pair (a, b) coded
// in reverse (b first, then a): the state must lie in
// [(L >> 2n) f_a f_b, (L >> 2n) b f_a f_b) = [2^8 f_a f_b, 2^40 f_a f_b), so
// one word is pushed first if x >= 2^40 f_a f_b.  Tile bytes as above with
// states of 5 to 8 bytes (x >= 2^32), a length table of two little-endian u32
// bit planes (lane l takes 5 + bit l of the first + 2 x bit l of the second
// bytes), word boundary and words of 4 bytes.
//
// fp4 (dtype 5; [SB] s2.1 lists fp4 among the seven formats measured): e2m1
// codes stored like int4 (two per byte, element k even in the low nibble),
// symbol = the code (alphabet 16), value e2m1 times an optional per-row scale.
//
// bf16 whole (dtype 7; [SB] s4.1 implies bf16 coded as 16-bit symbols): the
// 16-bit pattern is the symbol (alphabet 65536, probability precision up to
// n = 16); the wide-state pair bound is 2^(64 - 2n) f_a f_b, so it holds for
// n = 16 as well (two steps from x >= 2^32 leave x >= 1, and one 32-bit word
// restores x >= 2^32).
//
// fp4 pairs (dtype 6): fp4 codes coded one symbol per packed byte, the byte
// itself (alphabet 256), in the int4 pairs' lane map.
//
// int8 (dtype 4; [SB] s2.1 lists int8 among the seven formats measured): one byte per
// weight, two's complement q in [-128, 127], symbol q + 128, alphabet 256;
// value q times an optional per-row scale.
//
// int4 pairs (dtype 3; the pages call any discrete unit of a layer a symbol and
// leave the unit open): one symbol per packed int4 byte, i.e. per pair of
// consecutive K elements (k even, k + 1): s = (q_k + 8) | (q_{k+1} + 8) << 4,
// which is the packed byte XOR 0x88; alphabet 256, half as many symbols per
// tile.  Lane l's j-th pair symbol covers row l + 32 (4 h + i) and columns
// 16 s + 2 kk, 16 s + 2 kk + 1 with g = j / 8, kk = j % 8, i = g % 4,
// h = (g / 4) % (tile_n / 128), s = g / (4 tile_n / 128).
//
// Build: g++ -O2 -std=c++17 -shared -fPIC -pthread ans_oracle.cpp -o liboracle.so

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

enum {
  DT_INT4 = 0,
  DT_BF16_SPLIT = 1,
  DT_FP8_E4M3 = 2,
  DT_INT4_PAIRS = 3,
  DT_INT8 = 4,
  DT_FP4_E2M1 = 5,
  DT_FP4_PAIRS = 6,
  DT_BF16_WHOLE = 7
};
enum { SC_NONE = 0, SC_ROW_BF16 = 1, SC_ROW_F32 = 2, SC_GROUP_BF16 = 3 };
enum {
  OK = 0, ERR_ARG = 1, ERR_SHAPE = 2, ERR_ALPHABET = 3, ERR_BUFFER_TOO_SMALL = 4,
  ERR_CORRUPT = 6
};

const uint32_t kLanes = 32;          // substreams per tile, one per warp lane
const uint64_t kL = 1ull << 16;      // lower bound of the state interval
const uint32_t kWordBits = 16;       // renormalisation word width (b = 2^16)
const uint64_t kLWide = 1ull << 32;  // wide variant: lower bound of the state interval
const uint32_t kWideWordBits = 32;   // wide variant: renormalisation word width (b = 2^32)

int alphabet_of(int dtype) {
  if (dtype == DT_BF16_WHOLE) return 65536;
  return (dtype == DT_INT4 || dtype == DT_FP4_E2M1) ? 16 : 256;
}
// packed two per byte, element k even in the low nibble
bool is_nibble(int dtype) {
  return dtype == DT_INT4 || dtype == DT_INT4_PAIRS || dtype == DT_FP4_E2M1 || dtype == DT_FP4_PAIRS;
}
// one symbol per packed byte (two consecutive K elements)
bool is_pairs(int dtype) { return dtype == DT_INT4_PAIRS || dtype == DT_FP4_PAIRS; }
bool is_fp4(int dtype) { return dtype == DT_FP4_E2M1 || dtype == DT_FP4_PAIRS; }
bool is_int4(int dtype) { return dtype == DT_INT4 || dtype == DT_INT4_PAIRS; }

// ---- 1. Symbols: what is treated as "a sequence of discrete symbols" ---------
// [SB s2.1]: a layer is a sequence of symbols (int4 value, fp8 code, ...).
// [DF11 framework]: for bf16 only the exponent is entropy coded; sign and
// mantissa stay raw.
//   int4 : packed two per byte, element k even in the low nibble; the stored
//          nibble is the two's-complement code q in [-8, 7]; symbol = q + 8.
//   bf16 : symbol = exponent byte e = (bits >> 7) & 0xFF;
//          raw byte = sign << 7 | mantissa (7 bits).
//   fp8  : symbol = the e4m3 code byte.
int int4_code(const uint8_t* w, uint64_t idx) {
  uint8_t byte = w[idx / 2];
  int nib = (idx % 2 == 0) ? (byte & 0xF) : (byte >> 4);
  return nib >= 8 ? nib - 16 : nib;
}

// int4 pairs (the "higher-rate" reading of a symbol): one symbol per pair of
// consecutive K elements (idx even), low nibble = the even element's code + 8,
// high nibble = the odd element's code + 8; alphabet 256.
uint32_t pair_symbol_at(const void* w, uint64_t idx) {
  uint32_t lo = (uint32_t)(int4_code((const uint8_t*)w, idx) + 8);
  uint32_t hi = (uint32_t)(int4_code((const uint8_t*)w, idx + 1) + 8);
  return lo | (hi << 4);
}
uint32_t symbol_at(int dtype, const void* w, uint64_t idx) {
  if (dtype == DT_INT4) return (uint32_t)(int4_code((const uint8_t*)w, idx) + 8);
  if (dtype == DT_INT4_PAIRS) return pair_symbol_at(w, idx);
  // fp4 pairs: the packed byte itself (low nibble: the even element's code)
  if (dtype == DT_FP4_PAIRS) return ((const uint8_t*)w)[idx / 2];
  // fp4 e2m1: the 4-bit code itself
  if (dtype == DT_FP4_E2M1) {
    const uint8_t byte = ((const uint8_t*)w)[idx / 2];
    return (idx % 2 == 0) ? (byte & 0xF) : (byte >> 4);
  }
  // int8: two's complement code q in [-128, 127]; symbol q + 128 (the byte
  // with its top bit flipped)
  if (dtype == DT_INT8) return (uint32_t)((int)(int8_t)((const uint8_t*)w)[idx] + 128);
  if (dtype == DT_BF16_WHOLE) return ((const uint16_t*)w)[idx];  // the whole 16-bit pattern
  if (dtype == DT_BF16_SPLIT) {
    uint16_t bits = ((const uint16_t*)w)[idx];
    return (bits >> 7) & 0xFFu;
  }
  return ((const uint8_t*)w)[idx];
}

uint8_t bf16_raw_byte(uint16_t bits) {
  uint32_t sign = (bits >> 15) & 1u;
  uint32_t mant = bits & 0x7Fu;
  return (uint8_t)((sign << 7) | mant);
}

uint16_t bf16_from_parts(uint32_t exponent, uint8_t raw) {
  uint32_t sign = (raw >> 7) & 1u;
  uint32_t mant = raw & 0x7Fu;
  return (uint16_t)((sign << 15) | (exponent << 7) | mant);
}

// ---- 4/5. Tiling and lane map -------------------------------------------------
// [SB s3.1]: W is cut into tiles shaped like the consuming GEMM's tiles; every
// tile is coded on its own; each tile is split into 32 substreams, one per lane.
// Tile t = rb * (K / tile_k) + kt covers rows [rb*tile_n, +tile_n) of W (the
// output / N axis) and columns [kt*tile_k, +tile_k) (the K axis).
// Lane l's j-th symbol: g = j / 8 (a group of 8 consecutive K elements),
// kk = j % 8; with H = tile_n / 128 row halves,
//   i = g % 4, c = (g / 4) % 2, h = (g / 8) % H, s = g / (8 H),
//   row = l + 32 (4 h + i),  col = 16 s + 8 c + kk.
// So every 64 steps a 128-row x 16-column slab of the tile is complete.
void lane_map(uint32_t tile_n, uint32_t l, uint32_t j, uint32_t* row, uint32_t* col) {
  uint32_t g = j / 8, kk = j % 8;
  uint32_t H = tile_n / 128;
  uint32_t i = g % 4;
  uint32_t c = (g / 4) % 2;
  uint32_t h = (g / 8) % H;
  uint32_t s = g / (8 * H);
  *row = l + 32 * (4 * h + i);
  *col = 16 * s + 8 * c + kk;
}

// int4 pairs: lane l's j-th symbol covers the two elements at (row, col) and
// (row, col + 1): g = j / 8, kk = j % 8, i = g % 4, h = (g / 4) % H,
// s = g / (4 H); row = l + 32 (4 h + i), col = 16 s + 2 kk.  Eight symbols of a
// lane are 16 consecutive K elements of one row, so every 32 steps a 128-row
// x 16-column slab is complete.
void lane_map_pairs(uint32_t tile_n, uint32_t l, uint32_t j, uint32_t* row, uint32_t* col) {
  uint32_t g = j / 8, kk = j % 8;
  uint32_t H = tile_n / 128;
  uint32_t i = g % 4;
  uint32_t h = (g / 4) % H;
  uint32_t s = g / (4 * H);
  *row = l + 32 * (4 * h + i);
  *col = 16 * s + 2 * kk;
}

bool layout_ok(uint32_t N, uint32_t K, uint32_t tile_n, uint32_t tile_k) {
  if (N == 0 || K == 0) return false;
  if (tile_n != 128 && tile_n != 256) return false;
  if (tile_k == 0 || tile_k % 16 != 0 || tile_k > 256) return false;
  if (N % tile_n != 0 || K % tile_k != 0) return false;
  return true;
}

struct Codebook {
  uint32_t M = 0, n = 0;
  std::vector<uint32_t> f, c;        // frequency and cumulative frequency
  std::vector<int> slot_symbol;      // slot -> symbol (inverse of c/f), -1 if none
};

int make_codebook(const uint32_t* freq, int A, int prob_bits, Codebook* cb) {
  if (prob_bits < 1 || prob_bits > 16 || A < 1 || A > 65536) return ERR_ARG;
  cb->n = (uint32_t)prob_bits;
  cb->M = 1u << prob_bits;
  cb->f.assign(freq, freq + A);
  cb->c.assign(A + 1, 0);
  uint64_t sum = 0;
  for (int s = 0; s < A; ++s) { cb->c[s] = (uint32_t)sum; sum += freq[s]; }
  cb->c[A] = (uint32_t)sum;
  if (sum != cb->M) return ERR_ALPHABET;
  cb->slot_symbol.assign(cb->M, -1);
  for (int s = 0; s < A; ++s)
    for (uint32_t slot = cb->c[s]; slot < cb->c[s] + cb->f[s]; ++slot) cb->slot_symbol[slot] = s;
  return OK;
}

// ---- 6. rANS encode step (textbook; [SB s2.2] picks rANS) -------------------
// Before coding s the state must lie in [ (L >> n) f_s, (L >> n) b f_s ); if it
// is at or above the top, one 16-bit word (the low bits) is emitted first.
// Then x <- floor(x / f_s) M + (x mod f_s) + c_s.
uint64_t encode_step(uint64_t x, uint32_t f, uint32_t c, const Codebook& cb,
                     std::vector<uint16_t>* pushed) {
  uint64_t x_max = ((kL >> cb.n) << kWordBits) * (uint64_t)f;
  if (x >= x_max) {
    pushed->push_back((uint16_t)(x & 0xFFFFu));
    x >>= kWordBits;
  }
  return (x / f) * cb.M + (x % f) + c;
}

// Decode step: slot = x mod M selects s with c_s <= slot < c_s + f_s, then
// x <- f_s floor(x / M) + slot - c_s; a word is read afterwards if x < L.
uint64_t decode_symbol(uint64_t x, const Codebook& cb, int* sym) {
  uint32_t slot = (uint32_t)(x & (cb.M - 1));
  int s = cb.slot_symbol[slot];
  *sym = s;
  return (uint64_t)cb.f[s] * (x >> cb.n) + slot - cb.c[s];
}

// Wide variant, one pair (a = the earlier symbol, b = the later one) coded in
// reverse: push one 32-bit word if x >= 2^(64 - 2n) f_a f_b (2^40 f_a f_b for
// n = 12; compared in 128 bits: the bound is 2^64 when f_a = f_b = M), then
// code b, then a.
uint64_t encode_pair_wide(uint64_t x, uint32_t fa, uint32_t ca, uint32_t fb, uint32_t cb_,
                          const Codebook& cb, std::vector<uint32_t>* pushed) {
  unsigned __int128 x_max = ((unsigned __int128)fa * fb) << (64 - 2 * cb.n);
  if ((unsigned __int128)x >= x_max) {
    pushed->push_back((uint32_t)(x & 0xFFFFFFFFull));
    x >>= kWideWordBits;
  }
  x = (x / fb) * cb.M + (x % fb) + cb_;
  x = (x / fa) * cb.M + (x % fa) + ca;
  return x;
}

struct Layout {
  int dtype;
  uint32_t N, K, tile_n, tile_k;
  int state_bits;  // 32, or 64 for the wide-state variant
  uint64_t n_tiles() const { return (uint64_t)(N / tile_n) * (K / tile_k); }
  uint64_t tile_symbols() const { return (uint64_t)tile_n * tile_k / (is_pairs(dtype) ? 2 : 1); }
  uint64_t tile_weights() const { return (uint64_t)tile_n * tile_k; }
};

// ---- Final-state flush --------------------------------------------------------
// Byte count of a final state: the fewest whole bytes that hold x (x >= L, so
// at least 3 for 32-bit states and 5 for 64-bit ones).
uint32_t flush_bytes(uint64_t x) {
  uint32_t n = 0;
  while (x != 0) { ++n; x >>= 8; }
  return n;
}

// Appends the length table, the 32 final states and the zero bytes up to the
// word boundary to an empty `out`.
void put_final_states(const uint64_t* x, bool wide, std::vector<uint8_t>* out) {
  const uint32_t least = wide ? 5 : 3, planes = wide ? 2 : 1, word = wide ? 4 : 2;
  uint32_t plane[2] = {0, 0};
  for (uint32_t l = 0; l < kLanes; ++l) {
    const uint32_t extra = flush_bytes(x[l]) - least;  // 0..1 or 0..3
    plane[0] |= (extra & 1u) << l;
    plane[1] |= (extra >> 1) << l;
  }
  for (uint32_t p = 0; p < planes; ++p)
    for (int b = 0; b < 4; ++b) out->push_back((uint8_t)(plane[p] >> (8 * b)));
  for (uint32_t l = 0; l < kLanes; ++l)
    for (uint32_t b = 0; b < flush_bytes(x[l]); ++b) out->push_back((uint8_t)(x[l] >> (8 * b)));
  while (out->size() % word != 0) out->push_back(0);
}

// Reads the length table and the final states of a tile of `len` bytes.
// Returns the offset of the first word, or 0 when the table points past the
// tile or the word-boundary bytes are not zero.
uint64_t get_final_states(const uint8_t* tile, uint64_t len, bool wide, uint64_t* x) {
  const uint32_t least = wide ? 5 : 3, planes = wide ? 2 : 1, word = wide ? 4 : 2;
  if (len < 4 * planes) return 0;
  uint32_t plane[2] = {0, 0};
  for (uint32_t p = 0; p < planes; ++p)
    for (int b = 0; b < 4; ++b) plane[p] |= (uint32_t)tile[4 * p + b] << (8 * b);
  uint64_t pos = 4 * planes;
  for (uint32_t l = 0; l < kLanes; ++l) {
    const uint32_t n = least + ((plane[0] >> l) & 1u) + 2 * ((plane[1] >> l) & 1u);
    if (pos + n > len) return 0;
    uint64_t v = 0;
    for (uint32_t b = 0; b < n; ++b) v |= (uint64_t)tile[pos + b] << (8 * b);
    x[l] = v;
    pos += n;
  }
  for (; pos % word != 0; ++pos)
    if (pos >= len || tile[pos] != 0) return 0;
  return pos;
}

// Encode one tile into `out` (states, words, padding).  Returns OK or
// ERR_ALPHABET when a symbol has no frequency in the codebook.
int encode_tile(const Layout& lay, const void* w, const Codebook& cb, uint64_t t,
                std::vector<uint8_t>* out, uint8_t* raw_tile) {
  const uint32_t kt_count = lay.K / lay.tile_k;
  const uint64_t n0 = (t / kt_count) * lay.tile_n;
  const uint64_t k0 = (t % kt_count) * lay.tile_k;
  const uint32_t steps = (uint32_t)(lay.tile_symbols() / kLanes);
  const bool wide = lay.state_bits == 64;
  auto sym_of = [&](uint32_t l, uint32_t j) {
    uint32_t row, col;
    if (is_pairs(lay.dtype)) lane_map_pairs(lay.tile_n, l, j, &row, &col);
    else lane_map(lay.tile_n, l, j, &row, &col);
    return symbol_at(lay.dtype, w, (n0 + row) * lay.K + (k0 + col));
  };
  uint64_t x[kLanes];
  for (uint32_t l = 0; l < kLanes; ++l) x[l] = wide ? kLWide : kL;
  std::vector<uint16_t> pushed;
  std::vector<uint32_t> pushed32;
  // Reverse order: last step first, and inside a step the highest lane first,
  // so that the decoder (first step first, lowest lane first) meets the words
  // in the reverse of the order in which they were pushed.  The wide variant
  // walks pairs of steps (2i, 2i + 1) the same way.
  if (!wide) {
    for (uint32_t jj = steps; jj-- > 0;) {
      for (uint32_t ll = kLanes; ll-- > 0;) {
        uint32_t s = sym_of(ll, jj);
        if (s >= cb.f.size() || cb.f[s] == 0) return ERR_ALPHABET;
        x[ll] = encode_step(x[ll], cb.f[s], cb.c[s], cb, &pushed);
      }
    }
  } else {
    for (uint32_t ii = steps / 2; ii-- > 0;) {
      for (uint32_t ll = kLanes; ll-- > 0;) {
        uint32_t sa = sym_of(ll, 2 * ii), sb = sym_of(ll, 2 * ii + 1);
        if (sa >= cb.f.size() || cb.f[sa] == 0 || sb >= cb.f.size() || cb.f[sb] == 0)
          return ERR_ALPHABET;
        x[ll] = encode_pair_wide(x[ll], cb.f[sa], cb.c[sa], cb.f[sb], cb.c[sb], cb, &pushed32);
      }
    }
  }
  out->clear();
  put_final_states(x, wide, out);
  for (size_t q = pushed.size(); q-- > 0;) {
    out->push_back((uint8_t)(pushed[q] & 0xFF));
    out->push_back((uint8_t)(pushed[q] >> 8));
  }
  for (size_t q = pushed32.size(); q-- > 0;)
    for (int b = 0; b < 4; ++b) out->push_back((uint8_t)((pushed32[q] >> (8 * b)) & 0xFF));
  while (out->size() % 16 != 0) out->push_back(0);
  // ---- 8. raw side stream (bf16): per tile, byte of (lane l, step j) at
  //         (j / 8) * 256 + l * 8 + (j % 8).
  if (lay.dtype == DT_BF16_SPLIT && raw_tile != nullptr) {
    for (uint32_t jj = 0; jj < steps; ++jj)
      for (uint32_t l = 0; l < kLanes; ++l) {
        uint32_t row, col;
        lane_map(lay.tile_n, l, jj, &row, &col);
        uint64_t idx = (n0 + row) * lay.K + (k0 + col);
        raw_tile[(jj / 8) * 256 + l * 8 + (jj % 8)] = bf16_raw_byte(((const uint16_t*)w)[idx]);
      }
  }
  return OK;
}

int resolve_threads(int threads) {
  if (threads > 0) return threads;
  unsigned h = std::thread::hardware_concurrency();
  return h == 0 ? 1 : (int)h;
}

template <class F>
void parallel_for(uint64_t begin, uint64_t end, int threads, F fn) {
  threads = resolve_threads(threads);
  if (end <= begin) return;
  uint64_t n = end - begin;
  if ((uint64_t)threads > n) threads = (int)n;
  std::vector<std::thread> pool;
  for (int w = 0; w < threads; ++w) {
    uint64_t a = begin + n * w / threads, b = begin + n * (w + 1) / threads;
    pool.emplace_back([=]() { for (uint64_t i = a; i < b; ++i) fn(i); });
  }
  for (auto& th : pool) th.join();
}

// e4m3fn value from the format definition: 1 sign, 4 exponent (bias 7),
// 3 mantissa bits; no infinities; S.1111.111 is NaN; exponent 0 is
// subnormal with value m * 2^-9.
double e4m3_value(uint8_t code) {
  int sign = code >> 7;
  int E = (code >> 3) & 0xF;
  int m = code & 0x7;
  if (E == 15 && m == 7) return std::nan("");
  double v = (E == 0) ? std::ldexp((double)m, -9) : std::ldexp(1.0 + m / 8.0, E - 7);
  return sign ? -v : v;
}

// fp4 e2m1 value from the format definition: 1 sign, 2 exponent (bias 1),
// 1 mantissa bit; exponent 0 is subnormal with value m * 0.5; no inf or NaN.
double e2m1_value(uint8_t code) {
  int sign = (code >> 3) & 1;
  int E = (code >> 1) & 3;
  int m = code & 1;
  double v = (E == 0) ? 0.5 * m : std::ldexp(1.0 + m / 2.0, E - 1);
  return sign ? -v : v;
}

double bf16_value(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

double f32_value(const void* p, uint64_t i) {
  float f;
  std::memcpy(&f, (const uint8_t*)p + 4 * i, 4);
  return (double)f;
}

}  // namespace

extern "C" {

int oracle_alphabet_size(int dtype) { return alphabet_of(dtype); }

double oracle_e4m3_value(uint8_t code) { return e4m3_value(code); }

double oracle_e2m1_value(uint8_t code) { return e2m1_value(code); }

// ---- 2. Histogram and Shannon entropy ([SB s2.1], [DF11 实验方法]) -----------
void oracle_histogram(int dtype, const void* w, uint64_t n_weights, uint64_t* counts) {
  int A = alphabet_of(dtype);
  for (int s = 0; s < A; ++s) counts[s] = 0;
  const uint64_t step = is_pairs(dtype) ? 2 : 1;  // one pair symbol per 2 weights
  for (uint64_t i = 0; i + step <= n_weights; i += step) counts[symbol_at(dtype, w, i)]++;
}

// Histogram of the raw sign/mantissa byte of bf16 weights (256 bins).
void oracle_histogram_bf16_raw(const uint16_t* w, uint64_t n_weights, uint64_t* counts) {
  for (int s = 0; s < 256; ++s) counts[s] = 0;
  for (uint64_t i = 0; i < n_weights; ++i) counts[bf16_raw_byte(w[i])]++;
}

// H = -sum_s p_s log2 p_s with p_s = c_s / sum(c); absent symbols contribute 0.
double oracle_entropy(const uint64_t* counts, int A) {
  long double total = 0;
  for (int s = 0; s < A; ++s) total += (long double)counts[s];
  if (total == 0) return 0.0;
  long double H = 0;
  for (int s = 0; s < A; ++s) {
    if (counts[s] == 0) continue;
    long double p = (long double)counts[s] / total;
    H -= p * log2l(p);
  }
  return (double)H;
}

// ---- 3. Frequency normalisation to 2^prob_bits ([SB s4.1]) -----------------
// Integer f_s summing to M with f_s >= 1 exactly for the present symbols, chosen
// to minimise the coded size sum_s c_s log2(M / f_s).  The cost is separable
// and convex, so: start at max(1, floor(c_s M / N)), add single units where the
// saving c_s log2((f_s+1)/f_s) is largest (or remove where the extra cost
// c_s log2(f_s/(f_s-1)) is smallest) until the sum is M, then move single units
// while a move still lowers the cost.  Ties go to the lower symbol index.
// Gains are evaluated as c * log2l((f + 1.0L) / f) in long double.
int oracle_normalize(const uint64_t* counts, int A, int prob_bits, uint32_t* freq) {
  if (A < 1 || A > 65536 || prob_bits < 1 || prob_bits > 16) return ERR_ARG;
  const uint64_t M = 1ull << prob_bits;
  uint64_t total = 0, present = 0;
  for (int s = 0; s < A; ++s) { total += counts[s]; present += counts[s] > 0; }
  // the loops below visit the present symbols only, in increasing order
  std::vector<int> live;
  for (int s = 0; s < A; ++s)
    if (counts[s] > 0) live.push_back(s);
  if (total == 0) return ERR_ARG;
  if (present > M) return ERR_ALPHABET;
  std::vector<uint64_t> f(A, 0);
  uint64_t sum = 0;
  for (int s = 0; s < A; ++s) {
    if (counts[s] == 0) continue;
    unsigned __int128 scaled = (unsigned __int128)counts[s] * M / total;
    f[s] = std::max<uint64_t>(1, (uint64_t)scaled);
    sum += f[s];
  }
  auto gain = [&](int s) -> long double {   // saving from f_s -> f_s + 1
    return (long double)counts[s] * log2l(((long double)f[s] + 1.0L) / (long double)f[s]);
  };
  auto loss = [&](int s) -> long double {   // extra cost from f_s -> f_s - 1
    return (long double)counts[s] * log2l((long double)f[s] / ((long double)f[s] - 1.0L));
  };
  while (sum < M) {
    int best = -1;
    for (int s : live)
      if (best < 0 || gain(s) > gain(best)) best = s;
    f[best]++;
    sum++;
  }
  while (sum > M) {
    int best = -1;
    for (int s : live)
      if (f[s] > 1 && (best < 0 || loss(s) < loss(best))) best = s;
    f[best]--;
    sum--;
  }
  for (;;) {
    int up = -1;
    for (int s : live)
      if (up < 0 || gain(s) > gain(up)) up = s;
    int down = -1;
    for (int s : live)
      if (s != up && f[s] > 1 && (down < 0 || loss(s) < loss(down))) down = s;
    if (up < 0 || down < 0 || !(gain(up) > loss(down))) break;
    f[up]++;
    f[down]--;
  }
  for (int s = 0; s < A; ++s) freq[s] = (uint32_t)f[s];
  return OK;
}

// Cost sum_s c_s log2(M / f_s) in bits (infinite if a present symbol has f=0).
double oracle_code_cost(const uint64_t* counts, const uint32_t* freq, int A, int prob_bits) {
  long double M = (long double)(1ull << prob_bits), cost = 0;
  for (int s = 0; s < A; ++s) {
    if (counts[s] == 0) continue;
    if (freq[s] == 0) return INFINITY;
    cost += (long double)counts[s] * log2l(M / (long double)freq[s]);
  }
  return (double)cost;
}

// ---- Single-lane coder, for hand-checkable examples --------------------------
// Encodes msg[0..len) in reverse starting from x = L; states[i] receives the
// state after coding msg[i] (so states[0] is the final state).  Words are
// returned in decoder consumption order.
int oracle_rans_encode_message(const uint8_t* msg, int len, const uint32_t* freq, int A,
                               int prob_bits, uint32_t* states, uint16_t* words,
                               int words_cap, int* n_words) {
  Codebook cb;
  int st = make_codebook(freq, A, prob_bits, &cb);
  if (st != OK) return st;
  uint64_t x = kL;
  std::vector<uint16_t> pushed;
  for (int i = len; i-- > 0;) {
    uint32_t s = msg[i];
    if (s >= (uint32_t)A || cb.f[s] == 0) return ERR_ALPHABET;
    x = encode_step(x, cb.f[s], cb.c[s], cb, &pushed);
    states[i] = (uint32_t)x;
  }
  if ((int)pushed.size() > words_cap) return ERR_BUFFER_TOO_SMALL;
  *n_words = (int)pushed.size();
  for (size_t q = 0; q < pushed.size(); ++q) words[q] = pushed[pushed.size() - 1 - q];
  return OK;
}

// Decodes len symbols from (state, words); states[i] receives the state
// entering step i (states[0] = the given state), states[len] the end state.
int oracle_rans_decode_message(uint32_t state, const uint16_t* words, int n_words,
                               const uint32_t* freq, int A, int prob_bits, int len,
                               uint8_t* msg, uint32_t* states) {
  Codebook cb;
  int st = make_codebook(freq, A, prob_bits, &cb);
  if (st != OK) return st;
  uint64_t x = state;
  int cursor = 0;
  for (int i = 0; i < len; ++i) {
    states[i] = (uint32_t)x;
    int s;
    x = decode_symbol(x, cb, &s);
    msg[i] = (uint8_t)s;
    if (x < kL) {
      if (cursor >= n_words) return ERR_CORRUPT;
      x = (x << kWordBits) | words[cursor++];
    }
  }
  states[len] = (uint32_t)x;
  if (x != kL || cursor != n_words) return ERR_CORRUPT;
  return OK;
}

// ---- Single-lane wide-state coder (state_bits = 64), for hand-checkable examples
// len must be even (pairs).  states[i] (i even) receives the state after coding
// the pair (msg[i], msg[i+1]), so states[0] is the final state; odd entries are
// left 0.  Words (u32) are returned in decoder consumption order.
int oracle_rans64_encode_message(const uint8_t* msg, int len, const uint32_t* freq, int A,
                                 uint64_t* states, uint32_t* words, int words_cap,
                                 int* n_words) {
  if (len % 2 != 0) return ERR_ARG;
  Codebook cb;
  int st = make_codebook(freq, A, 12, &cb);
  if (st != OK) return st;
  uint64_t x = kLWide;
  std::vector<uint32_t> pushed;
  for (int i = len - 2; i >= 0; i -= 2) {
    uint32_t a = msg[i], b = msg[i + 1];
    if (a >= (uint32_t)A || b >= (uint32_t)A || cb.f[a] == 0 || cb.f[b] == 0) return ERR_ALPHABET;
    x = encode_pair_wide(x, cb.f[a], cb.c[a], cb.f[b], cb.c[b], cb, &pushed);
    states[i] = x;
    states[i + 1] = 0;
  }
  if ((int)pushed.size() > words_cap) return ERR_BUFFER_TOO_SMALL;
  *n_words = (int)pushed.size();
  for (size_t q = 0; q < pushed.size(); ++q) words[q] = pushed[pushed.size() - 1 - q];
  return OK;
}

// Decodes len (even) symbols; states[i] receives the state entering symbol i
// (states[0] = the given state), states[len] the end state.  After every
// second symbol one word is read if x < 2^32.
int oracle_rans64_decode_message(uint64_t state, const uint32_t* words, int n_words,
                                 const uint32_t* freq, int A, int len, uint8_t* msg,
                                 uint64_t* states) {
  if (len % 2 != 0) return ERR_ARG;
  Codebook cb;
  int st = make_codebook(freq, A, 12, &cb);
  if (st != OK) return st;
  uint64_t x = state;
  int cursor = 0;
  for (int i = 0; i < len; ++i) {
    states[i] = x;
    int s;
    x = decode_symbol(x, cb, &s);
    msg[i] = (uint8_t)s;
    if (i % 2 == 1 && x < kLWide) {
      if (cursor >= n_words) return ERR_CORRUPT;
      x = (x << kWideWordBits) | words[cursor++];
    }
  }
  states[len] = x;
  if (x != kLWide || cursor != n_words) return ERR_CORRUPT;
  return OK;
}

// Worst-case stream size: every symbol may push one word, plus the length
// table, full-width states, the word boundary and padding per tile.
// (Wide variant: 8-byte states and at most one 4-byte word per pair of
// symbols, so the same 2 bytes per symbol.)
uint64_t oracle_encode_bound(uint32_t N, uint32_t K, uint32_t tile_n, uint32_t tile_k,
                             int state_bits) {
  if (!layout_ok(N, K, tile_n, tile_k)) return 0;
  if (state_bits != 32 && state_bits != 64) return 0;
  uint64_t S = (uint64_t)tile_n * tile_k;
  uint64_t n_tiles = (uint64_t)(N / tile_n) * (K / tile_k);
  const uint64_t table = state_bits == 64 ? 8 : 4;
  return n_tiles * (table + (uint64_t)(state_bits / 8) * kLanes + 4 + 2 * S + 16);
}

// ---- Layer encode ([SB s3.1]): tiles, one shared codebook, offset index -----
// stream: concatenated tiles, each padded to 16 bytes; offsets[t] is the byte
// start of tile t and offsets[n_tiles] the end; raw (bf16 only) holds
// tile_n*tile_k bytes per tile at t * tile_n * tile_k.
int oracle_encode(int dtype, const void* w, uint32_t N, uint32_t K, uint32_t tile_n,
                  uint32_t tile_k, const uint32_t* freq, int prob_bits, uint8_t* stream,
                  uint64_t cap, uint64_t* stream_bytes, uint64_t* offsets, uint8_t* raw,
                  int threads, int state_bits) {
  if (dtype < 0 || dtype > 7) return ERR_ARG;
  if (state_bits != 32 && state_bits != 64) return ERR_ARG;
  if (!layout_ok(N, K, tile_n, tile_k)) return ERR_SHAPE;
  if (state_bits == 64 && prob_bits != 12 && prob_bits != 16) return ERR_ARG;  // pair bound: n = 12 or 16
  Codebook cb;
  int st = make_codebook(freq, alphabet_of(dtype), prob_bits, &cb);
  if (st != OK) return st;
  Layout lay{dtype, N, K, tile_n, tile_k, state_bits};
  const uint64_t T = lay.n_tiles();
  std::vector<std::vector<uint8_t>> tiles(T);
  std::vector<int> status(T, OK);
  parallel_for(0, T, threads, [&](uint64_t t) {
    uint8_t* raw_tile = (dtype == DT_BF16_SPLIT && raw) ? raw + t * lay.tile_symbols() : nullptr;
    status[t] = encode_tile(lay, w, cb, t, &tiles[t], raw_tile);
  });
  for (uint64_t t = 0; t < T; ++t)
    if (status[t] != OK) return status[t];
  uint64_t pos = 0;
  for (uint64_t t = 0; t < T; ++t) { offsets[t] = pos; pos += tiles[t].size(); }
  offsets[T] = pos;
  *stream_bytes = pos;
  if (pos > cap) return ERR_BUFFER_TOO_SMALL;
  parallel_for(0, T, threads, [&](uint64_t t) {
    std::memcpy(stream + offsets[t], tiles[t].data(), tiles[t].size());
  });
  return OK;
}

// ---- Layer decode ------------------------------------------------------------
// Decodes tiles [tile_begin, tile_end) into w_out (original format, row-major
// N x K; int4 nibbles of decoded tiles are overwritten, others untouched).
// Integrity: every lane must end at x = L, the words must end exactly at the
// last non-padding byte and the padding must be zero; otherwise ERR_CORRUPT.
int oracle_decode(int dtype, const uint8_t* stream, uint64_t stream_bytes,
                  const uint64_t* offsets, const uint8_t* raw, uint32_t N, uint32_t K,
                  uint32_t tile_n, uint32_t tile_k, const uint32_t* freq, int prob_bits,
                  void* w_out, uint64_t tile_begin, uint64_t tile_end, int threads,
                  int state_bits) {
  if (dtype < 0 || dtype > 7) return ERR_ARG;
  if (state_bits != 32 && state_bits != 64) return ERR_ARG;
  if (!layout_ok(N, K, tile_n, tile_k)) return ERR_SHAPE;
  if (state_bits == 64 && prob_bits != 12 && prob_bits != 16) return ERR_ARG;
  Codebook cb;
  int st = make_codebook(freq, alphabet_of(dtype), prob_bits, &cb);
  if (st != OK) return st;
  Layout lay{dtype, N, K, tile_n, tile_k, state_bits};
  const bool wide = state_bits == 64;
  const uint64_t L = wide ? kLWide : kL;
  const uint32_t word_bytes = wide ? 4 : 2;
  const uint64_t T = lay.n_tiles();
  if (tile_end > T) tile_end = T;
  if (tile_begin > tile_end) return ERR_ARG;
  if (dtype == DT_BF16_SPLIT && raw == nullptr) return ERR_ARG;
  const uint32_t kt_count = K / tile_k;
  const uint32_t steps = (uint32_t)(lay.tile_symbols() / kLanes);
  std::vector<int> status(tile_end - tile_begin, OK);
  parallel_for(tile_begin, tile_end, threads, [&](uint64_t t) {
    int& result = status[t - tile_begin];
    uint64_t a = offsets[t], b = offsets[t + 1];
    if (b < a || b > stream_bytes || a % 16 != 0) {
      result = ERR_CORRUPT;
      return;
    }
    const uint8_t* tile = stream + a;
    const uint64_t len = b - a;
    uint64_t x[kLanes];
    uint64_t cursor = get_final_states(tile, len, wide, x);
    if (cursor == 0) { result = ERR_CORRUPT; return; }
    for (uint32_t l = 0; l < kLanes; ++l)
      if (x[l] < L) { result = ERR_CORRUPT; return; }
    const uint64_t n0 = (t / kt_count) * tile_n, k0 = (t % kt_count) * tile_k;
    for (uint32_t j = 0; j < steps; ++j) {
      for (uint32_t l = 0; l < kLanes; ++l) {
        int s;
        x[l] = decode_symbol(x[l], cb, &s);
        // a word after every symbol (narrow), after the second of a pair (wide)
        const bool test = !wide || (j % 2 == 1);
        if (test && x[l] < L) {
          if (cursor + word_bytes > len) { result = ERR_CORRUPT; return; }
          uint64_t word = 0;
          for (uint32_t q = 0; q < word_bytes; ++q) word |= (uint64_t)tile[cursor + q] << (8 * q);
          cursor += word_bytes;
          x[l] = (x[l] << (8 * word_bytes)) | word;
        }
        uint32_t row, col;
        if (is_pairs(dtype)) lane_map_pairs(tile_n, l, j, &row, &col);
        else lane_map(tile_n, l, j, &row, &col);
        uint64_t idx = (n0 + row) * K + (k0 + col);
        if (is_pairs(dtype)) {
          // idx is even: the pair is exactly one packed byte
          ((uint8_t*)w_out)[idx / 2] = (uint8_t)(dtype == DT_INT4_PAIRS ? s ^ 0x88 : s);
        } else if (dtype == DT_INT4 || dtype == DT_FP4_E2M1) {
          uint8_t* out = (uint8_t*)w_out;
          uint8_t nib = (uint8_t)((dtype == DT_INT4 ? s - 8 : s) & 0xF);
          if (idx % 2 == 0) out[idx / 2] = (uint8_t)((out[idx / 2] & 0xF0) | nib);
          else out[idx / 2] = (uint8_t)((out[idx / 2] & 0x0F) | (nib << 4));
        } else if (dtype == DT_INT8) {
          ((uint8_t*)w_out)[idx] = (uint8_t)(int8_t)(s - 128);
        } else if (dtype == DT_BF16_WHOLE) {
          ((uint16_t*)w_out)[idx] = (uint16_t)s;
        } else if (dtype == DT_BF16_SPLIT) {
          uint8_t r = raw[t * lay.tile_symbols() + (j / 8) * 256 + l * 8 + (j % 8)];
          ((uint16_t*)w_out)[idx] = bf16_from_parts((uint32_t)s, r);
        } else {
          ((uint8_t*)w_out)[idx] = (uint8_t)s;
        }
      }
    }
    for (uint32_t l = 0; l < kLanes; ++l)
      if (x[l] != L) { result = ERR_CORRUPT; return; }
    if (len - cursor >= 16) { result = ERR_CORRUPT; return; }
    for (uint64_t q = cursor; q < len; ++q)
      if (tile[q] != 0) { result = ERR_CORRUPT; return; }
  });
  for (int s : status)
    if (s != OK) return s;
  return OK;
}

// ---- 9. Dequantise and GEMM in fp64 ------------------------------------------
// Y[m, i] = sum_k X[m, k] * w(rows[i], k) for the listed W rows (all rows when
// rows == NULL), X given as bf16 bits (M x K row-major).  w(n, k):
//   int4 : q * 1 (SC_NONE), q * s_n (SC_ROW_BF16, s bf16[N]),
//          q * s[n][k / group_k] (SC_GROUP_BF16, s bf16[N][K/group_k])
//   bf16 : the bf16 value (no scale)
//   fp8  : e4m3_value(code) (SC_NONE) or e4m3_value(code) * s_n (SC_ROW_F32)
//   int8 : q (SC_NONE) or q * s_n (SC_ROW_F32 or SC_ROW_BF16)
//   fp4  : e2m1_value(code) (SC_NONE) or e2m1_value(code) * s_n (SC_ROW_F32 or SC_ROW_BF16)
// Y is M x n_rows row-major doubles.
int oracle_gemm(int dtype, const uint16_t* X, uint32_t M, uint32_t K, const void* W,
                uint32_t N, int scale_kind, const void* scales, uint32_t group_k,
                const uint32_t* rows, uint32_t n_rows, double* Y, int threads) {
  if (dtype < 0 || dtype > 7) return ERR_ARG;
  if (scale_kind == SC_GROUP_BF16 && (group_k == 0 || K % group_k != 0)) return ERR_ARG;
  if (scale_kind != SC_NONE && scales == nullptr) return ERR_ARG;
  if (rows == nullptr) n_rows = N;
  std::vector<double> xv((uint64_t)M * K);
  for (uint64_t i = 0; i < xv.size(); ++i) xv[i] = bf16_value(X[i]);
  parallel_for(0, n_rows, threads, [&](uint64_t i) {
    uint64_t n = rows ? rows[i] : i;
    std::vector<double> wrow(K);
    for (uint32_t k = 0; k < K; ++k) {
      uint64_t idx = n * K + k;
      double v;
      if (is_int4(dtype)) {
        v = (double)int4_code((const uint8_t*)W, idx);
        if (scale_kind == SC_ROW_BF16) v *= bf16_value(((const uint16_t*)scales)[n]);
        else if (scale_kind == SC_GROUP_BF16)
          v *= bf16_value(((const uint16_t*)scales)[n * (K / group_k) + k / group_k]);
        else if (scale_kind == SC_ROW_F32) v *= f32_value(scales, n);
      } else if (is_fp4(dtype)) {
        const uint8_t byte = ((const uint8_t*)W)[idx / 2];
        v = e2m1_value((idx % 2 == 0) ? (byte & 0xF) : (byte >> 4));
        if (scale_kind == SC_ROW_F32) v *= f32_value(scales, n);
        else if (scale_kind == SC_ROW_BF16) v *= bf16_value(((const uint16_t*)scales)[n]);
      } else if (dtype == DT_INT8) {
        v = (double)(int8_t)((const uint8_t*)W)[idx];
        if (scale_kind == SC_ROW_F32) v *= f32_value(scales, n);
        else if (scale_kind == SC_ROW_BF16) v *= bf16_value(((const uint16_t*)scales)[n]);
      } else if (dtype == DT_BF16_SPLIT || dtype == DT_BF16_WHOLE) {
        v = bf16_value(((const uint16_t*)W)[idx]);
        if (scale_kind == SC_ROW_BF16) v *= bf16_value(((const uint16_t*)scales)[n]);
        else if (scale_kind == SC_ROW_F32) v *= f32_value(scales, n);
      } else {
        v = e4m3_value(((const uint8_t*)W)[idx]);
        if (scale_kind == SC_ROW_F32) v *= f32_value(scales, n);
        else if (scale_kind == SC_ROW_BF16) v *= bf16_value(((const uint16_t*)scales)[n]);
      }
      wrow[k] = v;
    }
    for (uint32_t m = 0; m < M; ++m) {
      double acc = 0;
      const double* xr = &xv[(uint64_t)m * K];
      for (uint32_t k = 0; k < K; ++k) acc += xr[k] * wrow[k];
      Y[(uint64_t)m * n_rows + i] = acc;
    }
  });
  return OK;
}

}  // extern "C"
