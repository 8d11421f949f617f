// rans_core.cuh -- warp-parallel tile rANS decoding shared by the standalone
// decode kernel and the fused decode + GEMM kernel.
//
// "Approaching Shannon Bound with Lossless LLM Weight Compression", s3.1
// "整体执行模型": each GEMM-shaped tile is one self-contained substream set;
// its bitstream is split into R = 32 substreams and every warp lane keeps its
// own rANS state, so one warp decodes one tile.  Symbols are looked up in a
// shared-memory slot table built from the layer's shared codebook.
//
// Per lane and step: slot = x & 4095; e = lut[slot] packs (f, symbol,
// slot - cdf); x = f * (x >> 12) + (slot - cdf); if x < 2^16 the lane takes
// the next 16-bit word of the tile's interleaved word stream (lanes in
// increasing order, found with a ballot + prefix popcount).
//
// Wide-state variant (LayerDev::wide): 64-bit states in [2^32, 2^64) and
// 32-bit words; a lane decodes two symbols (two slot lookups and updates)
// before one renormalisation test, so the ballot, prefix count and word load
// are made half as often.
//
// Compressed bytes reach shared memory through a per-warp ring of four
// 1 KB slots filled by 1-D bulk copies (no multicast) that complete on
// one mbarrier per slot; the ring runs up to three chunks ahead of the read
// cursor, across tile boundaries.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace ansdev {

constexpr uint32_t kLanes = 32;
constexpr uint32_t kSlots = 4096;        // 2^12 probability slots
constexpr uint32_t kStateLow = 1u << 16; // L
constexpr uint32_t kChunkBytes = 1024;
constexpr uint32_t kRingBytes = 4096;
// A ring occupies kRingStride bytes: after its kRingBytes the first
// kRingMirror bytes of slot 0 are repeated, so the words one decode step
// reads (at most 32 lanes x 4 bytes from the cursor) never wrap around.
constexpr uint32_t kRingMirror = 128;
constexpr uint64_t kStateLowWide = 1ull << 32;  // L of the wide-state variant
constexpr uint32_t kRingStride = kRingBytes + kRingMirror;
constexpr uint32_t kNoSymbol = kNoSymbolHost;

constexpr uint32_t kStatusCorrupt = 0x1u;
constexpr uint32_t kStatusTimeout = 0x2u;
constexpr uint32_t kStatusBadOffsets = 0x4u;
constexpr uint32_t kStatusSmemAlign = 0x8u;

// The fused kernels lay out W slabs and X stages at 1024-byte multiples of
// the dynamic shared-memory base and describe them to the tensor cores (and
// TMA) with 32-byte swizzle, whose pattern is taken from the absolute shared
// address: the base must be 1024-byte aligned.  Checked once per CTA, after
// griddepcontrol.wait (it writes global memory); a misaligned base is
// reported, not trapped on.
__device__ __forceinline__ void check_smem_base(const void* smem_base, uint32_t* status) {
  if (threadIdx.x == 0 && (smem_u32(smem_base) & 1023u) != 0) atomicOr(status, kStatusSmemAlign);
}

enum : uint32_t {
  kDtInt4 = 0,
  kDtBf16Split = 1,
  kDtFp8 = 2,
  kDtInt4Pairs = 3,
  kDtInt8 = 4,
  kDtFp4 = 5,
  kDtFp4Pairs = 6
};


// Budget of the waits that the pipeline's own progress ends (wait_live and
// its variants), in clock64() cycles: kWaitBudgetCycles unless the internal
// test hook shortened it (one copy per translation unit, set by the
// set_live_wait_budget_* functions).  Drains of copies already in flight
// always wait kWaitBudgetCycles: those copies land on their own, and a CTA
// must not exit while one is still writing its shared memory.
// Constant memory (one copy per translation unit, filled with
// cudaMemcpyToSymbol): a wait reads it once, before its spin loop, from the
// constant cache -- a spin loop must not wait on a memory load between polls.
static __constant__ long long g_live_wait_budget = kWaitBudgetCycles;

// Abort-aware bounded wait.  Returns false if the wait ran out (then sets the
// CTA's abort flag and the TIMEOUT status bit) or if the CTA already aborted.
// site: which wait (diagnostic bit 8 + site is set next to TIMEOUT).
// backoff_ns > 0: sleep between polls, for waiters off the critical path, so
// that they leave issue slots to the warps that are doing the work.
__device__ __forceinline__ bool wait_live(uint64_t* bar, uint32_t parity, volatile uint32_t* abort,
                                          uint32_t* status, uint32_t site = 0,
                                          uint32_t backoff_ns = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long budget = g_live_wait_budget;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort) return false;
    if (clock64() - t0 > budget) {
      *abort = 1u;
      atomicOr(status, kStatusTimeout | (1u << (8 + site)));
      return false;
    }
    if (backoff_ns) __nanosleep(backoff_ns);
  }
  return true;
}

// wait_live on a barrier given by its 32-bit shared-memory address.
__device__ __forceinline__ bool wait_live_s(uint32_t bar_s, uint32_t parity, volatile uint32_t* abort,
                                            uint32_t* status, uint32_t site = 0) {
  if (mbar_try_wait_s(bar_s, parity)) return true;
  const long long budget = g_live_wait_budget;
  const long long t0 = clock64();
  while (!mbar_try_wait_s(bar_s, parity)) {
    if (*abort) return false;
    if (clock64() - t0 > budget) {
      *abort = 1u;
      atomicOr(status, kStatusTimeout | (1u << (8 + site)));
      return false;
    }
  }
  return true;
}

// wait_live for n consecutive barriers (bars[0 .. n-1]).  Each pass tests
// them four at a time with independent instructions instead of one dependent
// wait after another: a test's latency is a few hundred cycles, so testing
// barriers that are already complete one by one costs more than the work
// that follows.
__device__ __forceinline__ bool wait_all_live(uint64_t* bars, uint32_t n, uint32_t parity,
                                              volatile uint32_t* abort, uint32_t* status,
                                              uint32_t site, uint32_t backoff_ns) {
  const uint32_t b0 = smem_u32(bars);
  const long long budget = g_live_wait_budget;
  long long t0 = 0;
  for (uint32_t pass = 0;; ++pass) {
    bool all = true;
    uint32_t k = 0;
    for (; k + 4 <= n; k += 4) all = mbar_test4_s(b0 + 8 * k, parity) && all;
    for (; k < n; ++k) all = mbar_test_s(b0 + 8 * k, parity) && all;
    if (all) return true;
    if (pass == 0) t0 = clock64();
    if (*abort) return false;
    if (clock64() - t0 > budget) {
      *abort = 1u;
      atomicOr(status, kStatusTimeout | (1u << (8 + site)));
      return false;
    }
    if (backoff_ns) __nanosleep(backoff_ns);
  }
}

// Bounded wait used when draining copies before exit; ignores the abort flag
// (bulk copies always complete on their own).
__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity, uint32_t* status) {
  if (!mbar_wait(bar, parity)) atomicOr(status, kStatusTimeout);
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Slot table: entry = (f & 0xFFF) << 20 | symbol << 12 | (slot - cdf[symbol]).
// A single-symbol codebook (f = 4096) is decoded by a separate path.
// Per-symbol build: warp w of nwarps fills the slots of symbols w, w + nwarps,
// ... (no barrier needed; used where a warp of the CTA has other prologue work).
__device__ __forceinline__ void build_lut(uint32_t* lut, const LayerDev& L, uint32_t warp,
                                          uint32_t nwarps, uint32_t lane) {
  for (uint32_t s = warp; s < L.alphabet; s += nwarps) {
    uint32_t f = L.freq[s], c = L.cdf[s];
    uint32_t hi = ((f & 0xFFFu) << 20) | (s << 12);
    for (uint32_t k = lane; k < f; k += 32) lut[c + k] = hi | k;
  }
}

// Search build, in two phases around a CTA barrier, from the kernel parameters only:
// lut_stage_cdf copies cdf[0 .. alphabet] into shared scratch; lut_fill gives
// thread tid the slots tid, tid + nthr, ... and finds the symbol of each by a
// binary search of the cdf for the largest s with cdf[s] <= slot (a symbol of
// zero frequency is never the largest), four searches in flight per thread.
// Every thread does the same few steps, whatever the frequencies: no loop
// over the alphabet, no warp left with the most frequent symbols.
__device__ __forceinline__ void lut_stage_cdf(uint32_t* cdf_s, const LayerDev& L, uint32_t tid,
                                              uint32_t nthr) {
  for (uint32_t s = tid; s <= L.alphabet; s += nthr) cdf_s[s] = L.cdf[s];
}

__device__ __forceinline__ void lut_fill(uint32_t* lut, const uint32_t* cdf_s, uint32_t alphabet,
                                         uint32_t tid, uint32_t nthr) {
  for (uint32_t base = tid; base < kSlots; base += 4 * nthr) {
    uint32_t lo[4] = {0, 0, 0, 0};
    // the answer stays in [lo, lo + n); n shrinks to ceil(n / 2) each step
    for (uint32_t n = alphabet; n > 1;) {
      const uint32_t half = n >> 1;
#pragma unroll
      for (uint32_t q = 0; q < 4; ++q)
        if (cdf_s[lo[q] + half] <= base + q * nthr) lo[q] += half;
      n -= half;
    }
#pragma unroll
    for (uint32_t q = 0; q < 4; ++q) {
      const uint32_t slot = base + q * nthr;
      if (slot < kSlots) {
        const uint32_t c = cdf_s[lo[q]], f = cdf_s[lo[q] + 1] - c;
        lut[slot] = ((f & 0xFFFu) << 20) | (lo[q] << 12) | (slot - c);
      }
    }
  }
}

// A tile opens with its final-state block: a table of the lanes' state byte
// counts (one u32 bit plane; two for the wide-state variant, whose counts are
// 5 + plane0 bit + 2 x plane1 bit), the 32 lane states in lane order, each
// little-endian in the fewest whole bytes that hold it (3..4, or 5..8), and
// zero bytes up to the word boundary.  Its least size (every state at L) and
// its greatest (every state at full width, before the word boundary):
__device__ __forceinline__ uint32_t flush_min_bytes(const LayerDev& L) {
  return L.wide ? 8u + 5u * kLanes : 4u + 3u * kLanes;
}
__device__ __forceinline__ uint32_t flush_max_bytes(const LayerDev& L) {
  return L.wide ? 8u + 8u * kLanes : 4u + 4u * kLanes;
}
// Greatest size of a tile: block, word boundary, at most 2 bytes of words a
// symbol, padding.
__device__ __forceinline__ uint64_t tile_max_bytes(const LayerDev& L) {
  return flush_max_bytes(L) + 4ull + 2ull * L.tile_n * L.tile_k + 16ull;
}
// A tile of a single-symbol codebook is its block with every state at L.
__device__ __forceinline__ uint32_t single_tile_bytes(const LayerDev& L) {
  return (flush_min_bytes(L) + 15u) & ~15u;
}

// Byte extent of tile t, validated against the format's rules.
__device__ __forceinline__ bool tile_extent(const LayerDev& L, uint32_t t, uint64_t* start,
                                            uint32_t* bytes) {
  uint64_t a = __ldg(reinterpret_cast<const unsigned long long*>(L.offsets) + t);
  uint64_t b = __ldg(reinterpret_cast<const unsigned long long*>(L.offsets) + t + 1);
  bool ok = (a % 16 == 0) && (b % 16 == 0) && b >= a + flush_min_bytes(L) && b <= L.stream_bytes &&
            (b - a) <= tile_max_bytes(L);
  *start = a;
  *bytes = ok ? static_cast<uint32_t>(b - a) : 0u;
  return ok;
}

// Tiles handled by one warp: units first, first + stride, ... while < end;
// unit u is tile u % modulo (units run over several token passes).
struct TileSeq {
  uint32_t first, stride, end, modulo;
  __device__ __forceinline__ bool has(uint32_t r) const {
    return static_cast<uint64_t>(first) + static_cast<uint64_t>(r) * stride < end;
  }
  __device__ __forceinline__ uint32_t at(uint32_t r) const { return (first + r * stride) % modulo; }
};

// Per-warp compressed-byte pipeline.  All lanes hold the same values; lane 0
// issues the copies.
struct ChunkPipe {
  uint8_t* ring;      // kRingBytes of shared memory (generic pointer, for copies)
  uint32_t ring_s;    // the same ring as a shared address (kRingStride bytes)
  uint64_t* bars;     // 4 mbarriers (count 1)
  uint32_t issued;    // chunks issued so far (global index over the warp's tiles)
  uint32_t ready;     // chunks known to have landed
  uint32_t it_r;      // next sequence position to issue from
  uint32_t it_chunk, it_nch, it_bytes;
  uint64_t it_start;
};

__device__ __forceinline__ void pipe_init(ChunkPipe& p, uint8_t* ring, uint64_t* bars) {
  p.ring = ring;
  p.ring_s = smem_u32(ring);
  p.bars = bars;
  p.issued = p.ready = 0;
  p.it_r = 0;
  p.it_chunk = p.it_nch = p.it_bytes = 0;
  p.it_start = 0;
}

// Issue chunks while issued < limit.  Tiles whose offsets are invalid
// contribute no chunks (their consumer skips them).
__device__ __forceinline__ void pipe_issue(ChunkPipe& p, const LayerDev& L, const TileSeq& seq,
                                           uint32_t limit, uint32_t lane) {
  while (p.issued < limit) {
    if (p.it_chunk >= p.it_nch) {
      if (!seq.has(p.it_r)) return;
      uint32_t t = seq.at(p.it_r);
      p.it_r++;
      tile_extent(L, t, &p.it_start, &p.it_bytes);
      p.it_chunk = 0;
      p.it_nch = (p.it_bytes + kChunkBytes - 1) / kChunkBytes;
      continue;
    }
    uint32_t off = p.it_chunk * kChunkBytes;
    uint32_t n = min(kChunkBytes, p.it_bytes - off);
    uint32_t slot = p.issued & 3u;
    if (lane == 0) {
      // the stream is read once per token pass: evicted from L2 first
      const uint64_t pol = l2_evict_first();
      const uint32_t bar = smem_u32(&p.bars[slot]);
      const uint32_t nm = slot == 0 ? min(n, kRingMirror) : 0u;  // mirror of slot 0's head
      mbar_arrive_expect_tx_s(bar, n + nm);
      bulk_g2s_hint_s(smem_u32(p.ring + slot * kChunkBytes), L.stream + p.it_start + off, n, bar, pol);
      if (nm) bulk_g2s_hint_s(smem_u32(p.ring + kRingBytes), L.stream + p.it_start + off, nm, bar, pol);
    }
    p.it_chunk++;
    p.issued++;
  }
}

// Make chunks [.., need] resident (need is a global chunk index).
__device__ __forceinline__ void pipe_wait(ChunkPipe& p, uint32_t need, volatile uint32_t* abort,
                                          uint32_t* status) {
  while (p.ready <= need && p.ready < p.issued) {
    if (!wait_live(&p.bars[p.ready & 3u], (p.ready >> 2) & 1u, abort, status)) return;
    p.ready++;
  }
}

__device__ __forceinline__ void pipe_drain(ChunkPipe& p, uint32_t* status) {
  while (p.ready < p.issued) {
    wait_drain(&p.bars[p.ready & 3u], (p.ready >> 2) & 1u, status);
    p.ready++;
  }
}

// Keeps the ring full and the chunks that the next groups can touch
// resident.  Called when the read position enters chunk c: afterwards chunks
// up to min(c + 1, last_chunk) are resident (a group of 8 steps reads at most
// 512 bytes) and up to three chunks beyond c are in flight.
__device__ __forceinline__ void pipe_enter_chunk(ChunkPipe& p, const LayerDev& L,
                                                 const TileSeq& seq, uint32_t c,
                                                 uint32_t last_chunk, uint32_t lane,
                                                 volatile uint32_t* abort, uint32_t* status) {
  uint32_t limit = min(c, p.ready) + 4u;
  if (p.issued < limit && !*abort) pipe_issue(p, L, seq, limit, lane);
  uint32_t need = min(c + 1u, last_chunk);
  if (p.ready <= need) pipe_wait(p, need, abort, status);
  limit = min(c, p.ready) + 4u;
  if (p.issued < limit && !*abort) pipe_issue(p, L, seq, limit, lane);
}

// Decode position inside the current tile of a warp.
struct TileCursor {
  uint32_t x;      // lane state
  uint64_t xw;     // lane state of the wide-state variant
  uint32_t pos;    // ring read position (bytes, unwrapped)
  uint32_t chunk;  // chunk holding pos when the pipeline was last consulted
  uint32_t cb;     // first chunk of the tile
  uint32_t last;   // last chunk of the tile
  uint32_t bytes;  // tile bytes (padded)
};

// Lane states from the final-state block at ring position pos (a tile start,
// 16-byte aligned; the block must be resident).  Every lane reads the table,
// finds its byte count and, by popcounts of the table below its bit, its
// offset, then reads its bytes one by one; each load wraps on its own.
// Returns the position of the first word.
__device__ __forceinline__ uint32_t load_states(const LayerDev& L, uint32_t ring_s, uint32_t pos,
                                                uint32_t lane, TileCursor& tc) {
  uint32_t p0, p1 = 0;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(p0) : "r"((pos & (kRingBytes - 1)) + ring_s) : "memory");
  if (L.wide)
    asm volatile("ld.shared.u32 %0, [%1];"
                 : "=r"(p1)
                 : "r"(((pos + 4) & (kRingBytes - 1)) + ring_s)
                 : "memory");
  const uint32_t least = L.wide ? 5u : 3u, table = L.wide ? 8u : 4u, word = L.wide ? 4u : 2u;
  const uint32_t below = (1u << lane) - 1u;
  const uint32_t n = least + ((p0 >> lane) & 1u) + 2u * ((p1 >> lane) & 1u);
  const uint32_t at = pos + table + least * lane + __popc(p0 & below) + 2u * __popc(p1 & below);
  uint64_t v = 0;
#pragma unroll
  for (uint32_t b = 0; b < 8; ++b) {
    if (b < n) {
      uint32_t byte;
      asm volatile("ld.shared.u8 %0, [%1];"
                   : "=r"(byte)
                   : "r"(((at + b) & (kRingBytes - 1)) + ring_s)
                   : "memory");
      v |= static_cast<uint64_t>(byte) << (8 * b);
    }
  }
  tc.x = static_cast<uint32_t>(v);
  tc.xw = v;
  const uint32_t block = table + least * kLanes + __popc(p0) + 2u * __popc(p1);
  return pos + ((block + word - 1u) & ~(word - 1u));
}

// A tile ends well when every lane is back at L and the cursor sits in the
// last 16 bytes of the (padded) tile; a tile of a single-symbol codebook is
// its states alone.
__device__ __forceinline__ bool lanes_at_start(const LayerDev& L, const TileCursor& tc) {
  return L.wide ? tc.xw == kStateLowWide : tc.x == kStateLow;
}


// Per-warp pipeline over a RUN: tiles that follow one another in the stream
// (a warp that owns a contiguous range of tiles streams one contiguous byte
// range, so no per-tile bookkeeping is needed to keep the ring full).  Bytes
// are addressed by an unwrapped position: a run starts on a chunk boundary
// (run_c0 * kChunkBytes) and byte b of the run sits at that start + b; the
// ring slot of a position is position % kRingBytes.  Same ring, chunk size
// and barriers as ChunkPipe.
struct RunPipe {
  uint32_t ring_s;     // the ring (kRingStride bytes) as a shared-memory address
  uint32_t bars_s;     // its 4 mbarriers (count 1), shared-memory address
  const uint8_t* src;  // first byte of the current run in global memory
  uint32_t run_c0;     // global chunk index of the run's first chunk
  uint32_t run_end;    // global chunk index one past the run's last chunk
  uint32_t run_bytes;
  uint32_t issued, ready;  // global chunk counters
  uint32_t cur;            // chunk the cursor was last seen in
};

__device__ __forceinline__ void rp_init(RunPipe& p, uint8_t* ring, uint64_t* bars) {
  p.ring_s = smem_u32(ring);
  p.bars_s = smem_u32(bars);
  p.src = nullptr;
  p.run_c0 = p.run_end = p.run_bytes = 0;
  p.issued = p.ready = 0;
  p.cur = 0xFFFFFFFFu;
}

// Starts a run of `bytes` bytes at `src`; returns its base position.  Chunks
// of earlier runs that are still in flight keep their slots until waited.
__device__ __forceinline__ uint32_t rp_run_begin(RunPipe& p, const uint8_t* src, uint32_t bytes) {
  p.src = src;
  p.run_bytes = bytes;
  p.run_c0 = p.issued;
  p.run_end = p.issued + (bytes + kChunkBytes - 1) / kChunkBytes;
  p.cur = 0xFFFFFFFFu;
  return p.run_c0 * kChunkBytes;
}

// Issue chunks while fewer than lim have been issued (lim <= the run's end).
// A slot is re-armed only after the chunk that last used it was waited for.
__device__ __forceinline__ void rp_issue(RunPipe& p, uint32_t lim, uint32_t lane,
                                         volatile uint32_t* abort, uint32_t* status) {
  while (p.issued < lim && !*abort) {
    while (p.ready + 4u <= p.issued) {
      if (!wait_live_s(p.bars_s + 8 * (p.ready & 3u), (p.ready >> 2) & 1u, abort, status)) return;
      p.ready++;
    }
    const uint32_t off = (p.issued - p.run_c0) * kChunkBytes;
    const uint32_t n = min(kChunkBytes, p.run_bytes - off);
    const uint32_t slot = p.issued & 3u;
    if (lane == 0) {
      // the stream is read once per token pass: evicted from L2 first
      const uint64_t pol = l2_evict_first();
      const uint32_t nm = slot == 0 ? min(n, kRingMirror) : 0u;  // mirror of slot 0's head
      const uint32_t bar = p.bars_s + 8 * slot;
      mbar_arrive_expect_tx_s(bar, n + nm);
      bulk_g2s_hint_s(p.ring_s + slot * kChunkBytes, p.src + off, n, bar, pol);
      if (nm) bulk_g2s_hint_s(p.ring_s + kRingBytes, p.src + off, nm, bar, pol);
    }
    p.issued++;
  }
}

// Start the copies of the chunks from position pos on (up to 4 chunks), without
// waiting: called at the start of a run so its first bytes are in flight early.
__device__ __forceinline__ void rp_prefetch(RunPipe& p, uint32_t pos, uint32_t lane,
                                            volatile uint32_t* abort, uint32_t* status) {
  rp_issue(p, min(pos / kChunkBytes + 4u, p.run_end), lane, abort, status);
}

// Called when the cursor enters chunk c: afterwards chunk c + 1 (or the run's
// last chunk) has landed and chunks up to c + 3 are in flight.
__device__ __forceinline__ void rp_enter(RunPipe& p, uint32_t c, uint32_t lane,
                                         volatile uint32_t* abort, uint32_t* status) {
  p.cur = c;
  rp_issue(p, min(c + 4u, p.run_end), lane, abort, status);
  const uint32_t need = min(c + 1u, p.run_end - 1u);
  while (p.ready <= need && p.ready < p.issued) {
    if (!wait_live_s(p.bars_s + 8 * (p.ready & 3u), (p.ready >> 2) & 1u, abort, status)) return;
    p.ready++;
  }
}

__device__ __forceinline__ void rp_drain(RunPipe& p, uint32_t* status) {
  while (p.ready < p.issued) {
    long long t0 = clock64();
    while (!mbar_try_wait_s(p.bars_s + 8 * (p.ready & 3u), (p.ready >> 2) & 1u)) {
      if (clock64() - t0 > kWaitBudgetCycles) {
        atomicOr(status, kStatusTimeout);
        break;
      }
    }
    p.ready++;
  }
}

// Before each group of 8 steps (at most 512 bytes read): keep the chunk after
// the cursor's resident.
__device__ __forceinline__ void rp_group(RunPipe& p, uint32_t pos, uint32_t lane,
                                         volatile uint32_t* abort, uint32_t* status) {
  const uint32_t c = pos / kChunkBytes;
  if (c != p.cur) rp_enter(p, c, lane, abort, status);
}

// Offsets of a run of tiles [t0, t1] (inclusive), validated as a whole: the
// run's copies stay inside the stream whatever the offsets say.
__device__ __forceinline__ bool run_extent(const LayerDev& L, uint32_t t0, uint32_t t1,
                                           uint64_t* start, uint32_t* bytes) {
  const unsigned long long* off = reinterpret_cast<const unsigned long long*>(L.offsets);
  const uint64_t a = __ldg(off + t0), b = __ldg(off + t1 + 1);
  const uint64_t max_tile = tile_max_bytes(L);
  const bool ok = (a % 16 == 0) && (b % 16 == 0) && b >= a + 1ull * flush_min_bytes(L) * (t1 - t0 + 1) &&
                  b <= L.stream_bytes && (b - a) <= max_tile * (t1 - t0 + 1) &&
                  (b - a) < (1ull << 31);
  *start = a;
  *bytes = ok ? static_cast<uint32_t>(b - a) : 0u;
  return ok;
}

// Tile inside a run: [a, b) are its stream offsets, run_start the run's first
// stream offset, base the run's base position.  Checks the tile's extent
// against the run, makes its first bytes resident and loads the lane states.
// Returns false for a tile whose offsets are invalid (the rest of the run is
// then skipped by the caller).
__device__ __forceinline__ bool run_tile_begin(RunPipe& p, const LayerDev& L, uint64_t a,
                                               uint64_t b, uint64_t run_start, uint32_t base,
                                               TileCursor& tc, uint32_t lane,
                                               volatile uint32_t* abort, uint32_t* status) {
  const uint64_t max_tile = tile_max_bytes(L);
  if (b % 16 != 0 || b < a + flush_min_bytes(L) || b - a > max_tile || a < run_start ||
      b > run_start + p.run_bytes)
    return false;
  tc.bytes = static_cast<uint32_t>(b - a);
  tc.cb = base + static_cast<uint32_t>(a - run_start);  // tile start position
  tc.pos = tc.cb;
  rp_group(p, tc.pos, lane, abort, status);
  tc.pos = load_states(L, p.ring_s, tc.pos, lane, tc);
  return true;
}

// Ends a tile of a run (same integrity rule as tile_end).
__device__ __forceinline__ bool run_tile_end(const LayerDev& L, const TileCursor& tc, bool single) {
  const uint32_t used = tc.pos - tc.cb;
  bool bad = !lanes_at_start(L, tc) || used > tc.bytes || tc.bytes - used >= 16;
  if (single) bad = !lanes_at_start(L, tc) || tc.bytes != single_tile_bytes(L);
  return !__any_sync(0xFFFFFFFFu, bad);
}



// Starts tile t: validates its extent, makes its first chunks resident and
// loads the lane states.  Returns false for a tile with invalid offsets.
__device__ __forceinline__ bool tile_begin(ChunkPipe& p, const LayerDev& L, const TileSeq& seq,
                                           uint32_t t, TileCursor& tc, uint32_t lane,
                                           volatile uint32_t* abort, uint32_t* status) {
  uint64_t start;
  if (!tile_extent(L, t, &start, &tc.bytes)) return false;
  const uint32_t nch = (tc.bytes + kChunkBytes - 1) / kChunkBytes;
  tc.last = tc.cb + nch - 1;
  tc.pos = tc.cb * kChunkBytes;
  tc.chunk = tc.cb;
  pipe_enter_chunk(p, L, seq, tc.chunk, tc.last, lane, abort, status);
  tc.pos = load_states(L, p.ring_s, tc.pos, lane, tc);
  return true;
}

// Before each group of 8 steps: consult the pipeline when a new chunk starts.
__device__ __forceinline__ void tile_group(ChunkPipe& p, const LayerDev& L, const TileSeq& seq,
                                           TileCursor& tc, uint32_t lane, volatile uint32_t* abort,
                                           uint32_t* status) {
  const uint32_t c = tc.pos / kChunkBytes;
  if (c != tc.chunk) {
    tc.chunk = c;
    pipe_enter_chunk(p, L, seq, c, tc.last, lane, abort, status);
  }
}

// Ends a tile: rANS integrity (every lane back at L, words ending inside the
// padding; a single-symbol tile holds only its states) and advances to the
// next tile's first chunk.
__device__ __forceinline__ bool tile_end(const LayerDev& L, TileCursor& tc, bool single) {
  const uint32_t used = tc.pos - tc.cb * kChunkBytes;
  bool bad = !lanes_at_start(L, tc) || used > tc.bytes || tc.bytes - used >= 16;
  if (single) bad = !lanes_at_start(L, tc) || tc.bytes != single_tile_bytes(L);
  tc.cb = tc.last + 1;
  return !__any_sync(0xFFFFFFFFu, bad);
}

// One decode step of the calling lane (see the file comment), as explicit
// PTX on 32-bit shared-memory addresses.  x: state; pos: ring read position
// (bytes, unwrapped; advanced by the words the whole warp consumed); lut_s:
// slot-table address; ring_s: ring address; lt: %lanemask_lt.  Slot lookup,
// state update, ballot of the lanes that need a word, prefix count, word
// merge by one byte permute (x << 16 | w, valid because a lane needing a word
// has x < 2^16, or x unchanged) whose selector is picked while the word load
// is in flight.  The ring base of the step, ring_s + pos mod 4096, is
// computed beside the state chain; the lane's word is at base + 2 * prefix
// with no wrap test, the mirror behind the ring covering the at most 62 bytes
// a step can run past its end.  Every lane loads the word at its prefix
// position (all in one 64-byte window, so lanes that need no word cost no
// extra wavefront).  Returns the slot-table entry of the decoded symbol.
__device__ __forceinline__ uint32_t decode_step(uint32_t& x, uint32_t& pos, uint32_t lut_s,
                                                uint32_t ring_s, uint32_t lt) {
  uint32_t e;
  asm volatile(
      "{\n\t"
      ".reg .pred p;\n\t"
      ".reg .b32 a, q, f, b, bal, t, pre, cnt, off, w, sel, pb;\n\t"
      "and.b32 a, %0, 4095;\n\t"
      "shl.b32 a, a, 2;\n\t"
      "add.u32 a, a, %3;\n\t"
      "ld.shared.u32 %2, [a];\n\t"
      "and.b32 pb, %1, 4095;\n\t"
      "add.u32 pb, pb, %4;\n\t"
      "shr.u32 q, %0, 12;\n\t"
      "shr.u32 f, %2, 20;\n\t"
      "and.b32 b, %2, 4095;\n\t"
      "mad.lo.u32 %0, f, q, b;\n\t"
      "setp.lt.u32 p, %0, 65536;\n\t"
      "vote.sync.ballot.b32 bal, p, 0xffffffff;\n\t"
      "selp.b32 sel, 0x5410, 0x7654, p;\n\t"
      "and.b32 t, bal, %5;\n\t"
      "popc.b32 pre, t;\n\t"
      "popc.b32 cnt, bal;\n\t"
      "mad.lo.u32 off, pre, 2, pb;\n\t"
      "ld.shared.u16 w, [off];\n\t"
      "prmt.b32 %0, w, %0, sel;\n\t"
      "mad.lo.u32 %1, cnt, 2, %1;\n\t"
      "}"
      : "+r"(x), "+r"(pos), "=&r"(e)
      : "r"(lut_s), "r"(ring_s), "r"(lt));
  return e;
}

// Two decode steps of the calling lane in the wide-state variant, then one
// renormalisation test: slot lookup and 64-bit state update for the first
// symbol, the same for the second, then the lanes with x < 2^32 take the next
// 32-bit words of the shared stream in lane order (ballot, prefix count,
// x = x << 32 | w).  Two decoded symbols from x >= 2^32 leave x >= 2^8, so one
// word always suffices.  The ring base is computed as in decode_step; a step
// reads at most 32 x 4 bytes past the cursor, inside the ring's mirror.
__device__ __forceinline__ void decode_pair(uint64_t& x, uint32_t& pos, uint32_t lut_s,
                                            uint32_t ring_s, uint32_t lt, uint32_t& e1,
                                            uint32_t& e2) {
  asm volatile(
      "{\n\t"
      ".reg .pred p;\n\t"
      ".reg .b32 a, f, b, bal, t, pre, cnt, off, w, pb, xl, xh;\n\t"
      ".reg .b64 q, f6, b6;\n\t"
      "cvt.u32.u64 xl, %0;\n\t"
      "and.b32 a, xl, 4095;\n\t"
      "shl.b32 a, a, 2;\n\t"
      "add.u32 a, a, %4;\n\t"
      "ld.shared.u32 %2, [a];\n\t"
      "and.b32 pb, %1, 4095;\n\t"
      "add.u32 pb, pb, %5;\n\t"
      "shr.u64 q, %0, 12;\n\t"
      "shr.u32 f, %2, 20;\n\t"
      "and.b32 b, %2, 4095;\n\t"
      "cvt.u64.u32 b6, b;\n\t"
      "cvt.u64.u32 f6, f;\n\t"
      "mul.lo.u64 q, q, f6;\n\t"
      "add.u64 %0, q, b6;\n\t"
      "cvt.u32.u64 xl, %0;\n\t"
      "and.b32 a, xl, 4095;\n\t"
      "shl.b32 a, a, 2;\n\t"
      "add.u32 a, a, %4;\n\t"
      "ld.shared.u32 %3, [a];\n\t"
      "shr.u64 q, %0, 12;\n\t"
      "shr.u32 f, %3, 20;\n\t"
      "and.b32 b, %3, 4095;\n\t"
      "cvt.u64.u32 b6, b;\n\t"
      "cvt.u64.u32 f6, f;\n\t"
      "mul.lo.u64 q, q, f6;\n\t"
      "add.u64 %0, q, b6;\n\t"
      "mov.b64 {xl, xh}, %0;\n\t"
      "setp.eq.u32 p, xh, 0;\n\t"
      "vote.sync.ballot.b32 bal, p, 0xffffffff;\n\t"
      "and.b32 t, bal, %6;\n\t"
      "popc.b32 pre, t;\n\t"
      "popc.b32 cnt, bal;\n\t"
      "mad.lo.u32 off, pre, 4, pb;\n\t"
      "ld.shared.u32 w, [off];\n\t"
      "@p mov.b64 %0, {w, xl};\n\t"
      "mad.lo.u32 %1, cnt, 4, %1;\n\t"
      "}"
      : "+l"(x), "+r"(pos), "=&r"(e1), "=&r"(e2)
      : "r"(lut_s), "r"(ring_s), "r"(lt));
}

// The eight slot-table entries of one group of a lane: eight decode steps, or
// (wide-state variant) four pair steps.
template <bool kWide>
__device__ __forceinline__ void decode_group(TileCursor& tc, uint32_t lut_s, uint32_t ring_s,
                                             uint32_t lt, uint32_t (&e)[8]) {
  if (kWide) {
#pragma unroll
    for (int k = 0; k < 8; k += 2) decode_pair(tc.xw, tc.pos, lut_s, ring_s, lt, e[k], e[k + 1]);
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) e[k] = decode_step(tc.x, tc.pos, lut_s, ring_s, lt);
  }
}

// ---- symbol -> MMA operand formatting ---------------------------------------
// Inputs are slot-table entries (symbol at bits 12..19); outputs are packed
// 16-bit pairs for 16-byte shared-memory stores.

// bf16 split: exponent from the symbol, sign and mantissa from the raw byte.
// raw8: 8 raw bytes for the group (byte k belongs to symbol k).
__device__ __forceinline__ void fmt_bf16_split(const uint32_t (&e)[8], uint64_t raw8,
                                               uint32_t (&out)[4]) {
  uint32_t rlo = static_cast<uint32_t>(raw8), rhi = static_cast<uint32_t>(raw8 >> 32);
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    uint32_t a = e[2 * p] >> 5;        // exponent -> bits 7..14
    uint32_t b = e[2 * p + 1] << 11;   // exponent -> bits 23..30
    uint32_t ab = (a & 0x0000FFFFu) | (b & 0xFFFF0000u);
    uint32_t r = (p < 2) ? rlo : rhi;
    uint32_t sel = (p & 1) ? 0x3322u : 0x1100u;   // [r0,r0,r1,r1] of the pair
    uint32_t rr = __byte_perm(r, 0u, sel);
    out[p] = (ab & 0x7F807F80u) | (rr & 0x807F807Fu);
  }
}

// int4 codes as exact bf16: bf16(128 + s) has bits 0x4300 | s; subtract 136.
__device__ __forceinline__ void fmt_int4_bf16(const uint32_t (&e)[8], uint32_t (&out)[4]) {
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    uint32_t a = e[2 * p] >> 12, b = e[2 * p + 1] << 4;
    uint32_t v = ((a & 0x0000FFFFu) | (b & 0xFFFF0000u)) & 0x00FF00FFu;
    v |= 0x43004300u;
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&v);
    const __nv_bfloat162 bias = __floats2bfloat162_rn(136.0f, 136.0f);
    h = __hsub2(h, bias);
    out[p] = *reinterpret_cast<uint32_t*>(&h);
  }
}

// int4 pair symbols (symbol = (q_even + 8) | (q_odd + 8) << 4, in bits 12..19 of
// the entry) as two exact bf16: the even code's nibble goes to the low half,
// the odd one's (already at bits 16..19) to the high half.  8 symbols -> 16
// consecutive K elements.
__device__ __forceinline__ void fmt_int4pair_bf16(const uint32_t (&e)[8], uint32_t (&out)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint32_t v = ((e[k] >> 12) & 0x0000000Fu) | (e[k] & 0x000F0000u) | 0x43004300u;
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&v);
    h = __hsub2(h, __floats2bfloat162_rn(136.0f, 136.0f));
    out[k] = *reinterpret_cast<uint32_t*>(&h);
  }
}

// int4 pair symbols times a per-row group scale, exact in f16.
__device__ __forceinline__ void fmt_int4pair_f16_scaled(const uint32_t (&e)[8], __half2 scale,
                                                        uint32_t (&out)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint32_t v = ((e[k] >> 12) & 0x0000000Fu) | (e[k] & 0x000F0000u) | 0x64006400u;
    __half2 h = *reinterpret_cast<__half2*>(&v);
    h = __hmul2(__hsub2(h, __floats2half2_rn(1032.0f, 1032.0f)), scale);
    out[k] = *reinterpret_cast<uint32_t*>(&h);
  }
}

// int4 codes times a per-row scale, exact in f16: f16(1024 + s) has bits
// 0x6400 | s; subtract 1032, multiply by the scale (|q * s| <= 11 bits).
__device__ __forceinline__ void fmt_int4_f16_scaled(const uint32_t (&e)[8], __half2 scale,
                                                    uint32_t (&out)[4]) {
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    uint32_t a = e[2 * p] >> 12, b = e[2 * p + 1] << 4;
    uint32_t v = ((a & 0x0000FFFFu) | (b & 0xFFFF0000u)) & 0x00FF00FFu;
    v |= 0x64006400u;
    __half2 h = *reinterpret_cast<__half2*>(&v);
    h = __hmul2(__hsub2(h, __floats2half2_rn(1032.0f, 1032.0f)), scale);
    out[p] = *reinterpret_cast<uint32_t*>(&h);
  }
}

// int8 codes (symbol q + 128) as exact f16: f16(1024 + s) has bits
// 0x6400 | s for s < 1024; subtract 1152.
__device__ __forceinline__ void fmt_int8_f16(const uint32_t (&e)[8], uint32_t (&out)[4]) {
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    uint32_t v = ((e[2 * p] >> 12) & 0xFFu) | ((e[2 * p + 1] << 4) & 0x00FF0000u) | 0x64006400u;
    __half2 h = *reinterpret_cast<__half2*>(&v);
    h = __hsub2(h, __floats2half2_rn(1152.0f, 1152.0f));
    out[p] = *reinterpret_cast<uint32_t*>(&h);
  }
}

// e2m1 codes as exact bf16: the magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 are the
// bf16 patterns 0x0000, 0x3F00, 0x3F80, 0x3FC0, 0x4000, 0x4040, 0x4080, 0x40C0,
// looked up bytewise with two byte permutes (the low and the high byte of
// both codes at once), interleaved with a third; bit 3 of a code is the sign.
__device__ __forceinline__ uint32_t e2m1x2_bf16x2(uint32_t c0, uint32_t c1) {
  const uint32_t sel = (c0 & 7u) | ((c1 & 7u) << 4);
  const uint32_t lo = __byte_perm(0xC0800000u, 0xC0804000u, sel);  // low bytes, codes 0-7
  const uint32_t hi = __byte_perm(0x3F3F3F00u, 0x40404040u, sel);  // high bytes
  return __byte_perm(lo, hi, 0x5140u) | ((c0 & 8u) << 12) | ((c1 & 8u) << 28);
}
__device__ __forceinline__ void fmt_fp4_bf16(const uint32_t (&e)[8], uint32_t (&out)[4]) {
#pragma unroll
  for (int p = 0; p < 4; ++p) out[p] = e2m1x2_bf16x2((e[2 * p] >> 12) & 0xFu, (e[2 * p + 1] >> 12) & 0xFu);
}
// fp4 pair symbols (the packed byte, in bits 12..19 of the entry): 8 symbols ->
// 16 consecutive K elements.
__device__ __forceinline__ void fmt_fp4pair_bf16(const uint32_t (&e)[8], uint32_t (&out)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) out[k] = e2m1x2_bf16x2((e[k] >> 12) & 0xFu, (e[k] >> 16) & 0xFu);
}

// e4m3 codes to exact f16 pairs with the hardware converter.
__device__ __forceinline__ uint32_t cvt_e4m3x2_f16x2(uint32_t two_codes) {
  uint32_t r;
  asm("{\n\t.reg .b16 t;\n\t"
      "cvt.u16.u32 t, %1;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
      : "=r"(r)
      : "r"(two_codes));
  return r;
}
__device__ __forceinline__ void fmt_fp8_f16(const uint32_t (&e)[8], uint32_t (&out)[4]) {
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    // low byte: code of symbol 2p, high byte: code of symbol 2p+1
    uint32_t v = __byte_perm(e[2 * p] >> 12, e[2 * p + 1] >> 4, 0x0050u);
    out[p] = cvt_e4m3x2_f16x2(v);
  }
}

}  // namespace ansdev
