// decode16.cu -- standalone GPU decode of bf16 weights coded as whole 16-bit
// symbols ("Approaching Shannon Bound with Lossless LLM Weight Compression",
// s4.1 "压缩率": bf16's large symbol table).  The stream format is the
// library's (tiles, 32 lanes, the one-symbol-per-element lane map, both state
// widths) with 2^n slots, n <= 16, instead of 2^12.
//
// A 2^16-slot table of 4-byte entries (256 KB) does not fit in shared
// memory, so the slot lookup is two-level: first[slot >> (n - 12)] names the
// first present symbol whose slot range reaches the slot's 2^(n-12)-slot
// bucket, and the lane steps forward through the present symbols (sorted,
// one 4-byte entry each: cdf | (f - 1) << 16) until the slot lies in one's
// range.  With a few thousand present symbols over 4,096 buckets that is
// about one step.  The table image (built on the host) is copied into shared
// memory once per CTA; its size limits the present symbols to kMaxPresent16.
// One warp decodes one tile, the stream arriving through the same chunk ring
// as the other decoders.
#include <cuda_runtime.h>

#include "kernels.h"
#include "launch.h"
#include "rans_core.cuh"

namespace ansdev {

constexpr uint32_t kDec16Warps = 16;
constexpr uint32_t kTable16Max = (8 + 2 * 4096 + 6 * kMaxPresent16 + 15) & ~15u;
// [table image][align slack][rings W x kRingStride][barriers W x 4 x 8 B]
constexpr uint32_t kDec16Smem = kTable16Max + 128 + kDec16Warps * kRingStride + kDec16Warps * 4 * 8;

struct Table16 {
  uint32_t last;          // n_present - 1
  uint32_t shift;         // n - 12
  uint32_t mask;          // 2^n - 1
  uint32_t first_s;       // shared address of first[4096] (u16)
  uint32_t ent_s;         // shared address of entry[n_present] (u32)
  uint32_t sym_s;         // shared address of symbol[n_present] (u16)
};

// The present symbol k holding slot, and its entry.
__device__ __forceinline__ uint32_t slot_symbol(const Table16& T, uint32_t slot, uint32_t& e) {
  uint32_t k;
  asm volatile("ld.shared.u16 %0, [%1];" : "=r"(k) : "r"(T.first_s + 2 * (slot >> T.shift)));
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(e) : "r"(T.ent_s + 4 * k));
  // slot - cdf > f - 1: past this symbol's range (cdf <= slot always holds)
  while (slot - (e & 0xFFFFu) > (e >> 16) && k < T.last) {
    ++k;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(e) : "r"(T.ent_s + 4 * k));
  }
  return k;
}

__device__ __forceinline__ uint32_t symbol_of(const Table16& T, uint32_t k) {
  uint32_t s;
  asm volatile("ld.shared.u16 %0, [%1];" : "=r"(s) : "r"(T.sym_s + 2 * k));
  return s;
}

// One step of a lane, 32-bit states: x = f (x >> n) + slot - cdf, then the
// lanes with x < 2^16 take the next 16-bit words of the shared stream in lane
// order (ballot, prefix count).  Returns the symbol.
__device__ __forceinline__ uint32_t step16(const Table16& T, uint32_t& x, uint32_t& pos,
                                           uint32_t ring_s, uint32_t lt, uint32_t n) {
  const uint32_t slot = x & T.mask;
  uint32_t e;
  const uint32_t k = slot_symbol(T, slot, e);
  x = ((e >> 16) + 1) * (x >> n) + slot - (e & 0xFFFFu);
  const bool need = x < 65536u;
  const uint32_t bal = __ballot_sync(0xFFFFFFFFu, need);
  const uint32_t addr = ring_s + (pos & (kRingBytes - 1)) + 2 * __popc(bal & lt);
  uint32_t w;
  asm volatile("ld.shared.u16 %0, [%1];" : "=r"(w) : "r"(addr));
  if (need) x = (x << 16) | w;
  pos += 2 * __popc(bal);
  return symbol_of(T, k);
}

// Two steps of a lane, 64-bit states, then one renormalisation test: the
// lanes with x < 2^32 take the next 32-bit words (two steps from x >= 2^32
// leave x >= 1, so one word restores x >= 2^32).
__device__ __forceinline__ void pair16(const Table16& T, uint64_t& x, uint32_t& pos,
                                       uint32_t ring_s, uint32_t lt, uint32_t n, uint32_t& sa,
                                       uint32_t& sb) {
  uint32_t e;
  uint32_t slot = static_cast<uint32_t>(x) & T.mask;
  uint32_t k = slot_symbol(T, slot, e);
  x = static_cast<uint64_t>((e >> 16) + 1) * (x >> n) + (slot - (e & 0xFFFFu));
  sa = symbol_of(T, k);
  slot = static_cast<uint32_t>(x) & T.mask;
  k = slot_symbol(T, slot, e);
  x = static_cast<uint64_t>((e >> 16) + 1) * (x >> n) + (slot - (e & 0xFFFFu));
  sb = symbol_of(T, k);
  const bool need = (x >> 32) == 0;
  const uint32_t bal = __ballot_sync(0xFFFFFFFFu, need);
  const uint32_t addr = ring_s + (pos & (kRingBytes - 1)) + 4 * __popc(bal & lt);
  uint32_t w;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w) : "r"(addr));
  if (need) x = (x << 32) | w;
  pos += 4 * __popc(bal);
}

template <bool kWide>
__global__ void __launch_bounds__(kDec16Warps * 32, 1)
    decode16_kernel(const __grid_constant__ LayerDev L, const uint8_t* __restrict__ table,
                    uint32_t table_bytes, uint16_t* __restrict__ out, uint32_t* __restrict__ status) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint32_t abort_flag;
  const uint32_t nwarps = blockDim.x / 32;
  const uint32_t warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t ring_base_s = (smem_u32(smem + kTable16Max) + 127) & ~127u;
  uint8_t* rings = smem + (ring_base_s - smem_u32(smem));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kTable16Max + 128 + kDec16Warps * kRingStride);
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (uint32_t i = 0; i < nwarps * 4; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  griddep_wait();
  griddep_launch_dependents();
  // the table image into shared memory (16-byte pieces)
  for (uint32_t i = threadIdx.x; i < table_bytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem)[i] = __ldg(reinterpret_cast<const uint4*>(table) + i);
  __syncthreads();
  const uint32_t n_present = reinterpret_cast<const uint32_t*>(smem)[0];
  const uint32_t n = reinterpret_cast<const uint32_t*>(smem)[1];
  // a table image that does not describe itself consistently decodes nothing
  if (n < 12 || n > 16 || n_present == 0 || n_present > kMaxPresent16 ||
      8 + 2 * 4096 + 6 * n_present > table_bytes) {
    if (threadIdx.x == 0) atomicOr(status, kStatusCorrupt);
    return;
  }
  Table16 T;
  T.last = n_present - 1;
  T.shift = n - 12;
  T.mask = (1u << n) - 1;
  T.first_s = smem_u32(smem + 8);
  T.ent_s = T.first_s + 2 * 4096;
  T.sym_s = T.ent_s + 4 * n_present;

  volatile uint32_t* abort = &abort_flag;
  const uint32_t lt = lanemask_lt();
  const uint32_t n_kt = L.n_kt, K = L.K, tile_n = L.tile_n, tile_k = L.tile_k;
  const uint32_t H = tile_n / 128, C = tile_k / 16;
  TileSeq seq{blockIdx.x * nwarps + warp, gridDim.x * nwarps, L.n_tiles, L.n_tiles};
  ChunkPipe pipe;
  pipe_init(pipe, rings + warp * kRingStride, bars + warp * 4);
  TileCursor tc;
  tc.cb = 0;
  const uint64_t row_step = 32ull * K;

  for (uint32_t r = 0; seq.has(r); ++r) {
    const uint32_t t = seq.at(r);
    if (!tile_begin(pipe, L, seq, t, tc, lane, abort, status)) {
      if (lane == 0) atomicOr(status, kStatusBadOffsets);
      continue;
    }
    const uint32_t rb = t / n_kt, kt = t - rb * n_kt;
    const uint64_t base = static_cast<uint64_t>(rb * tile_n + lane) * K + kt * tile_k;
    // groups in the lane map's order: slab s, half h, chunk c, row quarter i
    for (uint32_t s = 0; s < C; ++s) {
      for (uint32_t h = 0; h < H; ++h) {
#pragma unroll 1
        for (uint32_t ci = 0; ci < 8; ++ci) {
          const uint32_t c = ci >> 2, i = ci & 3;
          tile_group(pipe, L, seq, tc, lane, abort, status);
          uint32_t v[8];
          if (kWide) {
#pragma unroll
            for (int q = 0; q < 8; q += 2) pair16(T, tc.xw, tc.pos, pipe.ring_s, lt, n, v[q], v[q + 1]);
          } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) v[q] = step16(T, tc.x, tc.pos, pipe.ring_s, lt, n);
          }
          const uint64_t idx = base + (4 * h + i) * row_step + 16 * s + 8 * c;
          *reinterpret_cast<uint4*>(out + idx) =
              make_uint4(v[0] | v[1] << 16, v[2] | v[3] << 16, v[4] | v[5] << 16, v[6] | v[7] << 16);
        }
      }
    }
    if (!tile_end(L, tc, false) && lane == 0) atomicOr(status, kStatusCorrupt);
  }
  pipe_drain(pipe, status);
}

template <bool kWide>
static cudaError_t launch_dec16(const LayerDev& L, const uint8_t* table, uint32_t table_bytes,
                                uint16_t* out, uint32_t* status, cudaStream_t stream, uint32_t blocks,
                                uint32_t warps) {
  cudaError_t e = cudaFuncSetAttribute(decode16_kernel<kWide>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kDec16Smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode16_kernel<kWide>, dim3(blocks), dim3(warps * 32), kDec16Smem, stream, L,
                    table, table_bytes, out, status);
}

cudaError_t launch_decode_tiles16(const LayerDev& L, const uint8_t* table, uint32_t table_bytes,
                                  uint16_t* out, uint32_t* status, cudaStream_t stream, int num_sms) {
  if (L.n_tiles == 0) return cudaSuccess;
  if (table_bytes > kTable16Max || table_bytes % 16 != 0) return cudaErrorInvalidValue;
  // one block of up to 16 warps per SM (the table takes most of the shared memory)
  const uint32_t sms = num_sms > 0 ? static_cast<uint32_t>(num_sms) : 148;
  uint32_t warps = (L.n_tiles + sms - 1) / sms;
  if (warps > kDec16Warps) warps = kDec16Warps;
  if (warps < 1) warps = 1;
  uint32_t blocks = (L.n_tiles + warps - 1) / warps;
  if (blocks > sms) blocks = sms;
  return L.wide ? launch_dec16<true>(L, table, table_bytes, out, status, stream, blocks, warps)
                : launch_dec16<false>(L, table, table_bytes, out, status, stream, blocks, warps);
}

cudaError_t set_live_wait_budget_decode16(long long cycles) {
  return cudaMemcpyToSymbol(g_live_wait_budget, &cycles, sizeof(cycles));
}

}  // namespace ansdev
