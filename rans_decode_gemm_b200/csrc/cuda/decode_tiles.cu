// decode_tiles.cu -- standalone GPU decode of a tile-coded layer into HBM in
// the weights' original format, plus the GPU symbol histogram.
//
// The decode is the layer-level path that "Approaching Shannon Bound with
// Lossless LLM Weight Compression" (s2.2 "为什么大家不用无损压缩？", s4.2
// "kernel 层面") contrasts with the fused kernel: the whole layer is
// materialised in global memory before a dense GEMM runs.  Here it serves as
// the bit-exactness check and as the first half of the two-pass baseline.
// One warp decodes one tile (32 lanes = 32 substreams, s3.1 "整体执行模型").
#include <cuda_runtime.h>

#include "kernels.h"
#include "launch.h"
#include "rans_core.cuh"

namespace ansdev {

constexpr uint32_t kDecMaxWarps = 16;
constexpr uint32_t kDecLutBytes = kSlots * 4;
// [lut 16 KB][align slack 2 KB][rings W x 2 KB][barriers W x 4 x 8 B]
constexpr uint32_t kDecSmem = kDecLutBytes + 128 + kDecMaxWarps * kRingStride + kDecMaxWarps * 4 * 8;

// The 8 symbols of one lane's group in the original storage format: 8
// consecutive columns of one row, or 16 for pair symbols (one byte each).
template <uint32_t DT>
__device__ __forceinline__ void store_group(void* out, uint64_t idx, const uint32_t (&e)[8],
                                            uint64_t raw8) {
  if (DT == kDtBf16Split) {
    uint32_t o[4];
    fmt_bf16_split(e, raw8, o);
    *reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + idx) = make_uint4(o[0], o[1], o[2], o[3]);
  } else if (DT == kDtInt4 || DT == kDtFp4) {
    uint32_t w = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) w |= (((e[k] >> 12) ^ (DT == kDtInt4 ? 8u : 0u)) & 0xFu) << (4 * k);
    *reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(out) + idx / 2) = w;
  } else {
    // one byte per symbol: the e4m3 code, the int8 code (symbol ^ 0x80) or the
    // packed int4 pair (symbol ^ 0x88)
    uint32_t lo = __byte_perm(__byte_perm(e[0] >> 12, e[1] >> 4, 0x0050u),
                              __byte_perm(e[2] >> 12, e[3] >> 4, 0x0050u), 0x5410u);
    uint32_t hi = __byte_perm(__byte_perm(e[4] >> 12, e[5] >> 4, 0x0050u),
                              __byte_perm(e[6] >> 12, e[7] >> 4, 0x0050u), 0x5410u);
    if (DT == kDtInt4Pairs) {
      lo ^= 0x88888888u;
      hi ^= 0x88888888u;
    } else if (DT == kDtInt8) {
      lo ^= 0x80808080u;
      hi ^= 0x80808080u;
    }
    // idx counts bytes for fp8 and K elements (two per byte) for int4 pairs
    *reinterpret_cast<uint2*>(static_cast<uint8_t*>(out) +
                              ((DT == kDtInt4Pairs || DT == kDtFp4Pairs) ? idx / 2 : idx)) =
        make_uint2(lo, hi);
  }
}

template <uint32_t DT, bool kWide>
__global__ void __launch_bounds__(kDecMaxWarps * 32, 2)
    decode_tiles_kernel(const __grid_constant__ LayerDev L, void* __restrict__ out,
                        uint32_t* __restrict__ status) {
  extern __shared__ __align__(2048) uint8_t smem[];
  __shared__ uint32_t abort_flag;
  const uint32_t nwarps = blockDim.x / 32;
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem);
  // rings on a 128-byte aligned shared address
  const uint32_t ring_base_s = (smem_u32(smem + kDecLutBytes) + 127) & ~127u;
  uint8_t* rings = smem + (ring_base_s - smem_u32(smem));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kDecLutBytes + 128 + kDecMaxWarps * kRingStride);
  const uint32_t warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const bool single = L.single_symbol != kNoSymbol;
  const uint32_t single_e = L.single_symbol << 12;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (uint32_t i = 0; i < nwarps * 4; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  // slot table; the cdf is staged in its own array: staged in the ring area,
  // which bulk copies fill next, the decode read wrong words even with a
  // proxy fence and a CTA barrier between the two
  __shared__ uint32_t cdf_s[257];
  if (!single) lut_stage_cdf(cdf_s, L, threadIdx.x, blockDim.x);
  __syncthreads();
  if (!single) lut_fill(lut, cdf_s, L.alphabet, threadIdx.x, blockDim.x);
  __syncthreads();
  // the prologue above read only kernel parameters: from here on global
  // memory, after the previous grid in the stream has completed
  griddep_wait();
  griddep_launch_dependents();

  volatile uint32_t* abort = &abort_flag;
  const uint32_t lt = lanemask_lt();
  const uint32_t lut_s = smem_u32(lut);
  const uint32_t n_tiles = L.n_tiles, n_kt = L.n_kt, K = L.K;
  const uint32_t tile_n = L.tile_n, tile_k = L.tile_k;
  const uint32_t H = tile_n / 128, C = tile_k / 16;
  const uint32_t S = tile_n * tile_k;
  const uint8_t* raw = L.raw;
  TileSeq seq{blockIdx.x * nwarps + warp, gridDim.x * nwarps, n_tiles, n_tiles};
  ChunkPipe pipe;
  pipe_init(pipe, rings + warp * kRingStride, bars + warp * 4);
  TileCursor tc;
  tc.cb = 0;
  const uint64_t row_step = 32ull * K;  // next row of the same lane

  for (uint32_t r = 0; seq.has(r); ++r) {
    const uint32_t t = seq.at(r);
    if (!tile_begin(pipe, L, seq, t, tc, lane, abort, status)) {
      if (lane == 0) atomicOr(status, kStatusBadOffsets);
      continue;
    }
    const uint32_t rb = t / n_kt, kt = t - rb * n_kt;
    const uint64_t base = static_cast<uint64_t>(rb * tile_n + lane) * K + kt * tile_k;
    const unsigned long long* raw_tile =
        reinterpret_cast<const unsigned long long*>(raw + static_cast<uint64_t>(t) * S) + lane;
    const uint32_t groups = S / 256;
    // raw bytes of groups g, g+1, g+2 in flight
    uint64_t r0 = 0, r1 = 0, r2 = 0;
    if (DT == kDtBf16Split) {
      r0 = __ldg(raw_tile);
      r1 = __ldg(raw_tile + 32);
      r2 = __ldg(raw_tile + 64);
    }
    uint32_t g = 0;
    // group order (slab s, half h, chunk c, row i) matches the stream's lane
    // map; an int4 pair group covers both 8-column chunks of its row
    constexpr uint32_t kGroups = (DT == kDtInt4Pairs || DT == kDtFp4Pairs) ? 4 : 8;
    for (uint32_t s = 0; s < C; ++s) {
      for (uint32_t h = 0; h < H; ++h) {
#pragma unroll
        for (uint32_t ci = 0; ci < kGroups; ++ci, ++g) {
          const uint32_t c = ci >> 2, i = ci & 3;
          const uint64_t raw8 = r0;
          if (DT == kDtBf16Split) {
            r0 = r1;
            r1 = r2;
            if (g + 3 < groups) r2 = __ldg(raw_tile + 32 * (g + 3));
          }
          uint32_t e[8];
          if (single) {
#pragma unroll
            for (int k = 0; k < 8; ++k) e[k] = single_e;
          } else {
            tile_group(pipe, L, seq, tc, lane, abort, status);
            decode_group<kWide>(tc, lut_s, pipe.ring_s, lt, e);
          }
          const uint64_t idx = base + (4 * h + i) * row_step + 16 * s + 8 * c;
          store_group<DT>(out, idx, e, raw8);
        }
      }
    }
    if (!tile_end(L, tc, single) && lane == 0) atomicOr(status, kStatusCorrupt);
  }
  pipe_drain(pipe, status);
}

// Privatised per-warp histogram in shared memory, then one 64-bit atomic per
// bin and block.  Integer counts: the result is independent of scheduling.
constexpr uint32_t kHistWarps = 8;
__global__ void __launch_bounds__(kHistWarps * 32)
    histogram_kernel(const uint8_t* __restrict__ w, uint64_t n_bytes, uint32_t dtype,
                     unsigned long long* __restrict__ hist) {
  __shared__ uint32_t h[kHistWarps][256];
  const uint32_t warp = threadIdx.x / 32;
  for (uint32_t i = threadIdx.x; i < kHistWarps * 256; i += blockDim.x) (&h[0][0])[i] = 0;
  __syncthreads();
  uint32_t* mine = h[warp];
  const uint64_t n16 = n_bytes / 16;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (uint64_t v = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < n16; v += stride) {
    uint4 q = __ldg(reinterpret_cast<const uint4*>(w) + v);
    uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t u = words[k];
      if (dtype == kDtInt4 || dtype == kDtFp4) {
        const uint32_t flip = dtype == kDtInt4 ? 8u : 0u;
#pragma unroll
        for (int n = 0; n < 8; ++n) atomicAdd(&mine[((u >> (4 * n)) & 0xFu) ^ flip], 1u);
      } else if (dtype == kDtInt4Pairs || dtype == kDtInt8 || dtype == kDtFp4Pairs) {
        const uint32_t flip = dtype == kDtInt8 ? 0x80u : (dtype == kDtInt4Pairs ? 0x88u : 0u);
#pragma unroll
        for (int n = 0; n < 4; ++n) atomicAdd(&mine[((u >> (8 * n)) & 0xFFu) ^ flip], 1u);
      } else if (dtype == kDtBf16Split) {
        atomicAdd(&mine[(u >> 7) & 0xFFu], 1u);
        atomicAdd(&mine[(u >> 23) & 0xFFu], 1u);
      } else {
#pragma unroll
        for (int n = 0; n < 4; ++n) atomicAdd(&mine[(u >> (8 * n)) & 0xFFu], 1u);
      }
    }
  }
  // tail (n_bytes % 16 bytes), handled by block 0
  if (blockIdx.x == 0) {
    for (uint64_t b = n16 * 16 + threadIdx.x * (dtype == kDtBf16Split ? 2 : 1); b < n_bytes;
         b += blockDim.x * (dtype == kDtBf16Split ? 2 : 1)) {
      if (dtype == kDtInt4 || dtype == kDtFp4) {
        const uint32_t flip = dtype == kDtInt4 ? 8u : 0u;
        atomicAdd(&mine[(w[b] & 0xFu) ^ flip], 1u);
        atomicAdd(&mine[((w[b] >> 4) & 0xFu) ^ flip], 1u);
      } else if (dtype == kDtInt4Pairs || dtype == kDtInt8 || dtype == kDtFp4Pairs) {
        atomicAdd(&mine[w[b] ^ (dtype == kDtInt8 ? 0x80u : (dtype == kDtInt4Pairs ? 0x88u : 0u))], 1u);
      } else if (dtype == kDtBf16Split) {
        uint32_t u = w[b] | (static_cast<uint32_t>(w[b + 1]) << 8);
        atomicAdd(&mine[(u >> 7) & 0xFFu], 1u);
      } else {
        atomicAdd(&mine[w[b]], 1u);
      }
    }
  }
  __syncthreads();
  const uint32_t A = (dtype == kDtInt4 || dtype == kDtFp4) ? 16 : 256;
  for (uint32_t s = threadIdx.x; s < A; s += blockDim.x) {
    uint64_t sum = 0;
    for (uint32_t k = 0; k < kHistWarps; ++k) sum += h[k][s];
    if (sum) atomicAdd(&hist[s], static_cast<unsigned long long>(sum));
  }
}

template <uint32_t DT, bool kWide>
static cudaError_t launch_decode_variant(const LayerDev& L, void* out, uint32_t* status,
                                         cudaStream_t stream, uint32_t blocks, uint32_t warps) {
  cudaError_t e = cudaFuncSetAttribute(decode_tiles_kernel<DT, kWide>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmem);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_tiles_kernel<DT, kWide>, dim3(blocks), dim3(warps * 32), kDecSmem, stream, L,
                    out, status);
}

cudaError_t launch_decode_tiles(const LayerDev& L, void* out, uint32_t* status,
                                cudaStream_t stream, int num_sms) {
  if (L.n_tiles == 0) return cudaSuccess;
  // One warp decodes one tile at a time, so the tiles are the unit of
  // parallelism: spread them evenly, up to 2 blocks x 16 warps per SM.
  const uint32_t sms = num_sms > 0 ? static_cast<uint32_t>(num_sms) : 148;
  uint32_t warps = (L.n_tiles + sms - 1) / sms;
  if (warps > kDecMaxWarps) warps = kDecMaxWarps;
  if (warps < 1) warps = 1;
  uint32_t blocks = (L.n_tiles + warps - 1) / warps;
  // Two blocks per SM keep more tiles in flight when a warp gets only a few;
  // with many tiles per warp (8 or more at two blocks per SM) one block per SM
  // is faster: fewer warps contend for the shared-memory pipe, and the
  // rounding of tiles to warps costs little (405B-shaped fp8 layer: 1943 ->
  // 1737 us; layers of a few tiles per warp lose 10-20 % with one block).
  const uint64_t per_warp2 = (static_cast<uint64_t>(L.n_tiles) + 2ull * sms * warps - 1) / (2ull * sms * warps);
  const uint32_t per_sm = per_warp2 >= 8 ? 1u : 2u;
  if (blocks > per_sm * sms) blocks = per_sm * sms;
  if (L.wide) {
    if (L.dtype == kDtBf16Split) return launch_decode_variant<kDtBf16Split, true>(L, out, status, stream, blocks, warps);
    if (L.dtype == kDtInt4) return launch_decode_variant<kDtInt4, true>(L, out, status, stream, blocks, warps);
    if (L.dtype == kDtInt4Pairs) return launch_decode_variant<kDtInt4Pairs, true>(L, out, status, stream, blocks, warps);
    if (L.dtype == kDtInt8) return launch_decode_variant<kDtInt8, true>(L, out, status, stream, blocks, warps);
    if (L.dtype == kDtFp4) return launch_decode_variant<kDtFp4, true>(L, out, status, stream, blocks, warps);
    if (L.dtype == kDtFp4Pairs) return launch_decode_variant<kDtFp4Pairs, true>(L, out, status, stream, blocks, warps);
    return launch_decode_variant<kDtFp8, true>(L, out, status, stream, blocks, warps);
  }
  if (L.dtype == kDtBf16Split) return launch_decode_variant<kDtBf16Split, false>(L, out, status, stream, blocks, warps);
  if (L.dtype == kDtInt4) return launch_decode_variant<kDtInt4, false>(L, out, status, stream, blocks, warps);
  if (L.dtype == kDtInt4Pairs) return launch_decode_variant<kDtInt4Pairs, false>(L, out, status, stream, blocks, warps);
  if (L.dtype == kDtInt8) return launch_decode_variant<kDtInt8, false>(L, out, status, stream, blocks, warps);
  if (L.dtype == kDtFp4) return launch_decode_variant<kDtFp4, false>(L, out, status, stream, blocks, warps);
  if (L.dtype == kDtFp4Pairs) return launch_decode_variant<kDtFp4Pairs, false>(L, out, status, stream, blocks, warps);
  return launch_decode_variant<kDtFp8, false>(L, out, status, stream, blocks, warps);
}

cudaError_t launch_histogram(const void* w, uint64_t n_bytes, uint32_t dtype, uint64_t* hist,
                             cudaStream_t stream, int num_sms) {
  uint32_t A = (dtype == kDtInt4 || dtype == kDtFp4) ? 16 : 256;
  cudaError_t e = cudaMemsetAsync(hist, 0, A * sizeof(uint64_t), stream);
  if (e != cudaSuccess) return e;
  uint64_t n16 = n_bytes / 16;
  uint64_t want = (n16 + kHistWarps * 32 - 1) / (kHistWarps * 32);
  uint32_t blocks = static_cast<uint32_t>(want < 1 ? 1 : want);
  uint32_t cap = 4u * static_cast<uint32_t>(num_sms);
  if (blocks > cap) blocks = cap;
  histogram_kernel<<<blocks, kHistWarps * 32, 0, stream>>>(
      static_cast<const uint8_t*>(w), n_bytes, dtype, reinterpret_cast<unsigned long long*>(hist));
  return cudaGetLastError();
}

// Internal test kernel: one thread makes one bounded wait, as the kernels'
// waits run (wait_live), on an mbarrier that nothing ever arrives on; when the
// budget runs out the status word gets the TIMEOUT bit and the kernel returns.
__global__ void wait_probe_kernel(uint32_t* status) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) wait_live(&bar, 0, &abort_flag, status, 0);
}

cudaError_t launch_wait_probe(uint32_t* status, cudaStream_t stream) {
  wait_probe_kernel<<<1, 32, 0, stream>>>(status);
  return cudaGetLastError();
}

cudaError_t set_live_wait_budget_decode(long long cycles) {
  return cudaMemcpyToSymbol(g_live_wait_budget, &cycles, sizeof(cycles));
}

}  // namespace ansdev
