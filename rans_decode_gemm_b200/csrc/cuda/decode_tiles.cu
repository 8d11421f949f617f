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
#include "rans_core.cuh"

namespace ansdev {

constexpr uint32_t kDecWarps = 16;
constexpr uint32_t kDecLutBytes = kSlots * 4;
constexpr uint32_t kDecSmem = kDecLutBytes + kDecWarps * kRingBytes + kDecWarps * 4 * 8;

__global__ void __launch_bounds__(kDecWarps * 32, 2)
    decode_tiles_kernel(const __grid_constant__ LayerDev L, void* __restrict__ out,
                        uint32_t* __restrict__ status) {
  extern __shared__ __align__(2048) uint8_t smem[];
  __shared__ uint32_t abort_flag;
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem);
  uint8_t* rings = smem + kDecLutBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kDecLutBytes + kDecWarps * kRingBytes);
  const uint32_t warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const bool single = L.single_symbol != kNoSymbol;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (uint32_t i = 0; i < kDecWarps * 4; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  if (!single) build_lut(lut, L, warp, kDecWarps, lane);
  __syncthreads();

  volatile uint32_t* abort = &abort_flag;
  const uint32_t lt = lanemask_lt();
  TileSeq seq{blockIdx.x * kDecWarps + warp, gridDim.x * kDecWarps, L.n_tiles, L.n_tiles};
  ChunkPipe pipe;
  pipe_init(pipe, rings + warp * kRingBytes, bars + warp * 4);
  const uint32_t H = L.tile_n / 128;
  const uint32_t groups = L.tile_n * L.tile_k / 256;
  const uint32_t S = L.tile_n * L.tile_k;
  uint32_t cb = 0;  // first chunk of the current tile

  for (uint32_t r = 0; seq.has(r); ++r) {
    const uint32_t t = seq.at(r);
    uint64_t start;
    uint32_t bytes;
    if (!tile_extent(L, t, &start, &bytes)) {
      if (lane == 0) atomicOr(status, kStatusBadOffsets);
      continue;
    }
    const uint32_t nch = (bytes + kChunkBytes - 1) / kChunkBytes;
    const uint32_t last = cb + nch - 1;
    uint32_t pos = cb * kChunkBytes;
    const uint8_t* ring = pipe.ring;
    pipe_before_group(pipe, L, seq, pos, last, lane, abort, status);
    uint32_t x = *reinterpret_cast<const uint32_t*>(ring + ((pos + 4 * lane) & (kRingBytes - 1)));
    pos += 4 * kLanes;
    const uint32_t n0 = (t / L.n_kt) * L.tile_n, k0 = (t % L.n_kt) * L.tile_k;
    const uint8_t* raw_tile = L.raw + static_cast<uint64_t>(t) * S + lane * 8;
    uint64_t raw_next = 0;
    if (L.dtype == kDtBf16Split) raw_next = __ldg(reinterpret_cast<const unsigned long long*>(raw_tile));

    for (uint32_t g = 0; g < groups; ++g) {
      uint64_t raw8 = raw_next;
      if (L.dtype == kDtBf16Split && g + 1 < groups)
        raw_next = __ldg(reinterpret_cast<const unsigned long long*>(raw_tile + (g + 1) * 256));
      uint32_t e[8];
      if (single) {
#pragma unroll
        for (int k = 0; k < 8; ++k) e[k] = L.single_symbol << 12;
      } else {
        pipe_before_group(pipe, L, seq, pos, last, lane, abort, status);
#pragma unroll
        for (int k = 0; k < 8; ++k) e[k] = decode_step(x, pos, lut, ring, lt);
      }
      const uint32_t i = g & 3, c = (g >> 2) & 1, h = (g >> 3) % H, s = g / (8 * H);
      const uint64_t row = n0 + lane + 32 * (4 * h + i);
      const uint64_t col = k0 + 16 * s + 8 * c;
      const uint64_t idx = row * L.K + col;
      if (L.dtype == kDtBf16Split) {
        uint32_t o[4];
        fmt_bf16_split(e, raw8, o);
        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + idx) = make_uint4(o[0], o[1], o[2], o[3]);
      } else if (L.dtype == kDtInt4) {
        uint32_t w = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) w |= (((e[k] >> 12) ^ 8u) & 0xFu) << (4 * k);
        *reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(out) + idx / 2) = w;
      } else {
        uint32_t lo = __byte_perm(__byte_perm(e[0] >> 12, e[1] >> 4, 0x0050u),
                                  __byte_perm(e[2] >> 12, e[3] >> 4, 0x0050u), 0x5410u);
        uint32_t hi = __byte_perm(__byte_perm(e[4] >> 12, e[5] >> 4, 0x0050u),
                                  __byte_perm(e[6] >> 12, e[7] >> 4, 0x0050u), 0x5410u);
        *reinterpret_cast<uint2*>(static_cast<uint8_t*>(out) + idx) = make_uint2(lo, hi);
      }
    }
    // rANS integrity: every lane back at L, words ending within the padding.
    const uint32_t used = pos - cb * kChunkBytes;
    bool bad = (x != kStateLow) || used > bytes || bytes - used >= 16;
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) atomicOr(status, kStatusCorrupt);
    cb += nch;
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
      if (dtype == kDtInt4) {
#pragma unroll
        for (int n = 0; n < 8; ++n) atomicAdd(&mine[((u >> (4 * n)) & 0xFu) ^ 8u], 1u);
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
      if (dtype == kDtInt4) {
        atomicAdd(&mine[(w[b] & 0xFu) ^ 8u], 1u);
        atomicAdd(&mine[((w[b] >> 4) & 0xFu) ^ 8u], 1u);
      } else if (dtype == kDtBf16Split) {
        uint32_t u = w[b] | (static_cast<uint32_t>(w[b + 1]) << 8);
        atomicAdd(&mine[(u >> 7) & 0xFFu], 1u);
      } else {
        atomicAdd(&mine[w[b]], 1u);
      }
    }
  }
  __syncthreads();
  const uint32_t A = dtype == kDtInt4 ? 16 : 256;
  for (uint32_t s = threadIdx.x; s < A; s += blockDim.x) {
    uint64_t sum = 0;
    for (uint32_t k = 0; k < kHistWarps; ++k) sum += h[k][s];
    if (sum) atomicAdd(&hist[s], static_cast<unsigned long long>(sum));
  }
}

cudaError_t launch_decode_tiles(const LayerDev& L, void* out, uint32_t* status,
                                cudaStream_t stream, int num_sms) {
  cudaError_t e = cudaFuncSetAttribute(decode_tiles_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmem);
  if (e != cudaSuccess) return e;
  uint32_t blocks = (L.n_tiles + kDecWarps - 1) / kDecWarps;
  uint32_t cap = 2u * static_cast<uint32_t>(num_sms);
  if (blocks > cap) blocks = cap;
  if (blocks == 0) return cudaSuccess;
  decode_tiles_kernel<<<blocks, kDecWarps * 32, kDecSmem, stream>>>(L, out, status);
  return cudaGetLastError();
}

cudaError_t launch_histogram(const void* w, uint64_t n_bytes, uint32_t dtype, uint64_t* hist,
                             cudaStream_t stream, int num_sms) {
  uint32_t A = dtype == kDtInt4 ? 16 : 256;
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

}  // namespace ansdev
