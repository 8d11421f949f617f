// gemm_dense.cu -- dense tcgen05 GEMM on 16-bit weights that are already
// decoded: Y[m][n] = s_n * sum_k X[m][k] W[n][k], fp32 out.
//
// Used for the tokens past the first pass of a large-M call.  The fused
// kernel decodes every tile once while it computes the first 16 tokens, and
// stores each decoded slab's image (16-bit, W16) into the workspace.  The
// remaining tokens meet those weights here, at tensor-core rate, instead of
// decoding the layer again per token pass.  The uncompressed variant runs the same
// kernel on the same operands (its weights formatted the same way), so the
// two variants stay bit-identical.
//
// B200 design:
//   * Output tile 128 W rows x 256 tokens (swap-AB: A = W, B = X), full K per
//     tile (no split-K), fp32 accumulators in TMEM, two accumulator sets so
//     that the epilogue of one tile overlaps the MMAs of the next.
//   * K stages of 64 columns (48 KB a stage, 4 stages).  A is four consecutive
//     W16 slab images (128 rows x 16 columns, 32-byte swizzle), contiguous in
//     W16, so one 16 KB bulk copy brings them.  B is a TMA box of X, 256 x 64,
//     128-byte swizzle.  The MMA thread issues the stage's four K = 16 MMAs
//     back to back and releases the stage with one commit.
//   * Warp roles: 0 loads (bulk copy of A, TMA box of B), 1 MMA issue (and TMEM owner), 2-5
//     epilogue (warp w reads TMEM lanes 32 (w % 4) .. + 31).
//   * Persistent CTAs take tiles t = blockIdx.x + i * gridDim.x, W row block
//     major (t / m_blocks), so the CTAs running at one time share W rows
//     through L2 and every W row block streams from HBM about once.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstring>

#include "gemm_common.cuh"
#include "kernels.h"
#include "launch.h"
#include "rans_core.cuh"

namespace ansdev {

constexpr uint32_t kDenseStages = 4;
constexpr uint32_t kDenseBM = 128, kDenseBN = 256, kDenseBK = 64;
constexpr uint32_t kDenseABytes = kDenseBM * kDenseBK * 2;  // 16 KB
constexpr uint32_t kDenseBBytes = kDenseBN * kDenseBK * 2;  // 32 KB
constexpr uint32_t kDenseStageBytes = kDenseABytes + kDenseBBytes;
constexpr uint32_t kDenseThreads = 6 * 32;
constexpr uint32_t kDenseSmem = kDenseStages * kDenseStageBytes + 1024;  // + alignment slack

__global__ void __launch_bounds__(kDenseThreads, 1) dense_gemm_kernel(const __grid_constant__ DenseDev P) {
  extern __shared__ __align__(1024) uint8_t dsmem_raw[];
  __shared__ __align__(8) uint64_t full[kDenseStages], empty[kDenseStages];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], mma_done;
  __shared__ uint32_t tmem_slot;
  __shared__ uint32_t abort_flag;

  const uint32_t warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // stage buffers on a 1024-byte boundary (the 128-byte swizzle atom)
  uint8_t* smem = dsmem_raw + ((1024u - (smem_u32(dsmem_raw) & 1023u)) & 1023u);
  const uint32_t smem_s = smem_u32(smem);
  const uint32_t n_kb = P.K / kDenseBK;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (uint32_t i = 0; i < kDenseStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (uint32_t i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);  // one arrival per epilogue warp
    }
    mbar_init(&mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  } else if (warp == 0 && lane == 0) {
    prefetch_tmap(&P.tmap_b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  volatile uint32_t* abort = &abort_flag;
  // global memory only after the previous grid in the stream has completed
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    // ======================= loads =======================
    if (lane == 0) {
      uint32_t it = 0;
      for (uint32_t t = blockIdx.x; t < P.n_tiles && !*abort; t += gridDim.x) {
        const uint32_t nb = t / P.m_blocks, mb = t - nb * P.m_blocks;
        for (uint32_t kb = 0; kb < n_kb; ++kb, ++it) {
          const uint32_t s = it % kDenseStages;
          if (it >= kDenseStages &&
              !wait_live(&empty[s], ((it / kDenseStages) + 1) & 1u, abort, P.status, 20))
            break;
          const uint32_t bar = smem_u32(&full[s]);
          const uint32_t a_s = smem_s + s * kDenseStageBytes, b_s = a_s + kDenseABytes;
          mbar_arrive_expect_tx_s(bar, kDenseABytes + P.b_box_rows * kDenseBK * 2);
          bulk_g2s_s(a_s, P.w16 + (static_cast<uint64_t>(nb) * P.k_slabs + 4 * kb) * kSlabBytes,
                     kDenseABytes, bar);
          tma_load_2d_s(b_s, &P.tmap_b, static_cast<int32_t>(kb * kDenseBK),
                        static_cast<int32_t>(mb * kDenseBN), bar);
        }
      }
      // loads still in flight (only after an abort) land before exit
      const uint32_t first = it > kDenseStages ? it - kDenseStages : 0;
      for (uint32_t q = first; q < it; ++q)
        wait_drain(&full[q % kDenseStages], (q / kDenseStages) & 1u, P.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================= MMA issue =======================
    if (lane == 0) {
      // descriptor fields.  A: LBO 16 B, SBO 256 B (8 rows of 32 bytes),
      // version 1, 32-byte swizzle; slab j of a stage is the K = 16 slice j.
      // B: SBO 1024 B (8 rows of 128 bytes), 128-byte swizzle; the K = 16
      // slice j starts 32 j bytes into each swizzled row.
      const uint64_t da = (1ull << 16) | (16ull << 32) | (1ull << 46) | (6ull << 61);
      const uint64_t db = (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
      uint32_t it = 0, acc = 0;
      bool live = true;
      for (uint32_t t = blockIdx.x; t < P.n_tiles && live; t += gridDim.x, ++acc) {
        const uint32_t b = acc & 1u;
        if (acc >= 2 && !wait_live(&acc_empty[b], ((acc >> 1) + 1) & 1u, abort, P.status, 21)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * kDenseBN;
        // the last token block is narrower when M is not a multiple of 256
        const uint32_t idesc = (t % P.m_blocks == P.m_blocks - 1) ? P.idesc_tail : P.idesc;
        for (uint32_t kb = 0; kb < n_kb; ++kb, ++it) {
          const uint32_t s = it % kDenseStages;
          if (!wait_live(&full[s], (it / kDenseStages) & 1u, abort, P.status, 22)) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint32_t a16 = (smem_s + s * kDenseStageBytes) >> 4, b16 = a16 + (kDenseABytes >> 4);
#pragma unroll
          for (uint32_t j = 0; j < kDenseBK / 16; ++j)
            umma_f16(d_tmem, da | (a16 + j * (kSlabBytes >> 4)), db | (b16 + 2 * j), idesc,
                     (kb | j) != 0 ? 1u : 0u);
          umma_commit(&empty[s]);
        }
        if (live) umma_commit(&acc_full[b]);
      }
      umma_commit(&mma_done);
      wait_drain(&mma_done, 0, P.status);
    }
    __syncwarp();
  } else {
    // ======================= epilogue (warps 2-5) =======================
    const uint32_t quad = warp & 3u;
    const uint32_t row = 32 * quad + lane;
    uint32_t acc = 0;
    for (uint32_t t = blockIdx.x; t < P.n_tiles; t += gridDim.x, ++acc) {
      const uint32_t nb = t / P.m_blocks, mb = t - nb * P.m_blocks;
      const uint32_t b = acc & 1u;
      const bool ok = wait_live(&acc_full[b], (acc >> 1) & 1u, abort, P.status, 23, 128);
      tc_fence_after();
      const uint32_t n = nb * kDenseBM + row;
      float scale = 1.0f;
      if (P.scale_kind == 1) scale = bf16_to_f32(__ldg(static_cast<const uint16_t*>(P.scales) + n));
      else if (P.scale_kind == 2) scale = __ldg(static_cast<const float*>(P.scales) + n);
      const uint32_t m0 = mb * kDenseBN;
      const uint32_t cols = min(kDenseBN, P.M - m0);
      if (ok) {
        for (uint32_t c0 = 0; c0 < cols; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(tmem_base + ((32 * quad) << 16) + b * kDenseBN + c0, v);
          tmem_ld_wait();
          float* y = P.Y + static_cast<uint64_t>(m0 + c0) * P.N + n;
#pragma unroll
          for (uint32_t j = 0; j < 32; ++j) {
            if (c0 + j < cols) *y = __uint_as_float(v[j]) * scale;
            y += P.N;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
      if (!ok) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

cudaError_t set_live_wait_budget_dense(long long cycles) {
  return cudaMemcpyToSymbol(g_live_wait_budget, &cycles, sizeof(cycles));
}

cudaError_t launch_dense_gemm(const DenseDev& P, uint32_t sms, cudaStream_t stream) {
  if (P.M == 0 || P.n_tiles == 0) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::atomic<uint64_t> attr_set{0};
  if (dev < 64 && !(attr_set.load() & (1ull << dev))) {
    e = cudaFuncSetAttribute(dense_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kDenseSmem);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(1ull << dev);
  }
  const uint32_t grid = P.n_tiles < sms ? P.n_tiles : sms;
  return launch_pdl(dense_gemm_kernel, dim3(grid), dim3(kDenseThreads), kDenseSmem, stream, P);
}

}  // namespace ansdev
