// gemm.cu -- fused tile-rANS decode + GEMM on sm_100a (tcgen05 / TMEM / TMA).
//
// "Approaching Shannon Bound with Lossless LLM Weight Compression", s3.1
// "整体执行模型": producer warps decode compressed weight tiles straight into
// shared memory while other warps feed the tensor cores; decoding tile k+1
// overlaps the MMA on tile k; shared-memory stages are released in a fixed
// order given by the traversal, with no run-time reference counting.
//
// B200 design (swap-AB, Y^T = W X^T):
//   * A operand = a 128-row x 16-column slab of W (K-major, 32-byte swizzle),
//     written by a producer warp with 16-byte st.shared; B operand = X slab
//     (T tokens x 16 columns) brought in by TMA; fp32 accumulators in TMEM
//     (128 lanes = W rows, T columns = tokens).
//   * Warp roles: 0-3 epilogue (TMEM -> registers -> Y or split-K partial),
//     4 MMA issue (one thread), 5 X loader (TMA, one thread), 6.. producers
//     (rANS decoders in ans_gemm, plain copies in ans_gemm_uncompressed).
//   * Each producer owns a two-slot ring of 4 KB slabs; every pipeline edge is
//     an mbarrier (tcgen05.commit releases slabs and X stages).
//   * Static schedule: the tile units (token pass, W row block, K tile) are
//     split into one contiguous range per CTA; inside a CTA, round r gives
//     unit u_begin + r*D + d to producer d; the MMA thread consumes slabs in a
//     fixed order, so accumulation order (hence every bit of Y) does not
//     depend on timing and matches ans_gemm_uncompressed exactly.
//   * A W row block split over several CTAs is reduced by the last CTA to
//     finish it, in ascending CTA order (deterministic, no float atomics).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "gemm_common.cuh"
#include "kernels.h"
#include "launch.h"
#include "rans_core.cuh"

namespace ansdev {

constexpr uint32_t kFixedWarps = 6;
// 6 fixed warps + 14 producers = 20 warps (640 threads): about 100 registers
// a thread, so that the issuing warp and the producers run without spills
// (16 producers at 80 registers spill and run a few per cent slower)
constexpr uint32_t kMaxProducers = 14;
constexpr uint32_t kMaxThreads = (kFixedWarps + kMaxProducers) * 32;

// Barriers of one CTA, one array in this order:
//   w_full[2 D]   producer d's slot k holds a slab (count 1)
//   w_empty[2 D]  the MMAs that read producer d's slot k are done (one
//                 commit per slab)
//   x_full[XS]    X stage holds its slab (TMA bytes)
//   x_empty[XS]   the MMAs that read X stage k are done (one commit per stage)
//   acc_full[2], acc_empty[2], mma_done, chunk[4 D] (compressed-stream rings)
struct Bars {
  uint64_t *w_full, *w_empty, *x_full, *x_empty, *acc_full, *acc_empty, *mma_done, *chunk;
};
__device__ __forceinline__ Bars carve_bars(uint8_t* base, uint32_t D, uint32_t XS) {
  uint64_t* b = reinterpret_cast<uint64_t*>(base);
  Bars r;
  r.w_full = b;
  r.w_empty = b + 2 * D;
  r.x_full = b + 4 * D;
  r.x_empty = b + 4 * D + XS;
  r.acc_full = b + 4 * D + 2 * XS;
  r.acc_empty = r.acc_full + 2;
  r.mma_done = r.acc_empty + 2;
  r.chunk = r.mma_done + 1;
  return r;
}
__host__ __device__ inline uint32_t num_bars(uint32_t D, uint32_t XS) {
  return 4 * D + 2 * XS + 5 + 4 * D;
}
// Where a unit sits: K tile, token pass and W row-block segment, plus
// whether it opens / closes its segment within this CTA's range.
struct UnitInfo {
  uint32_t kt, p, lseg;
  bool seg_first, seg_last;
};

// Calls f(u, s, d, r, info) in the order the MMA thread consumes (unit, slab)
// pairs.  With two accumulator sets a round is consumed slab-major across
// all its units; with one set, the units of each segment of the round are
// finished before the next segment starts (so its accumulator can be drained
// first).  Either way the order within one segment is (slab, unit)
// ascending.  Unit coordinates are tracked incrementally (two divisions per
// round) so the single issuing threads stay cheap.
template <class F>
__device__ __forceinline__ void for_each_mma_step(const GemmDev& P, uint32_t u_begin,
                                                  uint32_t u_end, F&& f) {
  const uint32_t n_kt = P.L.n_kt, n_rb = P.n_rb;
  const uint32_t seg_begin = u_begin / n_kt;
  uint32_t r = 0;
  for (uint32_t u0 = u_begin; u0 < u_end; u0 += P.D, ++r) {
    const uint32_t nd = min(P.D, u_end - u0);
    const uint32_t seg0 = u0 / n_kt, kt0 = u0 - seg0 * n_kt;
    const uint32_t p0 = seg0 / n_rb, p1 = (seg0 + 1) / n_rb;
    auto info = [&](uint32_t d) {
      UnitInfo I;
      uint32_t kt = kt0 + d;
      const bool wrap = kt >= n_kt;
      kt -= wrap ? n_kt : 0;
      const uint32_t seg = seg0 + (wrap ? 1u : 0u);
      const uint32_t u = u0 + d;
      I.kt = kt;
      I.p = wrap ? p1 : p0;
      I.lseg = seg - seg_begin;
      I.seg_first = (u == u_begin) || (kt == 0);
      I.seg_last = (u + 1 == u_end) || (kt + 1 == n_kt);
      return I;
    };
    if (P.n_bufs == 2) {
      for (uint32_t s = 0; s < P.C; ++s)
        for (uint32_t d = 0; d < nd; ++d) f(u0 + d, s, d, r, info(d));
    } else {
      const uint32_t nA = min(nd, n_kt - kt0);
      for (uint32_t s = 0; s < P.C; ++s)
        for (uint32_t d = 0; d < nA; ++d) f(u0 + d, s, d, r, info(d));
      for (uint32_t s = 0; s < P.C; ++s)
        for (uint32_t d = nA; d < nd; ++d) f(u0 + d, s, d, r, info(d));
    }
  }
}

// ---------------------------------------------------------------------------
// ---------------------------------------------------------------------------
// Producer side of one W slab in copy mode (ans_gemm_uncompressed): the slab
// (rows n0 + 128 h .. + 127, columns k0 + 16 s .. + 15) formatted like the
// decoded one.  kCopyLoads: per-lane global loads of the packed nibbles.
template <uint32_t kFmt>
__device__ __forceinline__ void copy_loads(const GemmDev& P, uint32_t n0, uint32_t k0, uint32_t h,
                                           uint32_t s, uint32_t lane, uint4 (&cp)[8]) {
#pragma unroll
  for (int gg = 0; gg < 8; ++gg) {
    const uint32_t i = gg & 3, c = gg >> 2;
    const uint64_t row = n0 + lane + 32 * (4 * h + i);
    const uint64_t idx = row * P.L.K + k0 + 16 * s + 8 * c;
    const uint32_t v =
        __ldg(reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(P.w_plain) + idx / 2));
    cp[gg] = make_uint4(v, 0, 0, 0);
  }
}

// Eight packed-nibble codes (one 32-bit word, element k in bits 4k..4k+3) as
// slot-table-like entries (symbol at bits 12..19), then the format's operand.
template <uint32_t kFmt>
__device__ __forceinline__ void copy_nibbles_fmt(uint32_t v, __half2 gs, uint32_t (&o)[4]) {
  uint32_t e[8];
#pragma unroll
  for (int k = 0; k < 8; ++k)
    e[k] = (((v >> (4 * k)) & 0xFu) ^ (kFmt == kFmtFp4Bf16 ? 0u : 8u)) << 12;
  if constexpr (kFmt == kFmtFp4Bf16) fmt_fp4_bf16(e, o);
  else if constexpr (kFmt == kFmtInt4Bf16) fmt_int4_bf16(e, o);
  else fmt_int4_f16_scaled(e, gs, o);
}

// Eight 1-byte codes (two 32-bit words) as the format's operand.
template <uint32_t kFmt>
__device__ __forceinline__ void copy_bytes_fmt(uint32_t lo, uint32_t hi, uint32_t (&o)[4]) {
  const uint32_t flip = kFmt == kFmtInt8F16 ? 0x80u : 0u;  // int8: symbol = byte ^ 0x80
  uint32_t e[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    e[k] = (((lo >> (8 * k)) & 0xFFu) ^ flip) << 12;
    e[k + 4] = (((hi >> (8 * k)) & 0xFFu) ^ flip) << 12;
  }
  if constexpr (kFmt == kFmtInt8F16) fmt_int8_f16(e, o);
  else fmt_fp8_f16(e, o);
}

// Uncompressed weights (N x K codes) into W16, the slab images of the 16-bit
// operand format (see GemmDev::w16; the same values and layout the producers
// write into their slabs): thread i formats the eight elements 8 i .. 8 i + 7
// of row-major W and stores them as one 16-byte piece of their slab.
template <uint32_t kFmt>
__global__ void format_w16_kernel(const void* w, const void* scales, uint32_t K, uint32_t group_k,
                                  uint32_t n_groups_k, uint8_t* w16, uint64_t n8) {
  griddep_wait();
  griddep_launch_dependents();
  for (uint64_t i = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
    uint32_t o[4];
    if constexpr (kFmt == kFmtBf16Split) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(w) + i);
      o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    } else if constexpr (kFmt == kFmtFp8F16 || kFmt == kFmtInt8F16) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(w) + i);
      copy_bytes_fmt<kFmt>(v.x, v.y, o);
    } else {
      const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(w) + i);
      __half2 gs = __float2half2_rn(0.f);
      if constexpr (fmt_group(kFmt)) {
        const uint64_t e0 = i * 8;
        const uint64_t row = e0 / K;
        const uint32_t g = static_cast<uint32_t>(e0 - row * K) / group_k;
        gs = __float2half2_rn(bf16_to_f32(
            __ldg(static_cast<const uint16_t*>(scales) + row * n_groups_k + g)));
      }
      copy_nibbles_fmt<kFmt>(v, gs, o);
    }
    // row r, columns 8 c8 .. 8 c8 + 7 -> slab (r / 128, c8 / 2), row r % 128,
    // 16-byte chunk c8 % 2 under the 32-byte swizzle
    const uint64_t e0 = i * 8;
    const uint64_t r = e0 / K;
    const uint32_t col = static_cast<uint32_t>(e0 - r * K);
    const uint32_t rr = static_cast<uint32_t>(r & 127), c = (col >> 3) & 1u;
    const uint64_t slab = (r >> 7) * (K >> 4) + (col >> 4);
    const uint32_t off = rr * 32 + ((c << 4) ^ (((rr >> 2) & 1u) << 4));
    *reinterpret_cast<uint4*>(w16 + slab * kSlabBytes + off) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ---------------------------------------------------------------------------
template <bool kDecode, uint32_t kFmt, bool kWide>
__global__ void __launch_bounds__(kMaxThreads, 1)
    fused_gemm_kernel(const __grid_constant__ GemmDev P) {
  extern __shared__ __align__(2048) uint8_t smem[];
  __shared__ uint32_t tmem_slot;
  __shared__ uint32_t abort_flag;
  __shared__ uint32_t reduce_flag;
  __shared__ uint32_t red_n, red_seg[2];  // split-K segments of this CTA

  const uint32_t warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t D = P.D, XS = P.x_stages;
  const uint32_t G = gridDim.x;
  const uint32_t u_begin = cta_begin(static_cast<uint32_t>(P.n_units), G, blockIdx.x);
  const uint32_t u_end = cta_begin(static_cast<uint32_t>(P.n_units), G, blockIdx.x + 1);
  const uint32_t n_kt = P.L.n_kt;

  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + P.off_lut);
  uint8_t* wring = smem + P.off_w;
  // chunk rings start on a 128-byte aligned shared address (the plan leaves slack)
  uint8_t* chunks = smem + (((smem_u32(smem + P.off_chunk) + 127) & ~127u) - smem_u32(smem));
  uint8_t* xring = smem + P.off_x;
  Bars B = carve_bars(smem + P.off_bars, D, XS);
  const uint32_t x_stage_bytes = P.T_pass * 32;

  // barriers initialised by all threads, TMEM allocated by warp 0 while the
  // other warps build the slot table (see the local schedule's prologue)
  if (threadIdx.x == 0) {
    abort_flag = 0;
    red_n = 0;
    reduce_flag = 0;
  }
  {
    uint64_t* b0 = B.w_full;  // the barriers are one array, in carve_bars order
    const uint32_t n_bars = num_bars(D, XS);
    for (uint32_t i = threadIdx.x; i < n_bars; i += blockDim.x)
      mbar_init(&b0[i], (b0 + i >= B.acc_empty && b0 + i < B.acc_empty + 2) ? 4u : 1u);
    if (threadIdx.x < n_bars) fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, P.tmem_cols);
    tmem_relinquish();
  } else if (kDecode && P.L.single_symbol == kNoSymbol) {
    build_lut(lut, P.L, warp - 1, blockDim.x / 32 - 1, lane);
  } else if (warp == 5 && lane == 0) {
    prefetch_tmap(&P.tmap_x);
    if (!kDecode && copy_mode_of(kFmt) != kCopyLoads) prefetch_tmap(&P.tmap_w);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  volatile uint32_t* abort = &abort_flag;
  // the prologue above read only kernel parameters: from here on global
  // memory, after the previous grid in the stream has completed
  griddep_wait();
  griddep_launch_dependents();
  check_smem_base(smem, P.status);
  if (threadIdx.x == 0) trace_mark(P, 0);

  if (warp >= kFixedWarps) {
    // ======================= producer warps =======================
    const uint32_t d = warp - kFixedWarps;
    const LayerDev& L = P.L;
    const uint32_t H = P.H;
    const uint32_t n_us = P.H * P.C;  // slabs per unit
    TileSeq seq{static_cast<uint32_t>(u_begin) + d, D, static_cast<uint32_t>(u_end), L.n_tiles};
    const uint32_t swz = ((lane >> 2) & 1u) << 4;
    const uint32_t wslots_s = smem_u32(wring + 2 * d * kSlabBytes);
    constexpr uint32_t kCopy = kDecode ? kCopyLoads : copy_mode_of(kFmt);

    if constexpr (!kDecode && kCopy == kCopyTmaSlab) {
      // ---- bf16 weights: one TMA box per slab, straight into the slot (the
      // box's 32-byte swizzle is the slab layout); one lane works
      if (lane == 0) {
        uint32_t q = 0;  // slabs issued
        for (uint32_t r = 0; seq.has(r) && !*abort; ++r) {
          const uint32_t t = seq.at(r);
          const uint32_t n0 = (t / n_kt) * L.tile_n, k0 = (t % n_kt) * L.tile_k;
          for (uint32_t us = 0; us < n_us; ++us, ++q) {
            const uint32_t h = us % H, s = us / H, slot = q & 1u;
            if (q >= 2 && !wait_live(&B.w_empty[2 * d + slot], ((q >> 1) + 1) & 1u, abort, P.status, 1))
              break;
            const uint32_t bar = smem_u32(&B.w_full[2 * d + slot]);
            mbar_arrive_expect_tx_s(bar, kSlabBytes);
            tma_load_2d_s(wslots_s + slot * kSlabBytes, &P.tmap_w, static_cast<int32_t>(k0 + 16 * s),
                          static_cast<int32_t>(n0 + 128 * h), bar);
          }
          if (*abort) break;
        }
        // copies still in flight (only after an abort) land before exit
        for (uint32_t k = q > 2 ? q - 2 : 0; k < q; ++k)
          wait_drain(&B.w_full[2 * d + (k & 1u)], (k >> 1) & 1u, P.status);
      }
      __syncwarp();
    } else if constexpr (!kDecode && kCopy == kCopyTmaRaw) {
      // ---- 1-byte codes: the raw 128 x 16-byte box of each slab lands in a
      // two-stage ring (the decode variant's chunk ring), the lanes format it
      // into the slot: lane l owns rows l, l + 32, l + 64, l + 96
      const uint32_t raw_s = smem_u32(chunks + d * kRingStride);
      uint64_t* raw_bar = B.chunk + 4 * d;
      uint32_t n_slabs = 0;
      for (uint32_t r = 0; seq.has(r); ++r) n_slabs += n_us;
      auto issue_raw = [&](uint32_t q) {  // lane 0: the raw box of slab q into stage q & 1
        const uint32_t r = q / n_us, us = q - r * n_us;
        const uint32_t t = seq.at(r);
        const uint32_t n0 = (t / n_kt) * L.tile_n, k0 = (t % n_kt) * L.tile_k;
        const uint32_t h = us % H, s = us / H;
        const uint32_t bar = smem_u32(&raw_bar[q & 1u]);
        mbar_arrive_expect_tx_s(bar, 128 * 16);
        tma_load_2d_s(raw_s + (q & 1u) * 2048, &P.tmap_w, static_cast<int32_t>(k0 + 16 * s),
                      static_cast<int32_t>(n0 + 128 * h), bar);
      };
      uint32_t issued = 0;
      if (lane == 0)
        for (; issued < 2 && issued < n_slabs; ++issued) issue_raw(issued);
      issued = __shfl_sync(0xFFFFFFFFu, issued, 0);
      uint32_t q = 0;
      for (; q < n_slabs; ++q) {
        const uint32_t slot = q & 1u;
        const bool got = wait_live(&raw_bar[slot], (q >> 1) & 1u, abort, P.status, 7);
        if (__any_sync(0xFFFFFFFFu, !got)) break;  // warp-uniform exit
        uint4 v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v[i].x), "=r"(v[i].y), "=r"(v[i].z), "=r"(v[i].w)
                       : "r"(raw_s + slot * 2048 + (32 * i + lane) * 16)
                       : "memory");
        // the stage is free once every lane has read it: refill it
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && q + 2 < n_slabs && !*abort) {
          issue_raw(q + 2);
          issued = q + 3;
        }
        issued = __shfl_sync(0xFFFFFFFFu, issued, 0);
        uint32_t o[4][2][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          copy_bytes_fmt<kFmt>(v[i].x, v[i].y, o[i][0]);
          copy_bytes_fmt<kFmt>(v[i].z, v[i].w, o[i][1]);
        }
        const bool free_slot =
            q < 2 || wait_live(&B.w_empty[2 * d + slot], ((q >> 1) + 1) & 1u, abort, P.status, 1);
        if (__any_sync(0xFFFFFFFFu, !free_slot)) break;
        const uint32_t slab_s = wslots_s + slot * kSlabBytes;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t row_s = slab_s + (32 * i + lane) * 32;
#pragma unroll
          for (uint32_t c = 0; c < 2; ++c)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row_s + ((c << 4) ^ swz)),
                         "r"(o[i][c][0]), "r"(o[i][c][1]), "r"(o[i][c][2]), "r"(o[i][c][3])
                         : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.w_full[2 * d + slot]);
      }
      // raw boxes still in flight (only after an abort) land before exit
      if (lane == 0)
        for (uint32_t k = q; k < issued; ++k) wait_drain(&raw_bar[k & 1u], (k >> 1) & 1u, P.status);
      __syncwarp();
    } else {
      // ---- decode (ans_gemm), or per-lane loads of packed nibbles (copy)
      const uint32_t lt = lanemask_lt();
      const bool single = L.single_symbol != kNoSymbol;
      const uint32_t n_slabs = P.H * P.C;
      const uint32_t groups = n_slabs * 8;  // 8 groups of 8 symbols per lane fill one slab
      const uint32_t lut_s = smem_u32(lut);
      ChunkPipe pipe;
      pipe_init(pipe, chunks + d * kRingStride, B.chunk + 4 * d);
      TileCursor tc;
      tc.cb = 0;
      uint32_t sc = 0;  // unit slabs produced

      for (uint32_t r = 0; seq.has(r); ++r) {
        const uint32_t t = seq.at(r);
        const uint32_t n0 = (t / n_kt) * L.tile_n, k0 = (t % n_kt) * L.tile_k;
        bool zero_tile = false;
        if (kDecode) {
          if (!tile_begin(pipe, L, seq, t, tc, lane, abort, P.status)) {
            zero_tile = true;
            if (lane == 0) atomicOr(P.status, kStatusBadOffsets);
          }
        }
        __half2 gscale[8];
        if (fmt_group(kFmt)) {
          const uint32_t gk = k0 / P.group_k;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t hh = q / 4, ii = q % 4;
            float sv = 0.f;
            if (hh < H) {
              const uint32_t row = n0 + lane + 32 * (4 * hh + ii);
              sv = bf16_to_f32(__ldg(static_cast<const uint16_t*>(P.scales) +
                                     static_cast<uint64_t>(row) * P.n_groups_k + gk));
            }
            gscale[q] = __float2half2_rn(sv);
          }
        }
        // raw sign/mantissa bytes of groups g, g+1, g+2 in flight (bf16, decode)
        const unsigned long long* raw_tile = nullptr;
        uint64_t r0 = 0, r1 = 0, r2 = 0;
        if (kDecode && kFmt == kFmtBf16Split && !zero_tile) {
          raw_tile = reinterpret_cast<const unsigned long long*>(
                         L.raw + static_cast<uint64_t>(t) * (L.tile_n * L.tile_k)) + lane;
          r0 = __ldg(raw_tile);
          r1 = __ldg(raw_tile + 32);
          r2 = __ldg(raw_tile + 64);
        }

        for (uint32_t us = 0; us < n_slabs; ++us) {
          const uint32_t h = us % H, s = us / H;
          const uint32_t slot = sc & 1u;
          // group scales of this lane's four rows in half h (int4 x group scale)
          __half2 gs0, gs1, gs2, gs3;
          if (fmt_group(kFmt)) {
            gs0 = h ? gscale[4] : gscale[0];
            gs1 = h ? gscale[5] : gscale[1];
            gs2 = h ? gscale[6] : gscale[2];
            gs3 = h ? gscale[7] : gscale[3];
          }
          // copy mode: fetch the slab's 8 groups before waiting for the slot
          uint4 cp[8];
          if constexpr (!kDecode) copy_loads<kFmt>(P, n0, k0, h, s, lane, cp);
          if (sc >= 2) wait_live(&B.w_empty[2 * d + slot], ((sc >> 1) + 1) & 1u, abort, P.status, 1, 64);
          if (kDecode && P.w16 != nullptr) {
            // the store of the slot's previous slab has read it
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
          }
          const uint32_t slab_s = wslots_s + slot * kSlabBytes;
          // a group is 8 columns of one row, or both 8-column halves of it for
          // int4 pair symbols (4 groups per slab)
          constexpr bool kPair = fmt_pair(kFmt);
          constexpr uint32_t kGroups = kPair ? 4 : 8, kOut = kPair ? 8 : 4;
#pragma unroll 1
          for (uint32_t gg = 0; gg < kGroups; ++gg) {
            const uint32_t g = us * 8 + gg;
            const uint32_t i = gg & 3, c = gg >> 2;
            uint32_t o[kOut];
            if (kDecode) {
              const uint64_t raw8 = r0;
              if (kFmt == kFmtBf16Split && !zero_tile) {
                r0 = r1;
                r1 = r2;
                if (g + 3 < groups) r2 = __ldg(raw_tile + 32 * (g + 3));
              }
              uint32_t e[8];
              if (zero_tile) {
#pragma unroll
                for (int k = 0; k < 8; ++k) e[k] = 0;
              } else if (single) {
#pragma unroll
                for (int k = 0; k < 8; ++k) e[k] = L.single_symbol << 12;
              } else {
                tile_group(pipe, L, seq, tc, lane, abort, P.status);
                decode_group<kWide>(tc, lut_s, pipe.ring_s, lt, e);
              }
              if constexpr (kFmt == kFmtInt4PairBf16) fmt_int4pair_bf16(e, o);
              else if constexpr (kFmt == kFmtFp4PairBf16) fmt_fp4pair_bf16(e, o);
              else if constexpr (kFmt == kFmtInt4PairF16Group)
                fmt_int4pair_f16_scaled(e, i == 0 ? gs0 : i == 1 ? gs1 : i == 2 ? gs2 : gs3, o);
              else if constexpr (kFmt == kFmtBf16Split) fmt_bf16_split(e, raw8, o);
              else if constexpr (kFmt == kFmtInt4Bf16) fmt_int4_bf16(e, o);
              else if constexpr (kFmt == kFmtInt4F16Group)
                fmt_int4_f16_scaled(e, i == 0 ? gs0 : i == 1 ? gs1 : i == 2 ? gs2 : gs3, o);
              else if constexpr (kFmt == kFmtInt8F16) fmt_int8_f16(e, o);
              else if constexpr (kFmt == kFmtFp4Bf16) fmt_fp4_bf16(e, o);
              else fmt_fp8_f16(e, o);
              if (zero_tile) {
#pragma unroll
                for (uint32_t k = 0; k < kOut; ++k) o[k] = 0;
              }
            } else if constexpr (!kPair) {
              uint4 v = cp[0];
#pragma unroll
              for (int q = 1; q < 8; ++q)
                if (gg == static_cast<uint32_t>(q)) v = cp[q];
              copy_nibbles_fmt<kFmt>(v.x, i == 0 ? gs0 : i == 1 ? gs1 : i == 2 ? gs2 : gs3, o);
            }
            const uint32_t row_s = slab_s + (32 * i + lane) * 32;
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row_s + ((c << 4) ^ swz)),
                         "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3])
                         : "memory");
            if constexpr (kPair)
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row_s + (16u ^ swz)),
                           "r"(o[kOut - 4]), "r"(o[kOut - 3]), "r"(o[kOut - 2]), "r"(o[kOut - 1])
                           : "memory");
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&B.w_full[2 * d + slot]);
          // first token pass of a large-M call: the slab also goes to W16
          if (kDecode && P.w16 != nullptr && lane == 0)
            bulk_s2g_s(P.w16 + ((static_cast<uint64_t>((n0 >> 7) + h) * (L.K >> 4)) + (k0 >> 4) + s) *
                                   kSlabBytes,
                       slab_s, kSlabBytes);
          if (lane == 0 && sc == 0) trace_mark(P, 2 + d);
          ++sc;
        }
        if (kDecode && !zero_tile) {
          if (!tile_end(L, tc, single) && lane == 0) atomicOr(P.status, kStatusCorrupt);
        }
      }
      if (kDecode) pipe_drain(pipe, P.status);
      if (kDecode && P.w16 != nullptr && lane == 0) bulk_wait_all();
    }
    if (lane == 0) trace_mark(P, 18 + d);
  } else if (warp == 4) {
    // ======================= MMA issue =======================
    // Slabs are consumed in a fixed order (round, part, slab, producer, half),
    // so the accumulation order does not depend on timing.  For every (round,
    // part, slab) group the warp's lanes first test the W barriers of all its
    // producers at once (one round trip instead of one per producer), then
    // lane 0 issues the group's MMAs, X stage by X stage.
    const uint32_t ub = static_cast<uint32_t>(u_begin), ue = static_cast<uint32_t>(u_end);
    const uint32_t seg_begin = ub / n_kt;
    const uint32_t H = P.H;
    // descriptor fields shared by every operand: LBO 16 B, SBO 256 B,
    // version 1, 32-byte swizzle; only the start address varies
    const uint64_t dhi = (1ull << 16) | (16ull << 32) | (1ull << 46) | (6ull << 61);
    const uint32_t a_base = smem_u32(wring) >> 4, x_base = smem_u32(xring) >> 4;
    const uint32_t slab16 = kSlabBytes >> 4, xstage16 = x_stage_bytes >> 4, t16 = (P.T * 32) >> 4;
    uint32_t fresh = 0;  // bit (buf * 2 + h): next MMA into that accumulator starts it
    uint32_t xs = 0, xpar = 0;
    uint32_t r = 0;
    bool live = true;
    for (uint32_t u0 = ub; u0 < ue && live; u0 += D, ++r) {
      const uint32_t nd = min(D, ue - u0);
      const uint32_t seg0 = u0 / n_kt, kt0 = u0 - seg0 * n_kt;
      const uint32_t nA = P.n_bufs == 2 ? nd : min(nd, n_kt - kt0);
      for (uint32_t part = 0; part < 2 && live; ++part) {
        const uint32_t d_lo = part == 0 ? 0 : nA, d_hi = part == 0 ? nA : nd;
        if (d_lo == d_hi) continue;
        for (uint32_t s = 0; s < P.C && live; ++s) {
          // readiness of every W slab of the group, one lane per (producer, half)
          bool ok = true;
          const uint32_t ng = (d_hi - d_lo) * H;
          if (lane < ng) {
            const uint32_t dd = d_lo + lane / H, hh = lane % H;
            const uint32_t idx = (r * P.C + s) * H + hh;
            ok = wait_live(&B.w_full[2 * dd + (idx & 1u)], (idx >> 1) & 1u, abort, P.status, 3);
          }
          if (__ballot_sync(0xFFFFFFFFu, !ok) != 0) live = false;
          if (!live) break;
          if (lane == 0) {
            tc_fence_after();
            for (uint32_t d = d_lo; d < d_hi; ++d) {
              const uint32_t kt = kt0 + d;
              const bool wrap = kt >= n_kt;
              const uint32_t ktw = wrap ? kt - n_kt : kt;
              const uint32_t lseg = seg0 + (wrap ? 1u : 0u) - seg_begin;
              const uint32_t buf = P.n_bufs == 2 ? (lseg & 1u) : 0u;
              if (s == 0 && (u0 + d == ub || ktw == 0)) {
                const uint32_t k = P.n_bufs == 2 ? (lseg >> 1) : lseg;
                if (k >= 1 && !wait_live(&B.acc_empty[buf], (k - 1) & 1u, abort, P.status, 4)) {
                  live = false;
                  break;
                }
                tc_fence_after();
                fresh |= 3u << (2 * buf);
              }
              if (!wait_live(&B.x_full[xs], xpar, abort, P.status, 2)) {
                live = false;
                break;
              }
              tc_fence_after();
              for (uint32_t h = 0; h < H; ++h) {
                const uint32_t idx = (r * P.C + s) * H + h;
                const uint32_t slot = idx & 1u;
                const uint64_t adesc = dhi | (a_base + (2 * d + slot) * slab16);
                const uint32_t acc_bit = 1u << (2 * buf + h);
                const uint32_t accumulate = (fresh & acc_bit) ? 0u : 1u;
                for (uint32_t j = 0; j < P.NT; ++j) {
                  const uint64_t bdesc = dhi | (x_base + xs * xstage16 + j * t16);
                  const uint32_t col = ((buf * H + h) * P.NT + j) * P.T;
                  umma_f16(tmem_base + col, adesc, bdesc, P.idesc, accumulate);
                }
                fresh &= ~acc_bit;
                umma_commit(&B.w_empty[2 * d + slot]);
              }
              umma_commit(&B.x_empty[xs]);
              if (++xs == XS) { xs = 0; xpar ^= 1u; }
              if (s == P.C - 1 && (u0 + d + 1 == ue || ktw + 1 == n_kt))
                umma_commit(&B.acc_full[buf]);
            }
          }
          live = __shfl_sync(0xFFFFFFFFu, live ? 1u : 0u, 0) != 0;
        }
      }
    }
    if (lane == 0) {
      umma_commit(B.mma_done);
      trace_mark(P, 34);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ============ X loader (TMA from the tensor map, one thread) ============
    // X slab (token pass p, columns kx .. kx + 15) is the tensor map's box at
    // (kx, p * T_pass + j * T) for j < NT; rows past M land as zeros.
    if (lane == 0) {
      uint32_t xc = 0;
      uint32_t n_issued = 0;  // loads issued: steps [0, n_issued) (none after an abort)
      const uint32_t xring_s = smem_u32(xring);
      for_each_mma_step(P, static_cast<uint32_t>(u_begin), static_cast<uint32_t>(u_end),
                        [&](uint32_t, uint32_t s, uint32_t, uint32_t, const UnitInfo& I) {
        const uint32_t xs = xc % XS;
        if (xc >= XS) wait_live(&B.x_empty[xs], ((xc / XS) + 1) & 1u, abort, P.status, 5, 32);
        if (!*abort && n_issued == xc) {
          const uint32_t kx = I.kt * P.L.tile_k + 16 * s;
          const uint32_t bar = smem_u32(&B.x_full[xs]);
          mbar_arrive_expect_tx_s(bar, x_stage_bytes);
          for (uint32_t j = 0; j < P.NT; ++j)
            tma_load_2d_s(xring_s + xs * x_stage_bytes + j * P.T * 32, &P.tmap_x,
                          static_cast<int32_t>(kx), static_cast<int32_t>(I.p * P.T_pass + j * P.T),
                          bar);
          n_issued = xc + 1;
        }
        ++xc;
      });
      trace_mark(P, 42);
      // drain: the last load issued into every stage must have landed
      const uint32_t first = n_issued > XS ? n_issued - XS : 0;
      for (uint32_t q = first; q < n_issued; ++q)
        wait_drain(&B.x_full[q % XS], (q / XS) & 1u, P.status);
      trace_mark(P, 35);
    }
    __syncwarp();
  } else {
    // ======================= epilogue (warps 0-3, 128 threads) =======================
    const uint32_t e = threadIdx.x;  // TMEM lane = row within the 128-row half
    const uint32_t seg_first = u_begin / n_kt, seg_last = (u_end - 1) / n_kt;
    uint32_t pend[2], npend = 0;  // segments shared with other CTAs (first, last)
    for (uint32_t seg = seg_first; seg <= seg_last; ++seg) {
      const uint32_t lseg = static_cast<uint32_t>(seg - seg_first);
      const uint32_t buf = lseg % P.n_bufs;
      // after an abort the accumulator holds no valid sum, but the epilogue
      // still takes part in split-K so that the counters return to zero
      wait_live(&B.acc_full[buf], (lseg / P.n_bufs) & 1u, abort, P.status, 6, 256);
      tc_fence_after();
      if (e == 0 && lseg < 2) trace_mark(P, 36 + lseg);
      const uint32_t p = static_cast<uint32_t>(seg / P.n_rb);
      const uint32_t rb = static_cast<uint32_t>(seg % P.n_rb);
      const uint32_t s_lo = seg * n_kt, s_hi = s_lo + n_kt;
      const bool complete = u_begin <= s_lo && u_end >= s_hi;
      const uint32_t slot = (seg == seg_first) ? 0u : 1u;
      float* part = P.partials + (static_cast<uint64_t>(blockIdx.x) * 2 + slot) * P.H * P.T_pass * 128;
      for (uint32_t h = 0; h < P.H; ++h) {
        const uint32_t n = rb * P.L.tile_n + h * 128 + e;
        const float scale = complete ? row_scale(P, n) : 1.0f;
        for (uint32_t j = 0; j < P.NT; ++j) {
          const uint32_t col0 = ((buf * P.H + h) * P.NT + j) * P.T;
          // tokens past M are padding: stop at the last 16-column chunk holding one
          const uint32_t m0 = p * P.T_pass + j * P.T;
          const uint32_t t_end = P.M > m0 ? min(P.T, P.M - m0) : 0u;
          for (uint32_t cc = 0; cc < t_end; cc += 32) {
            uint32_t v[2][16];
            tmem_ld16(tmem_base + ((32 * warp) << 16) + col0 + cc, v[0]);
            if (cc + 16 < t_end) tmem_ld16(tmem_base + ((32 * warp) << 16) + col0 + cc + 16, v[1]);
            tmem_ld_wait();
#pragma unroll
            for (uint32_t k = 0; k < 2; ++k) {
              if (cc + 16 * k >= t_end) break;
              float f[16];
#pragma unroll
              for (int q = 0; q < 16; ++q) f[q] = __uint_as_float(v[k][q]);
              epi_emit16(P, f, complete, scale, part, p, h, j * P.T + cc + 16 * k, n, e);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.acc_empty[buf]);
      if (!complete) pend[npend++] = seg;
    }
    // split-K arrival once every partial of this CTA is written; the
    // reductions this CTA owns run after the CTA barrier, on every thread
    if (npend) splitk_arrive(P, G, pend, npend, e, &reduce_flag);
    if (e == 0) {
      red_n = npend;
      red_seg[0] = pend[0];
      red_seg[1] = pend[1];
    }
  }

  // ---- teardown: every MMA retired before TMEM is released
  if (threadIdx.x == 0) trace_mark(P, 40);
  __syncthreads();
  if (threadIdx.x == 0) trace_mark(P, 41);
  if (warp == 0) {
    wait_drain(B.mma_done, 0, P.status);
    tc_fence_after();
    tmem_dealloc(tmem_base, P.tmem_cols);
  }
  // the split-K reductions this CTA arrived last for, on every thread
  if (reduce_flag) {
    fence_acq_rel_gpu();  // acquire: the counter showed every contributor arrived
    for (uint32_t k = 0; k < red_n; ++k)
      if ((reduce_flag >> k) & 1u) splitk_reduce(P, G, red_seg[k], threadIdx.x, blockDim.x);
  }
}

// f16 copy of X for the formats whose MMA runs in f16 (X row-major M x K,
// bf16 bits in, f16 out; 8 elements per thread step).
__global__ void x_to_f16_kernel(const uint16_t* __restrict__ X, uint16_t* __restrict__ X16,
                                uint64_t n8) {
  griddep_wait();
  griddep_launch_dependents();
  for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(X) + i);
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      __half2 hv = __floats2half2_rn(__uint_as_float(in[k] << 16), __uint_as_float(in[k] & 0xFFFF0000u));
      out[k] = *reinterpret_cast<uint32_t*>(&hv);
    }
    reinterpret_cast<uint4*>(X16)[i] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// =============================== host side ===============================

static uint32_t round_up(uint32_t a, uint32_t b) { return (a + b - 1) / b * b; }

static unsigned long long* g_trace = nullptr;
void set_trace_buffer(void* d_buf, size_t bytes) {
  g_trace = bytes >= 64 * sizeof(unsigned long long) ? static_cast<unsigned long long*>(d_buf) : nullptr;
}

cudaError_t set_live_wait_budget_gemm(long long cycles) {
  return cudaMemcpyToSymbol(g_live_wait_budget, &cycles, sizeof(cycles));
}

static std::atomic<uint32_t> g_cap_ctas{0}, g_cap_producers{0}, g_force_shared{0};
void set_plan_limits(uint32_t max_ctas, uint32_t max_producers, uint32_t force_shared) {
  g_cap_ctas.store(max_ctas, std::memory_order_relaxed);
  g_cap_producers.store(max_producers, std::memory_order_relaxed);
  g_force_shared.store(force_shared ? 1u : 0u, std::memory_order_relaxed);
}

// Accumulator slots the local schedule needs in the busiest CTA: one per
// (producer warp, W row-block segment) pair that holds units.
static uint32_t local_slots(uint32_t U, uint32_t G, uint32_t D, uint32_t n_kt) {
  uint32_t mx = 0;
  for (uint32_t c = 0; c < G; ++c) {
    const uint32_t ub = cta_begin(U, G, c), ue = cta_begin(U, G, c + 1);
    uint32_t cnt = 0;
    for (uint32_t d = 0; d < D; ++d) {
      const uint32_t b = ub + cta_begin(ue - ub, D, d), e = ub + cta_begin(ue - ub, D, d + 1);
      if (e > b) cnt += (e - 1) / n_kt - b / n_kt + 1;
    }
    if (cnt > mx) mx = cnt;
  }
  return mx;
}

// The schedule (grid, producers, token passes) depends only on the shape, the
// format and the device, never on whether the weights arrive compressed, so
// ans_gemm and ans_gemm_uncompressed add the same products in the same order.
bool make_gemm_plan(const LayerDev& L, uint32_t M, uint32_t scale_kind, bool decode, int num_sms,
                    GemmPlan* plan) {
  GemmPlan p;
  std::memset(&p, 0, sizeof(p));
  if (L.dtype == 1) p.fmt = kFmtBf16Split;
  else if (L.dtype == 0) p.fmt = (scale_kind == 3) ? kFmtInt4F16Group : kFmtInt4Bf16;
  else if (L.dtype == 3)
    // int4 pair symbols fill the same slabs as per-element int4 symbols; the
    // uncompressed weights take the per-element copy path
    p.fmt = decode ? ((scale_kind == 3) ? kFmtInt4PairF16Group : kFmtInt4PairBf16)
                   : ((scale_kind == 3) ? kFmtInt4F16Group : kFmtInt4Bf16);
  else if (L.dtype == 4) p.fmt = kFmtInt8F16;
  else if (L.dtype == 5) p.fmt = kFmtFp4Bf16;
  else if (L.dtype == 6) p.fmt = decode ? kFmtFp4PairBf16 : kFmtFp4Bf16;  // same slabs
  else p.fmt = kFmtFp8F16;
  p.ab_f16 = (fmt_group(p.fmt) || p.fmt == kFmtFp8F16 || p.fmt == kFmtInt8F16) ? 1 : 0;
  p.M = M;
  p.H = L.tile_n / 128;
  p.C = L.tile_k / 16;
  const uint32_t Mp = round_up(M < 1 ? 1 : M, 16);
  uint64_t sms = num_sms > 0 ? static_cast<uint64_t>(num_sms) : 148;
  // test limits (set_plan_limits): cap the CTA count and the producer warps
  // per CTA, force the shared-accumulator schedule
  const uint32_t cap_ctas = g_cap_ctas.load(std::memory_order_relaxed);
  if (cap_ctas > 0 && cap_ctas < sms) sms = cap_ctas;
  p.sms = static_cast<uint32_t>(sms);
  const uint32_t cap_prod = g_cap_producers.load(std::memory_order_relaxed);
  // unit indices are 32-bit in the kernels
  if (static_cast<uint64_t>(L.n_tiles) * ((M + 15) / 16) >= (1ull << 31)) return false;
  // The small-M schedule keeps a private accumulator of H * T columns per
  // producer and accumulator slot.  256-row tiles at 17-32 tokens (64
  // columns: about 7 producers fit TMEM) take it only with pair symbols,
  // whose cheaper decode keeps up with fewer producers; the choice depends on
  // the layout alone, so both variants plan the same schedule.
  const bool pair_layout = L.dtype == 3 || L.dtype == 6;
  bool want_local = p.H * Mp <= 32 || (pair_layout && Mp <= 32 && p.H * Mp <= 64);
  if (g_force_shared.load(std::memory_order_relaxed)) want_local = false;
  const uint32_t lut_bytes = kSlots * 4;

  // More tokens than one pass of the shared-accumulator schedule (512 / H):
  // the first kDenseFirstTokens tokens run fused on the small-M schedule,
  // whose decoders are the fastest, and store every decoded slab into W16;
  // the other tokens run as one dense GEMM on W16 (gemm_dense.cu).  The plan
  // is the first pass's, with the call's token count and the workspace of
  // the whole call.
  // (When the first pass does not fit the small-M schedule -- a device of
  // very few SMs -- every pass runs on the shared-accumulator schedule.)
  GemmPlan first;
  if (M > 512 / p.H && L.K % 64 == 0 && !g_force_shared.load(std::memory_order_relaxed) &&
      make_gemm_plan(L, kDenseFirstTokens, scale_kind, decode, num_sms, &first) && first.local) {
    const uint32_t T_pass = 512 / p.H;
    p = first;
    p.M = M;
    p.dense = 1;
    p.M_first = kDenseFirstTokens;
    p.T_pass = T_pass;
    p.n_pass = (M + T_pass - 1) / T_pass;
    p.ws_x16_bytes = p.ab_f16 ? static_cast<size_t>(M) * L.K * 2 : 0;
    // W16: decoded by the first pass, or the uncompressed weights formatted
    p.ws_w16_bytes = static_cast<size_t>(L.N) * L.K * 2;
    p.ws_bytes = p.ws_counters_bytes + (p.ws_partials_bytes + 255) / 256 * 256 +
                 (p.ws_x16_bytes + 255) / 256 * 256 + p.ws_w16_bytes;
    *plan = p;
    return true;
  }

  if (want_local) {
    // ---- local schedule: every producer issues its own MMAs (gemm_local.cu)
    p.T = p.T_pass = Mp;
    p.NT = 1;
    p.n_pass = 1;
    p.n_bufs = 1;
    p.n_units = L.n_tiles;
    p.n_segments = L.N / L.tile_n;
    p.grid = static_cast<uint32_t>(p.n_units < sms ? p.n_units : sms);
    const uint64_t per_cta = (p.n_units + p.grid - 1) / p.grid;
    uint32_t D = (cap_prod > 0 && cap_prod < kLocalProducersMax) ? cap_prod : kLocalProducersMax;
    if (D > per_cta) D = static_cast<uint32_t>(per_cta);
    for (; D >= 1; --D) {
      const uint32_t slots = local_slots(static_cast<uint32_t>(p.n_units), p.grid, D, L.n_kt);
      const uint32_t cols = slots * p.H * p.T;
      uint32_t off = lut_bytes;
      off = round_up(off, 1024);
      const uint32_t off_w = off;
      off += 2 * D * kSlabBytes;  // two W slabs per producer
      off = round_up(off, 128);
      const uint32_t off_chunk = off;
      off += D * kRingStride + 128;
      off = round_up(off, 1024);
      const uint32_t off_x = off;
      off += 2 * D * p.T * 32;  // two X slabs per producer
      off = round_up(off, 8);
      const uint32_t off_bars = off;
      off += (8 * D + 1 + slots) * 8;
      if (cols <= 512 && off <= kSmemLimit) {
        p.local = 1;
        p.D = D;
        p.n_slots = slots;
        p.tmem_cols = 32;
        while (p.tmem_cols < cols) p.tmem_cols <<= 1;
        p.off_lut = 0;
        p.off_w = off_w;
        p.off_chunk = off_chunk;
        p.off_x = off_x;
        p.off_bars = off_bars;
        p.smem_bytes = off;
        p.ws_partials_bytes = static_cast<size_t>(p.grid) * 2 * p.H * p.T_pass * 128 * sizeof(float);
        p.ws_counters_bytes = round_up(p.n_segments * 4, 256);
        p.ws_x16_bytes = 0;
        p.ws_bytes = p.ws_counters_bytes + (p.ws_partials_bytes + 255) / 256 * 256;
        *plan = p;
        return true;
      }
    }
    // no fit: fall through to the shared-accumulator schedule
  }

  // ---- shared-accumulator schedule: one MMA-issuing warp per CTA
  const uint32_t max_cols = 512;
  if (2 * p.H * Mp <= max_cols) {
    p.n_bufs = 2;
    p.T_pass = Mp;
  } else if (p.H * Mp <= max_cols) {
    p.n_bufs = 1;
    p.T_pass = Mp;
  } else {
    p.n_bufs = 1;
    p.T_pass = max_cols / p.H;
  }
  p.NT = (p.T_pass + 255) / 256;
  p.T = round_up((p.T_pass + p.NT - 1) / p.NT, 16);
  p.T_pass = p.T * p.NT;
  p.n_pass = (M + p.T_pass - 1) / p.T_pass;
  if (p.n_pass == 0) p.n_pass = 1;
  const uint32_t cols = p.n_bufs * p.H * p.T_pass;
  p.tmem_cols = 32;
  while (p.tmem_cols < cols) p.tmem_cols <<= 1;
  if (p.tmem_cols > 512) return false;

  p.n_units = static_cast<uint64_t>(p.n_pass) * L.n_tiles;
  p.n_segments = p.n_pass * (L.N / L.tile_n);
  p.grid = static_cast<uint32_t>(p.n_units < sms ? p.n_units : sms);
  uint64_t per_cta = (p.n_units + p.grid - 1) / p.grid;

  // Producers against X stages.  Every MMA step waits for its X slab, loaded
  // by TMA from L2 a microsecond or more before; the decode variant consumes
  // a slab about every 1,000 cycles (one per producer every ~13,000), so a
  // few stages cover that latency: at least 3, and 32 KB of stages when they
  // are small.  The producer count is the largest that leaves them room.
  // Shared memory, decode variant: [slot table][W slots][chunk rings][X stages][barriers].
  const uint32_t x_stage = p.T_pass * 32;
  const uint32_t xs_min = std::max(3u, std::min(8u, 32768u / x_stage));
  uint32_t D = (cap_prod > 0 && cap_prod < kMaxProducers) ? cap_prod : kMaxProducers;
  if (D > L.n_kt) D = L.n_kt;  // a round spans at most two W row-block segments
  if (D > per_cta) D = static_cast<uint32_t>(per_cta);
  const uint32_t lut_bytes_c = lut_bytes;
  auto layout = [&](uint32_t Dn, bool with_lut, bool with_rings, uint32_t* off_w, uint32_t* off_chunk,
                    uint32_t* off_x) {
    uint32_t off = with_lut ? round_up(lut_bytes_c, 2048) : 0;
    *off_w = off;
    off += Dn * 2 * kSlabBytes;
    off = round_up(off, 128);
    *off_chunk = off;
    if (with_rings) off += Dn * kRingStride + 128;
    off = round_up(off, 1024);
    *off_x = off;
    return off;
  };
  for (;; --D) {
    if (D == 0) return false;
    uint32_t ow, oc, ox;
    const uint32_t off = layout(D, true, true, &ow, &oc, &ox);
    const uint32_t bars_max = num_bars(D, 64) * 8;
    const uint32_t room = kSmemLimit > off + bars_max ? kSmemLimit - off - bars_max : 0;
    if (room / x_stage >= xs_min) break;
  }
  p.D = D;
  // the layout of the variant asked for: the decode variant as above; the copy
  // variant has no slot table and (except for 1-byte codes, staged by TMA in
  // the chunk area) no chunk rings, so its X ring is deeper -- it consumes a
  // slab per MMA, not per decode
  const uint32_t cmode = copy_mode_of(p.fmt);
  const bool rings = decode || cmode == kCopyTmaRaw;
  {
    uint32_t ow, oc, ox;
    uint32_t off = layout(D, decode, rings, &ow, &oc, &ox);
    const uint32_t bars_max = num_bars(D, 64) * 8;
    const uint32_t room = kSmemLimit > off + bars_max ? kSmemLimit - off - bars_max : 0;
    uint32_t XS = room / x_stage;
    if (XS > 64) XS = 64;
    if (XS < 2) return false;
    off += XS * x_stage;
    off = round_up(off, 8);
    p.off_lut = 0;
    p.off_w = ow;
    p.off_chunk = oc;
    p.off_x = ox;
    p.off_bars = off;
    off += num_bars(D, XS) * 8;
    p.smem_bytes = off;
    p.x_stages = XS;
  }
  p.ws_partials_bytes = static_cast<size_t>(p.grid) * 2 * p.H * p.T_pass * 128 * sizeof(float);
  p.ws_counters_bytes = round_up(p.n_segments * 4, 256);
  p.ws_x16_bytes = p.ab_f16 ? static_cast<size_t>(M) * L.K * 2 : 0;  // f16 copy of X
  p.ws_bytes = p.ws_counters_bytes + (p.ws_partials_bytes + 255) / 256 * 256 +
               (p.ws_x16_bytes + 255) / 256 * 256;
  *plan = p;
  return true;
}

// ---- tensor maps (2-D, tiled, one destination CTA), encoded through the driver
// entry point the runtime hands out (no link-time dependence on libcuda)
static cudaError_t encode_tmap(CUtensorMap* map, CUtensorMapDataType type, const void* base,
                               uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
                               uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  static cudaError_t lookup = cudaSuccess;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    lookup = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q);
    if (lookup == cudaSuccess && (q != cudaDriverEntryPointSuccess || f == nullptr))
      lookup = cudaErrorSymbolNotFound;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  if (lookup != cudaSuccess) return lookup;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, type, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <bool kDecode, uint32_t kFmt, bool kWide = false>
static cudaError_t launch_variant(const GemmPlan& plan, const GemmDev& P, cudaStream_t stream) {
  auto kern = fused_gemm_kernel<kDecode, kFmt, kWide>;
  // the opt-in shared-memory size is a per-device function attribute: set it
  // once per device and variant
  static int attr_set[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    if (e != cudaSuccess) return e;
    attr_set[dev] = 1;
  }
  return launch_pdl(kern, dim3(plan.grid), dim3((kFixedWarps + plan.D) * 32), plan.smem_bytes,
                    stream, P);
}

// Kernel parameters of one layer's launch; ws is that layer's workspace.
static GemmDev make_gemm_dev(const GemmPlan& plan, const LayerDev& L, const void* w_plain,
                             const uint16_t* X, const void* scales, uint32_t scale_kind,
                             uint32_t group_k, float* Y, void* ws, uint32_t* status) {
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  GemmDev P;
  std::memset(&P, 0, sizeof(P));
  P.L = L;
  P.w_plain = w_plain;
  P.scales = scales;
  P.Y = Y;
  P.counters = reinterpret_cast<uint32_t*>(wsb);
  P.partials = reinterpret_cast<float*>(wsb + plan.ws_counters_bytes);
  P.xs = wsb + plan.ws_counters_bytes + ((plan.ws_partials_bytes + 255) / 256) * 256;
  P.status = status;
  P.scale_kind = scale_kind;
  P.group_k = group_k;
  P.n_groups_k = group_k ? L.K / group_k : 0;
  P.M = plan.M;
  P.T = plan.T;
  P.NT = plan.NT;
  P.T_pass = plan.T_pass;
  P.n_pass = plan.n_pass;
  P.H = plan.H;
  P.C = plan.C;
  P.D = plan.D;
  P.n_bufs = plan.n_bufs;
  P.x_stages = plan.x_stages;
  P.tmem_cols = plan.tmem_cols;
  P.n_rb = L.N / L.tile_n;
  P.n_units = plan.n_units;
  P.idesc = idesc_f16(plan.ab_f16 ? 0u : 1u, 128, plan.T);
  P.off_lut = plan.off_lut;
  P.off_w = plan.off_w;
  P.off_chunk = plan.off_chunk;
  P.off_x = plan.off_x;
  P.off_bars = plan.off_bars;
  P.trace = g_trace;
  P.X = X;
  P.x_f16 = plan.ab_f16;
  P.n_slots = plan.n_slots;
  P.n_cta = plan.grid;
  P.cta0 = 0;
  return P;
}

// Grid for an elementwise pass over n items, 256 threads a block.
static uint32_t stream_blocks(uint64_t n) {
  uint64_t b = (n + 255) / 256;
  if (b > 4096) b = 4096;
  return b == 0 ? 1u : static_cast<uint32_t>(b);
}

// X (M x K bf16) as f16 into x16, for the formats whose MMA operands are f16.
static cudaError_t convert_x(const uint16_t* X, uint32_t M, uint32_t K, uint8_t* x16,
                             cudaStream_t stream) {
  const uint64_t n8 = static_cast<uint64_t>(M) * K / 8;
  return launch_pdl(x_to_f16_kernel, dim3(stream_blocks(n8)), dim3(256), 0, stream, X,
                    reinterpret_cast<uint16_t*>(x16), n8);
}

// One launch of a single-pass plan.  x16_ready: this call's f16 copy of X,
// already made (null: made here when the format wants it).  w16: when set,
// the decode variant also stores every decoded slab there (N x K row-major).
static cudaError_t launch_single(const GemmPlan& plan, const LayerDev& L, bool decode,
                                 const void* w_plain, const uint16_t* X, const uint8_t* x16_ready,
                                 const void* scales, uint32_t scale_kind, uint32_t group_k, float* Y,
                                 void* ws, uint16_t* w16, uint32_t* status, cudaStream_t stream) {
  GemmDev P = make_gemm_dev(plan, L, w_plain, X, scales, scale_kind, group_k, Y, ws, status);
  if (decode && w16) P.w16 = reinterpret_cast<uint8_t*>(w16);  // the decoded slabs' images
  if (!plan.local) {
    // X for the MMA as a tensor map: the caller's bf16 X, or its f16 copy
    const void* xsrc = X;
    if (plan.ab_f16) {
      if (x16_ready) {
        P.xs = x16_ready;
      } else {
        cudaError_t e = convert_x(X, plan.M, L.K, const_cast<uint8_t*>(P.xs), stream);
        if (e != cudaSuccess) return e;
      }
      xsrc = P.xs;
    }
    cudaError_t e = encode_tmap(&P.tmap_x, CU_TENSOR_MAP_DATA_TYPE_UINT16, xsrc, L.K, plan.M,
                                static_cast<uint64_t>(L.K) * 2, 16, plan.T, CU_TENSOR_MAP_SWIZZLE_32B);
    if (e != cudaSuccess) return e;
    if (!decode) {
      const uint32_t cm = copy_mode_of(plan.fmt);
      if (cm == kCopyTmaSlab)
        e = encode_tmap(&P.tmap_w, CU_TENSOR_MAP_DATA_TYPE_UINT16, w_plain, L.K, L.N,
                        static_cast<uint64_t>(L.K) * 2, 16, 128, CU_TENSOR_MAP_SWIZZLE_32B);
      else if (cm == kCopyTmaRaw)
        e = encode_tmap(&P.tmap_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_plain, L.K, L.N, L.K, 16, 128,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
      if (e != cudaSuccess) return e;
    }
  }
  if (plan.local) return launch_gemm_local(plan, P, decode, stream);

  switch (plan.fmt | (decode ? 0u : 16u)) {  // 16 | fmt: the copy variants
    case kFmtBf16Split:
      return P.L.wide ? launch_variant<true, kFmtBf16Split, true>(plan, P, stream)
                      : launch_variant<true, kFmtBf16Split>(plan, P, stream);
    case kFmtInt4Bf16:
      return P.L.wide ? launch_variant<true, kFmtInt4Bf16, true>(plan, P, stream)
                      : launch_variant<true, kFmtInt4Bf16>(plan, P, stream);
    case kFmtInt4F16Group:
      return P.L.wide ? launch_variant<true, kFmtInt4F16Group, true>(plan, P, stream)
                      : launch_variant<true, kFmtInt4F16Group>(plan, P, stream);
    case kFmtInt4PairBf16:
      return P.L.wide ? launch_variant<true, kFmtInt4PairBf16, true>(plan, P, stream)
                      : launch_variant<true, kFmtInt4PairBf16>(plan, P, stream);
    case kFmtInt4PairF16Group:
      return P.L.wide ? launch_variant<true, kFmtInt4PairF16Group, true>(plan, P, stream)
                      : launch_variant<true, kFmtInt4PairF16Group>(plan, P, stream);
    case kFmtFp8F16:
      return P.L.wide ? launch_variant<true, kFmtFp8F16, true>(plan, P, stream)
                      : launch_variant<true, kFmtFp8F16>(plan, P, stream);
    case kFmtInt8F16:
      return P.L.wide ? launch_variant<true, kFmtInt8F16, true>(plan, P, stream)
                      : launch_variant<true, kFmtInt8F16>(plan, P, stream);
    case kFmtFp4Bf16:
      return P.L.wide ? launch_variant<true, kFmtFp4Bf16, true>(plan, P, stream)
                      : launch_variant<true, kFmtFp4Bf16>(plan, P, stream);
    case kFmtFp4PairBf16:
      return P.L.wide ? launch_variant<true, kFmtFp4PairBf16, true>(plan, P, stream)
                      : launch_variant<true, kFmtFp4PairBf16>(plan, P, stream);
    case 16 | kFmtBf16Split: return launch_variant<false, kFmtBf16Split>(plan, P, stream);
    case 16 | kFmtInt4Bf16: return launch_variant<false, kFmtInt4Bf16>(plan, P, stream);
    case 16 | kFmtInt4F16Group: return launch_variant<false, kFmtInt4F16Group>(plan, P, stream);
    case 16 | kFmtFp8F16: return launch_variant<false, kFmtFp8F16>(plan, P, stream);
    case 16 | kFmtInt8F16: return launch_variant<false, kFmtInt8F16>(plan, P, stream);
    case 16 | kFmtFp4Bf16: return launch_variant<false, kFmtFp4Bf16>(plan, P, stream);
  }
  return cudaErrorInvalidValue;
}

static cudaError_t format_w16(uint32_t fmt, const void* w, const void* scales, const LayerDev& L,
                              uint32_t group_k, uint8_t* w16, cudaStream_t stream) {
  const uint64_t n8 = static_cast<uint64_t>(L.N) * L.K / 8;
  const uint32_t ngk = group_k ? L.K / group_k : 0;
  const dim3 g(stream_blocks(n8)), b(256);
  switch (fmt) {
    case kFmtBf16Split:
      return launch_pdl(format_w16_kernel<kFmtBf16Split>, g, b, 0, stream, w, scales, L.K, group_k, ngk, w16, n8);
    case kFmtInt4Bf16:
      return launch_pdl(format_w16_kernel<kFmtInt4Bf16>, g, b, 0, stream, w, scales, L.K, group_k, ngk, w16, n8);
    case kFmtInt4F16Group:
      return launch_pdl(format_w16_kernel<kFmtInt4F16Group>, g, b, 0, stream, w, scales, L.K, group_k, ngk, w16, n8);
    case kFmtFp8F16:
      return launch_pdl(format_w16_kernel<kFmtFp8F16>, g, b, 0, stream, w, scales, L.K, group_k, ngk, w16, n8);
    case kFmtInt8F16:
      return launch_pdl(format_w16_kernel<kFmtInt8F16>, g, b, 0, stream, w, scales, L.K, group_k, ngk, w16, n8);
    case kFmtFp4Bf16:
      return launch_pdl(format_w16_kernel<kFmtFp4Bf16>, g, b, 0, stream, w, scales, L.K, group_k, ngk, w16, n8);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_gemm(const GemmPlan& plan, const LayerDev& L, bool decode, const void* w_plain,
                        const uint16_t* X, const void* scales, uint32_t scale_kind,
                        uint32_t group_k, float* Y, void* ws, uint32_t* status,
                        cudaStream_t stream) {
  if (plan.M == 0) return cudaSuccess;
  if (!plan.dense)
    return launch_single(plan, L, decode, w_plain, X, nullptr, scales, scale_kind, group_k, Y, ws,
                         nullptr, status, stream);
  // Large M: the first M_first tokens fused (the decode variant storing the
  // decoded weights into W16), then every other token in one dense GEMM on
  // W16 -- the uncompressed variant formats its codes into W16 the same way
  // (bf16 weights are used as they are), so both variants feed the dense
  // kernel the same operands.
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  uint8_t* x16 = wsb + plan.ws_counters_bytes + (plan.ws_partials_bytes + 255) / 256 * 256;
  uint16_t* w16 = reinterpret_cast<uint16_t*>(x16 + (plan.ws_x16_bytes + 255) / 256 * 256);
  cudaError_t e;
  if (plan.ab_f16) {
    e = convert_x(X, plan.M, L.K, x16, stream);
    if (e != cudaSuccess) return e;
  }
  GemmPlan first;
  if (!make_gemm_plan(L, plan.M_first, scale_kind, decode, static_cast<int>(plan.sms), &first))
    return cudaErrorInvalidValue;
  e = launch_single(first, L, decode, w_plain, X, plan.ab_f16 ? x16 : nullptr, scales, scale_kind,
                    group_k, Y, ws, decode ? w16 : nullptr, status, stream);
  if (e != cudaSuccess) return e;
  if (!decode) {
    e = format_w16(plan.fmt, w_plain, scales, L, group_k, reinterpret_cast<uint8_t*>(w16), stream);
    if (e != cudaSuccess) return e;
  }
  const uint32_t M_rest = plan.M - plan.M_first;
  const void* xr = plan.ab_f16 ? static_cast<const void*>(x16 + static_cast<uint64_t>(plan.M_first) * L.K * 2)
                               : static_cast<const void*>(X + static_cast<uint64_t>(plan.M_first) * L.K);
  DenseDev D;
  std::memset(&D, 0, sizeof(D));
  D.w16 = reinterpret_cast<const uint8_t*>(w16);
  D.k_slabs = L.K / 16;
  // a box of at most M_rest rows; the MMA's token columns past it hold stale
  // shared memory and are never stored
  e = encode_tmap(&D.tmap_b, CU_TENSOR_MAP_DATA_TYPE_UINT16, xr, L.K, M_rest,
                  static_cast<uint64_t>(L.K) * 2, 64, std::min(M_rest, 256u),
                  CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  D.Y = Y + static_cast<uint64_t>(plan.M_first) * L.N;
  D.scales = scales;
  D.status = status;
  D.scale_kind = scale_kind;
  D.M = M_rest;
  D.N = L.N;
  D.K = L.K;
  D.m_blocks = (M_rest + 255) / 256;
  D.n_tiles = D.m_blocks * (L.N / 128);
  D.b_box_rows = std::min(M_rest, 256u);
  D.idesc = idesc_f16(plan.ab_f16 ? 0u : 1u, 128, 256);
  const uint32_t tail = M_rest - (D.m_blocks - 1) * 256;
  D.idesc_tail = idesc_f16(plan.ab_f16 ? 0u : 1u, 128, (tail + 15) / 16 * 16);
  return launch_dense_gemm(D, plan.sms, stream);
}

cudaError_t launch_gemm_batched(const GemmPlan* plans, uint32_t n, const LayerDev* const* Ls,
                                const uint16_t* const* Xs, const void* const* scales,
                                uint32_t scale_kind, uint32_t group_k, float* const* Ys, void* ws,
                                const size_t* ws_off, uint32_t* status, cudaStream_t stream) {
  if (n == 0 || plans[0].M == 0) return cudaSuccess;
  if (n > kMaxBatch) return cudaErrorInvalidValue;
  static_assert(sizeof(BatchDev) <= 32000, "kernel parameter limit");
  BatchDev B;
  std::memset(&B, 0, sizeof(B));
  B.n_jobs = n;
  GemmPlan shape = plans[0];  // the launch: the largest producer count and shared memory
  uint32_t cta = 0;
  for (uint32_t j = 0; j < n; ++j) {
    if (!plans[j].local || plans[j].dense || plans[j].fmt != plans[0].fmt) return cudaErrorInvalidValue;
    B.job[j] = make_gemm_dev(plans[j], *Ls[j], nullptr, Xs[j], scales[j], scale_kind, group_k,
                             Ys[j], static_cast<uint8_t*>(ws) + ws_off[j], status);
    B.job[j].cta0 = cta;
    cta += plans[j].grid;
    shape.D = std::max(shape.D, plans[j].D);
    shape.smem_bytes = std::max(shape.smem_bytes, plans[j].smem_bytes);
  }
  return launch_gemm_local_batch(shape, B, cta, stream);
}

}  // namespace ansdev
