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
#include <cuda_runtime.h>

#include <cstdlib>
#include <cstring>

#include "gemm_common.cuh"
#include "kernels.h"
#include "launch.h"
#include "rans_core.cuh"

namespace ansdev {

constexpr uint32_t kFixedWarps = 6;
constexpr uint32_t kMaxProducers = 16;
constexpr uint32_t kMaxThreads = (kFixedWarps + kMaxProducers) * 32;

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
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  volatile uint32_t* abort = &abort_flag;
  // the prologue above read only kernel parameters: from here on global
  // memory, after the previous grid in the stream (X staging) has completed
  griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x == 0) trace_mark(P, 0);

  if (warp >= kFixedWarps) {
    // ======================= producer warps =======================
    const uint32_t d = warp - kFixedWarps;
    const uint32_t lt = lanemask_lt();
    const LayerDev& L = P.L;
    const bool single = L.single_symbol != kNoSymbol;
    const uint32_t H = P.H;
    const uint32_t n_slabs = P.H * P.C;
    const uint32_t groups = n_slabs * 8;  // 8 groups of 8 symbols per lane fill one slab
    const uint32_t lut_s = smem_u32(lut);
    TileSeq seq{static_cast<uint32_t>(u_begin) + d, D, static_cast<uint32_t>(u_end), L.n_tiles};
    ChunkPipe pipe;
    pipe_init(pipe, chunks + d * kRingStride, B.chunk + 4 * d);
    TileCursor tc;
    tc.cb = 0;
    uint32_t sc = 0;  // unit slabs produced
    const uint32_t swz = ((lane >> 2) & 1u) << 4;
    const uint32_t wslots_s = smem_u32(wring + 2 * d * kSlabBytes);

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
        if (!kDecode) {
#pragma unroll
          for (int gg = 0; gg < 8; ++gg) {
            const uint32_t i = gg & 3, c = gg >> 2;
            const uint64_t row = n0 + lane + 32 * (4 * h + i);
            const uint64_t idx = row * L.K + k0 + 16 * s + 8 * c;
            if (kFmt == kFmtBf16Split) {
              cp[gg] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(P.w_plain) + idx));
            } else if (kFmt == kFmtFp8F16 || kFmt == kFmtInt8F16) {
              uint2 v = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint8_t*>(P.w_plain) + idx));
              cp[gg] = make_uint4(v.x, v.y, 0, 0);
            } else {
              uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(P.w_plain) + idx / 2));
              cp[gg] = make_uint4(v, 0, 0, 0);
            }
          }
        }
        if (sc >= 2) wait_live(&B.w_empty[2 * d + slot], ((sc >> 1) + 1) & 1u, abort, P.status, 1, 64);
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
            if (kFmt == kFmtBf16Split) {
              o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
            } else {
              uint32_t e[8];
              if (kFmt == kFmtFp8F16 || kFmt == kFmtInt8F16) {
                  const uint32_t flip = kFmt == kFmtInt8F16 ? 0x80u : 0u;  // int8: symbol = byte ^ 0x80
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  e[k] = (((v.x >> (8 * k)) & 0xFFu) ^ flip) << 12;
                  e[k + 4] = (((v.y >> (8 * k)) & 0xFFu) ^ flip) << 12;
                }
                if constexpr (kFmt == kFmtInt8F16) fmt_int8_f16(e, o);
                else fmt_fp8_f16(e, o);
              } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) e[k] = (((v.x >> (4 * k)) & 0xFu) ^ (kFmt == kFmtFp4Bf16 ? 0u : 8u)) << 12;
                if (kFmt == kFmtFp4Bf16) fmt_fp4_bf16(e, o);
                else if (kFmt == kFmtInt4Bf16) fmt_int4_bf16(e, o);
                else fmt_int4_f16_scaled(e, i == 0 ? gs0 : i == 1 ? gs1 : i == 2 ? gs2 : gs3, o);
              }
            }
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
        if (lane == 0 && sc == 0) trace_mark(P, 2 + d);
        ++sc;
      }
      if (kDecode && !zero_tile) {
        if (!tile_end(L, tc, single) && lane == 0) atomicOr(P.status, kStatusCorrupt);
      }
    }
    if (kDecode) pipe_drain(pipe, P.status);
    if (lane == 0) trace_mark(P, 18 + d);
  } else if (warp == 4) {
    // ======================= MMA issue (one thread) =======================
    if (lane == 0) {
      const uint32_t ub = static_cast<uint32_t>(u_begin), ue = static_cast<uint32_t>(u_end);
      const uint32_t seg_begin = ub / n_kt;
      // descriptor fields shared by every operand: LBO 16 B, SBO 256 B,
      // version 1, 32-byte swizzle; only the start address varies
      const uint64_t dhi = (1ull << 16) | (16ull << 32) | (1ull << 46) | (6ull << 61);
      const uint32_t a_base = smem_u32(wring) >> 4, x_base = smem_u32(xring) >> 4;
      const uint32_t slab16 = kSlabBytes >> 4, xstage16 = x_stage_bytes >> 4, t16 = (P.T * 32) >> 4;
      uint32_t fresh = 0;  // bit (buf * 2 + h): next MMA into that accumulator starts it
      uint32_t xs = 0, xpar = 0;
      uint32_t r = 0;
      for (uint32_t u0 = ub; u0 < ue; u0 += D, ++r) {
        const uint32_t nd = min(D, ue - u0);
        const uint32_t seg0 = u0 / n_kt, kt0 = u0 - seg0 * n_kt;
        const uint32_t nA = P.n_bufs == 2 ? nd : min(nd, n_kt - kt0);
        for (uint32_t part = 0; part < 2; ++part) {
          const uint32_t d_lo = part == 0 ? 0 : nA, d_hi = part == 0 ? nA : nd;
          for (uint32_t s = 0; s < P.C; ++s) {
            for (uint32_t d = d_lo; d < d_hi; ++d) {
              const uint32_t kt = kt0 + d;
              const bool wrap = kt >= n_kt;
              const uint32_t ktw = wrap ? kt - n_kt : kt;
              const uint32_t lseg = seg0 + (wrap ? 1u : 0u) - seg_begin;
              const uint32_t buf = P.n_bufs == 2 ? (lseg & 1u) : 0u;
              if (s == 0 && (u0 + d == ub || ktw == 0)) {
                const uint32_t k = P.n_bufs == 2 ? (lseg >> 1) : lseg;
                if (k >= 1) wait_live(&B.acc_empty[buf], (k - 1) & 1u, abort, P.status, 4);
                tc_fence_after();
                fresh |= 3u << (2 * buf);
              }
              wait_live(&B.x_full[xs], xpar, abort, P.status, 2);
              for (uint32_t h = 0; h < P.H; ++h) {
                const uint32_t idx = (r * P.C + s) * P.H + h;
                const uint32_t slot = idx & 1u;
                wait_live(&B.w_full[2 * d + slot], (idx >> 1) & 1u, abort, P.status, 3);
                tc_fence_after();
                const uint64_t adesc = dhi | (a_base + (2 * d + slot) * slab16);
                const uint32_t acc_bit = 1u << (2 * buf + h);
                const uint32_t accumulate = (fresh & acc_bit) ? 0u : 1u;
                for (uint32_t j = 0; j < P.NT; ++j) {
                  const uint64_t bdesc = dhi | (x_base + xs * xstage16 + j * t16);
                  const uint32_t col = ((buf * P.H + h) * P.NT + j) * P.T;
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
          if (P.n_bufs == 2) break;  // one part: the whole round slab-major
        }
      }
      umma_commit(B.mma_done);
      trace_mark(P, 34);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ======================= X loader (TMA, one thread) =======================
    if (lane == 0) {
      uint32_t xc = 0;
      uint32_t n_issued = 0;  // loads issued: steps [0, n_issued) (none after an abort)
      long long xw = 0, xi = 0;
      const long long xb = clock64();
      for_each_mma_step(P, static_cast<uint32_t>(u_begin), static_cast<uint32_t>(u_end),
                        [&](uint32_t, uint32_t s, uint32_t, uint32_t, const UnitInfo& I) {
        const uint32_t xs = xc % XS;
        long long c0 = clock64();
        if (xc >= XS) wait_live(&B.x_empty[xs], ((xc / XS) + 1) & 1u, abort, P.status, 5);
        xw += clock64() - c0;
        c0 = clock64();
        const uint32_t p = I.p;
        const uint32_t kx = I.kt * P.L.tile_k + 16 * s;
        if (!*abort && n_issued == xc) {
          // X slab (pass p, 16-column slab kx/16) is T_pass x 32 contiguous,
          // pre-swizzled bytes in the staged copy: one bulk copy
          const uint64_t slab = static_cast<uint64_t>(p) * (P.L.K / 16) + kx / 16;
          mbar_arrive_expect_tx(&B.x_full[xs], P.T_pass * 32);
          bulk_g2s(xring + xs * x_stage_bytes, P.xs + slab * (P.T_pass * 32), P.T_pass * 32,
                   &B.x_full[xs]);
          n_issued = xc + 1;
        }
        xi += clock64() - c0;
        ++xc;
      });
      if (P.trace) {
        P.trace[blockIdx.x * 64 + 53] = xw;
        P.trace[blockIdx.x * 64 + 54] = xi;
        P.trace[blockIdx.x * 64 + 55] = clock64() - xb;
        P.trace[blockIdx.x * 64 + 56] = xc;
      }
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
          for (uint32_t cc = 0; cc < P.T; cc += 16) {
            uint32_t v[16];
            tmem_ld16(tmem_base + ((32 * warp) << 16) + col0 + cc, v);
            tmem_ld_wait();
            float f[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) f[q] = __uint_as_float(v[q]);
            epi_emit16(P, f, complete, scale, part, p, h, j * P.T + cc, n, e);
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

// Stages X for the fused kernel: for every token pass p and 16-column slab
// ks, a contiguous block of T_pass rows x 32 bytes holding X[p*T_pass + r]
// [16 ks .. 16 ks + 15] (zero for rows >= M), its two 16-byte chunks placed
// with the 32-byte swizzle the MMA descriptor expects (chunk c of row r at
// c ^ ((r >> 2) & 1)); optionally converted to f16.  One thread per chunk.
__global__ void x_stage_kernel(const uint16_t* __restrict__ X, uint8_t* __restrict__ xs,
                               uint32_t M, uint32_t K, uint32_t T_pass, uint32_t n_pass,
                               uint32_t to_f16) {
  griddep_wait();
  griddep_launch_dependents();
  const uint64_t n_chunks = static_cast<uint64_t>(n_pass) * (K / 16) * T_pass * 2;
  for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_chunks;
       i += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
    const uint32_t c = static_cast<uint32_t>(i & 1);
    const uint64_t rest = i >> 1;
    const uint32_t r = static_cast<uint32_t>(rest % T_pass);
    const uint64_t slab = rest / T_pass;  // p * (K / 16) + ks
    const uint32_t ks = static_cast<uint32_t>(slab % (K / 16));
    const uint32_t p = static_cast<uint32_t>(slab / (K / 16));
    const uint32_t m = p * T_pass + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (m < M) {
      v = __ldg(reinterpret_cast<const uint4*>(X + static_cast<uint64_t>(m) * K + 16 * ks + 8 * c));
      if (to_f16) {
        uint32_t in[4] = {v.x, v.y, v.z, v.w}, out[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          __half2 h = __floats2half2_rn(__uint_as_float(in[k] << 16), __uint_as_float(in[k] & 0xFFFF0000u));
          out[k] = *reinterpret_cast<uint32_t*>(&h);
        }
        v = make_uint4(out[0], out[1], out[2], out[3]);
      }
    }
    const uint64_t dst = slab * (static_cast<uint64_t>(T_pass) * 32) + r * 32 + ((c ^ ((r >> 2) & 1u)) << 4);
    *reinterpret_cast<uint4*>(xs + dst) = v;
  }
}

// =============================== host side ===============================

static uint32_t round_up(uint32_t a, uint32_t b) { return (a + b - 1) / b * b; }

static unsigned long long* g_trace = nullptr;
void set_trace_buffer(void* d_buf, size_t bytes) {
  g_trace = bytes >= 64 * sizeof(unsigned long long) ? static_cast<unsigned long long*>(d_buf) : nullptr;
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
  // Tuning / testing knobs: cap the CTA count and the producer warps per CTA,
  // force one of the two schedules.
  if (const char* v = std::getenv("ANS_GEMM_MAX_CTAS")) {
    long cap = std::strtol(v, nullptr, 10);
    if (cap > 0 && static_cast<uint64_t>(cap) < sms) sms = static_cast<uint64_t>(cap);
  }
  uint32_t D_cap = kMaxProducers;
  if (const char* v = std::getenv("ANS_GEMM_MAX_PRODUCERS")) {
    long cap = std::strtol(v, nullptr, 10);
    if (cap > 0 && static_cast<uint32_t>(cap) < D_cap) D_cap = static_cast<uint32_t>(cap);
  }
  // unit indices are 32-bit in the kernels
  if (static_cast<uint64_t>(L.n_tiles) * ((M + 15) / 16) >= (1ull << 31)) return false;
  bool want_local = p.H * Mp <= 32;
  if (const char* v = std::getenv("ANS_GEMM_SCHEDULE")) {
    if (std::strcmp(v, "central") == 0) want_local = false;
  }
  const uint32_t lut_bytes = kSlots * 4;

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
    uint32_t D = D_cap < kLocalProducersMax ? D_cap : kLocalProducersMax;
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

  // ---- shared-accumulator schedule: one MMA-issuing thread per CTA
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
  uint32_t cols = p.n_bufs * p.H * p.T_pass;
  p.tmem_cols = 32;
  while (p.tmem_cols < cols) p.tmem_cols <<= 1;
  if (p.tmem_cols > 512) return false;

  p.n_units = static_cast<uint64_t>(p.n_pass) * L.n_tiles;
  p.n_segments = p.n_pass * (L.N / L.tile_n);
  p.grid = static_cast<uint32_t>(p.n_units < sms ? p.n_units : sms);
  uint64_t per_cta = (p.n_units + p.grid - 1) / p.grid;

  // shared memory: [lut][w rings][chunk rings][x stages][barriers]
  const uint32_t x_stage = p.T_pass * 32;
  uint32_t D = D_cap;
  if (D > L.n_kt) D = L.n_kt;
  if (D > per_cta) D = static_cast<uint32_t>(per_cta);
  // X stages take whatever shared memory the producers leave (deep rings keep
  // every X slab of a round in flight at small M), at least 2, at most 64.
  uint32_t XS = 0;
  for (;;) {
    uint32_t off = lut_bytes;
    off = round_up(off, 2048);
    const uint32_t off_w = off;
    off += D * 2 * kSlabBytes;
    off = round_up(off, 128);
    const uint32_t off_chunk = off;
    off += D * kRingStride + 128;
    off = round_up(off, 1024);
    const uint32_t off_x = off;
    const uint32_t bars_max = num_bars(D, 64) * 8;
    const uint32_t room = kSmemLimit > off + bars_max ? kSmemLimit - off - bars_max : 0;
    XS = room / x_stage;
    if (XS > 64) XS = 64;
    if (XS >= 2) {
      off += XS * x_stage;
      off = round_up(off, 8);
      p.off_lut = 0;
      p.off_w = off_w;
      p.off_chunk = off_chunk;
      p.off_x = off_x;
      p.off_bars = off;
      off += num_bars(D, XS) * 8;
      p.smem_bytes = off;
      break;
    }
    if (D > 1) { --D; continue; }
    return false;
  }
  p.D = D;
  p.x_stages = XS;
  p.ws_partials_bytes = static_cast<size_t>(p.grid) * 2 * p.H * p.T_pass * 128 * sizeof(float);
  p.ws_counters_bytes = round_up(p.n_segments * 4, 256);
  p.ws_x16_bytes = static_cast<size_t>(p.n_pass) * p.T_pass * L.K * 2;  // staged X slabs
  p.ws_bytes = p.ws_counters_bytes + (p.ws_partials_bytes + 255) / 256 * 256 +
               (p.ws_x16_bytes + 255) / 256 * 256;
  *plan = p;
  return true;
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

cudaError_t launch_gemm(const GemmPlan& plan, const LayerDev& L, bool decode, const void* w_plain,
                        const uint16_t* X, const void* scales, uint32_t scale_kind,
                        uint32_t group_k, float* Y, void* ws, uint32_t* status,
                        cudaStream_t stream) {
  if (plan.M == 0) return cudaSuccess;
  const GemmDev P = make_gemm_dev(plan, L, w_plain, X, scales, scale_kind, group_k, Y, ws, status);
  if (!plan.local) {
    const uint64_t n_chunks = static_cast<uint64_t>(plan.n_pass) * (L.K / 16) * plan.T_pass * 2;
    uint32_t blocks = static_cast<uint32_t>((n_chunks + 255) / 256);
    if (blocks > 4096) blocks = 4096;
    if (blocks == 0) blocks = 1;
    cudaError_t e = launch_pdl(x_stage_kernel, dim3(blocks), dim3(256), 0, stream, X,
                               const_cast<uint8_t*>(P.xs), plan.M, L.K, plan.T_pass,
                               plan.n_pass, plan.ab_f16);
    if (e != cudaSuccess) return e;
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

cudaError_t launch_gemm_batched(const GemmPlan& plan, uint32_t n, const LayerDev* const* Ls,
                                const uint16_t* const* Xs, const void* const* scales,
                                uint32_t scale_kind, uint32_t group_k, float* const* Ys, void* ws,
                                uint32_t* status, cudaStream_t stream) {
  if (plan.M == 0 || n == 0) return cudaSuccess;
  if (!plan.local || n > kMaxBatch) return cudaErrorInvalidValue;
  static_assert(sizeof(BatchDev) <= 32000, "kernel parameter limit");
  BatchDev B;
  std::memset(&B, 0, sizeof(B));
  B.n_jobs = n;
  const size_t ws_job = ((plan.ws_bytes + 255) / 256) * 256;
  for (uint32_t j = 0; j < n; ++j) {
    B.job[j] = make_gemm_dev(plan, *Ls[j], nullptr, Xs[j], scales[j], scale_kind, group_k, Ys[j],
                             static_cast<uint8_t*>(ws) + j * ws_job, status);
    B.job[j].cta0 = j * plan.grid;
  }
  return launch_gemm_local_batch(plan, B, n * plan.grid, stream);
}

}  // namespace ansdev
