// gemm_local.cu -- fused tile-rANS decode + GEMM for small token counts
// (M <= 32): private accumulators per producer warp, one issuing warp.
//
// "Approaching Shannon Bound with Lossless LLM Weight Compression", s3.1
// "整体执行模型": decoder warps decode compressed tiles straight into shared
// memory and the decoded tile is consumed there by the GEMM; decoding of the
// next slab overlaps the MMA on the current one; buffers are released in an
// order fixed by the traversal.
//
// Schedule (swap-AB, Y^T = W X^T, as in gemm.cu):
//   * The units (tiles) are split into one contiguous range per CTA and,
//     inside it, one contiguous sub-range per producer warp, so a producer
//     streams one contiguous run of compressed bytes (RunPipe).
//   * A producer decodes a 128 x 16 slab of W into one of its two
//     shared-memory slots, writes the matching 16-column slab of X next to
//     it and signals the slab on an mbarrier.  The store of each group of 8
//     decoded columns is deferred until the next group's first decode step
//     has been issued, so it overlaps the decode chain.
//   * One issuing warp (one lane per producer) hands every ready slab to the
//     tensor core as soon as it is signalled -- tcgen05.mma issues are
//     serialised per SM, so producers never wait in that queue -- into the
//     producer's own TMEM accumulator, in that producer's slab order; the
//     MMA's completion (tcgen05.commit) frees the slot.
//   * A producer owns one accumulator per W row-block segment it touches, so
//     an accumulator is written in a fixed order and read once; no warp waits
//     for the epilogue.  The epilogue sums the accumulators of a segment in
//     ascending unit order, then stores Y or takes part in the deterministic
//     split-K reduction (gemm_common.cuh).  Every addition happens in an
//     order fixed by the schedule, so Y is bit-identical to the same kernel
//     fed uncompressed weights.
// Warps: 0-3 epilogue (TMEM lanes 0-127), 4 MMA issue, 5 .. 5 + D - 1 producers.
#include <cuda_runtime.h>

#include <cstring>
#include <type_traits>

#include "gemm_common.cuh"
#include "kernels.h"
#include "launch.h"
#include "rans_core.cuh"

namespace ansdev {

// 5 + 15 = 20 warps: five per SM sub-partition leaves 96 registers a thread
constexpr uint32_t kLocalMaxProducers = kLocalProducersMax;
constexpr uint32_t kLocalFixedWarps = 5;
constexpr uint32_t kLocalThreads = (kLocalFixedWarps + kLocalMaxProducers) * 32;
constexpr uint32_t kLocalMaxSlots = 32;  // 512 TMEM columns / (H * T >= 16) per accumulator
constexpr uint32_t kRawAhead = 3;        // raw-byte groups loaded ahead of their use

// Contiguous sub-range of producer d inside the CTA's range [ub, ue) (the
// same balanced split as the CTA ranges).
__device__ __forceinline__ void producer_range(uint32_t ub, uint32_t ue, uint32_t D, uint32_t d,
                                               uint32_t* b, uint32_t* e) {
  *b = ub + cta_begin(ue - ub, D, d);
  *e = ub + cta_begin(ue - ub, D, d + 1);
}

// First accumulator slot of producer d: slots are numbered in unit order, so
// it follows the segments touched by producers 0 .. d-1.
__device__ __forceinline__ uint32_t producer_first_slot(uint32_t ub, uint32_t ue, uint32_t D,
                                                        uint32_t d, uint32_t n_kt) {
  uint32_t slot = 0;
  for (uint32_t q = 0; q < d; ++q) {
    uint32_t b, e;
    producer_range(ub, ue, D, q, &b, &e);
    if (e > b) slot += (e - 1) / n_kt - b / n_kt + 1;
  }
  return slot;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
__device__ __forceinline__ void sts128(uint32_t addr, const uint32_t (&o)[4]) {
  sts128(addr, o[0], o[1], o[2], o[3]);
}

// One CTA of the launch that P describes: CTA blockIdx.x - P.cta0 of the
// P.n_cta that share P's layer (kBatch), or of the whole grid.
template <bool kDecode, uint32_t kFmt, bool kWide, bool kBatch>
__device__ __forceinline__ void local_cta(const GemmDev& P) {
  extern __shared__ __align__(2048) uint8_t smem[];
  __shared__ uint32_t tmem_slot;
  __shared__ uint32_t abort_flag;
  __shared__ uint32_t reduce_flag;
  __shared__ uint32_t red_n, red_seg[2];  // split-K segments of this CTA
  __shared__ uint32_t slot_seg[kLocalMaxSlots];
  __shared__ uint32_t n_cta_slots;

  const uint32_t warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t D = P.D, H = P.H, C = P.C, T = P.T;
  const uint32_t G = kBatch ? P.n_cta : gridDim.x;
  const uint32_t cta = kBatch ? blockIdx.x - P.cta0 : blockIdx.x;
  const uint32_t ub = cta_begin(static_cast<uint32_t>(P.n_units), G, cta);
  const uint32_t ue = cta_begin(static_cast<uint32_t>(P.n_units), G, cta + 1);
  const uint32_t n_kt = P.L.n_kt, n_tiles = P.L.n_tiles;

  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + P.off_lut);
  uint8_t* wslots = smem + P.off_w;   // 2 per producer, kSlabBytes each
  uint8_t* chunks = smem + (((smem_u32(smem + P.off_chunk) + 127) & ~127u) - smem_u32(smem));
  uint8_t* xslots = smem + P.off_x;   // 2 per producer, T * 32 bytes each
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P.off_bars);
  uint64_t* w_full = bars;                // 2 per producer: slab written
  uint64_t* w_empty = bars + 2 * D;       // 2 per producer: slab consumed by its MMA
  uint64_t* chunk_bars = bars + 4 * D;    // 4 per producer: compressed-stream ring
  uint64_t* mma_done = bars + 8 * D;      // every MMA of the CTA retired
  uint64_t* acc_full = bars + 8 * D + 1;  // one per accumulator slot

  // Prologue, on the critical path of every CTA that starts after a CTA of
  // the previous launch left its SM: the barriers are initialised by all
  // threads (one thread initialising them in turn took ~3,300 cycles), warp 0
  // allocates TMEM while the other warps build the slot table.
  if (threadIdx.x == 0) {
    abort_flag = 0;
    red_n = 0;
    reduce_flag = 0;
  }
  const uint32_t n_bars = 8 * D + 1 + P.n_slots;
  for (uint32_t i = threadIdx.x; i < n_bars; i += blockDim.x) mbar_init(&bars[i], i == 8 * D ? 32u : 1u);
  if (threadIdx.x < n_bars) fence_mbar_init();
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
  // memory, after the previous grid in the stream has completed
  griddep_wait();
  griddep_launch_dependents();
  check_smem_base(smem, P.status);
  if (threadIdx.x == 0) trace_mark(P, 0);

  if (warp >= kLocalFixedWarps + D) {
    // a batched launch is shaped for its job with the most producer warps;
    // the warps beyond this job's producers have no work
  } else if (warp >= kLocalFixedWarps) {
    // ============================ producer warps ============================
    const uint32_t d = warp - kLocalFixedWarps;
    uint32_t pb, pe;
    producer_range(ub, ue, D, d, &pb, &pe);
    const LayerDev& L = P.L;
    const bool single = L.single_symbol != kNoSymbol;
    const uint32_t lt = lanemask_lt();
    const uint32_t lut_s = smem_u32(lut);
    const uint32_t swz = ((lane >> 2) & 1u) << 4;
    const uint32_t w_s0 = smem_u32(wslots + 2 * d * kSlabBytes);
    const uint32_t x_s0 = smem_u32(xslots + 2 * d * T * 32);
    const unsigned long long* offsets = reinterpret_cast<const unsigned long long*>(L.offsets);
    const uint32_t S = L.tile_n * L.tile_k;
    const uint32_t n_xch = T / 16;  // 16-byte X chunks per lane per slab (1 or 2)
    RunPipe pipe;
    rp_init(pipe, chunks + d * kRingStride, chunk_bars + 4 * d);
    TileCursor tc;
    tc.x = tc.pos = tc.cb = tc.bytes = 0;
    uint32_t nw = 0;  // slabs signalled to the issuing warp

    uint32_t u = pb;
    while (u < pe) {
      const uint32_t p = u / n_tiles;
      const uint32_t run_e = min(pe, (p + 1) * n_tiles);
      const uint32_t t0 = u - p * n_tiles;
      const uint32_t t1 = run_e - 1 - p * n_tiles;
      bool run_ok = true;
      uint64_t run_start = 0, a_next = 0;
      uint32_t run_bytes = 0, base = 0;
      if (kDecode) {
        run_ok = run_extent(L, t0, t1, &run_start, &run_bytes);
        if (run_ok) {
          base = rp_run_begin(pipe, L.stream + run_start, run_bytes);
          rp_prefetch(pipe, base, lane, abort, P.status);
        }
        a_next = run_start;
      }
      // raw sign/mantissa bytes (bf16, decode; read once, so loaded with the
      // evict-first hint): groups g .. g + kRawAhead - 1 of the current tile in
      // flight.  A run's tiles are consecutive, so their
      // raw blocks are too: the loads run on into the next tile's first groups,
      // and the first tile's are issued here, before its first chunk is awaited.
      const uint32_t groups = H * C * 8;
      uint64_t rq[kRawAhead];
#pragma unroll
      for (uint32_t k = 0; k < kRawAhead; ++k) rq[k] = 0;
      bool rq_ready = false;  // rq holds groups 0 .. kRawAhead - 1 of tile u
      if (kDecode && kFmt == kFmtBf16Split && run_ok) {
        const unsigned long long* r0 =
            reinterpret_cast<const unsigned long long*>(L.raw + static_cast<uint64_t>(t0) * S) + lane;
#pragma unroll
        for (uint32_t k = 0; k < kRawAhead; ++k) rq[k] = __ldcs(r0 + 32 * k);
        rq_ready = true;
      }
      for (; u < run_e; ++u) {
        const uint32_t t = u - p * n_tiles;
        const uint32_t rb = t / n_kt, kt = t - rb * n_kt;
        const uint32_t n0 = rb * L.tile_n, k0 = kt * L.tile_k;
        bool zero_tile = false;
        if (kDecode) {
          zero_tile = !run_ok;
          if (run_ok) {
            const uint64_t a = a_next, b = __ldg(offsets + t + 1);
            a_next = b;
            if (!run_tile_begin(pipe, L, a, b, run_start, base, tc, lane, abort, P.status)) {
              run_ok = false;
              zero_tile = true;
            }
          }
          if (zero_tile && lane == 0) atomicOr(P.status, kStatusBadOffsets);
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
        const unsigned long long* raw_tile = nullptr;
        // the loads may run into the next tile's raw block while one exists
        const uint32_t raw_lim = (t + 1 < n_tiles) ? groups + kRawAhead : groups;
        if (kDecode && kFmt == kFmtBf16Split && !zero_tile) {
          raw_tile = reinterpret_cast<const unsigned long long*>(L.raw + static_cast<uint64_t>(t) * S) + lane;
          if (!rq_ready) {
#pragma unroll
            for (uint32_t k = 0; k < kRawAhead; ++k) rq[k] = __ldcs(raw_tile + 32 * k);
          }
        }
        // the slabs of this tile; a tile of constant symbols (single-symbol
        // codebook, or zeros for a tile with bad offsets) takes a separate
        // instantiation so the decoding path carries no per-group branches
        const uint32_t const_e = zero_tile ? 0u : (single ? L.single_symbol << 12 : 0u);
        auto run_slabs = [&](auto const_sym) {
          constexpr bool kConst = decltype(const_sym)::value;
          for (uint32_t us = 0; us < H * C; ++us) {
            const uint32_t h = us % H, s = us / H;
            const uint32_t slot = nw & 1u;
            const uint32_t w_s = w_s0 + slot * kSlabBytes, x_s = x_s0 + slot * T * 32;
            __half2 gsc[4];
            if (fmt_group(kFmt)) {
              gsc[0] = h ? gscale[4] : gscale[0];
              gsc[1] = h ? gscale[5] : gscale[1];
              gsc[2] = h ? gscale[6] : gscale[2];
              gsc[3] = h ? gscale[7] : gscale[3];
            }
            // X slab s of this unit (T rows x 16 columns): this lane's chunks,
            // fetched now and stored next to the W slab at its end
            uint4 xv[2];
#pragma unroll
            for (uint32_t j = 0; j < 2; ++j) {
              xv[j] = make_uint4(0, 0, 0, 0);
              const uint32_t r = (lane >> 1) + 16 * j, c = lane & 1u;
              const uint32_t m = p * P.T_pass + r;
              if (j < n_xch && m < P.M)
                xv[j] = __ldg(reinterpret_cast<const uint4*>(P.X + static_cast<uint64_t>(m) * L.K + k0 +
                                                             16 * s + 8 * c));
            }
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
            // the store of group gg - 1 (deferred); the first store into the
            // slot waits for the MMA that last read it (slab nw - 2).  A group
            // is 8 columns of one row, or both 8-column halves of it for int4
            // pair symbols (4 groups per slab).
            constexpr bool kPair = fmt_pair(kFmt);
            constexpr uint32_t kGroups = kPair ? 4 : 8, kOut = kPair ? 8 : 4;
            uint32_t o_prev[kOut];
#pragma unroll
            for (uint32_t k = 0; k < kOut; ++k) o_prev[k] = 0;
            auto store_prev = [&](uint32_t gg) {
              if (gg == 1 && nw >= 2) {
                wait_live(&w_empty[2 * d + slot], ((nw >> 1) + 1) & 1u, abort, P.status, 1);
                if (kDecode && P.w16 != nullptr) {
                  // the W16 store of the slot's previous slab has read it
                  if (lane == 0) bulk_wait_read<1>();
                  __syncwarp();
                }
              }
              const uint32_t row_s = w_s + (32 * ((gg - 1) & 3) + lane) * 32;
              if constexpr (kPair) {
                sts128(row_s + swz, o_prev[0], o_prev[1], o_prev[2], o_prev[3]);
                sts128(row_s + (16u ^ swz), o_prev[4], o_prev[5], o_prev[6], o_prev[7]);
              } else {
                sts128(row_s + ((((gg - 1) >> 2) << 4) ^ swz), o_prev[0], o_prev[1], o_prev[2], o_prev[3]);
              }
            };
#pragma unroll
            for (uint32_t gg = 0; gg < kGroups; ++gg) {
              const uint32_t g = us * 8 + gg;
              [[maybe_unused]] const uint32_t i = gg & 3;  // row quarter (group scales)
              uint32_t o[kOut];
              if (kDecode) {
                [[maybe_unused]] const uint64_t raw8 = rq[0];
                if (kFmt == kFmtBf16Split && (!kConst || !zero_tile)) {
#pragma unroll
                  for (uint32_t k = 0; k + 1 < kRawAhead; ++k) rq[k] = rq[k + 1];
                  if (g + kRawAhead < raw_lim) rq[kRawAhead - 1] = __ldcs(raw_tile + 32 * (g + kRawAhead));
                }
                uint32_t e[8];
                if (kConst) {
#pragma unroll
                  for (int k = 0; k < 8; ++k) e[k] = const_e;
                  if (gg > 0) store_prev(gg);
                } else {
                  rp_group(pipe, tc.pos, lane, abort, P.status);
                  if (kWide) {
                    decode_pair(tc.xw, tc.pos, lut_s, pipe.ring_s, lt, e[0], e[1]);
                    if (gg > 0) store_prev(gg);
#pragma unroll
                    for (int k = 2; k < 8; k += 2)
                      decode_pair(tc.xw, tc.pos, lut_s, pipe.ring_s, lt, e[k], e[k + 1]);
                  } else {
                    e[0] = decode_step(tc.x, tc.pos, lut_s, pipe.ring_s, lt);
                    if (gg > 0) store_prev(gg);
#pragma unroll
                    for (int k = 1; k < 8; ++k) e[k] = decode_step(tc.x, tc.pos, lut_s, pipe.ring_s, lt);
                  }
                }
                if constexpr (kFmt == kFmtInt4PairBf16) fmt_int4pair_bf16(e, o);
                else if constexpr (kFmt == kFmtFp4PairBf16) fmt_fp4pair_bf16(e, o);
                else if constexpr (kFmt == kFmtInt4PairF16Group) fmt_int4pair_f16_scaled(e, gsc[i], o);
                else if constexpr (kFmt == kFmtBf16Split) fmt_bf16_split(e, raw8, o);
                else if constexpr (kFmt == kFmtInt4Bf16) fmt_int4_bf16(e, o);
                else if constexpr (kFmt == kFmtInt4F16Group) fmt_int4_f16_scaled(e, gsc[i], o);
                else if constexpr (kFmt == kFmtInt8F16) fmt_int8_f16(e, o);
                else if constexpr (kFmt == kFmtFp4Bf16) fmt_fp4_bf16(e, o);
                else fmt_fp8_f16(e, o);
                if (kConst && zero_tile) {
#pragma unroll
                  for (uint32_t k = 0; k < kOut; ++k) o[k] = 0;
                }
              } else if constexpr (!kPair) {
                const uint4 v = cp[gg];
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
                    else fmt_int4_f16_scaled(e, gsc[i], o);
                  }
                }
                if (gg > 0) store_prev(gg);
              }
#pragma unroll
              for (uint32_t k = 0; k < kOut; ++k) o_prev[k] = o[k];
            }
            store_prev(kGroups);
            // X slab, then hand the slab to the issuing warp
#pragma unroll
            for (uint32_t j = 0; j < 2; ++j) {
              if (j >= n_xch) break;
              uint4 v = xv[j];
              if (P.x_f16) {
                uint32_t in[4] = {v.x, v.y, v.z, v.w}, out[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  __half2 hv = __floats2half2_rn(__uint_as_float(in[k] << 16),
                                                 __uint_as_float(in[k] & 0xFFFF0000u));
                  out[k] = *reinterpret_cast<uint32_t*>(&hv);
                }
                v = make_uint4(out[0], out[1], out[2], out[3]);
              }
              const uint32_t r = (lane >> 1) + 16 * j, c = lane & 1u;
              const uint32_t xo[4] = {v.x, v.y, v.z, v.w};
              sts128(x_s + r * 32 + ((c ^ ((r >> 2) & 1u)) << 4), xo);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&w_full[2 * d + slot]);
            // first pass of a large-M call: the slab also goes to W16
            if (kDecode && P.w16 != nullptr && lane == 0)
              bulk_s2g_s(P.w16 + ((static_cast<uint64_t>((n0 >> 7) + h) * (L.K >> 4)) + (k0 >> 4) + s) *
                                     kSlabBytes,
                         w_s, kSlabBytes);
            ++nw;
          }
        };
        if (kDecode && (zero_tile || single)) run_slabs(std::true_type{});
        else run_slabs(std::false_type{});
        // groups 0 .. kRawAhead - 1 of tile t + 1 are in rq if this tile's
        // loads ran on into it
        rq_ready = kDecode && kFmt == kFmtBf16Split && !zero_tile && t + 1 < n_tiles;
        if (kDecode && !zero_tile && !run_tile_end(L, tc, single) && lane == 0)
          atomicOr(P.status, kStatusCorrupt);
      }
    }
    if (kDecode) rp_drain(pipe, P.status);
    if (kDecode && P.w16 != nullptr && lane == 0) bulk_wait_all();
    if (lane == 0) trace_mark(P, 18 + d);
  } else if (warp == 4) {
    // ================== MMA issue (lane q follows producer q) ==================
    // Every lane whose producer has a slab ready issues that slab's MMA and
    // commits itself: the ready lanes issue in the same instructions, which
    // the tensor core takes about twice as fast as one thread issuing them in
    // turn.  Each producer's MMAs come from one lane, in slab order, into that
    // producer's own accumulators, so the accumulation order is fixed.
    const uint32_t q = lane;
    uint32_t pb = 0, pe = 0;
    if (q < D) producer_range(ub, ue, D, q, &pb, &pe);
    uint32_t acc_slot = q < D ? producer_first_slot(ub, ue, D, q, n_kt) : 0u;
    uint32_t u = pb, us = 0, nslab = 0, n_issued = 0;
    uint32_t cur_seg = pb / n_kt;
    uint32_t fresh = (1u << H) - 1u;  // bit h: next MMA into half h starts the accumulator
    const uint32_t n_us = H * C;
    // descriptor fields shared by both operands: LBO 16 B, SBO 256 B,
    // version 1, 32-byte swizzle; only the start address differs
    const uint64_t dhi = (1ull << 16) | (16ull << 32) | (1ull << 46) | (6ull << 61);
    const uint32_t a_s = smem_u32(wslots) + 2 * q * kSlabBytes;
    const uint32_t b_s = smem_u32(xslots) + 2 * q * T * 32;
    long long idle_since = clock64();
    const long long idle_budget = g_live_wait_budget;
    for (;;) {
      const bool has = q < D && u < pe;
      if (__ballot_sync(0xFFFFFFFFu, has) == 0) break;
      const uint32_t slot = nslab & 1u;
      const bool ready = has && mbar_try_wait(&w_full[2 * q + slot], (nslab >> 1) & 1u);
      const uint32_t rmask = __ballot_sync(0xFFFFFFFFu, ready);
      if (rmask == 0) {
        if (*abort) break;
        if (clock64() - idle_since > idle_budget) {
          if (lane == 0) {
            *abort = 1u;
            atomicOr(P.status, kStatusTimeout | (1u << (8 + 2)));
          }
          break;
        }
        __nanosleep(32);
        continue;
      }
      idle_since = clock64();
      if (lane == 0 && P.trace) {
        unsigned long long tnow;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(tnow));
        if (P.trace[blockIdx.x * 64 + 36] == 0) P.trace[blockIdx.x * 64 + 36] = tnow;
        P.trace[blockIdx.x * 64 + 37] += __popc(rmask);
        P.trace[blockIdx.x * 64 + 39] += 1;
        P.trace[blockIdx.x * 64 + 42] = tnow;
        P.trace[blockIdx.x * 64 + 43] = __popc(rmask);
      }
      // this lane's slab: accumulator columns, accumulate flag, segment end
      const uint32_t h = us % H;
      const uint32_t col = (acc_slot * H + h) * T;
      const bool accum = ((fresh >> h) & 1u) == 0u;
      const uint32_t d_tmem = tmem_base + col;
      const uint64_t a_desc = dhi | ((a_s + slot * kSlabBytes) >> 4);
      const uint64_t b_desc = dhi | ((b_s + slot * T * 32) >> 4);
      // the lanes that start an accumulator and the lanes that add to one
      // issue in separate instructions, so that the accumulate flag of an
      // instruction is the same on every lane issuing it
      if (ready && !accum) {
        tc_fence_after();
        umma_f16(d_tmem, a_desc, b_desc, P.idesc, 0u);
      }
      __syncwarp();
      if (ready && accum) {
        tc_fence_after();
        umma_f16(d_tmem, a_desc, b_desc, P.idesc, 1u);
      }
      __syncwarp();
      if (ready) {
        const bool seg_end = (us + 1 == n_us) && (u + 1 == pe || (u + 1) / n_kt != cur_seg);
        // the producer reuses this slot only if it has a slab nslab + 2
        const bool reuse = nslab + 2 < (pe - pb) * n_us;
        if (reuse) umma_commit(&w_empty[2 * q + slot]);
        if (seg_end) umma_commit(&acc_full[acc_slot]);
        ++n_issued;
        fresh &= ~(1u << h);
        ++nslab;
        if (++us == n_us) {
          us = 0;
          ++u;
          if (u < pe && u / n_kt != cur_seg) {
            cur_seg = u / n_kt;
            ++acc_slot;
            fresh = (1u << H) - 1u;
          }
        }
      }
      __syncwarp();
    }
    if (lane == 0) trace_mark(P, 35);
    // retirement of every MMA this CTA issued (waited for before TMEM is
    // freed): 32 arrivals, a commit from each lane that issued MMAs (it
    // fires once they are done) and a plain arrival from the others
    if (n_issued) umma_commit(mma_done);
    else mbar_arrive(mma_done);
    __syncwarp();
  } else {
    // ===================== epilogue (warps 0-3, 128 threads) =====================
    const uint32_t e = threadIdx.x;   // TMEM lane = row within the 128-row half
    const uint32_t nck = H * T / 16;  // 16-column chunks per accumulator (1, 2 or 4)
    const uint32_t seg_first = ub / n_kt;
    // W row-block segment of every accumulator slot, in slot (= unit) order
    if (e == 0) {
      uint32_t k = 0;
      for (uint32_t d = 0; d < D; ++d) {
        uint32_t b, en;
        producer_range(ub, ue, D, d, &b, &en);
        if (en <= b) continue;
        for (uint32_t seg = b / n_kt; seg <= (en - 1) / n_kt && k < kLocalMaxSlots; ++seg) slot_seg[k++] = seg;
      }
      n_cta_slots = k;
    }
    named_bar_sync(1, 128);
    const uint32_t ns = n_cta_slots;
    uint32_t nflush = 0;
    uint32_t pend[2], npend = 0;  // segments shared with other CTAs (first, last)
    for (uint32_t sa = 0; sa < ns;) {
      const uint32_t seg = slot_seg[sa];
      uint32_t sb = sa + 1;
      while (sb < ns && slot_seg[sb] == seg) ++sb;
      // sum the segment's accumulators in slot order, two 16-column TMEM
      // loads in flight per wait.  The accumulators of a segment complete
      // close together (at the end of the producers' work): the first one is
      // polled for alone (a cheap poll while the producers still decode),
      // then all of them are tested together with overlapping tests.
      wait_live(&acc_full[sa], 0, abort, P.status, 6, 64);
      wait_all_live(&acc_full[sa], sb - sa, 0, abort, P.status, 6, 32);
      tc_fence_after();
      // store: Y for a segment this CTA holds whole, else split-K partials
      const uint32_t p = seg / P.n_rb, rb = seg % P.n_rb;
      const uint32_t s_lo = seg * n_kt, s_hi = s_lo + n_kt;
      const bool complete = ub <= s_lo && ue >= s_hi;
      const uint32_t pslot = (seg == seg_first) ? 0u : 1u;
      float* part = P.partials + (static_cast<uint64_t>(cta) * 2 + pslot) * H * P.T_pass * 128;
      // the accumulators' 16-column chunks, two at a time (one pass unless a
      // 256-row tile meets more than 16 tokens)
      for (uint32_t c0 = 0; c0 < nck; c0 += 2) {
        const uint32_t ncc = min(2u, nck - c0);
        float acc[2][16];
        for (uint32_t k = sa; k < sb;) {
          // one chunk per accumulator: two accumulators per wait
          const uint32_t nb = (ncc == 1 && k + 1 < sb) ? 2u : 1u;
          uint32_t v[2][16];
          const uint32_t taddr = tmem_base + ((32 * warp) << 16) + k * H * T + 16 * c0;
          tmem_ld16(taddr, v[0]);
          if (nb == 2) tmem_ld16(taddr + H * T, v[1]);
          else if (ncc == 2) tmem_ld16(taddr + 16, v[1]);
          tmem_ld_wait();
          if (ncc == 1) {
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              float x = __uint_as_float(v[0][q]);
              if (k > sa) x = acc[0][q] + x;
              if (nb == 2) x = x + __uint_as_float(v[1][q]);
              acc[0][q] = x;
            }
          } else {
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              acc[0][q] = (k > sa) ? acc[0][q] + __uint_as_float(v[0][q]) : __uint_as_float(v[0][q]);
              acc[1][q] = (k > sa) ? acc[1][q] + __uint_as_float(v[1][q]) : __uint_as_float(v[1][q]);
            }
          }
          k += nb;
        }
#pragma unroll
        for (uint32_t ck = 0; ck < 2; ++ck) {
          if (ck >= ncc) break;
          const uint32_t c = c0 + ck, per_h = T / 16;
          const uint32_t h = c / per_h, tok0 = (c % per_h) * 16;
          const uint32_t n = rb * P.L.tile_n + h * 128 + e;
          const float scale = complete ? row_scale(P, n) : 1.0f;
          epi_emit16(P, acc[ck], complete, scale, part, p, h, tok0, n, e);
        }
      }
      if (e == 0) trace_mark(P, 60 + min(nflush, 1u));
      if (!complete) pend[npend++] = seg;
      ++nflush;
      sa = sb;
    }
    // split-K arrival once every partial of this CTA is written; the
    // reductions this CTA owns run after the CTA barrier, on every thread
    if (npend) splitk_arrive(P, G, pend, npend, e, &reduce_flag);
    if (e == 0) {
      trace_mark(P, 62);
      red_n = npend;
      red_seg[0] = pend[0];
      red_seg[1] = pend[1];
    }
  }

  // ---- teardown: every MMA retired before TMEM is released
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) trace_mark(P, 41);
  if (warp == 0) {
    wait_drain(mma_done, 0, P.status);
    tc_fence_after();
    tmem_dealloc(tmem_base, P.tmem_cols);
  }
  // the split-K reductions this CTA arrived last for, on every thread
  if (reduce_flag) {
    fence_acq_rel_gpu();  // acquire: the counter showed every contributor arrived
    const uint32_t both[2] = {red_seg[0], red_seg[1]};
    if (!(reduce_flag == 3u && splitk_reduce2(P, G, both, threadIdx.x, blockDim.x)))
      for (uint32_t k = 0; k < red_n; ++k)
        if ((reduce_flag >> k) & 1u) splitk_reduce(P, G, red_seg[k], threadIdx.x, blockDim.x);
  }
}

template <bool kDecode, uint32_t kFmt, bool kWide>
__global__ void __launch_bounds__(kLocalThreads, 1)
    fused_gemm_local_kernel(const __grid_constant__ GemmDev P) {
  local_cta<kDecode, kFmt, kWide, false>(P);
}

// Several layers of one shape in one launch (decode only): the CTAs of job j
// run the kernel above on job j's layer.
template <uint32_t kFmt, bool kWide>
__global__ void __launch_bounds__(kLocalThreads, 1)
    fused_gemm_local_batch_kernel(const __grid_constant__ BatchDev B) {
  uint32_t j = 0;
  while (j + 1 < B.n_jobs && blockIdx.x >= B.job[j + 1].cta0) ++j;
  local_cta<true, kFmt, kWide, true>(B.job[j]);
}

template <bool kDecode, uint32_t kFmt, bool kWide = false>
static cudaError_t launch_local_variant(const GemmPlan& plan, const GemmDev& P, cudaStream_t stream) {
  auto kern = fused_gemm_local_kernel<kDecode, kFmt, kWide>;
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
  return launch_pdl(kern, dim3(plan.grid), dim3((kLocalFixedWarps + plan.D) * 32), plan.smem_bytes,
                    stream, P);
}

cudaError_t launch_gemm_local(const GemmPlan& plan, const GemmDev& P, bool decode,
                              cudaStream_t stream) {
  switch (plan.fmt | (decode ? 0u : 16u)) {  // 16 | fmt: the copy variants
    case kFmtBf16Split:
      return P.L.wide ? launch_local_variant<true, kFmtBf16Split, true>(plan, P, stream)
                      : launch_local_variant<true, kFmtBf16Split>(plan, P, stream);
    case kFmtInt4Bf16:
      return P.L.wide ? launch_local_variant<true, kFmtInt4Bf16, true>(plan, P, stream)
                      : launch_local_variant<true, kFmtInt4Bf16>(plan, P, stream);
    case kFmtInt4F16Group:
      return P.L.wide ? launch_local_variant<true, kFmtInt4F16Group, true>(plan, P, stream)
                      : launch_local_variant<true, kFmtInt4F16Group>(plan, P, stream);
    case kFmtInt4PairBf16:
      return P.L.wide ? launch_local_variant<true, kFmtInt4PairBf16, true>(plan, P, stream)
                      : launch_local_variant<true, kFmtInt4PairBf16>(plan, P, stream);
    case kFmtInt4PairF16Group:
      return P.L.wide ? launch_local_variant<true, kFmtInt4PairF16Group, true>(plan, P, stream)
                      : launch_local_variant<true, kFmtInt4PairF16Group>(plan, P, stream);
    case kFmtFp8F16:
      return P.L.wide ? launch_local_variant<true, kFmtFp8F16, true>(plan, P, stream)
                      : launch_local_variant<true, kFmtFp8F16>(plan, P, stream);
    case kFmtInt8F16:
      return P.L.wide ? launch_local_variant<true, kFmtInt8F16, true>(plan, P, stream)
                      : launch_local_variant<true, kFmtInt8F16>(plan, P, stream);
    case kFmtFp4Bf16:
      return P.L.wide ? launch_local_variant<true, kFmtFp4Bf16, true>(plan, P, stream)
                      : launch_local_variant<true, kFmtFp4Bf16>(plan, P, stream);
    case kFmtFp4PairBf16:
      return P.L.wide ? launch_local_variant<true, kFmtFp4PairBf16, true>(plan, P, stream)
                      : launch_local_variant<true, kFmtFp4PairBf16>(plan, P, stream);
    case 16 | kFmtBf16Split: return launch_local_variant<false, kFmtBf16Split>(plan, P, stream);
    case 16 | kFmtInt4Bf16: return launch_local_variant<false, kFmtInt4Bf16>(plan, P, stream);
    case 16 | kFmtInt4F16Group: return launch_local_variant<false, kFmtInt4F16Group>(plan, P, stream);
    case 16 | kFmtFp8F16: return launch_local_variant<false, kFmtFp8F16>(plan, P, stream);
    case 16 | kFmtInt8F16: return launch_local_variant<false, kFmtInt8F16>(plan, P, stream);
    case 16 | kFmtFp4Bf16: return launch_local_variant<false, kFmtFp4Bf16>(plan, P, stream);
  }
  return cudaErrorInvalidValue;
}

template <uint32_t kFmt, bool kWide>
static cudaError_t launch_local_batch_variant(const GemmPlan& plan, const BatchDev& B, uint32_t grid,
                                              cudaStream_t stream) {
  auto kern = fused_gemm_local_batch_kernel<kFmt, kWide>;
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
  return launch_pdl(kern, dim3(grid), dim3((kLocalFixedWarps + plan.D) * 32), plan.smem_bytes,
                    stream, B);
}

cudaError_t launch_gemm_local_batch(const GemmPlan& plan, const BatchDev& B, uint32_t grid,
                                    cudaStream_t stream) {
  const bool wide = B.job[0].L.wide != 0;
  switch (plan.fmt) {
    case kFmtBf16Split:
      return wide ? launch_local_batch_variant<kFmtBf16Split, true>(plan, B, grid, stream)
                  : launch_local_batch_variant<kFmtBf16Split, false>(plan, B, grid, stream);
    case kFmtInt4Bf16:
      return wide ? launch_local_batch_variant<kFmtInt4Bf16, true>(plan, B, grid, stream)
                  : launch_local_batch_variant<kFmtInt4Bf16, false>(plan, B, grid, stream);
    case kFmtInt4F16Group:
      return wide ? launch_local_batch_variant<kFmtInt4F16Group, true>(plan, B, grid, stream)
                  : launch_local_batch_variant<kFmtInt4F16Group, false>(plan, B, grid, stream);
    case kFmtInt4PairBf16:
      return wide ? launch_local_batch_variant<kFmtInt4PairBf16, true>(plan, B, grid, stream)
                  : launch_local_batch_variant<kFmtInt4PairBf16, false>(plan, B, grid, stream);
    case kFmtInt4PairF16Group:
      return wide ? launch_local_batch_variant<kFmtInt4PairF16Group, true>(plan, B, grid, stream)
                  : launch_local_batch_variant<kFmtInt4PairF16Group, false>(plan, B, grid, stream);
    case kFmtFp8F16:
      return wide ? launch_local_batch_variant<kFmtFp8F16, true>(plan, B, grid, stream)
                  : launch_local_batch_variant<kFmtFp8F16, false>(plan, B, grid, stream);
    case kFmtInt8F16:
      return wide ? launch_local_batch_variant<kFmtInt8F16, true>(plan, B, grid, stream)
                  : launch_local_batch_variant<kFmtInt8F16, false>(plan, B, grid, stream);
    case kFmtFp4Bf16:
      return wide ? launch_local_batch_variant<kFmtFp4Bf16, true>(plan, B, grid, stream)
                  : launch_local_batch_variant<kFmtFp4Bf16, false>(plan, B, grid, stream);
    case kFmtFp4PairBf16:
      return wide ? launch_local_batch_variant<kFmtFp4PairBf16, true>(plan, B, grid, stream)
                  : launch_local_batch_variant<kFmtFp4PairBf16, false>(plan, B, grid, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t set_live_wait_budget_local(long long cycles) {
  return cudaMemcpyToSymbol(g_live_wait_budget, &cycles, sizeof(cycles));
}

}  // namespace ansdev
