// gemm_common.cuh -- pieces shared by the two schedules of the fused decode +
// GEMM kernel (gemm.cu: one MMA-issuing thread per CTA feeding a shared
// accumulator; gemm_local.cu: every producer warp issues its own MMAs into
// private accumulators).  Unit ranges, the epilogue's output stores and the
// deterministic split-K reduction live here.
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"
#include "rans_core.cuh"

namespace ansdev {

constexpr uint32_t kSlabBytes = 128 * 32;       // 128 rows x 16 bf16 (one MMA A operand)
constexpr uint32_t kSmemLimit = 232448 - 4096;  // sm_100 per-block maximum, less static smem

// Units (token pass, tile; fewer than 2^31) are split into one contiguous
// range per CTA, the first U % G CTAs taking one unit more than the others.
// 32-bit arithmetic only: 64-bit divisions are long software routines here.
__host__ __device__ __forceinline__ uint32_t cta_begin(uint32_t U, uint32_t G, uint32_t c) {
  const uint32_t q = U / G, r = U % G;
  return q * c + (c < r ? c : r);
}

// CTA whose range contains unit u (G <= U, so q >= 1 past the longer ranges).
__host__ __device__ __forceinline__ uint32_t cta_of(uint32_t U, uint32_t G, uint32_t u) {
  const uint32_t q = U / G, r = U % G;
  const uint32_t big = r * (q + 1);
  return u < big ? u / (q + 1) : r + (u - big) / q;
}

__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void trace_mark(const GemmDev& P, uint32_t slot) {
  if (P.trace) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    P.trace[blockIdx.x * 64 + slot] = t;
  }
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Per-row output scale (row n of W), 1 when the format has none or applies
// it before the MMA.
__device__ __forceinline__ float row_scale(const GemmDev& P, uint32_t n) {
  if (P.scale_kind == 1) return bf16_to_f32(__ldg(static_cast<const uint16_t*>(P.scales) + n));
  if (P.scale_kind == 2) return __ldg(static_cast<const float*>(P.scales) + n);
  return 1.0f;
}

// Epilogue output of NV accumulator columns (tokens tok0 .. tok0 + NV - 1 of
// token pass p) for W row n = rb * tile_n + h * 128 + e.  A segment that this
// CTA holds completely goes to Y (scaled); otherwise the values go to this
// CTA's partial-sum slot for the split-K reduction.
template <uint32_t NV>
__device__ __forceinline__ void epi_emit(const GemmDev& P, const float (&v)[NV], bool complete,
                                         float scale, float* part, uint32_t p, uint32_t h,
                                         uint32_t tok0, uint32_t n, uint32_t e) {
  // tokens past M are padding: neither stored nor reduced
  const uint32_t m0 = p * P.T_pass + tok0;
  const uint32_t nv = P.M > m0 ? min(NV, P.M - m0) : 0u;
  if (complete) {
    float* y = P.Y + static_cast<uint64_t>(m0) * P.L.N + n;
#pragma unroll
    for (uint32_t q = 0; q < NV; ++q) {
      if (q < nv) *y = v[q] * scale;
      y += P.L.N;
    }
  } else {
    float* d = part + (static_cast<uint64_t>(h) * P.T_pass + tok0) * 128 + e;
#pragma unroll
    for (uint32_t q = 0; q < NV; ++q)
      if (q < nv) d[q * 128] = v[q];
  }
}
__device__ __forceinline__ void epi_emit16(const GemmDev& P, const float (&v)[16], bool complete,
                                           float scale, float* part, uint32_t p, uint32_t h,
                                           uint32_t tok0, uint32_t n, uint32_t e) {
  epi_emit<16>(P, v, complete, scale, part, p, h, tok0, n, e);
}

// Split-K over CTAs.  A W row block's segment seg (token pass p, row block
// rb) that spans several CTAs is summed in a fixed order: every contributor
// writes its partial sums, then counts itself in counters[seg]; the last CTA
// to arrive adds the contributors' partials in ascending CTA order (so the
// result does not depend on timing) and writes Y.  A CTA holds at most two
// such segments: its first (partial slot 0) and its last (slot 1); only the
// first contributor of a segment can hold it in its slot 1, when its range
// started before the segment.

// Arrival: run by the 128 epilogue threads once all of this CTA's partials
// are written, for at most two segments.  Returns (to every thread) a bit per
// segment for which this CTA arrived last and must reduce; the reducing CTA
// runs fence_acq_rel_gpu() before it reads the other CTAs' partials.
__device__ __forceinline__ uint32_t splitk_arrive(const GemmDev& P, uint32_t G, const uint32_t* segs,
                                                  uint32_t n, uint32_t e,
                                                  volatile uint32_t* reduce_flag) {
  const uint32_t n_kt = P.L.n_kt, U = static_cast<uint32_t>(P.n_units);
  named_bar_sync(1, 128);
  if (e == 0) {
    // release: one gpu-scope acq_rel fence after the barrier covers the
    // partials every epilogue thread wrote before it (fences are cumulative);
    // both counters are incremented before either result is looked at
    fence_acq_rel_gpu();
    uint32_t bits = 0;
    uint32_t old[2] = {0, 0}, need[2] = {0, 0};
#pragma unroll
    for (uint32_t k = 0; k < 2; ++k) {
      if (k < n) {
        const uint32_t s_lo = segs[k] * n_kt;
        need[k] = cta_of(U, G, s_lo + n_kt - 1) - cta_of(U, G, s_lo);
        old[k] = atomicAdd(&P.counters[segs[k]], 1u);
      }
    }
#pragma unroll
    for (uint32_t k = 0; k < 2; ++k)
      if (k < n && old[k] == need[k]) bits |= 1u << k;
    *reduce_flag = bits;
  }
  named_bar_sync(1, 128);
  return *reduce_flag;
}

// Reduction of segment seg by the CTA that arrived last, run by threads
// tid = 0 .. nthr - 1 of that CTA (the whole CTA, once its other work is
// done).
__device__ __forceinline__ void splitk_reduce(const GemmDev& P, uint32_t G, uint32_t seg, uint32_t tid,
                                              uint32_t nthr) {
  const uint32_t n_kt = P.L.n_kt, U = static_cast<uint32_t>(P.n_units);
  const uint32_t p = seg / P.n_rb, rb = seg % P.n_rb;
  const uint32_t s_lo = seg * n_kt, s_hi = s_lo + n_kt;
  const uint32_t c_first = cta_of(U, G, s_lo);
  const uint32_t c_last = cta_of(U, G, s_hi - 1);
  const uint32_t sl_first = (cta_begin(U, G, c_first) < s_lo) ? 1u : 0u;
  const uint64_t cta_stride = 2ull * P.H * P.T_pass * 128;
  const uint32_t t_valid = min(P.T_pass, P.M - p * P.T_pass);
  const uint32_t n_items = P.H * t_valid * 32;  // float4 items: (h, token, 4 rows)
  const float* first = P.partials + c_first * cta_stride + sl_first * (cta_stride / 2);
  // an output item is 4 rows of one token (a float4).  Few items (small M):
  // one per thread, the loads of up to 8 contributors in flight together;
  // many items: 4 per thread and pass, 2 contributors at a time.  Either way
  // the contributors are added in ascending CTA order.
  auto item_off = [&](uint32_t it, uint32_t* h, uint32_t* tok, uint32_t* q) {
    *q = it & 31;
    const uint32_t ht = it >> 5;
    *h = ht / t_valid;
    *tok = ht - *h * t_valid;
    return (static_cast<uint64_t>(*h) * P.T_pass + *tok) * 128 + 4 * *q;
  };
  auto store = [&](float4 acc, uint32_t h, uint32_t tok, uint32_t q) {
    const uint32_t n = rb * P.L.tile_n + h * 128 + 4 * q;
    if (P.scale_kind == 1) {
      const uint2 sb = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(P.scales) + n));
      acc.x *= __uint_as_float(sb.x << 16);
      acc.y *= __uint_as_float(sb.x & 0xFFFF0000u);
      acc.z *= __uint_as_float(sb.y << 16);
      acc.w *= __uint_as_float(sb.y & 0xFFFF0000u);
    } else if (P.scale_kind == 2) {
      const float4 sf = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(P.scales) + n));
      acc.x *= sf.x; acc.y *= sf.y; acc.z *= sf.z; acc.w *= sf.w;
    }
    const uint32_t m = p * P.T_pass + tok;
    *reinterpret_cast<float4*>(P.Y + static_cast<uint64_t>(m) * P.L.N + n) = acc;
  };
  if (n_items <= nthr) {
    for (uint32_t it = tid; it < n_items; it += nthr) {
      uint32_t h, tok, q;
      const uint64_t off = item_off(it, &h, &tok, &q);
      float4 acc = __ldcg(reinterpret_cast<const float4*>(first + off));
      for (uint32_t c0 = c_first + 1; c0 <= c_last; c0 += 8) {
        float4 v[8];
#pragma unroll
        for (uint32_t k = 0; k < 8; ++k) {
          const uint32_t cc = min(c0 + k, c_last);
          v[k] = __ldcg(reinterpret_cast<const float4*>(P.partials + cc * cta_stride + off));
        }
#pragma unroll
        for (uint32_t k = 0; k < 8; ++k) {
          if (c0 + k > c_last) break;
          acc.x += v[k].x; acc.y += v[k].y; acc.z += v[k].z; acc.w += v[k].w;
        }
      }
      store(acc, h, tok, q);
    }
  } else {
    for (uint32_t it0 = tid; it0 < n_items; it0 += 4 * nthr) {
      uint64_t off[4];
      uint32_t hh[4], tt[4], qq[4];
      float4 acc[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        off[u] = item_off(min(it0 + nthr * u, n_items - 1), &hh[u], &tt[u], &qq[u]);
        acc[u] = __ldcg(reinterpret_cast<const float4*>(first + off[u]));
      }
      for (uint32_t c2 = c_first + 1; c2 <= c_last; c2 += 2) {
        const uint32_t cb = min(c2 + 1, c_last);
        float4 v0[4], v1[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          v0[u] = __ldcg(reinterpret_cast<const float4*>(P.partials + c2 * cta_stride + off[u]));
          v1[u] = __ldcg(reinterpret_cast<const float4*>(P.partials + cb * cta_stride + off[u]));
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          acc[u].x += v0[u].x; acc[u].y += v0[u].y; acc[u].z += v0[u].z; acc[u].w += v0[u].w;
        }
        if (c2 + 1 <= c_last) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            acc[u].x += v1[u].x; acc[u].y += v1[u].y; acc[u].z += v1[u].z; acc[u].w += v1[u].w;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (it0 + nthr * u < n_items) store(acc[u], hh[u], tt[u], qq[u]);
    }
  }
  if (tid == 0) P.counters[seg] = 0;
  if (tid == 0) trace_mark(P, 38);
}

// Two segments reduced by the same CTA at once (its first and its last), when
// each has at most nthr items: thread tid takes item tid of both, with the
// loads of up to 8 contributors of each in flight together, so both
// reductions cost one round trip instead of two.  The additions per item are
// the same, in the same order, as in splitk_reduce.
__device__ __forceinline__ bool splitk_reduce2(const GemmDev& P, uint32_t G, const uint32_t (&seg)[2],
                                               uint32_t tid, uint32_t nthr) {
  const uint32_t n_kt = P.L.n_kt, U = static_cast<uint32_t>(P.n_units);
  const uint64_t cta_stride = 2ull * P.H * P.T_pass * 128;
  uint32_t p[2], rb[2], c_first[2], c_last[2], t_valid[2], n_items[2];
  const float* first[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    p[k] = seg[k] / P.n_rb;
    rb[k] = seg[k] % P.n_rb;
    const uint32_t s_lo = seg[k] * n_kt;
    c_first[k] = cta_of(U, G, s_lo);
    c_last[k] = cta_of(U, G, s_lo + n_kt - 1);
    const uint32_t sl_first = (cta_begin(U, G, c_first[k]) < s_lo) ? 1u : 0u;
    t_valid[k] = min(P.T_pass, P.M - p[k] * P.T_pass);
    n_items[k] = P.H * t_valid[k] * 32;
    first[k] = P.partials + c_first[k] * cta_stride + sl_first * (cta_stride / 2);
  }
  if (n_items[0] > nthr || n_items[1] > nthr) return false;
  float4 acc[2];
  uint64_t off[2];
  uint32_t hh[2], tt[2], qq[2];
  bool has[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    has[k] = tid < n_items[k];
    const uint32_t it = has[k] ? tid : 0u;
    qq[k] = it & 31;
    const uint32_t ht = it >> 5;
    hh[k] = ht / t_valid[k];
    tt[k] = ht - hh[k] * t_valid[k];
    off[k] = (static_cast<uint64_t>(hh[k]) * P.T_pass + tt[k]) * 128 + 4 * qq[k];
    acc[k] = __ldcg(reinterpret_cast<const float4*>(first[k] + off[k]));
  }
  const uint32_t rounds = max((c_last[0] - c_first[0] + 7) / 8, (c_last[1] - c_first[1] + 7) / 8);
  for (uint32_t r = 0; r < rounds; ++r) {
    float4 v[2][8];
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (uint32_t j = 0; j < 8; ++j) {
        const uint32_t cc = min(c_first[k] + 1 + 8 * r + j, c_last[k]);
        v[k][j] = __ldcg(reinterpret_cast<const float4*>(P.partials + cc * cta_stride + off[k]));
      }
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (uint32_t j = 0; j < 8; ++j) {
        if (c_first[k] + 1 + 8 * r + j > c_last[k]) break;
        acc[k].x += v[k][j].x; acc[k].y += v[k][j].y; acc[k].z += v[k][j].z; acc[k].w += v[k][j].w;
      }
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    if (!has[k]) continue;
    const uint32_t n = rb[k] * P.L.tile_n + hh[k] * 128 + 4 * qq[k];
    float4 a = acc[k];
    if (P.scale_kind == 1) {
      const uint2 sb = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(P.scales) + n));
      a.x *= __uint_as_float(sb.x << 16);
      a.y *= __uint_as_float(sb.x & 0xFFFF0000u);
      a.z *= __uint_as_float(sb.y << 16);
      a.w *= __uint_as_float(sb.y & 0xFFFF0000u);
    } else if (P.scale_kind == 2) {
      const float4 sf = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(P.scales) + n));
      a.x *= sf.x; a.y *= sf.y; a.z *= sf.z; a.w *= sf.w;
    }
    const uint32_t m = p[k] * P.T_pass + tt[k];
    *reinterpret_cast<float4*>(P.Y + static_cast<uint64_t>(m) * P.L.N + n) = a;
  }
  if (tid == 0) {
    P.counters[seg[0]] = 0;
    P.counters[seg[1]] = 0;
    trace_mark(P, 38);
  }
  return true;
}

}  // namespace ansdev
