// kernels.h -- plain structs and launch entry points shared between the C-ABI
// layer (host C++) and the CUDA kernels.  No device code here.
#pragma once
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace ansdev {

constexpr uint32_t kNoSymbolHost = 0xFFFFFFFFu;

// A compressed layer as the kernels see it (passed by value as a kernel
// parameter; the codebook travels with it).
struct LayerDev {
  const uint8_t* stream;
  const uint64_t* offsets;
  const uint8_t* raw;
  uint64_t stream_bytes;
  uint32_t N, K, tile_n, tile_k;
  uint32_t n_kt, n_tiles, dtype, alphabet;
  uint32_t single_symbol;  // the symbol when the codebook has exactly one, else kNoSymbolHost
  uint32_t wide;           // 1: wide-state variant (64-bit states, 32-bit words, pair steps)
  uint16_t freq[256];
  uint16_t cdf[257];
};

// Output formats of the producer warps (what lands in the MMA operand slab).
enum : uint32_t {
  kFmtBf16Split = 0,   // bf16 weights: exponent symbol + raw sign/mantissa byte -> bf16
  kFmtInt4Bf16 = 1,    // int4 code -> exact bf16 (row scale applied in the epilogue)
  kFmtInt4F16Group = 2,// int4 code * group scale -> exact f16
  kFmtFp8F16 = 3,      // e4m3 code -> exact f16 (row scale applied in the epilogue)
  kFmtInt4PairBf16 = 4,     // int4 pair symbol -> two exact bf16 (row scale in the epilogue)
  kFmtInt4PairF16Group = 5, // int4 pair symbol * group scale -> two exact f16
  kFmtInt8F16 = 6,          // int8 code -> exact f16 (row scale applied in the epilogue)
  kFmtFp4Bf16 = 7,          // e2m1 code -> exact bf16 (row scale applied in the epilogue)
  kFmtFp4PairBf16 = 8       // e2m1 pair symbol (a packed byte) -> two exact bf16
};
// int4 pair symbols: 8 symbols of a lane fill 16 columns of one slab row
__host__ __device__ constexpr bool fmt_pair(uint32_t f) {
  return f == kFmtInt4PairBf16 || f == kFmtInt4PairF16Group || f == kFmtFp4PairBf16;
}
// a per-(row, K group) scale is applied while the slab is written
__host__ __device__ constexpr bool fmt_group(uint32_t f) { return f == kFmtInt4F16Group || f == kFmtInt4PairF16Group; }

// Static schedule of one fused GEMM launch, computed on the host.
struct GemmPlan {
  uint32_t fmt;        // kFmt*
  uint32_t ab_f16;     // MMA operand type: 1 = f16, 0 = bf16
  uint32_t M, T, NT, T_pass, n_pass;
  uint32_t H, C;       // 128-row halves per tile, 16-column slabs per tile
  uint32_t D;          // producer warps per CTA
  uint32_t n_bufs;     // TMEM accumulator sets (1 or 2)
  uint32_t x_stages;
  uint32_t tmem_cols;
  uint32_t local;      // 1: every producer warp issues its own MMAs (gemm_local.cu)
  uint32_t n_slots;    // local schedule: TMEM accumulators per CTA (max over CTAs)
  uint32_t grid;       // CTAs
  uint64_t n_units;    // n_pass * n_tiles
  uint32_t n_segments; // n_pass * (N / tile_n)
  uint32_t smem_bytes;
  uint32_t off_lut, off_w, off_chunk, off_x, off_bars;
  size_t ws_partials_bytes, ws_counters_bytes, ws_x16_bytes, ws_bytes;
};

struct GemmDev {
  LayerDev L;
  const void* w_plain;   // copy mode: uncompressed weights
  const void* scales;
  float* Y;
  float* partials;
  uint32_t* counters;
  uint32_t* status;
  uint32_t scale_kind, group_k, n_groups_k;
  uint32_t M, T, NT, T_pass, n_pass;
  uint32_t H, C, D, n_bufs, x_stages, tmem_cols;
  uint32_t n_rb;
  uint64_t n_units;
  uint32_t idesc;
  uint32_t off_lut, off_w, off_chunk, off_x, off_bars;
  unsigned long long* trace;  // optional per-CTA event timestamps (internal profiling)
  const uint8_t* xs;          // X staged as pre-swizzled 16-column slabs (workspace)
  const uint16_t* X;          // local schedule: X as given (bf16, M x K row-major)
  uint32_t x_f16;             // local schedule: convert X to f16 for the MMA
  uint32_t n_slots;           // local schedule: accumulator slots (barriers) per CTA
  uint32_t n_cta;             // CTAs that share this layer's units (the grid, or a batch job's share)
  uint32_t cta0;              // first CTA of this layer in the grid (0 unless batched)
};

// Several layers of one shape in one launch of the local schedule: job j
// owns CTAs [job[j].cta0, job[j].cta0 + job[j].n_cta).  Passed by value as
// the kernel parameter (well under the 32 KB parameter limit).
constexpr uint32_t kMaxBatch = 8;
struct BatchDev {
  uint32_t n_jobs;
  GemmDev job[kMaxBatch];
};

// Internal profiling hook: when set, every fused-GEMM CTA writes globaltimer
// stamps of its phases to trace[cta * 64 + slot].
void set_trace_buffer(void* d_buf, size_t bytes);

// Scratch capacity of the allocation-free entry point (16 MiB per device).
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
// Device address of that scratch on the current device (looked up once per
// device; see noalloc.cu).
cudaError_t noalloc_scratch(void** ptr);

// Producer warps per CTA of the local schedule (gemm_local.cu).
constexpr uint32_t kLocalProducersMax = 15;

// Local schedule (gemm_local.cu): launches the kernel for an already filled
// GemmDev.
cudaError_t launch_gemm_local(const GemmPlan& plan, const GemmDev& P, bool decode,
                              cudaStream_t stream);

// Local schedule, batched: one launch of grid CTAs over B's jobs.
cudaError_t launch_gemm_local_batch(const GemmPlan& plan, const BatchDev& B, uint32_t grid,
                                    cudaStream_t stream);

// Fills a plan; returns false if the shape cannot be scheduled.
bool make_gemm_plan(const LayerDev& L, uint32_t M, uint32_t scale_kind, bool decode,
                    int num_sms, GemmPlan* plan);

cudaError_t launch_decode_tiles(const LayerDev& L, void* out, uint32_t* status,
                                cudaStream_t stream, int num_sms);
cudaError_t launch_histogram(const void* w, uint64_t n_bytes, uint32_t dtype, uint64_t* hist,
                             cudaStream_t stream, int num_sms);
// X: bf16 M x K.  ws must hold plan.ws_bytes (partials, counters, f16 X copy).
cudaError_t launch_gemm(const GemmPlan& plan, const LayerDev& L, bool decode, const void* w_plain,
                        const uint16_t* X, const void* scales, uint32_t scale_kind,
                        uint32_t group_k, float* Y, void* ws, uint32_t* status,
                        cudaStream_t stream);
// n layers of one shape (plan made for one of them with a CTA cap of grid / n;
// plan.local), each with its own X, scales and Y, in one launch; ws holds n
// consecutive workspaces of round_up(plan.ws_bytes, 256) bytes.
cudaError_t launch_gemm_batched(const GemmPlan& plan, uint32_t n, const LayerDev* const* Ls,
                                const uint16_t* const* Xs, const void* const* scales,
                                uint32_t scale_kind, uint32_t group_k, float* const* Ys, void* ws,
                                uint32_t* status, cudaStream_t stream);

}  // namespace ansdev
