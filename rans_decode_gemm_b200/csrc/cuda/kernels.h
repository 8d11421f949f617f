// kernels.h -- plain structs and launch entry points shared between the C-ABI
// layer (host C++) and the CUDA kernels.  No device code here.
#pragma once
#include <cuda.h>  // CUtensorMap (the type only: maps are encoded through the runtime's driver entry point)
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace ansdev {

constexpr uint32_t kNoSymbolHost = 0xFFFFFFFFu;
// Default budget of the kernels' bounded waits (about 1.5 s at 1.9 GHz; the
// device side's kWaitBudgetCycles).
constexpr long long kWaitBudgetCyclesHost = 3000000000LL;

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
  uint32_t x_stages;    // X stages of the shared-accumulator schedule (differs between the
                        // decode and copy variants; the accumulation order does not depend on it)
  uint32_t tmem_cols;
  uint32_t local;      // 1: every producer warp issues its own MMAs (gemm_local.cu)
  uint32_t n_slots;    // local schedule: TMEM accumulators per CTA (max over CTAs)
  uint32_t grid;       // CTAs
  uint64_t n_units;    // n_pass * n_tiles
  uint32_t n_segments; // n_pass * (N / tile_n)
  uint32_t smem_bytes;
  uint32_t off_lut, off_w, off_chunk, off_x, off_bars;
  uint32_t sms;        // SMs the plan was made for
  // large M: a fused first pass of M_first tokens (the small-M schedule,
  // storing the decoded weights into W16), then a dense GEMM for the other
  // M - M_first tokens; the other fields describe the first pass's launch
  uint32_t dense, M_first;
  // workspace: [counters][partials][f16 copy of X][W16]; W16 (the weights
  // decoded or formatted to the 16-bit operand format, N x K row-major) only
  // when the call has several token passes (see launch_gemm)
  size_t ws_partials_bytes, ws_counters_bytes, ws_x16_bytes, ws_w16_bytes, ws_bytes;
};

// How the producers of the shared-accumulator schedule fill W slabs from
// uncompressed weights (ans_gemm_uncompressed).
enum : uint32_t {
  kCopyLoads = 0,    // per-lane global loads, formatted in registers (packed nibbles)
  kCopyTmaSlab = 1,  // bf16: one TMA box per slab, straight into the slot (32-byte swizzle)
  kCopyTmaRaw = 2    // 1-byte codes: TMA box of the raw bytes, formatted shared -> shared
};
__host__ __device__ constexpr uint32_t copy_mode_of(uint32_t fmt) {
  return fmt == kFmtBf16Split ? kCopyTmaSlab
         : (fmt == kFmtFp8F16 || fmt == kFmtInt8F16) ? kCopyTmaRaw : kCopyLoads;
}

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
  const uint8_t* xs;          // f16 copy of X (M x K row-major, workspace) for the f16 formats
  const uint16_t* X;          // local schedule: X as given (bf16, M x K row-major)
  uint32_t x_f16;             // local schedule: convert X to f16 for the MMA
  uint32_t n_slots;           // local schedule: accumulator slots (barriers) per CTA
  uint32_t n_cta;             // CTAs that share this layer's units (the grid, or a batch job's share)
  uint32_t cta0;              // first CTA of this layer in the grid (0 unless batched)
  // shared-accumulator schedule: X (or its f16 copy) as a 2-D tensor map,
  // box 16 columns x T rows, 32-byte swizzle; copy variant: W as a 2-D
  // tensor map (bf16: box 16 x 128, 32-byte swizzle; 1-byte codes: box
  // 16 bytes x 128 rows, no swizzle)
  CUtensorMap tmap_x;
  CUtensorMap tmap_w;
  // first token pass of a large-M call (decode variant): every decoded slab
  // is also stored into W16 for the dense kernel that takes the remaining
  // tokens, or null.  W16 holds the weights in the MMA operand format as 4 KB
  // slab images (128 rows x 16 columns, 32-byte swizzle, the shared-memory
  // layout): the image of rows 128 b .. + 127, columns 16 j .. + 15 at byte
  // (b * K / 16 + j) * 4096.
  uint8_t* w16;
};

// Dense GEMM on 16-bit weights that are already in the MMA operand format
// (gemm_dense.cu): Y[m][n] = s_n * sum_k X[m][k] W[n][k] for m < M, fp32 Y
// (M x N row-major).  W is W16 (slab images, see GemmDev::w16); X (M x K,
// 16-bit row-major) is a 2-D tensor map with 64 x 256 boxes, 128-byte
// swizzle; tiles of 128 W rows x 256 tokens, W-row-block major.
struct DenseDev {
  const uint8_t* w16;   // W
  CUtensorMap tmap_b;   // X
  float* Y;
  const void* scales;   // scale_kind 1: bf16 per row, 2: fp32 per row, else none
  uint32_t* status;
  uint32_t scale_kind;
  uint32_t M, N, K;
  uint32_t m_blocks, n_tiles;
  uint32_t k_slabs;     // K / 16: W16 slab images per 128-row block
  uint32_t b_box_rows;  // rows of X a box brings (256, or M when smaller)
  uint32_t idesc;       // MMA 128 x 256 x 16
  uint32_t idesc_tail;  // the last token block: N = its tokens rounded up to 16
};
cudaError_t launch_dense_gemm(const DenseDev& P, uint32_t sms, cudaStream_t stream);

// Several layers in one launch of the local schedule (shapes may differ; one
// operand format): job j owns CTAs [job[j].cta0, job[j].cta0 + job[j].n_cta)
// and runs with its own plan's producers, slots and shared-memory layout.
// Passed by value as the kernel parameter (under the 32 KB parameter limit).
constexpr uint32_t kMaxBatch = 8;
struct BatchDev {
  uint32_t n_jobs;
  GemmDev job[kMaxBatch];
};

// Internal profiling hook: when set, every fused-GEMM CTA writes globaltimer
// stamps of its phases to trace[cta * 64 + slot].
void set_trace_buffer(void* d_buf, size_t bytes);

// Internal test hook: caps on the CTAs and producer warps a fused-GEMM plan
// may use, and a switch that sends every token count to the shared-
// accumulator schedule (0 = no cap, default schedule).  Process-wide; the
// tests use it to force many rounds, long producer runs and both schedules
// on small shapes.
void set_plan_limits(uint32_t max_ctas, uint32_t max_producers, uint32_t force_shared);

// Internal test hooks: the budget (clock64 cycles) of the waits that the
// pipeline's progress ends, per translation unit, on the current device
// (kWaitBudgetCycles by default); and a kernel that makes one such wait on a
// barrier nothing arrives on (status gets the TIMEOUT bit).
cudaError_t set_live_wait_budget_gemm(long long cycles);
cudaError_t set_live_wait_budget_local(long long cycles);
cudaError_t set_live_wait_budget_decode(long long cycles);
cudaError_t set_live_wait_budget_dense(long long cycles);
cudaError_t set_live_wait_budget_decode16(long long cycles);
cudaError_t launch_wait_probe(uint32_t* status, cudaStream_t stream);

// Scratch capacity of the allocation-free entry point (16 MiB per device).
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
// Device address of that scratch on the current device (looked up once per
// device; see noalloc.cu).
cudaError_t noalloc_scratch(void** ptr);

// bf16 as whole 16-bit symbols (decode16.cu): the decoder's table image
// (built on the host) holds at most this many present symbols.
constexpr uint32_t kMaxPresent16 = 16384;
cudaError_t launch_decode_tiles16(const LayerDev& L, const uint8_t* table, uint32_t table_bytes,
                                  uint16_t* out, uint32_t* status, cudaStream_t stream, int num_sms);

// Tokens of the fused first pass of a large-M call (see GemmPlan::dense).
constexpr uint32_t kDenseFirstTokens = 16;

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
// n layers in one launch of the small-M schedule: layer j runs plans[j]
// (every plan local, one operand format) on CTAs [sum of the earlier grids,
// + plans[j].grid), each with its own X, scales, Y and workspace
// (ws + ws_off[j], round_up(plans[j].ws_bytes, 256) bytes at least).
cudaError_t launch_gemm_batched(const GemmPlan* plans, uint32_t n, const LayerDev* const* Ls,
                                const uint16_t* const* Xs, const void* const* scales,
                                uint32_t scale_kind, uint32_t group_k, float* const* Ys, void* ws,
                                const size_t* ws_off, uint32_t* status, cudaStream_t stream);

}  // namespace ansdev
