/*
 * ans.h -- C ABI of the tile-granular rANS weight codec and its fused
 *          decode + GEMM for NVIDIA B200 (sm_100a).
 *
 * The operations follow "Approaching Shannon Bound with Lossless LLM Weight
 * Compression" (blog summary, marsggbo.github.io, 2026-07-22):
 *   s2.1  "熵分析：逐层算直方图"  a layer is a sequence of discrete symbols;
 *         its histogram gives the Shannon entropy (ans_histogram, ans_entropy);
 *   s2.2  "为什么大家不用无损压缩？"  rANS; tiles must decode independently;
 *         decoded weights go to shared memory, never to global memory;
 *   s3.1  "整体执行模型"  W is cut into GEMM-shaped tiles, all tiles of a layer
 *         share one compact codebook, each tile's start is kept in an offset
 *         index, each tile is split into R substreams with one rANS state per
 *         warp lane (ans_encode_tiles, ans_gemm);
 *   s4.1  "压缩率"  frequencies are normalised to a finite precision
 *         (ans_build_codebook);
 *   s4.2  "kernel 层面"  the layer-level decompress-then-GEMM baseline
 *         (ans_decode_tiles followed by a dense GEMM).
 * The bf16 split into an entropy-coded exponent and a raw sign/mantissa byte
 * follows the DFloat11 summary "70%大小，100%准确！...", section
 * "无损LLM压缩框架，实现高效GPU推理" (EncodedExponent / PackedSignMantissa).
 *
 * Stream format (fixed by this library; the pages leave these constants open):
 *   probability precision 12 bits (frequencies sum to 4096), 32 lanes per
 *   tile, 32-bit lane states in [2^16, 2^32), 16-bit renormalisation words.
 *   Tile t = rb * (K / tile_k) + kt covers W rows [rb*tile_n, +tile_n) and
 *   columns [kt*tile_k, +tile_k).  Lane l's j-th symbol is element
 *     row = l + 32*(4h + i), col = 16s + 8c + kk   where  g = j/8, kk = j%8,
 *     i = g%4, c = (g/4)%2, h = (g/8)%(tile_n/128), s = g/(8*(tile_n/128)).
 *   Tile bytes: the final-state block, then the u16 words in decoder order
 *   (step by step; within a step, lanes that need a word take the next one in
 *   increasing lane order), then zero bytes to a 16-byte boundary.
 *   offsets[t] = byte start of tile t (16-byte aligned), offsets[n_tiles] =
 *   total stream bytes.
 *   Final-state block (a variable-length flush): a length table, one
 *   little-endian u32 whose bit l is set when lane l's state takes 4 bytes
 *   (else 3; states are >= 2^16), then the 32 final encoder states in lane
 *   order, each little-endian in its byte count, then zero bytes up to an
 *   even offset.  A single-symbol tile is 112 bytes: a zero table, 32 states
 *   2^16 (00 00 01) and 12 bytes of padding.
 *   Wide-state variant (ans_layout.state_bits = 64): 64-bit lane states in
 *   [2^32, 2^64), 32-bit renormalisation words, and the renormalisation test
 *   made once per pair of symbols (steps 2i, 2i+1) instead of after every
 *   symbol: the decoder decodes both symbols of a pair, then a lane with
 *   x < 2^32 takes one word (x = x << 32 | w).  The encoder pushes a word
 *   before coding a pair (a, b) if x >= 2^40 * f_a * f_b.  Tile bytes: the
 *   final-state block with states of 5 to 8 bytes (states are >= 2^32) and a
 *   length table of two little-endian u32 bit planes (lane l takes 5 + bit l
 *   of the first + 2 * bit l of the second bytes), zero bytes up to a multiple
 *   of 4, then the u32 words in decoder order, then zero padding.  About 16
 *   more bits per lane and tile than the default format (the initial state
 *   2^32 instead of 2^16), in exchange for half as many renormalisation steps.
 *   bf16 raw side stream: tile_n*tile_k bytes per tile at t*tile_n*tile_k,
 *   the raw byte (sign << 7 | 7-bit mantissa) of lane l's j-th symbol at
 *   (j/8)*256 + l*8 + j%8.
 *
 * Weight storage ("original format"), row-major N x K:
 *   ANS_INT4       packed nibbles, element k even in the low nibble, two's
 *                  complement code q in [-8, 7]; coded symbol q + 8 (A = 16).
 *   ANS_BF16_SPLIT uint16 bf16 bits; coded symbol = exponent byte (A = 256).
 *   ANS_FP8_E4M3   e4m3fn code bytes; coded symbol = the code (A = 256).
 *   ANS_FP4_E2M1   e2m1 codes packed like ANS_INT4 (element k even in the low
 *                  nibble); coded symbol = the code (A = 16).
 *   ANS_FP4_PAIRS  the same storage as ANS_FP4_E2M1, coded one symbol per packed
 *                  byte (the byte itself, A = 256), in the lane map of
 *                  ANS_INT4_PAIRS.
 *   ANS_INT8       int8 code bytes q in [-128, 127]; coded symbol q + 128,
 *                  i.e. the byte XOR 0x80 (A = 256).
 *   ANS_BF16_WHOLE uint16 bf16 bits; coded symbol = the whole 16-bit pattern
 *                  (A = 65536), probability precision up to 16 bits, the lane
 *                  map of the one-symbol-per-element formats.  Only the
 *                  16-bit-symbol entry points (ans_*16) take it.
 *   ANS_INT4_PAIRS the same storage as ANS_INT4, coded one symbol per packed
 *                  byte (two consecutive K elements): symbol = byte ^ 0x88,
 *                  i.e. (q_k + 8) | (q_{k+1} + 8) << 4 (A = 256), half as
 *                  many symbols per tile.  Lane l's j-th symbol covers row
 *                  l + 32 (4 h + i), columns 16 s + 2 kk and 16 s + 2 kk + 1,
 *                  with g = j / 8, kk = j % 8, i = g % 4,
 *                  h = (g / 4) % (tile_n / 128), s = g / (4 tile_n / 128).
 *
 * Conventions.  Every buffer belongs to the caller; the library allocates no
 * device memory.  "d_" pointers are device pointers, "h_" host pointers.  GPU
 * calls are asynchronous and stream-ordered on `stream` (a cudaStream_t; NULL
 * is the legacy default stream).  Argument errors are returned synchronously;
 * launch failures return ANS_ERR_CUDA (text via ans_last_error()).  Faults
 * found while the kernel runs (a corrupt stream, a wait that ran out) are
 * OR-ed into the caller's device word *d_status as ANS_STATUS_* bits; read it
 * after synchronising.  No call traps or asserts on the device.
 */
#ifndef ANS_H_
#define ANS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* ans_stream_t; /* same type as cudaStream_t */

typedef enum {
  ANS_OK = 0,
  ANS_ERR_ARG = 1,              /* null pointer, bad enum, misaligned pointer */
  ANS_ERR_SHAPE = 2,            /* tile does not divide N/K, unsupported tile */
  ANS_ERR_ALPHABET = 3,         /* bad codebook / symbol absent from it */
  ANS_ERR_BUFFER_TOO_SMALL = 4, /* output or workspace capacity too small */
  ANS_ERR_CUDA = 5,             /* a CUDA runtime call failed */
  ANS_ERR_CORRUPT = 6,          /* host-side check found a corrupt stream */
  ANS_ERR_TIMEOUT = 7,          /* reserved for host-side waits */
  ANS_ERR_UNSUPPORTED = 8       /* no sm_100 device, or a size the kernels refuse */
} ans_status;

/* Bits OR-ed into *d_status by the device. */
#define ANS_STATUS_CORRUPT 0x1u     /* a tile did not end at x = L (2^16, or 2^32 for the
                                       wide-state variant) in every lane, or
                                       its words did not end at its last byte */
#define ANS_STATUS_TIMEOUT 0x2u     /* a bounded wait inside a kernel ran out */
#define ANS_STATUS_BAD_OFFSETS 0x4u /* an offset was unaligned, decreasing or past the end */
#define ANS_STATUS_SMEM_ALIGN 0x8u  /* a fused-GEMM CTA's dynamic shared memory did not start
                                       on the 1024-byte boundary its tensor-core operand
                                       layout assumes (its Y is not valid) */

typedef enum {
  ANS_INT4 = 0,
  ANS_BF16_SPLIT = 1,
  ANS_FP8_E4M3 = 2,
  ANS_INT4_PAIRS = 3,
  ANS_INT8 = 4,
  ANS_FP4_E2M1 = 5,
  ANS_FP4_PAIRS = 6,
  ANS_BF16_WHOLE = 7  /* the 16-bit-symbol entry points only (ans_*16 below) */
} ans_dtype;

typedef enum {
  ANS_SCALE_NONE = 0,
  ANS_SCALE_ROW_BF16 = 1,  /* scales: bf16[N]; w = q * s[n]            (int4) */
  ANS_SCALE_ROW_F32 = 2,   /* scales: f32[N];  w = value * s[n]       (fp8, int4) */
  ANS_SCALE_GROUP_BF16 = 3 /* scales: bf16[N][K/group_k]; w = q * s[n][k/group_k] (int4) */
} ans_scale_kind;

/* Shared per-layer codebook ("Approaching Shannon Bound", s3.1 and s4.1).
 * freq[s] > 0 exactly for the symbols present in the layer; the freq sum to
 * 2^prob_bits; cdf[s] = sum of freq[t] for t < s, cdf[alphabet] = 2^prob_bits. */
typedef struct {
  uint32_t alphabet;  /* 16 (ANS_INT4, ANS_FP4_E2M1) or 256 */
  uint32_t prob_bits; /* 12 for the stream format; 1..15 accepted by ans_build_codebook */
  uint16_t freq[256];
  uint16_t cdf[257];
  uint16_t reserved;
} ans_codebook;

typedef struct {
  uint32_t dtype;      /* ans_dtype */
  uint32_t N, K;       /* W is N x K (N = output features, K = reduction) */
  uint32_t tile_n;     /* 128 or 256 */
  uint32_t tile_k;     /* multiple of 16, at most 256 */
  uint32_t state_bits; /* lane state width: 32 (also 0) or 64 (the wide-state variant) */
} ans_layout;

/* A compressed layer.  For GPU calls the three pointers are device pointers;
 * the struct itself lives on the host and is read during the call only. */
typedef struct {
  ans_layout layout;
  ans_codebook codebook;
  const uint8_t* stream;   /* offsets[n_tiles] bytes, 16-byte aligned */
  uint64_t stream_bytes;
  const uint64_t* offsets; /* n_tiles + 1 entries */
  const uint8_t* raw;      /* ANS_BF16_SPLIT only: N*K bytes, 16-byte aligned; else NULL */
} ans_tiles;

/* Human-readable name of a status code (static storage). */
const char* ans_status_string(ans_status s);

/* Text of the last CUDA error seen by this thread (static per thread). */
const char* ans_last_error(void);

/* Number of tiles of a layout, or 0 when the layout is invalid. */
uint64_t ans_num_tiles(const ans_layout* layout);

/* Validates a layout: N, K > 0, tile_n in {128, 256}, tile_k % 16 == 0,
 * tile_k <= 256, N % tile_n == 0, K % tile_k == 0.  Returns ANS_ERR_SHAPE
 * (or ANS_ERR_ARG for a bad dtype / NULL). */
ans_status ans_layout_check(const ans_layout* layout);

/* GPU histogram of the coded symbols of a layer ("Approaching Shannon Bound",
 * s2.1: empirical histogram per layer).  d_w: the N*K weights in their
 * original format; d_hist: uint64[alphabet], overwritten (zeroed first on
 * `stream`).  Integer counts, so the result does not depend on scheduling. */
ans_status ans_histogram(const void* d_w, const ans_layout* layout, uint64_t* d_hist,
                         ans_stream_t stream);

/* Host counterpart of ans_histogram for offline use without a GPU: h_w the
 * N*K weights in their original format (host memory), hist uint64[alphabet]
 * overwritten.  Multithreaded over rows; integer counts. */
ans_status ans_histogram_host(const void* h_w, const ans_layout* layout, uint64_t* hist);

/* Shannon entropy H = -sum p log2 p of a histogram of up to 65,536 bins,
 * bits per symbol (DFloat11 summary, section "实验方法").  Host. */
ans_status ans_entropy(const uint64_t* hist, uint32_t alphabet, double* bits_per_symbol);

/* Normalises a histogram to integer frequencies summing to 2^prob_bits with
 * freq > 0 exactly for the present symbols, minimising the coded size
 * sum_s hist[s] * log2(2^prob_bits / freq[s]) ("Approaching Shannon Bound",
 * s4.1).  Ties are broken towards the lower symbol index.  Host.
 * Errors: ANS_ERR_ARG (empty histogram, alphabet not 16/256, prob_bits out of
 * 1..15), ANS_ERR_ALPHABET (more present symbols than 2^prob_bits). */
ans_status ans_build_codebook(const uint64_t* hist, uint32_t alphabet, uint32_t prob_bits,
                              ans_codebook* out);

/* Upper bound of the stream size ans_encode_tiles can produce for a layout. */
ans_status ans_encode_bound(const ans_layout* layout, uint64_t* max_stream_bytes);

/* Offline host encoder ("Approaching Shannon Bound", s3.1): codes every tile
 * independently against `codebook` (prob_bits must be 12), writes the stream
 * (h_stream, capacity `cap` bytes), the offset index (h_offsets, n_tiles + 1
 * entries) and, for ANS_BF16_SPLIT, the raw side stream (h_raw, N*K bytes;
 * may be NULL otherwise).  Multithreaded over tiles; the output does not
 * depend on the thread count.  *stream_bytes receives the size even when
 * ANS_ERR_BUFFER_TOO_SMALL is returned.  ANS_ERR_ALPHABET if a weight's
 * symbol has zero frequency. */
ans_status ans_encode_tiles(const void* h_w, const ans_layout* layout,
                            const ans_codebook* codebook, uint8_t* h_stream, uint64_t cap,
                            uint64_t* stream_bytes, uint64_t* h_offsets, uint8_t* h_raw);

/* Standalone GPU decode to HBM: writes the original weights (format of the
 * layout's dtype, row-major N x K) to d_out.  One warp per tile.  This is the
 * bit-exactness check and the first half of the layer-level two-pass baseline
 * ("Approaching Shannon Bound", s2.2 and s4.2).  d_status: device uint32. */
ans_status ans_decode_tiles(const ans_tiles* tiles, void* d_out, uint32_t* d_status,
                            ans_stream_t stream);

/* ---- bf16 as whole 16-bit symbols ("Approaching Shannon Bound", s4.1:
 * bf16's large symbol table makes the precision of the normalised
 * frequencies cost more than for low-bit formats).  The stream format above
 * with symbol = the bf16 bit pattern, 2^n slots (n <= 16; 16 is the reading
 * used here), no raw side stream.  The codebook is a host array
 * uint32 freq[65536] summing to 2^n.  Decode only: the fused GEMM takes the
 * split format (ANS_BF16_SPLIT). */

/* hist: uint64[65536], overwritten.  Host, multithreaded. */
ans_status ans_histogram16_host(const uint16_t* h_w, uint64_t n_weights, uint64_t* hist);

/* The normalisation of ans_build_codebook over 65,536 symbols: freq[65536]
 * summing to 2^prob_bits (1..16), freq > 0 exactly for the present symbols.
 * ANS_ERR_ALPHABET: more present symbols than 2^prob_bits. */
ans_status ans_build_codebook16(const uint64_t* hist, uint32_t prob_bits, uint32_t* freq);

/* Offline encoder for an ANS_BF16_WHOLE layout (either state width; the
 * wide-state format only at prob_bits 12 or 16, else ANS_ERR_ARG); the
 * stream capacity from ans_encode_bound.  Same outputs and errors as
 * ans_encode_tiles (no raw stream). */
ans_status ans_encode_tiles16(const uint16_t* h_w, const ans_layout* layout, const uint32_t* freq,
                              uint32_t prob_bits, uint8_t* h_stream, uint64_t cap,
                              uint64_t* stream_bytes, uint64_t* h_offsets);

/* The decoder's lookup table for a codebook (host image, to be copied to the
 * device as is): *table_bytes receives its size (a multiple of 16); with
 * h_table NULL only the size is returned.  prob_bits 12..16; at most 16,384
 * present symbols (the table lives in shared memory), else
 * ANS_ERR_UNSUPPORTED. */
ans_status ans_decode_table16(const uint32_t* freq, uint32_t prob_bits, uint8_t* h_table,
                              uint64_t cap, uint64_t* table_bytes);

/* GPU decode of an ANS_BF16_WHOLE layer into its bf16 bits (uint16 N x K
 * row-major, 16-byte aligned).  d_table: the ans_decode_table16 image on the
 * device (16-byte aligned); d_stream / d_offsets as in ans_tiles.  Status
 * bits as for ans_decode_tiles. */
ans_status ans_decode_tiles16(const ans_layout* layout, const uint8_t* d_table, uint64_t table_bytes,
                              const uint8_t* d_stream, uint64_t stream_bytes,
                              const uint64_t* d_offsets, uint16_t* d_out, uint32_t* d_status,
                              ans_stream_t stream);

/* Bytes of device workspace ans_gemm / ans_gemm_uncompressed need for a
 * layout, M tokens and a scale kind.  The workspace must be zero-filled once
 * before its first use; the kernels return it to all-zero counters on
 * completion (after a run that set *d_status, zero it again).  Above one
 * token pass (M > 512 for 128-row tiles, M > 256 for 256-row tiles, with K a
 * multiple of 64) it also holds a 16-bit copy of the decoded weights, 2 N K
 * bytes (see ans_gemm). */
ans_status ans_gemm_workspace(const ans_layout* layout, uint32_t M, ans_scale_kind scale_kind,
                              size_t* bytes);

/* Fused decode + GEMM ("Approaching Shannon Bound", s3.1):
 *   Y[m][n] = sum_k X[m][k] * w(n, k),  Y fp32 M x N row-major,
 * with X bf16 M x K row-major (16-byte aligned) and w the dequantised weight:
 *   int4: q (NONE), q * s[n] (ROW_BF16 or ROW_F32), q * s[n][k/group_k]
 *         (GROUP_BF16, group_k a multiple of 16 dividing K);
 *   bf16: the bf16 value (NONE);  fp8: e4m3 value (NONE) or value * s[n] (ROW_F32);
 *   int8: q (NONE) or q * s[n] (ROW_BF16 or ROW_F32);
 *   fp4: e2m1 value (NONE) or value * s[n] (ROW_BF16 or ROW_F32).
 * W's tiles are decoded by producer warps straight into shared memory in the
 * tensor-core operand layout and consumed by tcgen05 MMAs.  Up to one token
 * pass (512 tokens for 128-row tiles, 256 for 256-row tiles) the decoded
 * weights never reach global memory.  Above it, the first pass runs fused
 * and also stores every decoded tile into the workspace, and the remaining
 * tokens run as one dense tensor-core GEMM on those stored weights.  Each
 * tile is then decoded once per call, not once per pass.  Accumulation is
 * fp32 in a fixed order, so the result is bit-identical to
 * ans_gemm_uncompressed on the same weights.  GROUP_BF16 runs
 * the MMA in f16 (X and q*s are exact in f16 when |X| < 65504 and the scales
 * lie in [2^-14, 2^12]), and so do fp8 and int8 (their codes are exact in
 * f16, the row scale is applied to the fp32 accumulator); the other kinds run
 * it in bf16.
 * M == 0 is a no-op.  d_ws: ans_gemm_workspace bytes, 256-byte aligned; d_X,
 * d_Y and d_scales 16-byte aligned (ANS_ERR_ARG otherwise). */
ans_status ans_gemm(const uint16_t* d_X, uint32_t M, const ans_tiles* W,
                    ans_scale_kind scale_kind, const void* d_scales, uint32_t group_k,
                    float* d_Y, void* d_ws, size_t ws_bytes, uint32_t* d_status,
                    ans_stream_t stream);

/* Allocation-free variant of ans_gemm (no counterpart in the paper; it exists
 * for callers of this library that cannot call cudaMalloc: code that runs
 * while a CUDA graph is being captured, plug-ins whose host framework owns all
 * device memory, or latency-critical paths that may not take an allocation's
 * implicit synchronisation).  Same arguments and result as ans_gemm, without
 * the workspace: the scratch (split-K counters and partials, the f16 copy of
 * X for the f16 formats and, above one token pass, the decoded copy of W)
 * lives in a fixed 16 MiB device array inside the
 * library, which every GPU that loads the library holds until the process
 * exits.  A shape whose ans_gemm_workspace exceeds 16 MiB returns
 * ANS_ERR_BUFFER_TOO_SMALL (text via ans_last_error).  Every argument check of
 * ans_gemm runs before anything is queued, so a refused call leaves the array
 * untouched.  The first call on a device looks the array's device address up
 * (cudaGetSymbolAddress with that device current) and keeps it for the life of
 * the process; make that first call before any stream capture, and do not
 * reset the device (cudaDeviceReset) while the library is loaded.  Each call
 * clears the split-K counters with a memset on `stream`; it never allocates.
 * All calls share the one array, which keeps the last call's contents: calls
 * that overlap on the GPU (other streams, other threads) race and must be
 * serialised by the caller. */
ans_status ans_gemm_noalloc(const uint16_t* d_X, uint32_t M, const ans_tiles* W,
                            ans_scale_kind scale_kind, const void* d_scales, uint32_t group_k,
                            float* d_Y, uint32_t* d_status, ans_stream_t stream);

/* The same kernel with the decoder warps replaced by a copy of the original
 * (uncompressed) weights d_W (format of layout->dtype, row-major N x K).
 * Above one token pass the weights are formatted into the workspace's 16-bit
 * copy for the dense GEMM, as ans_gemm's decoded ones are.  Bit-exact
 * reference for ans_gemm and the uncompressed baseline. */
ans_status ans_gemm_uncompressed(const uint16_t* d_X, uint32_t M, const void* d_W,
                                 const ans_layout* layout, ans_scale_kind scale_kind,
                                 const void* d_scales, uint32_t group_k, float* d_Y, void* d_ws,
                                 size_t ws_bytes, uint32_t* d_status, ans_stream_t stream);

/* One layer of a batched call: its X (bf16 M x K, 16-byte aligned), its
 * compressed weights, its scales (as for ans_gemm) and its Y (fp32 M x N,
 * 16-byte aligned).  The structs and the ans_tiles they point to are read
 * during the call only. */
typedef struct {
  const uint16_t* d_X;
  const ans_tiles* W;
  const void* d_scales;
  float* d_Y;
} ans_gemm_job;

#define ANS_MAX_BATCH 8

/* Bytes of device workspace for ans_gemm_batched over these n_jobs layers
 * (same conditions as ans_gemm_workspace, for each layer). */
ans_status ans_gemm_batched_workspace(const ans_gemm_job* jobs, uint32_t n_jobs, uint32_t M,
                                      ans_scale_kind scale_kind, size_t* bytes);

/* Several independent layers in one launch (the gate, up and down
 * projections of an MLP, say: block-level batched decompression of several
 * matrices, DFloat11's "两阶段Kernel"; "Approaching Shannon Bound", s3.1
 * applied to a list of layers): Y_j = X_j * dequant(W_j)^T for j < n_jobs,
 * with M, scale_kind and group_k shared.  1 <= n_jobs <= ANS_MAX_BATCH; every
 * W_j must have the same coded dtype and stream format (state width;
 * ANS_ERR_SHAPE otherwise) and its own codebook; N, K and the tile shape may
 * differ.  Layer j takes a share of the SMs proportional to its weight count
 * N_j * K_j: G_j = max(1, floor(SMs * w_j / sum w)), the largest share giving
 * SMs back while the shares add up to more than the device has, the SMs left
 * over going one each to the first layers.  When every layer takes the small-M
 * schedule on its share (M up to 32 for 128-row tiles, 16 for 256-row tiles)
 * the layers share one kernel launch, each on its share with its own launch
 * plan, so one kernel tail serves them all; otherwise they run as consecutive
 * ans_gemm launches.  Each Y_j is deterministic and within the error bound of
 * ans_gemm; in one launch it is bit-identical to ans_gemm on the same layer
 * confined to G_j SMs (the split-K partition depends on the SM count, so it
 * may differ from ans_gemm's on the whole device in the last bits).  d_ws:
 * ans_gemm_batched_workspace bytes, zero-filled once before first use (the
 * kernels leave it that way); d_status as for ans_gemm. */
ans_status ans_gemm_batched(const ans_gemm_job* jobs, uint32_t n_jobs, uint32_t M,
                            ans_scale_kind scale_kind, uint32_t group_k, void* d_ws,
                            size_t ws_bytes, uint32_t* d_status, ans_stream_t stream);

/* ---- Versioned on-disk container of a compressed layer ---------------------
 * "Approaching Shannon Bound", s3.1: the offline stage yields per layer a
 * shared codebook, a tile offset index and the tile stream (and, for the bf16
 * split, the raw side stream); the container holds them with the layout they
 * were coded for, so a layer is compressed once and loaded many times.
 * Bytes, all little-endian:
 *   [0, 96)  header: magic "RANSTILE", u32 version (1), u32 header size (96),
 *            u32 dtype, N, K, tile_n, tile_k, state_bits, prob_bits, alphabet,
 *            u64 n_tiles, stream bytes, raw bytes, payload bytes, checksum,
 *            reserved (0);
 *   payload: freq (alphabet x u32), offsets ((n_tiles + 1) x u64), stream,
 *            raw, each section starting on a 16-byte boundary of the
 *            container (zero bytes between them).
 * The checksum is 64-bit FNV-1a over the header (checksum field zero) and the
 * payload.  All of it is host memory; nothing is allocated. */
typedef struct {
  ans_layout layout;       /* state_bits 0 is written as 32 */
  uint32_t prob_bits;      /* 12; ANS_BF16_WHOLE: 12..16 (12 or 16 with 64-bit states) */
  uint32_t alphabet;       /* 16 or 256 as the dtype has it; 65,536 for ANS_BF16_WHOLE */
  uint64_t stream_bytes;
  uint64_t raw_bytes;      /* N*K for ANS_BF16_SPLIT, else 0 */
  const uint32_t* freq;    /* alphabet entries summing to 2^prob_bits */
  const uint64_t* offsets; /* n_tiles + 1 entries: 0, 16-byte aligned, non-decreasing,
                              the last = stream_bytes */
  const uint8_t* stream;
  const uint8_t* raw;      /* NULL when raw_bytes == 0 */
  ans_codebook codebook;   /* output of ans_container_read (one-byte formats; zero for
                              ANS_BF16_WHOLE); ignored by ans_container_write */
} ans_container;

/* Writes the container of `layer` to h_out (capacity `cap`); *bytes receives
 * its size (h_out NULL: only the size).  ANS_ERR_ARG / ANS_ERR_SHAPE for a bad
 * layout, a missing array, a raw size that does not match the dtype or
 * offsets that break their rule; ANS_ERR_ALPHABET for an alphabet or a
 * precision the dtype does not take or freq not summing to 2^prob_bits;
 * ANS_ERR_BUFFER_TOO_SMALL when cap < *bytes. */
ans_status ans_container_write(const ans_container* layer, uint8_t* h_out, uint64_t cap,
                               uint64_t* bytes);

/* Reads a container of exactly `bytes` bytes at h_buf (16-byte aligned, kept
 * alive by the caller while `layer` is used): checks the magic, the version,
 * the sizes, the checksum, the layout, the codebook and the offsets, then fills
 * `layer` with the header's fields, views into h_buf (stream and raw 16-byte
 * aligned) and, for the one-byte formats, the ans_codebook of freq.
 * ANS_ERR_ARG for a NULL or misaligned argument, ANS_ERR_UNSUPPORTED for
 * another version, ANS_ERR_CORRUPT for anything else that does not hold. */
ans_status ans_container_read(const uint8_t* h_buf, uint64_t bytes, ans_container* layer);

#ifdef __cplusplus
}
#endif

#endif /* ANS_H_ */
