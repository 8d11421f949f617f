// abi.cpp -- the extern "C" boundary declared in include/ans.h: argument
// validation, codebook checks, and dispatch to the host codec or the CUDA
// kernels.  No device memory is allocated here.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>

#include "../../include/ans.h"
#include "cuda/kernels.h"
#include "host/codec_host.h"

namespace {

thread_local char g_last_error[256] = "";

ans_status cuda_fail(cudaError_t e, const char* where) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where, cudaGetErrorString(e),
                static_cast<int>(e));
  return ANS_ERR_CUDA;
}

uint32_t alphabet_of(uint32_t dtype) { return (dtype == ANS_INT4 || dtype == ANS_FP4_E2M1) ? 16u : 256u; }
// packed-nibble storage (per-element or pair symbols)
bool is_int4(uint32_t dtype) { return dtype == ANS_INT4 || dtype == ANS_INT4_PAIRS; }
// two weights per byte
bool is_nibble(uint32_t dtype) {
  return is_int4(dtype) || dtype == ANS_FP4_E2M1 || dtype == ANS_FP4_PAIRS;
}

ans_status check_layout(const ans_layout* l) {
  if (!l) return ANS_ERR_ARG;
  if (l->dtype > ANS_FP4_PAIRS) return ANS_ERR_ARG;
  if (l->state_bits != 0 && l->state_bits != 32 && l->state_bits != 64) return ANS_ERR_ARG;
  if (!anshost::layout_valid(l->N, l->K, l->tile_n, l->tile_k)) return ANS_ERR_SHAPE;
  return ANS_OK;
}

// Layout of the 16-bit-symbol entry points: dtype ANS_BF16_WHOLE.
ans_status check_layout16(const ans_layout* l) {
  if (!l) return ANS_ERR_ARG;
  if (l->dtype != ANS_BF16_WHOLE) return ANS_ERR_ARG;
  if (l->state_bits != 0 && l->state_bits != 32 && l->state_bits != 64) return ANS_ERR_ARG;
  if (!anshost::layout_valid(l->N, l->K, l->tile_n, l->tile_k)) return ANS_ERR_SHAPE;
  return ANS_OK;
}

// A 16-bit codebook: 65,536 frequencies summing to 2^prob_bits.
ans_status check_freq16(const uint32_t* freq, uint32_t prob_bits) {
  if (!freq || prob_bits < 1 || prob_bits > 16) return ANS_ERR_ARG;
  uint64_t run = 0;
  for (uint32_t s = 0; s < 65536; ++s) run += freq[s];
  return run == (1ull << prob_bits) ? ANS_OK : ANS_ERR_ALPHABET;
}

// Either kind of layout: the one-byte-symbol formats, or the 16-bit-symbol
// layout of the ans_*16 entry points.
ans_status check_any_layout(const ans_layout* layout) {
  return layout && layout->dtype == ANS_BF16_WHOLE ? check_layout16(layout) : check_layout(layout);
}

// Stream-format codebook: alphabet of the dtype, 12-bit precision, freq
// summing to 4096, cdf consistent with freq.
ans_status check_codebook(const ans_codebook* cb, uint32_t dtype) {
  if (!cb) return ANS_ERR_ARG;
  if (cb->alphabet != alphabet_of(dtype) || cb->prob_bits != 12) return ANS_ERR_ALPHABET;
  uint32_t run = 0;
  for (uint32_t s = 0; s < cb->alphabet; ++s) {
    if (cb->cdf[s] != run) return ANS_ERR_ALPHABET;
    run += cb->freq[s];
  }
  if (run != 4096 || cb->cdf[cb->alphabet] != 4096) return ANS_ERR_ALPHABET;
  return ANS_OK;
}

ans_status device_info(int* num_sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  static int cached_sms[64];
  static int cached_major[64];
  if (dev < 0 || dev >= 64) return ANS_ERR_UNSUPPORTED;
  if (cached_sms[dev] == 0) {
    int sms = 0, major = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    cached_major[dev] = major;
    cached_sms[dev] = sms;
  }
  if (cached_major[dev] != 10) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "kernels are built for sm_100a; device major = %d", cached_major[dev]);
    return ANS_ERR_UNSUPPORTED;
  }
  *num_sms = cached_sms[dev];
  return ANS_OK;
}

void fill_layer(const ans_tiles* t, ansdev::LayerDev* L) {
  std::memset(L, 0, sizeof(*L));
  const ans_layout& ly = t->layout;
  L->stream = t->stream;
  L->offsets = t->offsets;
  L->raw = t->raw;
  L->stream_bytes = t->stream_bytes;
  L->N = ly.N;
  L->K = ly.K;
  L->tile_n = ly.tile_n;
  L->tile_k = ly.tile_k;
  L->n_kt = ly.K / ly.tile_k;
  L->n_tiles = (ly.N / ly.tile_n) * L->n_kt;
  L->dtype = ly.dtype;
  L->wide = ly.state_bits == 64 ? 1u : 0u;
  L->alphabet = t->codebook.alphabet;
  L->single_symbol = ansdev::kNoSymbolHost;
  for (uint32_t s = 0; s < t->codebook.alphabet; ++s) {
    L->freq[s] = t->codebook.freq[s];
    L->cdf[s] = t->codebook.cdf[s];
    if (t->codebook.freq[s] == 4096) L->single_symbol = s;
  }
  L->cdf[t->codebook.alphabet] = t->codebook.cdf[t->codebook.alphabet];
}

// Layout-only LayerDev (copy mode and planning).
void fill_layer_plain(const ans_layout* ly, ansdev::LayerDev* L) {
  std::memset(L, 0, sizeof(*L));
  L->N = ly->N;
  L->K = ly->K;
  L->tile_n = ly->tile_n;
  L->tile_k = ly->tile_k;
  L->n_kt = ly->K / ly->tile_k;
  L->n_tiles = (ly->N / ly->tile_n) * L->n_kt;
  L->dtype = ly->dtype;
  L->alphabet = alphabet_of(ly->dtype);
  L->single_symbol = ansdev::kNoSymbolHost;
}

ans_status check_scales(uint32_t dtype, ans_scale_kind kind, const void* scales, uint32_t group_k,
                        const ans_layout& ly) {
  switch (kind) {
    case ANS_SCALE_NONE: return ANS_OK;
    case ANS_SCALE_ROW_BF16:
    case ANS_SCALE_ROW_F32: return scales ? ANS_OK : ANS_ERR_ARG;
    case ANS_SCALE_GROUP_BF16:
      if (!is_int4(dtype) || !scales) return ANS_ERR_ARG;
      if (group_k == 0 || group_k % 16 != 0 || ly.K % group_k != 0) return ANS_ERR_ARG;
      if (group_k % ly.tile_k != 0) return ANS_ERR_UNSUPPORTED;
      return ANS_OK;
  }
  return ANS_ERR_ARG;
}

// Checks of the device buffers every fused-GEMM call takes (no device work).
ans_status check_gemm_io(const uint16_t* d_X, float* d_Y, uint32_t* d_status, const void* d_scales) {
  if (!d_X || !d_Y || !d_status) return ANS_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(d_X) % 16 != 0 || reinterpret_cast<uintptr_t>(d_Y) % 16 != 0 ||
      (d_scales && reinterpret_cast<uintptr_t>(d_scales) % 16 != 0))
    return ANS_ERR_ARG;
  return ANS_OK;
}

// Checks of a compressed layer as ans_gemm takes it (no device work).
ans_status check_gemm_tiles(const ans_tiles* W, ans_scale_kind scale_kind, const void* d_scales,
                            uint32_t group_k) {
  if (!W) return ANS_ERR_ARG;
  ans_status st = check_layout(&W->layout);
  if (st != ANS_OK) return st;
  st = check_codebook(&W->codebook, W->layout.dtype);
  if (st != ANS_OK) return st;
  st = check_scales(W->layout.dtype, scale_kind, d_scales, group_k, W->layout);
  if (st != ANS_OK) return st;
  if (!W->stream || !W->offsets) return ANS_ERR_ARG;
  if (W->layout.dtype == ANS_BF16_SPLIT && !W->raw) return ANS_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(W->stream) % 16 != 0 ||
      reinterpret_cast<uintptr_t>(W->offsets) % 8 != 0 ||
      (W->raw && reinterpret_cast<uintptr_t>(W->raw) % 16 != 0))
    return ANS_ERR_ARG;
  return ANS_OK;
}

// The launch plan of one call on the current device.
ans_status plan_gemm(const ansdev::LayerDev& L, uint32_t M, ans_scale_kind kind, bool decode,
                     ansdev::GemmPlan* plan) {
  int sms = 0;
  ans_status st = device_info(&sms);
  if (st != ANS_OK) return st;
  if (!ansdev::make_gemm_plan(L, M, kind, decode, sms, plan)) return ANS_ERR_UNSUPPORTED;
  return ANS_OK;
}

ans_status launch_planned(const ansdev::GemmPlan& plan, const uint16_t* d_X,
                          const ansdev::LayerDev& L, bool decode, const void* d_W,
                          ans_scale_kind kind, const void* d_scales, uint32_t group_k, float* d_Y,
                          void* d_ws, uint32_t* d_status, ans_stream_t stream) {
  cudaError_t e = ansdev::launch_gemm(plan, L, decode, d_W, d_X, d_scales, kind, group_k, d_Y,
                                      d_ws, d_status, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, decode ? "ans_gemm" : "ans_gemm_uncompressed");
  return ANS_OK;
}

ans_status run_gemm(const uint16_t* d_X, uint32_t M, const ansdev::LayerDev& L, bool decode,
                    const void* d_W, ans_scale_kind kind, const void* d_scales, uint32_t group_k,
                    float* d_Y, void* d_ws, size_t ws_bytes, uint32_t* d_status,
                    ans_stream_t stream) {
  if (M == 0) return ANS_OK;
  ans_status st = check_gemm_io(d_X, d_Y, d_status, d_scales);
  if (st != ANS_OK) return st;
  if (!d_ws || reinterpret_cast<uintptr_t>(d_ws) % 256 != 0) return ANS_ERR_ARG;
  ansdev::GemmPlan plan;
  st = plan_gemm(L, M, kind, decode, &plan);
  if (st != ANS_OK) return st;
  if (ws_bytes < plan.ws_bytes) return ANS_ERR_BUFFER_TOO_SMALL;
  return launch_planned(plan, d_X, L, decode, d_W, kind, d_scales, group_k, d_Y, d_ws, d_status,
                        stream);
}

// Layout, alphabet, precision and raw size of a container's layer: ANS_OK,
// or the status that ans_container_write reports.
ans_status check_container_fields(const ans_container* c) {
  ans_status st = check_any_layout(&c->layout);
  if (st != ANS_OK) return st;
  const uint32_t dtype = c->layout.dtype;
  const bool whole = dtype == ANS_BF16_WHOLE;
  if (c->alphabet != (whole ? 65536u : alphabet_of(dtype))) return ANS_ERR_ALPHABET;
  if (whole ? (c->prob_bits < 12 || c->prob_bits > 16 ||
               (c->layout.state_bits == 64 && c->prob_bits != 12 && c->prob_bits != 16))
            : c->prob_bits != 12)
    return ANS_ERR_ALPHABET;
  const uint64_t raw = dtype == ANS_BF16_SPLIT ? static_cast<uint64_t>(c->layout.N) * c->layout.K : 0;
  if (c->raw_bytes != raw) return ANS_ERR_ARG;
  const uint64_t bound = anshost::encode_bound(c->layout.N, c->layout.K, c->layout.tile_n,
                                               c->layout.tile_k, c->layout.state_bits == 64);
  if (c->stream_bytes > bound) return ANS_ERR_ARG;
  return ANS_OK;
}

anshost::ContainerLayer to_host_layer(const ans_container* c) {
  anshost::ContainerLayer h;
  h.dtype = c->layout.dtype;
  h.N = c->layout.N;
  h.K = c->layout.K;
  h.tile_n = c->layout.tile_n;
  h.tile_k = c->layout.tile_k;
  h.state_bits = c->layout.state_bits == 64 ? 64u : 32u;
  h.prob_bits = c->prob_bits;
  h.alphabet = c->alphabet;
  h.n_tiles = static_cast<uint64_t>(c->layout.N / c->layout.tile_n) * (c->layout.K / c->layout.tile_k);
  h.stream_bytes = c->stream_bytes;
  h.raw_bytes = c->raw_bytes;
  h.freq = c->freq;
  h.offsets = c->offsets;
  h.stream = c->stream;
  h.raw = c->raw;
  return h;
}

}  // namespace

extern "C" {

const char* ans_status_string(ans_status s) {
  switch (s) {
    case ANS_OK: return "ok";
    case ANS_ERR_ARG: return "invalid argument";
    case ANS_ERR_SHAPE: return "unsupported shape";
    case ANS_ERR_ALPHABET: return "invalid codebook or symbol outside it";
    case ANS_ERR_BUFFER_TOO_SMALL: return "buffer too small";
    case ANS_ERR_CUDA: return "CUDA error";
    case ANS_ERR_CORRUPT: return "corrupt stream";
    case ANS_ERR_TIMEOUT: return "timeout";
    case ANS_ERR_UNSUPPORTED: return "unsupported";
  }
  return "unknown status";
}

const char* ans_last_error(void) { return g_last_error; }

uint64_t ans_num_tiles(const ans_layout* layout) {
  if (check_any_layout(layout) != ANS_OK) return 0;
  return static_cast<uint64_t>(layout->N / layout->tile_n) * (layout->K / layout->tile_k);
}

ans_status ans_layout_check(const ans_layout* layout) { return check_any_layout(layout); }

ans_status ans_histogram(const void* d_w, const ans_layout* layout, uint64_t* d_hist,
                         ans_stream_t stream) {
  if (!layout || layout->dtype > ANS_FP4_PAIRS) return ANS_ERR_ARG;
  if (layout->N == 0 || layout->K == 0) return ANS_ERR_SHAPE;
  if (is_nibble(layout->dtype) && layout->K % 2 != 0) return ANS_ERR_SHAPE;
  if (!d_w || !d_hist || reinterpret_cast<uintptr_t>(d_w) % 16 != 0) return ANS_ERR_ARG;
  int sms = 0;
  ans_status st = device_info(&sms);
  if (st != ANS_OK) return st;
  const uint64_t n = static_cast<uint64_t>(layout->N) * layout->K;
  const uint64_t bytes = is_nibble(layout->dtype) ? n / 2 : (layout->dtype == ANS_BF16_SPLIT ? 2 * n : n);
  cudaError_t e = ansdev::launch_histogram(d_w, bytes, layout->dtype, d_hist,
                                           reinterpret_cast<cudaStream_t>(stream), sms);
  if (e != cudaSuccess) return cuda_fail(e, "ans_histogram");
  return ANS_OK;
}

ans_status ans_histogram_host(const void* h_w, const ans_layout* layout, uint64_t* hist) {
  if (!layout || layout->dtype > ANS_FP4_PAIRS) return ANS_ERR_ARG;
  if (layout->N == 0 || layout->K == 0) return ANS_ERR_SHAPE;
  if (is_nibble(layout->dtype) && layout->K % 2 != 0) return ANS_ERR_SHAPE;
  if (!h_w || !hist) return ANS_ERR_ARG;
  anshost::histogram(layout->dtype, h_w, static_cast<uint64_t>(layout->N) * layout->K, hist);
  return ANS_OK;
}

ans_status ans_entropy(const uint64_t* hist, uint32_t alphabet, double* bits_per_symbol) {
  if (!hist || !bits_per_symbol || alphabet == 0 || alphabet > 65536) return ANS_ERR_ARG;
  *bits_per_symbol = anshost::entropy_bits(hist, alphabet);
  return ANS_OK;
}

ans_status ans_build_codebook(const uint64_t* hist, uint32_t alphabet, uint32_t prob_bits,
                              ans_codebook* out) {
  if (!hist || !out || (alphabet != 16 && alphabet != 256)) return ANS_ERR_ARG;
  uint32_t freq[256] = {0};
  int r = anshost::normalize(hist, alphabet, prob_bits, freq);
  if (r == 1) return ANS_ERR_ARG;
  if (r == 3) return ANS_ERR_ALPHABET;
  std::memset(out, 0, sizeof(*out));
  out->alphabet = alphabet;
  out->prob_bits = prob_bits;
  uint32_t run = 0;
  for (uint32_t s = 0; s < alphabet; ++s) {
    out->freq[s] = static_cast<uint16_t>(freq[s]);
    out->cdf[s] = static_cast<uint16_t>(run);
    run += freq[s];
  }
  out->cdf[alphabet] = static_cast<uint16_t>(run);
  return ANS_OK;
}

ans_status ans_encode_bound(const ans_layout* layout, uint64_t* max_stream_bytes) {
  ans_status st = check_any_layout(layout);
  if (st != ANS_OK) return st;
  if (!max_stream_bytes) return ANS_ERR_ARG;
  *max_stream_bytes = anshost::encode_bound(layout->N, layout->K, layout->tile_n, layout->tile_k,
                                           layout->state_bits == 64);
  return ANS_OK;
}

ans_status ans_encode_tiles(const void* h_w, const ans_layout* layout,
                            const ans_codebook* codebook, uint8_t* h_stream, uint64_t cap,
                            uint64_t* stream_bytes, uint64_t* h_offsets, uint8_t* h_raw) {
  ans_status st = check_layout(layout);
  if (st != ANS_OK) return st;
  if (!h_w || !h_stream || !stream_bytes || !h_offsets) return ANS_ERR_ARG;
  if (layout->dtype == ANS_BF16_SPLIT && !h_raw) return ANS_ERR_ARG;
  st = check_codebook(codebook, layout->dtype);
  if (st != ANS_OK) return st;
  uint32_t freq[256] = {0};
  for (uint32_t s = 0; s < codebook->alphabet; ++s) freq[s] = codebook->freq[s];
  int r = anshost::encode(layout->dtype, h_w, layout->N, layout->K, layout->tile_n,
                          layout->tile_k, freq, h_stream, cap, stream_bytes, h_offsets, h_raw,
                          layout->state_bits == 64);
  if (r == 3) return ANS_ERR_ALPHABET;
  if (r == 4) return ANS_ERR_BUFFER_TOO_SMALL;
  return r == 0 ? ANS_OK : ANS_ERR_ARG;
}

ans_status ans_decode_tiles(const ans_tiles* tiles, void* d_out, uint32_t* d_status,
                            ans_stream_t stream) {
  if (!tiles || !d_out || !d_status) return ANS_ERR_ARG;
  ans_status st = check_layout(&tiles->layout);
  if (st != ANS_OK) return st;
  st = check_codebook(&tiles->codebook, tiles->layout.dtype);
  if (st != ANS_OK) return st;
  if (!tiles->stream || !tiles->offsets) return ANS_ERR_ARG;
  if (tiles->layout.dtype == ANS_BF16_SPLIT && !tiles->raw) return ANS_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(d_out) % 16 != 0 ||
      reinterpret_cast<uintptr_t>(tiles->stream) % 16 != 0 ||
      reinterpret_cast<uintptr_t>(tiles->offsets) % 8 != 0 ||
      (tiles->raw && reinterpret_cast<uintptr_t>(tiles->raw) % 16 != 0))
    return ANS_ERR_ARG;
  int sms = 0;
  st = device_info(&sms);
  if (st != ANS_OK) return st;
  ansdev::LayerDev L;
  fill_layer(tiles, &L);
  cudaError_t e = ansdev::launch_decode_tiles(L, d_out, d_status,
                                              reinterpret_cast<cudaStream_t>(stream), sms);
  if (e != cudaSuccess) return cuda_fail(e, "ans_decode_tiles");
  return ANS_OK;
}

ans_status ans_histogram16_host(const uint16_t* h_w, uint64_t n_weights, uint64_t* hist) {
  if (!h_w || !hist) return ANS_ERR_ARG;
  anshost::histogram16(h_w, n_weights, hist);
  return ANS_OK;
}

ans_status ans_build_codebook16(const uint64_t* hist, uint32_t prob_bits, uint32_t* freq) {
  if (!hist || !freq) return ANS_ERR_ARG;
  const int r = anshost::normalize16(hist, prob_bits, freq);
  if (r == 3) return ANS_ERR_ALPHABET;
  return r == 0 ? ANS_OK : ANS_ERR_ARG;
}

ans_status ans_encode_tiles16(const uint16_t* h_w, const ans_layout* layout, const uint32_t* freq,
                              uint32_t prob_bits, uint8_t* h_stream, uint64_t cap,
                              uint64_t* stream_bytes, uint64_t* h_offsets) {
  ans_status st = check_layout16(layout);
  if (st != ANS_OK) return st;
  if (!h_w || !h_stream || !stream_bytes || !h_offsets) return ANS_ERR_ARG;
  st = check_freq16(freq, prob_bits);
  if (st != ANS_OK) return st;
  const int r = anshost::encode16(h_w, layout->N, layout->K, layout->tile_n, layout->tile_k, freq,
                                  prob_bits, h_stream, cap, stream_bytes, h_offsets,
                                  layout->state_bits == 64);
  if (r == 3) return ANS_ERR_ALPHABET;
  if (r == 4) return ANS_ERR_BUFFER_TOO_SMALL;
  return r == 0 ? ANS_OK : ANS_ERR_ARG;
}

ans_status ans_decode_table16(const uint32_t* freq, uint32_t prob_bits, uint8_t* h_table,
                              uint64_t cap, uint64_t* table_bytes) {
  if (!table_bytes) return ANS_ERR_ARG;
  ans_status st = check_freq16(freq, prob_bits);
  if (st != ANS_OK) return st;
  if (prob_bits < 12) return ANS_ERR_UNSUPPORTED;
  uint64_t present = 0;
  for (uint32_t s = 0; s < 65536; ++s) present += freq[s] ? 1 : 0;
  if (present > ansdev::kMaxPresent16) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "ans_decode_table16: %llu present symbols, the decoder holds at most %u",
                  static_cast<unsigned long long>(present), ansdev::kMaxPresent16);
    return ANS_ERR_UNSUPPORTED;
  }
  *table_bytes = anshost::table16_bytes(freq);
  if (!h_table) return ANS_OK;
  const int r = anshost::table16(freq, prob_bits, h_table, cap);
  if (r == 4) return ANS_ERR_BUFFER_TOO_SMALL;
  return r == 0 ? ANS_OK : ANS_ERR_ALPHABET;
}

ans_status ans_decode_tiles16(const ans_layout* layout, const uint8_t* d_table, uint64_t table_bytes,
                              const uint8_t* d_stream, uint64_t stream_bytes,
                              const uint64_t* d_offsets, uint16_t* d_out, uint32_t* d_status,
                              ans_stream_t stream) {
  ans_status st = check_layout16(layout);
  if (st != ANS_OK) return st;
  if (!d_table || !d_stream || !d_offsets || !d_out || !d_status) return ANS_ERR_ARG;
  if (table_bytes == 0 || table_bytes % 16 != 0 ||
      table_bytes > 8 + 2 * 4096 + 6ull * ansdev::kMaxPresent16 + 15)
    return ANS_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(d_out) % 16 != 0 ||
      reinterpret_cast<uintptr_t>(d_table) % 16 != 0 ||
      reinterpret_cast<uintptr_t>(d_stream) % 16 != 0 ||
      reinterpret_cast<uintptr_t>(d_offsets) % 8 != 0)
    return ANS_ERR_ARG;
  int sms = 0;
  st = device_info(&sms);
  if (st != ANS_OK) return st;
  ansdev::LayerDev L;
  fill_layer_plain(layout, &L);
  L.stream = d_stream;
  L.stream_bytes = stream_bytes;
  L.offsets = d_offsets;
  L.wide = layout->state_bits == 64 ? 1u : 0u;
  cudaError_t e = ansdev::launch_decode_tiles16(L, d_table, static_cast<uint32_t>(table_bytes),
                                                d_out, d_status,
                                                reinterpret_cast<cudaStream_t>(stream), sms);
  if (e != cudaSuccess) return cuda_fail(e, "ans_decode_tiles16");
  return ANS_OK;
}

ans_status ans_gemm_workspace(const ans_layout* layout, uint32_t M, ans_scale_kind scale_kind,
                              size_t* bytes) {
  ans_status st = check_layout(layout);
  if (st != ANS_OK) return st;
  if (!bytes) return ANS_ERR_ARG;
  if (M == 0) { *bytes = 0; return ANS_OK; }
  int sms = 0;
  st = device_info(&sms);
  if (st != ANS_OK) return st;
  ansdev::LayerDev L;
  fill_layer_plain(layout, &L);
  ansdev::GemmPlan plan;
  if (!ansdev::make_gemm_plan(L, M, scale_kind, true, sms, &plan)) return ANS_ERR_UNSUPPORTED;
  *bytes = plan.ws_bytes;
  return ANS_OK;
}

ans_status ans_gemm(const uint16_t* d_X, uint32_t M, const ans_tiles* W,
                    ans_scale_kind scale_kind, const void* d_scales, uint32_t group_k,
                    float* d_Y, void* d_ws, size_t ws_bytes, uint32_t* d_status,
                    ans_stream_t stream) {
  ans_status st = check_gemm_tiles(W, scale_kind, d_scales, group_k);
  if (st != ANS_OK) return st;
  ansdev::LayerDev L;
  fill_layer(W, &L);
  return run_gemm(d_X, M, L, true, nullptr, scale_kind, d_scales, group_k, d_Y, d_ws, ws_bytes,
                  d_status, stream);
}

ans_status ans_gemm_uncompressed(const uint16_t* d_X, uint32_t M, const void* d_W,
                                 const ans_layout* layout, ans_scale_kind scale_kind,
                                 const void* d_scales, uint32_t group_k, float* d_Y, void* d_ws,
                                 size_t ws_bytes, uint32_t* d_status, ans_stream_t stream) {
  ans_status st = check_layout(layout);
  if (st != ANS_OK) return st;
  if (!d_W || reinterpret_cast<uintptr_t>(d_W) % 16 != 0) return ANS_ERR_ARG;
  st = check_scales(layout->dtype, scale_kind, d_scales, group_k, *layout);
  if (st != ANS_OK) return st;
  ansdev::LayerDev L;
  fill_layer_plain(layout, &L);
  return run_gemm(d_X, M, L, false, d_W, scale_kind, d_scales, group_k, d_Y, d_ws, ws_bytes,
                  d_status, stream);
}

ans_status ans_gemm_noalloc(const uint16_t* d_X, uint32_t M, const ans_tiles* W,
                            ans_scale_kind scale_kind, const void* d_scales, uint32_t group_k,
                            float* d_Y, uint32_t* d_status, ans_stream_t stream) {
  // every check of ans_gemm first: a refused call leaves the shared scratch
  // (and any call still running on it) untouched
  ans_status st = check_gemm_tiles(W, scale_kind, d_scales, group_k);
  if (st != ANS_OK) return st;
  if (M == 0) return ANS_OK;
  st = check_gemm_io(d_X, d_Y, d_status, d_scales);
  if (st != ANS_OK) return st;
  ansdev::LayerDev L;
  fill_layer(W, &L);
  ansdev::GemmPlan plan;
  st = plan_gemm(L, M, scale_kind, true, &plan);
  if (st != ANS_OK) return st;
  if (plan.ws_bytes > ansdev::kNoAllocScratchBytes) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "ans_gemm_noalloc: this shape needs %zu bytes of scratch, above the fixed "
                  "%zu-byte maximum; use ans_gemm with a caller workspace",
                  plan.ws_bytes, ansdev::kNoAllocScratchBytes);
    return ANS_ERR_BUFFER_TOO_SMALL;
  }
  void* scratch = nullptr;
  cudaError_t e = ansdev::noalloc_scratch(&scratch);
  if (e != cudaSuccess) return cuda_fail(e, "ans_gemm_noalloc scratch");
  // the split-K counters must start at zero: clear them on the caller's
  // stream (a memset, not an allocation)
  e = cudaMemsetAsync(scratch, 0, plan.ws_counters_bytes, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "ans_gemm_noalloc clear");
  return launch_planned(plan, d_X, L, true, nullptr, scale_kind, d_scales, group_k, d_Y, scratch,
                        d_status, stream);
}

// Internal profiling hook (not part of the public ABI in include/ans.h).
void ansdev_set_trace(void* d_buf, size_t bytes) { ansdev::set_trace_buffer(d_buf, bytes); }

// Internal test hooks (not part of the public ABI): the budget, in clock64
// cycles, of every wait in the library's kernels that the pipeline's own
// progress ends (0 restores the default of about 1.5 s), on the current
// device; and one bounded wait on a barrier that nothing arrives on, which
// leaves the TIMEOUT bit in *d_status.
int ansdev_set_wait_budget(long long cycles) {
  const long long c = cycles > 0 ? cycles : ansdev::kWaitBudgetCyclesHost;
  cudaError_t e = ansdev::set_live_wait_budget_gemm(c);
  if (e == cudaSuccess) e = ansdev::set_live_wait_budget_local(c);
  if (e == cudaSuccess) e = ansdev::set_live_wait_budget_decode(c);
  if (e == cudaSuccess) e = ansdev::set_live_wait_budget_dense(c);
  if (e == cudaSuccess) e = ansdev::set_live_wait_budget_decode16(c);
  return e == cudaSuccess ? ANS_OK : cuda_fail(e, "ansdev_set_wait_budget");
}

int ansdev_wait_probe(uint32_t* d_status, ans_stream_t stream) {
  if (!d_status) return ANS_ERR_ARG;
  cudaError_t e = ansdev::launch_wait_probe(d_status, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ANS_OK : cuda_fail(e, "ansdev_wait_probe");
}

// Internal test hook (not part of the public ABI): caps on the CTAs and
// producer warps of every later fused-GEMM plan in this process and a switch
// that forces the shared-accumulator schedule; 0, 0, 0 restores the defaults.
void ansdev_set_plan_limits(uint32_t max_ctas, uint32_t max_producers, uint32_t force_shared) {
  ansdev::set_plan_limits(max_ctas, max_producers, force_shared);
}

// Internal test hook (not part of the public ABI): the launch plan that
// ans_gemm (decode = 1) or ans_gemm_uncompressed (decode = 0) would use for a
// layout, M and scale kind on a device with num_sms SMs, without touching a
// device.  out[0..20] = local, grid, D, n_slots, tmem_cols, smem_bytes, T,
// T_pass, n_pass, NT, n_bufs, fmt, ab_f16, H, C, x_stages, n_units,
// n_segments, ws_bytes (low 32 bits), ws_bytes (high 32 bits), dense (1: a
// fused first pass of 16 tokens, then the dense GEMM; the other fields are
// the first pass's).
// Returns 1 if the shape can be scheduled, 0 if not, -1 for a bad layout.
int ansdev_gemm_plan(const ans_layout* layout, uint32_t M, uint32_t scale_kind, int decode,
                     int num_sms, uint32_t* out) {
  if (check_layout(layout) != ANS_OK || !out) return -1;
  ansdev::LayerDev L;
  fill_layer_plain(layout, &L);
  L.wide = layout->state_bits == 64 ? 1u : 0u;
  ansdev::GemmPlan p;
  if (!ansdev::make_gemm_plan(L, M, scale_kind, decode != 0, num_sms, &p)) return 0;
  const uint32_t v[21] = {p.local, p.grid, p.D, p.n_slots, p.tmem_cols, p.smem_bytes, p.T,
                          p.T_pass, p.n_pass, p.NT, p.n_bufs, p.fmt, p.ab_f16, p.H, p.C,
                          p.x_stages, static_cast<uint32_t>(p.n_units), p.n_segments,
                          static_cast<uint32_t>(p.ws_bytes),
                          static_cast<uint32_t>(static_cast<uint64_t>(p.ws_bytes) >> 32), p.dense};
  for (int i = 0; i < 21; ++i) out[i] = v[i];
  return 1;
}

}  // extern "C"

namespace {

// Shared checks of a batch: every layout valid, one coded dtype and one
// stream format (state width) for all jobs; shapes and tiles may differ.  On
// success *sms is the device's SM count.
ans_status check_batch(const ans_gemm_job* jobs, uint32_t n_jobs, int* sms) {
  if (!jobs || n_jobs == 0 || n_jobs > ANS_MAX_BATCH) return ANS_ERR_ARG;
  for (uint32_t j = 0; j < n_jobs; ++j) {
    if (!jobs[j].W) return ANS_ERR_ARG;
    ans_status st = check_layout(&jobs[j].W->layout);
    if (st != ANS_OK) return st;
    const ans_layout& a = jobs[0].W->layout;
    const ans_layout& b = jobs[j].W->layout;
    if (a.dtype != b.dtype || (a.state_bits == 64) != (b.state_bits == 64)) return ANS_ERR_SHAPE;
  }
  return device_info(sms);
}

// SM shares of a batch in one launch, proportional to the jobs' weight
// counts: G_j = max(1, floor(sms * w_j / sum w)); while the shares add up to
// more than sms the largest gives one back; what is left over goes one each
// to the first jobs.
void batch_shares(const ans_gemm_job* jobs, uint32_t n, int sms, uint32_t* G) {
  double total = 0;
  for (uint32_t j = 0; j < n; ++j)
    total += static_cast<double>(jobs[j].W->layout.N) * jobs[j].W->layout.K;
  uint32_t sum = 0;
  for (uint32_t j = 0; j < n; ++j) {
    const double w = static_cast<double>(jobs[j].W->layout.N) * jobs[j].W->layout.K;
    G[j] = static_cast<uint32_t>(static_cast<double>(sms) * w / total);
    if (G[j] < 1) G[j] = 1;
    sum += G[j];
  }
  while (sum > static_cast<uint32_t>(sms)) {
    uint32_t big = 0;
    for (uint32_t j = 1; j < n; ++j)
      if (G[j] > G[big]) big = j;
    if (G[big] <= 1) break;
    --G[big];
    --sum;
  }
  for (uint32_t j = 0; sum < static_cast<uint32_t>(sms) && j < n; ++j, ++sum) ++G[j];
}

// Plans of a batch: share[j] for job j on its share of the SMs (used when
// every job takes the small-M schedule there: all jobs in one launch),
// full[j] for job j on all SMs (consecutive launches otherwise); ws_off[j]
// the byte offset of job j's workspace, ws_off[n] the total, each job's part
// large enough for either plan.
ans_status batch_plan(const ans_gemm_job* jobs, uint32_t n_jobs, uint32_t M,
                      ans_scale_kind scale_kind, int sms, ansdev::GemmPlan* share,
                      ansdev::GemmPlan* full, size_t* ws_off, bool* one_launch) {
  uint32_t G[ANS_MAX_BATCH];
  batch_shares(jobs, n_jobs, sms, G);
  *one_launch = true;
  ws_off[0] = 0;
  for (uint32_t j = 0; j < n_jobs; ++j) {
    ansdev::LayerDev L;
    fill_layer_plain(&jobs[j].W->layout, &L);
    if (!ansdev::make_gemm_plan(L, M, scale_kind, true, static_cast<int>(G[j]), &share[j]))
      return ANS_ERR_UNSUPPORTED;
    if (!ansdev::make_gemm_plan(L, M, scale_kind, true, sms, &full[j])) return ANS_ERR_UNSUPPORTED;
    // one launch only when every job is a single pass of the small-M schedule
    // on its share (a large-M plan's fields describe its first pass alone)
    if (!share[j].local || share[j].dense || share[j].fmt != share[0].fmt) *one_launch = false;
    const size_t a = share[j].ws_bytes > full[j].ws_bytes ? share[j].ws_bytes : full[j].ws_bytes;
    ws_off[j + 1] = ws_off[j] + ((a + 255) / 256) * 256;
  }
  return ANS_OK;
}

}  // namespace

extern "C" {

ans_status ans_gemm_batched_workspace(const ans_gemm_job* jobs, uint32_t n_jobs, uint32_t M,
                                      ans_scale_kind scale_kind, size_t* bytes) {
  if (!bytes) return ANS_ERR_ARG;
  int sms = 0;
  ans_status st = check_batch(jobs, n_jobs, &sms);
  if (st != ANS_OK) return st;
  if (M == 0) { *bytes = 0; return ANS_OK; }
  ansdev::GemmPlan share[ANS_MAX_BATCH], full[ANS_MAX_BATCH];
  size_t ws_off[ANS_MAX_BATCH + 1];
  bool one = false;
  st = batch_plan(jobs, n_jobs, M, scale_kind, sms, share, full, ws_off, &one);
  if (st != ANS_OK) return st;
  *bytes = ws_off[n_jobs];
  return ANS_OK;
}

ans_status ans_gemm_batched(const ans_gemm_job* jobs, uint32_t n_jobs, uint32_t M,
                            ans_scale_kind scale_kind, uint32_t group_k, void* d_ws,
                            size_t ws_bytes, uint32_t* d_status, ans_stream_t stream) {
  int sms = 0;
  ans_status st = check_batch(jobs, n_jobs, &sms);
  if (st != ANS_OK) return st;
  ansdev::LayerDev Ls[ANS_MAX_BATCH];
  const ansdev::LayerDev* Lp[ANS_MAX_BATCH];
  const uint16_t* Xs[ANS_MAX_BATCH];
  const void* Ss[ANS_MAX_BATCH];
  float* Ys[ANS_MAX_BATCH];
  for (uint32_t j = 0; j < n_jobs; ++j) {
    const ans_tiles* W = jobs[j].W;
    st = check_gemm_tiles(W, scale_kind, jobs[j].d_scales, group_k);
    if (st != ANS_OK) return st;
    if (M > 0) {
      st = check_gemm_io(jobs[j].d_X, jobs[j].d_Y, d_status, jobs[j].d_scales);
      if (st != ANS_OK) return st;
    }
    fill_layer(W, &Ls[j]);
    Lp[j] = &Ls[j];
    Xs[j] = jobs[j].d_X;
    Ss[j] = jobs[j].d_scales;
    Ys[j] = jobs[j].d_Y;
  }
  if (M == 0) return ANS_OK;
  if (!d_ws || reinterpret_cast<uintptr_t>(d_ws) % 256 != 0) return ANS_ERR_ARG;
  ansdev::GemmPlan share[ANS_MAX_BATCH], full[ANS_MAX_BATCH];
  size_t ws_off[ANS_MAX_BATCH + 1];
  bool one = false;
  st = batch_plan(jobs, n_jobs, M, scale_kind, sms, share, full, ws_off, &one);
  if (st != ANS_OK) return st;
  if (ws_bytes < ws_off[n_jobs]) return ANS_ERR_BUFFER_TOO_SMALL;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (one) {
    cudaError_t e = ansdev::launch_gemm_batched(share, n_jobs, Lp, Xs, Ss, scale_kind, group_k, Ys,
                                                d_ws, ws_off, d_status, s);
    if (e != cudaSuccess) return cuda_fail(e, "ans_gemm_batched");
    return ANS_OK;
  }
  for (uint32_t j = 0; j < n_jobs; ++j) {
    cudaError_t e = ansdev::launch_gemm(full[j], Ls[j], true, nullptr, Xs[j], Ss[j], scale_kind,
                                        group_k, Ys[j], static_cast<uint8_t*>(d_ws) + ws_off[j],
                                        d_status, s);
    if (e != cudaSuccess) return cuda_fail(e, "ans_gemm_batched");
  }
  return ANS_OK;
}

ans_status ans_container_write(const ans_container* layer, uint8_t* h_out, uint64_t cap,
                               uint64_t* bytes) {
  if (!layer || !bytes) return ANS_ERR_ARG;
  ans_status st = check_container_fields(layer);
  if (st != ANS_OK) return st;
  const anshost::ContainerLayer h = to_host_layer(layer);
  const int r = anshost::container_check(h);
  if (r == 3) return ANS_ERR_ALPHABET;
  if (r != 0) return ANS_ERR_ARG;
  const int w = anshost::container_write(h, h_out, cap, bytes);
  if (w == 4) return ANS_ERR_BUFFER_TOO_SMALL;
  return w == 0 ? ANS_OK : ANS_ERR_ARG;
}

ans_status ans_container_read(const uint8_t* h_buf, uint64_t bytes, ans_container* layer) {
  if (!h_buf || !layer || reinterpret_cast<uintptr_t>(h_buf) % 16 != 0) return ANS_ERR_ARG;
  anshost::ContainerLayer h;
  const int r = anshost::container_read(h_buf, bytes, &h);
  if (r == 8) return ANS_ERR_UNSUPPORTED;
  if (r != 0) return ANS_ERR_CORRUPT;
  ans_container c;
  std::memset(&c, 0, sizeof(c));
  c.layout = ans_layout{h.dtype, h.N, h.K, h.tile_n, h.tile_k, h.state_bits};
  c.prob_bits = h.prob_bits;
  c.alphabet = h.alphabet;
  c.stream_bytes = h.stream_bytes;
  c.raw_bytes = h.raw_bytes;
  c.freq = h.freq;
  c.offsets = h.offsets;
  c.stream = h.stream;
  c.raw = h.raw;
  // a header that passed its checksum may still describe an impossible layer
  if ((h.state_bits != 32 && h.state_bits != 64) || check_container_fields(&c) != ANS_OK)
    return ANS_ERR_CORRUPT;
  if (to_host_layer(&c).n_tiles != h.n_tiles || anshost::container_check(h) != 0)
    return ANS_ERR_CORRUPT;
  if (c.alphabet <= 256) {
    c.codebook.alphabet = c.alphabet;
    c.codebook.prob_bits = c.prob_bits;
    uint32_t run = 0;
    for (uint32_t s = 0; s < c.alphabet; ++s) {
      c.codebook.freq[s] = static_cast<uint16_t>(c.freq[s]);
      c.codebook.cdf[s] = static_cast<uint16_t>(run);
      run += c.freq[s];
    }
    c.codebook.cdf[c.alphabet] = static_cast<uint16_t>(run);
  }
  *layer = c;
  return ANS_OK;
}

}  // extern "C"
