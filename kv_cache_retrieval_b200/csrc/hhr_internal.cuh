// Internal declarations shared by the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cstddef>
#include <atomic>
#include <cstdint>

#include <cuda_runtime.h>

#include "hhr.h"

namespace hhr {

constexpr int kD = 128;                 // head dimension handled by every kernel
constexpr int kDecodeThreads = 512;     // one decode CTA per SM, 16 warps
constexpr int kMaxCtasPerUnit = 64;     // CTAs that may share one (sequence, KV head)
constexpr int kMinPagesPerCta = 32;     // below this a unit uses fewer CTAs
constexpr int kBuckets = 2048;          // page top-P histogram bins
constexpr int kCandMax = 1024;          // boundary-bucket candidates held in shared memory
constexpr int kRankDirect = 48;         // at most this many are ranked without a second level
constexpr int kMaxTokensPerCta = 16384; // candidate tokens one CTA scores
constexpr int kLaneSlots = 16;         // ring slots per warp below the R / W buffer (8 KiB)
constexpr int kRingSlots = 24;         // ring slots per warp in all (12 KiB), the upper 8 over R / W
constexpr unsigned long long kSpinLimit = 1ull << 31;  // ~1 s at 2 GHz

inline __host__ __device__ size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Floats of one CTA's partial softmax state (r heads x (d outputs, max, sum)),
// padded to a multiple of four so it can be moved with 16-B accesses.
inline __host__ __device__ constexpr int part_stride(int r) { return (r * (kD + 2) + 3) / 4 * 4; }

// Bins of a token-distance histogram: distances 0 .. bits (min over the
// group's heads) or 0 .. r * bits (HHR_FLAG_GQA_SUM).
inline __host__ __device__ int hist_bins(int r, int bits, int flags) {
  return ((flags & HHR_FLAG_GQA_SUM) ? r * bits : bits) + 1;
}

// Workspace layout (bytes).  The status word sits at offset 0.
struct WsLayout {
  size_t status, counters, U, minmax, hist, part, total;
  int np_stride;  // floats per unit in the U area (multiple of 4)
};

inline __host__ __device__ WsLayout ws_layout(int units, int np_cap, int r, int hbins) {
  WsLayout L;
  size_t off = 0;
  L.status = off;   off += 256;
  L.counters = off; off += align_up(sizeof(uint32_t) * (size_t)units, 256);
  L.np_stride = (int)align_up((size_t)np_cap, 4);
  L.U = off;        off += align_up(sizeof(float) * (size_t)units * L.np_stride, 256);
  L.minmax = off;   off += align_up(sizeof(float) * 2 * (size_t)units * kMaxCtasPerUnit, 256);
  L.hist = off;     off += align_up(sizeof(int32_t) * (size_t)units * kMaxCtasPerUnit * hbins, 256);
  L.part = off;     off += align_up(sizeof(float) * (size_t)units * kMaxCtasPerUnit * part_stride(r), 256);
  L.total = off;
  return L;
}

enum DecodeMode : int { kModeSelect = 0, kModeFused = 1, kModeAttend = 2 };

struct DecodeArgs {
  // inputs
  const uint16_t* q;        // bf16 [B][Hq][d]
  const float* R;           // [Hkv][d][d]
  const float* W;           // [Hkv][d][bits]
  const uint32_t* codes;    // [B][Hkv][n_cap][w]
  const void* meta;         // bf16 (f32 if meta_f32) [B][Hkv][np_cap][2][d]
  const uint16_t* K;        // bf16 [B][Hkv][n_cap][d]
  const uint16_t* V;
  const int32_t* tok_in;    // attend-only: [B][Hkv][k]
  const int32_t* nsel_in;   // attend-only: [B][Hkv]
  // outputs
  int32_t* page_idx;        // [B][Hkv][P]
  int32_t* tok_idx;         // [B][Hkv][k]
  int32_t* n_sel;           // [B][Hkv]
  float* out;               // [B][Hq][d]
  float* dbg_U;             // nullable [B][Hkv][NP]
  int32_t* dbg_D;           // nullable [B][Hkv][P*page]
  // workspace
  uint32_t* status;
  uint32_t* counters;
  float* wsU;
  float* wsMinMax;
  int32_t* wsHist;
  float* wsPart;
  int np_stride;
  // sizes
  int B, Hq, Hkv, units, page, n_cap, np_cap, n_valid, NP, P, Pk, k, C, grid_units;
  int slice_pages;          // max kept pages one CTA scores (ceil(Pk / C))
  int slice_tokens;         // max tokens one CTA scores or attends
  float scale_log2;         // scale * log2(e)
  unsigned long long spin_limit;
  int test_extra_stage;     // test hook: unit barrier (1 or 2) that waits for one arrival too many; 0 = none
  int meta_f32;             // HHR_FLAG_META_F32: f32 metadata, bounds by SIMT
  int gqa_sum;              // HHR_FLAG_GQA_SUM: distance = sum over the group's heads
  int hbins;                // distance histogram bins (hist_bins)
  int dense;                // attend mode over all n_valid keys, no token list (hhr_dense_attend)
  int simt_bounds;          // HHR_FLAG_SIMT_BOUNDS: Eq. 3 on the CUDA cores (bf16 metadata)
};

struct EncodeArgs {
  const uint16_t* K;
  const float* R;
  const float* W;
  uint32_t* codes;
  void* meta;                      // bf16, or f32 when meta_f32
  int Hkv, units, bits, page, n_cap, np_cap, n_begin, n_end, tile_begin, n_tiles;
  int meta_f32;                    // HHR_FLAG_META_F32: unrounded f32 extrema
  unsigned long long spin_limit;   // clock cycles a pipeline wait may take
  int test_extra_arrival;          // test hook: the first stage waits for one producer arrival too many
};

// Shared-memory bytes of a decode CTA (host and device agree on the carve-up).
struct DecodeSmem {
  size_t qb, qf, qt, qc, my_pages, tokD, sel, scratch, total;
};

inline __host__ __device__ size_t decode_scratch_bytes(int NP, int C, int r, int mode, int hbins) {
  size_t sel = 0, hist = 0, attn = 0, stream = 0;
  if (mode != kModeAttend) {
    // per-warp metadata rings; their upper slots double as R / W staging
    stream = (size_t)(kDecodeThreads / 32) * kRingSlots * 512;
    sel = sizeof(float) * align_up((size_t)NP, 4)          // U of every page
        + sizeof(int) * kBuckets                             // histogram
        + sizeof(uint32_t) * align_up(((size_t)NP + 31) / 32, 4)  // kept bitmap
        + 2 * (sizeof(float) + sizeof(int)) * kCandMax       // boundary candidates, 2 levels
        + sizeof(float) * 2 * (kDecodeThreads / 32);          // level-2 min / max
    // distance histograms, their row prefixes, the unit totals (+ copy rounding)
    hist = sizeof(int) * ((size_t)C * hbins + (size_t)C * (hbins + 1) + hbins) + 16;
  }
  if (mode != kModeSelect) {
    // per warp: K and V of 16 tokens; then the 16-row query tile
    const size_t ring = (size_t)(kDecodeThreads / 32) * 2 * 16 * 2 * kD + 16 * 2 * kD;
    const size_t merge = sizeof(float) * (kDecodeThreads / 32) * (size_t)r * (kD + 2);  // the warps' states
    attn = ring > merge ? ring : merge;
  }
  size_t m = sel > hist ? sel : hist;
  m = m > stream ? m : stream;
  return m > attn ? m : attn;
}

inline __host__ __device__ DecodeSmem decode_smem(int NP, int C, int bits, int r, int slice_pages,
                                                  int slice_tokens, int mode, int hbins) {
  DecodeSmem s;
  size_t off = 0;
  s.qb = off;       off += (size_t)8 * ((r * 4 + 7) / 8) * 2 * kD * 2;  // bf16 terms of q~, [8 nb][2 d]
  s.qf = off;       off += align_up(sizeof(float) * r * kD, 16);
  s.qt = off;       off += align_up(sizeof(float) * r * kD, 16);          // q~ (f32-metadata bounds)
  s.qc = off;       off += align_up(sizeof(uint32_t) * r * (bits / 32), 16);
  s.my_pages = off; off += align_up(sizeof(int) * (size_t)(slice_pages + 1), 16);
  s.tokD = off;     off += align_up(sizeof(uint16_t) * (size_t)(slice_tokens + 1), 16);
  s.sel = off;      off += align_up(sizeof(int) * (size_t)(slice_tokens + 1), 16);
  s.scratch = off;  off += align_up(decode_scratch_bytes(NP, C, r, mode, hbins), 16);
  s.total = off;
  return s;
}

// Raises a kernel's dynamic shared-memory limit to at least `bytes` on the
// current device, calling cudaFuncSetAttribute only when the limit grows
// (one record per kernel and device: `raised` must be a zero-initialised
// static array of kMaxDevices entries).
constexpr int kMaxDevices = 64;
inline cudaError_t ensure_smem_limit(const void* kernel, size_t bytes, std::atomic<size_t>* raised) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < kMaxDevices && raised[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess && dev < kMaxDevices) {
    size_t cur = raised[dev].load(std::memory_order_relaxed);
    while (cur < bytes && !raised[dev].compare_exchange_weak(cur, bytes, std::memory_order_release)) {
    }
  }
  return e;
}

// hhr_decode_step's argument and size checks without launching (api.cu).
int32_t decode_step_check(const hhr_dims* dims, const void* q, const float* R, const float* W,
                          const uint32_t* codes, const void* meta, const void* K, const void* V,
                          int32_t n_valid, int32_t P, int32_t k, float scale, int32_t* page_idx,
                          int32_t* tok_idx, int32_t* n_sel, float* out, void* workspace,
                          size_t ws_bytes);

// Launchers (defined in decode.cu / encode.cu).  Return a cudaError_t.
cudaError_t launch_decode(const DecodeArgs& a, int r, int bits, int mode, size_t smem_bytes,
                          cudaStream_t stream);
cudaError_t launch_encode(const EncodeArgs& a, int sms, cudaStream_t stream);
size_t encode_smem_bytes();
// Copies the encode kernels' sticky error word to *out and clears it (synchronizes `stream`).
cudaError_t encode_read_status(uint32_t* out, cudaStream_t stream);
constexpr int kEncodeTileKeys = 128;   // keys per encode tile (tile starts are multiples of it)

}  // namespace hhr
