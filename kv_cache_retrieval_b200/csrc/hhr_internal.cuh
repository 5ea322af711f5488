// Internal declarations shared by the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cstddef>
#include <atomic>
#include <cstdint>

#include <cuda_runtime.h>

#include "hhr.h"

namespace hhr {

constexpr int kD = 128;                  // head dimension handled by every kernel
constexpr int kDecodeThreads = 512;      // one decode CTA per SM, 16 warps
constexpr int kMaxCtasPerUnit = 64;      // CTAs that may share one (sequence, KV head)
constexpr int kMinPagesPerCta = 32;      // below this a unit uses fewer CTAs
constexpr int kPageBytes = 2 * kD * 2;   // one page's bf16 [lower; upper] rows
constexpr int kChunkPages = 32;          // pages per bulk copy of the metadata ring
constexpr int kChunkBytes = kChunkPages * kPageBytes;  // 16 KiB
constexpr int kSlots = 8;                // metadata ring slots (128 KiB)
constexpr int kRingBytes = kSlots * kChunkBytes;
constexpr int kRWBytes = kD * kD * 4;    // R, or 128 columns of W, in float32
constexpr int kSample = 64;              // pages every CTA of a unit scores to fix common bins
constexpr int kLocalMaxPages = 256;      // at most this many pages: every CTA scores all of them
constexpr int kMaxSlicePages = 2560;     // pages one CTA scores
constexpr int kMaxTokensPerCta = 8192;   // candidate tokens one CTA ranks
constexpr int kWinMax = 512;             // list entries read around the expected cutoff, per side
constexpr unsigned long long kSpinLimit = 1ull << 31;  // ~1 s at 2 GHz

inline __host__ __device__ size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Floats of one CTA's partial softmax state (r heads x (d outputs, max, sum)),
// padded to a multiple of four so it can be moved with 16-B accesses.
inline __host__ __device__ constexpr int part_stride(int r) { return (r * (kD + 2) + 3) / 4 * 4; }

// Entries of the cumulative bin counts one CTA publishes for the page
// selection (kSample + 1 bins -> kSample + 2 prefix values), padded.
constexpr int kCumStride = (kSample + 2 + 3) / 4 * 4;

// Workspace layout (bytes).  The status word sits at offset 0, the per-unit
// barrier counters right after it.
struct WsLayout {
  size_t status, counters, cum, list, cumD, part, total;
  int list_stride;   // list entries (8 B) per unit
  int cumD_stride;   // int32 per (unit, CTA) in the distance area
};

inline __host__ __device__ WsLayout ws_layout(int units, int np_cap, int r, int bits) {
  WsLayout L;
  size_t off = 0;
  L.status = off;   off += 256;
  L.counters = off; off += align_up(sizeof(uint32_t) * (size_t)units, 256);
  L.cum = off;      off += align_up(sizeof(int32_t) * (size_t)units * kMaxCtasPerUnit * kCumStride, 256);
  // every CTA's list lives in [2 c s, 2 (c + 1) s) with s = ceil(NP / C) rounded up to even,
  // so 2 C s <= 2 (np_cap + 2 C)
  L.list_stride = (int)align_up(2 * ((size_t)np_cap + 2 * kMaxCtasPerUnit), 4);
  L.list = off;     off += align_up(8 * (size_t)units * L.list_stride, 256);
  L.cumD_stride = (int)align_up((size_t)bits + 2, 4);
  L.cumD = off;     off += align_up(sizeof(int32_t) * (size_t)units * kMaxCtasPerUnit * L.cumD_stride, 256);
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
  const uint16_t* meta;     // bf16 [B][Hkv][np_cap][2][d]
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
  int32_t* wsCum;           // [units][kMaxCtasPerUnit][kCumStride]
  int2* wsList;             // [units][list_stride] (float bits of U, page)
  int32_t* wsCumD;          // [units][kMaxCtasPerUnit][cumD_stride]
  float* wsPart;            // [units][kMaxCtasPerUnit][part_stride]
  int list_stride, cumD_stride;
  // sizes
  int B, Hq, Hkv, units, page, n_cap, np_cap, n_valid, NP, P, Pk, k, C, grid_units;
  int slice_pages;          // max pages one CTA scores (ceil(NP / C)), 0 in attend mode
  int slice_tokens;         // max tokens one CTA ranks or attends
  int local;                // 1: every CTA holds every bound (no page exchange)
  int n_sample;             // pages of the common sample (NP in local mode when C > 1)
  int b_exp;                // bin where the page cutoff is expected
  int win;                  // list entries read on each side of the expected cutoff (even)
  int list_half;            // half of each CTA's list area (slice_pages rounded up to even)
  float scale_log2;         // scale * log2(e)
  unsigned long long spin_limit;
  int test_extra_stage;     // test hook: unit barrier (1..3) that waits for one extra arrival, 0 = none
};

struct EncodeArgs {
  const uint16_t* K;
  const float* R;
  const float* W;
  uint32_t* codes;
  uint16_t* meta;
  int Hkv, units, bits, page, n_cap, np_cap, n_begin, n_end, tile_begin, n_tiles;
  unsigned long long spin_limit;
  int test_short_tx;        // test hook: expect 16 more bytes than a key tile delivers
};

// Shared-memory carve-up of a decode CTA (host and device agree on it).
struct DecodeSmem {
  size_t ring, rw, sS, sE, sU, sBin, qt, qraw, qc, total;
};

inline __host__ __device__ DecodeSmem decode_smem(int r, int bits, int slice_pages, int mode) {
  DecodeSmem s;
  size_t off = 0;
  s.ring = off;  off += kRingBytes;                 // metadata ring; later K/V tiles, lists, merges
  s.rw = off;    off += kRWBytes;                   // R, then W; later the selected tokens
  if (mode == kModeAttend) {
    s.sS = s.sE = s.sU = s.sBin = s.qt = s.qraw = s.qc = off;
    s.total = off;
    return s;
  }
  s.sS = off;    off += sizeof(float) * kLocalMaxPages;            // sample bounds (all, in local mode)
  s.sE = off;    off += sizeof(float) * kLocalMaxPages;            // sorted sample (bin edges)
  s.sU = off;    off += align_up(sizeof(float) * (size_t)slice_pages, 16);   // own bounds
  s.sBin = off;  off += align_up((size_t)slice_pages, 16);                  // own bins (u8)
  s.qt = off;    off += align_up(sizeof(float) * (size_t)r * kD, 16);      // q~ (float32)
  s.qraw = off;  off += align_up(sizeof(float) * (size_t)r * kD, 16);      // q (float32)
  s.qc = off;    off += align_up(sizeof(uint32_t) * (size_t)r * (bits / 32), 16);
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

// Launchers (defined in decode.cu / encode.cu).  Return a cudaError_t.
cudaError_t launch_decode(const DecodeArgs& a, int r, int bits, int mode, size_t smem_bytes,
                          cudaStream_t stream);
cudaError_t launch_encode(const EncodeArgs& a, int sms, cudaStream_t stream);
size_t encode_smem_bytes();
// Copies the encode kernels' sticky error word to *out and clears it (synchronizes `stream`).
cudaError_t encode_read_status(uint32_t* out, cudaStream_t stream);
constexpr int kEncodeTileKeys = 128;   // keys per encode tile (tile starts are multiples of it)
cudaError_t launch_wait_timeout(uint32_t* status, uint32_t* counter, unsigned long long spin,
                                cudaStream_t stream);

}  // namespace hhr
