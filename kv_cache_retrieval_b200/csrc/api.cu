// C ABI of the HHR decode-time retrieval library (declared in include/hhr.h).
// Host-side argument checks, launch configuration and workspace carving.

#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "hhr.h"
#include "hhr_internal.cuh"

namespace {

using namespace hhr;

constexpr int32_t kVersion = 100;  // 0.1.0

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Structural checks shared by every call.
int32_t check_dims(const hhr_dims* d) {
  if (!d) return HHR_ERR_INVALID_ARG;
  if (d->B < 1 || d->Hq < 1 || d->Hkv < 1 || d->d < 1 || d->bits < 1 || d->page < 1 || d->n_cap < 1)
    return HHR_ERR_INVALID_ARG;
  if (d->Hq % d->Hkv != 0) return HHR_ERR_INVALID_ARG;
  if (d->flags & ~(HHR_FLAG_META_F32 | HHR_FLAG_GQA_SUM | HHR_FLAG_SIMT_BOUNDS)) return HHR_ERR_INVALID_ARG;
  const int r = d->Hq / d->Hkv;
  if (d->d != kD) return HHR_ERR_UNSUPPORTED;
  if (d->bits != 128 && d->bits != 256) return HHR_ERR_UNSUPPORTED;
  if (!is_pow2(d->page) || d->page > 64) return HHR_ERR_UNSUPPORTED;
  if (r != 1 && r != 2 && r != 4 && r != 8) return HHR_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(d->B) * d->Hkv * d->n_cap;
  if (rows * kD >= (1ll << 40)) return HHR_ERR_UNSUPPORTED;
  return HHR_OK;
}

int np_cap_of(const hhr_dims* d) { return (d->n_cap + d->page - 1) / d->page; }

int hbins_of(const hhr_dims* d) { return hist_bins(d->Hq / d->Hkv, d->bits, d->flags); }

struct DeviceInfo {
  int sms = 0;
  size_t smem_optin = 0;
};

// SM count and opt-in shared memory of the current device, queried once per
// device.
int32_t device_info(DeviceInfo* info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HHR_ERR_CUDA;
  static std::mutex mu;
  static DeviceInfo cache[kMaxDevices];
  static bool known[kMaxDevices];
  if (dev < kMaxDevices) {
    std::lock_guard<std::mutex> lock(mu);
    if (known[dev]) {
      *info = cache[dev];
      return HHR_OK;
    }
  }
  int v = 0;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return HHR_ERR_CUDA;
  info->sms = v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return HHR_ERR_CUDA;
  info->smem_optin = static_cast<size_t>(v);
  if (dev < kMaxDevices) {
    std::lock_guard<std::mutex> lock(mu);
    cache[dev] = *info;
    known[dev] = true;
  }
  return HHR_OK;
}

// Picks the CTAs per unit and fills the size fields of `a`.  Returns the
// dynamic shared-memory bytes through *smem.
int32_t plan_decode(const hhr_dims* d, int mode, int n_valid, int P, int k, DecodeArgs* a,
                    size_t* smem, bool dense = false) {
  DeviceInfo info;
  if (int32_t st = device_info(&info)) return st;
  const int r = d->Hq / d->Hkv;
  const int units = d->B * d->Hkv;
  const int hbins = hbins_of(d);
  const int NP = (n_valid + d->page - 1) / d->page;
  const int Pk = P < NP ? P : NP;
  // one CTA per SM (512 threads, up to 128 registers each)
  const int resident = info.sms;
  int C = resident / units;
  if (C < 1) C = 1;
  if (C > kMaxCtasPerUnit) C = kMaxCtasPerUnit;
  if (dense) {
    const int by_tokens = (n_valid + 255) / 256;  // at least 256 keys per CTA
    if (C > by_tokens) C = by_tokens < 1 ? 1 : by_tokens;
  } else if (mode == kModeAttend) {
    const int by_tokens = (k + 63) / 64;  // at least 64 tokens per CTA
    if (C > by_tokens) C = by_tokens < 1 ? 1 : by_tokens;
  } else {
    const int by_pages = (NP + kMinPagesPerCta - 1) / kMinPagesPerCta;
    if (C > by_pages) C = by_pages < 1 ? 1 : by_pages;
    // the unit's C distance histograms, their row prefixes and the totals
    // share the scratch area with the metadata ring (192 KiB): with the wide
    // GQA-sum histograms that caps C
    const int by_hist = static_cast<int>((size_t{192} * 1024 / sizeof(int) - hbins - 4) / (2 * hbins + 1));
    if (C > by_hist) C = by_hist < 1 ? 1 : by_hist;
  }
  int slice_pages = 0, slice_tokens = 0;
  for (;;) {
    if (dense) {
      slice_pages = 0;
      slice_tokens = 1;   // no token list
    } else if (mode == kModeAttend) {
      slice_pages = 0;
      slice_tokens = (k + C - 1) / C + 1;
    } else {
      slice_pages = (Pk + C - 1) / C;
      slice_tokens = slice_pages * d->page;
    }
    if (slice_tokens <= kMaxTokensPerCta || C >= kMaxCtasPerUnit || C * units >= resident) break;
    ++C;
  }
  if (slice_tokens > kMaxTokensPerCta) return HHR_ERR_UNSUPPORTED;
  const DecodeSmem lay = decode_smem(NP, C, d->bits, r, slice_pages, slice_tokens, mode, hbins);
  if (lay.total > info.smem_optin) return HHR_ERR_UNSUPPORTED;
  int grid_units = resident / C;
  if (grid_units > units) grid_units = units;
  if (grid_units < 1) grid_units = 1;

  a->B = d->B;
  a->Hq = d->Hq;
  a->Hkv = d->Hkv;
  a->units = units;
  a->page = d->page;
  a->n_cap = d->n_cap;
  a->np_cap = np_cap_of(d);
  a->n_valid = n_valid;
  a->NP = NP;
  a->P = P;
  a->Pk = Pk;
  a->k = k;
  a->C = C;
  a->grid_units = grid_units;
  a->slice_pages = slice_pages;
  a->slice_tokens = slice_tokens;
  a->spin_limit = kSpinLimit;
  a->meta_f32 = (d->flags & HHR_FLAG_META_F32) ? 1 : 0;
  a->gqa_sum = (d->flags & HHR_FLAG_GQA_SUM) ? 1 : 0;
  a->simt_bounds = (d->flags & HHR_FLAG_SIMT_BOUNDS) ? 1 : 0;
  a->hbins = hbins;
  a->dense = dense ? 1 : 0;
  *smem = lay.total;
  return HHR_OK;
}

void carve_workspace(void* ws, const hhr_dims* d, DecodeArgs* a) {
  const WsLayout L = ws_layout(d->B * d->Hkv, np_cap_of(d), d->Hq / d->Hkv, hbins_of(d));
  unsigned char* base = static_cast<unsigned char*>(ws);
  a->status = reinterpret_cast<uint32_t*>(base + L.status);
  a->counters = reinterpret_cast<uint32_t*>(base + L.counters);
  a->wsU = reinterpret_cast<float*>(base + L.U);
  a->wsMinMax = reinterpret_cast<float*>(base + L.minmax);
  a->wsHist = reinterpret_cast<int32_t*>(base + L.hist);
  a->wsPart = reinterpret_cast<float*>(base + L.part);
  a->np_stride = L.np_stride;
}

int32_t check_workspace(const hhr_dims* d, void* ws, size_t ws_bytes) {
  if (!ws) return HHR_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return HHR_ERR_WORKSPACE;
  const WsLayout L = ws_layout(d->B * d->Hkv, np_cap_of(d), d->Hq / d->Hkv, hbins_of(d));
  if (ws_bytes < L.total) return HHR_ERR_WORKSPACE;
  return HHR_OK;
}

int32_t finish_launch(cudaError_t e) { return e == cudaSuccess ? HHR_OK : HHR_ERR_CUDA; }

// One-shot test hook (hhr_test_arm_timeout): which wait the next matching
// call makes unmeetable, and the spin limit it gets.
std::atomic<int> g_test_where{0};
std::atomic<unsigned long long> g_test_spin{0};

// Consumes the hook when it is armed for one of the given sites.
int take_test_hook(int lo, int hi, unsigned long long* spin) {
  int w = g_test_where.load();
  if (w < lo || w > hi) return 0;
  if (!g_test_where.compare_exchange_strong(w, 0)) return 0;
  *spin = g_test_spin.load();
  return w;
}

}  // namespace


extern "C" {

int32_t hhr_version(void) { return kVersion; }

const char* hhr_status_string(int32_t status) {
  switch (status) {
    case HHR_OK: return "ok";
    case HHR_ERR_INVALID_ARG: return "invalid argument";
    case HHR_ERR_UNSUPPORTED: return "unsupported size";
    case HHR_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case HHR_ERR_CUDA: return "CUDA error";
    case HHR_ERR_TIMEOUT: return "bounded inter-CTA wait timed out";
    default: return "unknown status";
  }
}

int32_t hhr_encode_keys(const hhr_dims* dims, const void* K, const float* R, const float* W,
                        int32_t n_begin, int32_t n_end, uint32_t* codes, void* meta, void* stream) {
  if (int32_t st = check_dims(dims)) return st;
  if (!K || !R || !W || !codes || !meta) return HHR_ERR_INVALID_ARG;
  if (n_begin < 0 || n_end < n_begin || n_end > dims->n_cap) return HHR_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(R) || !aligned16(W) || !aligned16(codes) || !aligned16(meta))
    return HHR_ERR_INVALID_ARG;
  if (n_begin == n_end) return HHR_OK;
  EncodeArgs a;
  a.K = static_cast<const uint16_t*>(K);
  a.R = R;
  a.W = W;
  a.codes = codes;
  a.meta = meta;
  a.meta_f32 = (dims->flags & HHR_FLAG_META_F32) ? 1 : 0;
  a.Hkv = dims->Hkv;
  a.units = dims->B * dims->Hkv;
  a.bits = dims->bits;
  a.page = dims->page;
  a.n_cap = dims->n_cap;
  a.np_cap = np_cap_of(dims);
  a.n_begin = n_begin;
  a.n_end = n_end;
  a.spin_limit = kSpinLimit;
  a.test_extra_arrival = 0;
  {
    unsigned long long spin = 0;
    if (take_test_hook(3, 3, &spin)) {
      a.test_extra_arrival = 1;
      a.spin_limit = spin;
    }
  }
  a.tile_begin = n_begin / kEncodeTileKeys * kEncodeTileKeys;
  a.n_tiles = (n_end - a.tile_begin + kEncodeTileKeys - 1) / kEncodeTileKeys;
  DeviceInfo info;
  if (int32_t st = device_info(&info)) return st;
  if (encode_smem_bytes() > info.smem_optin) return HHR_ERR_UNSUPPORTED;
  if (static_cast<long long>(a.units / a.Hkv) * a.n_tiles > 0x7FFFFFFFLL) return HHR_ERR_UNSUPPORTED;
  return finish_launch(launch_encode(a, info.sms, static_cast<cudaStream_t>(stream)));
}

size_t hhr_workspace_size(const hhr_dims* dims, int32_t P, int32_t k) {
  if (check_dims(dims) != HHR_OK || P < 1 || k < 1) return 0;
  const WsLayout L = ws_layout(dims->B * dims->Hkv, np_cap_of(dims), dims->Hq / dims->Hkv, hbins_of(dims));
  return L.total;
}

static int32_t decode_common(const hhr_dims* dims, int mode, const void* q, const float* R,
                             const float* W, const uint32_t* codes, const void* meta, const void* K,
                             const void* V, const int32_t* tok_in, const int32_t* nsel_in,
                             int32_t n_valid, int32_t P, int32_t k, float scale, int32_t* page_idx,
                             int32_t* tok_idx, int32_t* n_sel, float* out, float* dbg_U,
                             int32_t* dbg_D, void* workspace, size_t ws_bytes, void* stream,
                             bool check_only = false, bool dense = false) {
  if (int32_t st = check_dims(dims)) return st;
  if (np_cap_of(dims) > HHR_MAX_PAGES) return HHR_ERR_UNSUPPORTED;
  if (k < 1 || !q) return HHR_ERR_INVALID_ARG;
  if (mode != kModeAttend) {
    if (P < 1 || n_valid < 0 || n_valid > dims->n_cap) return HHR_ERR_INVALID_ARG;
    if (!R || !W || !codes || !meta || !page_idx || !tok_idx || !n_sel) return HHR_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(meta)) return HHR_ERR_INVALID_ARG;
  }
  if (mode != kModeSelect) {
    if (!K || !V || !out) return HHR_ERR_INVALID_ARG;
    if (!aligned16(K) || !aligned16(V)) return HHR_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return HHR_ERR_INVALID_ARG;
  }
  if (mode == kModeAttend && !dense && (!tok_in || !nsel_in)) return HHR_ERR_INVALID_ARG;
  if (dense && (n_valid < 0 || n_valid > dims->n_cap)) return HHR_ERR_INVALID_ARG;
  if (int32_t st = check_workspace(dims, workspace, ws_bytes)) return st;

  DecodeArgs a;
  std::memset(&a, 0, sizeof a);
  size_t smem = 0;
  if (int32_t st = plan_decode(dims, mode, n_valid, P, k, &a, &smem, dense)) return st;
  if (check_only) return HHR_OK;
  a.q = static_cast<const uint16_t*>(q);
  a.R = R;
  a.W = W;
  a.codes = codes;
  a.meta = meta;
  a.K = static_cast<const uint16_t*>(K);
  a.V = static_cast<const uint16_t*>(V);
  a.tok_in = tok_in;
  a.nsel_in = nsel_in;
  a.page_idx = page_idx;
  a.tok_idx = tok_idx;
  a.n_sel = n_sel;
  a.out = out;
  a.dbg_U = dbg_U;
  a.dbg_D = dbg_D;
  a.scale_log2 = scale * 1.4426950408889634f;
  if (mode != kModeAttend) {
    unsigned long long spin = 0;
    if (const int w = take_test_hook(1, 2, &spin)) {
      a.test_extra_stage = w;
      a.spin_limit = spin;
    }
  }
  carve_workspace(workspace, dims, &a);
  return finish_launch(launch_decode(a, dims->Hq / dims->Hkv, dims->bits, mode, smem,
                                     static_cast<cudaStream_t>(stream)));
}

int32_t hhr_select(const hhr_dims* dims, const void* q, const float* R, const float* W,
                   const uint32_t* codes, const void* meta, int32_t n_valid, int32_t P, int32_t k,
                   int32_t* page_idx, int32_t* tok_idx, int32_t* n_sel, float* dbg_U,
                   int32_t* dbg_D, void* workspace, size_t ws_bytes, void* stream) {
  return decode_common(dims, kModeSelect, q, R, W, codes, meta, nullptr, nullptr, nullptr, nullptr,
                       n_valid, P, k, 1.0f, page_idx, tok_idx, n_sel, nullptr, dbg_U, dbg_D,
                       workspace, ws_bytes, stream);
}

int32_t hhr_sparse_attend(const hhr_dims* dims, const void* q, const void* K, const void* V,
                          const int32_t* tok_idx, const int32_t* n_sel, int32_t k, float scale,
                          float* out, void* workspace, size_t ws_bytes, void* stream) {
  return decode_common(dims, kModeAttend, q, nullptr, nullptr, nullptr, nullptr, K, V, tok_idx,
                       n_sel, dims ? dims->n_cap : 0, 1, k, scale, nullptr, nullptr, nullptr, out,
                       nullptr, nullptr, workspace, ws_bytes, stream);
}

int32_t hhr_dense_attend(const hhr_dims* dims, const void* q, const void* K, const void* V,
                         int32_t n_valid, float scale, float* out, void* workspace, size_t ws_bytes,
                         void* stream) {
  return decode_common(dims, kModeAttend, q, nullptr, nullptr, nullptr, nullptr, K, V, nullptr,
                       nullptr, n_valid, 1, 1, scale, nullptr, nullptr, nullptr, out, nullptr, nullptr,
                       workspace, ws_bytes, stream, false, true);
}

int32_t hhr_decode_step(const hhr_dims* dims, const void* q, const float* R, const float* W,
                        const uint32_t* codes, const void* meta, const void* K, const void* V,
                        int32_t n_valid, int32_t P, int32_t k, float scale, int32_t* page_idx,
                        int32_t* tok_idx, int32_t* n_sel, float* out, void* workspace,
                        size_t ws_bytes, void* stream) {
  return decode_common(dims, kModeFused, q, R, W, codes, meta, K, V, nullptr, nullptr, n_valid, P,
                       k, scale, page_idx, tok_idx, n_sel, out, nullptr, nullptr, workspace,
                       ws_bytes, stream);
}

}  // extern "C"

namespace hhr {
// Every check hhr_decode_step makes before it enqueues work, without
// enqueuing any (the allocation-free variant validates before it touches its
// shared scratch).
int32_t decode_step_check(const hhr_dims* dims, const void* q, const float* R, const float* W,
                          const uint32_t* codes, const void* meta, const void* K, const void* V,
                          int32_t n_valid, int32_t P, int32_t k, float scale, int32_t* page_idx,
                          int32_t* tok_idx, int32_t* n_sel, float* out, void* workspace,
                          size_t ws_bytes) {
  return decode_common(dims, kModeFused, q, R, W, codes, meta, K, V, nullptr, nullptr, n_valid, P,
                       k, scale, page_idx, tok_idx, n_sel, out, nullptr, nullptr, workspace,
                       ws_bytes, nullptr, true);
}
}  // namespace hhr

extern "C" {

int32_t hhr_decode_step_host(const hhr_dims* dims, const void* q_host, void* q, const float* R,
                             const float* W, const uint32_t* codes, const void* meta, const void* K,
                             const void* V, int32_t n_valid, int32_t P, int32_t k, float scale,
                             int32_t* page_idx, int32_t* tok_idx, int32_t* n_sel, float* out,
                             float* out_host, void* workspace, size_t ws_bytes, void* stream) {
  if (!q_host || !out_host) return HHR_ERR_INVALID_ARG;
  if (int32_t st = hhr::decode_step_check(dims, q, R, W, codes, meta, K, V, n_valid, P, k, scale,
                                          page_idx, tok_idx, n_sel, out, workspace, ws_bytes))
    return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t qn = static_cast<size_t>(dims->B) * dims->Hq * dims->d;
  if (cudaMemcpyAsync(q, q_host, qn * 2, cudaMemcpyHostToDevice, s) != cudaSuccess) return HHR_ERR_CUDA;
  if (int32_t st = hhr_decode_step(dims, q, R, W, codes, meta, K, V, n_valid, P, k, scale, page_idx,
                                   tok_idx, n_sel, out, workspace, ws_bytes, stream))
    return st;
  if (cudaMemcpyAsync(out_host, out, qn * 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return HHR_ERR_CUDA;
  return cudaStreamSynchronize(s) == cudaSuccess ? HHR_OK : HHR_ERR_CUDA;
}

int32_t hhr_encode_status(void* stream) {
  uint32_t host = 0;
  if (encode_read_status(&host, static_cast<cudaStream_t>(stream)) != cudaSuccess) return HHR_ERR_CUDA;
  return static_cast<int32_t>(host);
}

int32_t hhr_read_status(void* workspace, void* stream) {
  if (!workspace) return HHR_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t host = 0;
  if (cudaMemcpyAsync(&host, workspace, sizeof host, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return HHR_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return HHR_ERR_CUDA;
  if (host != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof host, s) != cudaSuccess) return HHR_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return HHR_ERR_CUDA;
  }
  return static_cast<int32_t>(host);
}

int32_t hhr_test_arm_timeout(int32_t where, uint64_t spin_cycles) {
  if (where < 1 || where > 3) return HHR_ERR_INVALID_ARG;
  if (spin_cycles < 1000) spin_cycles = 1000;
  if (spin_cycles > (1ull << 32)) spin_cycles = 1ull << 32;
  g_test_spin.store(spin_cycles);
  g_test_where.store(where);
  return HHR_OK;
}

}  // extern "C"
