// Decode-time retrieval kernels for sm_100a.
//
// One (sequence, KV head) pair -- a "unit" -- is spread over C CTAs of a
// cooperative launch; CTA c owns the contiguous page range [c NP / C,
// (c + 1) NP / C).  A fused step runs these phases per unit:
//
//   0  query prep      R arrives by one bulk copy while the metadata ring
//                      fills; q~ = q R (Eq. 4) for the r query heads
//   1  page bounds     U_p = max_h sum_j max(q~_hj l_pj, q~_hj u_pj) (Eq. 3)
//                      for a common sample of the unit's pages and for the
//                      CTA's own pages.  The metadata streams through a ring
//                      of 16-KiB bulk copies (the warp that frees a slot
//                      refills it); warps score 8-page tasks with packed
//                      float32 FMAs and a butterfly reduction
//   2  publish         every CTA sorts the sample (identically), bins its own
//                      bounds by the sample values, publishes its cumulative
//                      bin counts and its bounds ordered by bin, and arrives
//                      at unit barrier 1; then forms the query codes (Eq. 10,
//                      sign) from W
//      -- unit barrier 1 --
//   3  page top-P      one read of every CTA's counts and of the stretch of
//                      its list around the expected cutoff bin gives the
//                      boundary bin, and an exact ranking of that bin's
//                      entries gives the cutoff (bound, page): a page is kept
//                      iff (U, -page) is not below it, ties to the lower page
//   4  Hamming         D_n = min_h popc(qcode_h xor code_n) (Eq. 2) for the
//                      tokens of the CTA's own kept pages; the cumulative
//                      histogram of D is published
//      -- unit barrier 2 --
//   5  token top-k     the histograms of all CTAs give the threshold distance,
//                      each CTA's quota of threshold ties (lower tokens first)
//                      and its output offset
//   6  attention       softmax(scale q.k) v over the CTA's selected tokens:
//                      K/V rows by bulk copy into per-warp double buffers,
//                      float32 dot products and online softmax
//      -- the last-arriving CTA merges the C partial softmax states --
//
// Units with at most kLocalMaxPages pages, or with a single CTA, skip the
// exchange of phase 3: every CTA scores every page.
//
// The kernel is launched as a programmatic dependent of the previous kernel
// on the stream and waits for it before touching memory.  Inter-CTA waits
// spin on workspace counters with a clock64() limit; on expiry the kernel
// records HHR_ERR_TIMEOUT and returns.  The last CTA of a unit resets its
// counter, so the workspace is zero again after each call.

#include <cuda_bf16.h>

#include <cfloat>
#include <climits>
#include <cstdint>

#include "hhr_internal.cuh"

namespace hhr {
namespace {

constexpr int NT = kDecodeThreads;
constexpr int NWARPS = NT / 32;
constexpr unsigned FULL = 0xFFFFFFFFu;
constexpr int kTaskPages = 8;                              // pages one warp scores per task
constexpr int kTasksPerChunk = kChunkPages / kTaskPages;   // 4
static_assert(NT == 4 * kD, "query products use four row quarters of 128 columns");
static_assert(kSlots * kChunkBytes == kRingBytes, "ring size");
static_assert(NWARPS * 8192 <= kRingBytes, "per-warp K/V double buffers live in the ring");

// ------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// CTA-scope acquire-release add on a shared-memory word.
__device__ __forceinline__ uint32_t smem_atom_add_acq_rel(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;"
               : "=r"(old) : "r"(smem_addr(p)), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes) : "memory");
}

// 1-D bulk copy global -> shared on the TMA unit; completion is signalled on
// the mbarrier as transferred bytes.  Both addresses 16-B aligned, size a
// multiple of 16.  This GPU's memory only; no multicast.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }

// The same copy with an L2 cache policy (createpolicy): evict-last for the
// small tensors every step re-reads (R, W).
__device__ __forceinline__ void bulk_g2s_hint(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                              uint64_t policy) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
               :: "r"(dst), "l"(src), "r"(bytes), "r"(bar), "l"(policy) : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Copies `rows` rows of `chunks` 16-B chunks from global (row stride
// src_stride bytes, read at L2) to shared memory (row stride dst_stride
// bytes) with cp.async; warp w takes rows w, w + 16, ...  Chunks whose index
// is outside [c_lo, c_hi) are skipped.  Commits one group; the caller waits
// (cp_async_wait<0>) and synchronises.
__device__ __forceinline__ void copy_rows_async(uint32_t dst, const char* src, int rows, int chunks,
                                                size_t src_stride, uint32_t dst_stride, int c_lo, int c_hi) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int r = warp; r < rows; r += NT / 32)
    for (int ch = lane; ch < chunks; ch += 32)
      if (ch >= c_lo && ch < c_hi)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                     :: "r"(dst + r * dst_stride + ch * 16), "l"(src + r * src_stride + ch * 16) : "memory");
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// Brings the 128-B line holding `p` into L2 (no register result).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" :: "l"(p));
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
               " selp.u32 %0, 1, 0, p;\n}" : "=r"(done) : "r"(bar), "r"(parity) : "memory");
  return done != 0;
}

// Waits for the mbarrier phase with the given parity; gives up (false) after
// `limit` clock cycles.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned long long limit) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  do {
    if (mbar_try(bar, parity)) return true;
  } while (static_cast<unsigned long long>(clock64() - t0) <= limit);
  return false;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// The two bf16 halves of a word, widened exactly to float32.
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ------------------------------------------------------- block primitives

// Exclusive prefix sum over the CTA.  Every thread must call it.
__device__ int block_excl_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(FULL, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int w = lane < NWARPS ? s_warp[lane] : 0;
    int wx = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(FULL, wx, o);
      if (lane >= o) wx += y;
    }
    if (lane < NWARPS) s_warp[lane] = wx - w;
    if (lane == NWARPS - 1) s_warp[NWARPS] = wx;
  }
  __syncthreads();
  const int res = s_warp[warp] + x - v;
  *total = s_warp[NWARPS];
  __syncthreads();
  return res;
}

// Exclusive prefix sum over the CTA with a single CTA barrier.  s_warp
// (NWARPS ints) must not be reused before the next CTA barrier.  Every
// thread must call it.
__device__ __forceinline__ int block_excl_scan1(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(FULL, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  int pre = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < NWARPS; ++w) {
    const int t = s_warp[w];
    pre += w < warp ? t : 0;
    tot += t;
  }
  *total = tot;
  return pre + x - v;
}

__device__ int block_sum(int v, int* s_warp) {
  int total;
  block_excl_scan(v, s_warp, &total);
  return total;
}

// Order-preserving map of a float to uint32 (-0 and +0 map together).
__device__ __forceinline__ uint32_t order_key(float u) {
  const uint32_t x = __float_as_uint(u + 0.0f);
  return (x & 0x80000000u) ? ~x : (x | 0x80000000u);
}

// ------------------------------------------------- page cutoff (top-P)
//
// The kept pages are the Pk largest in the order (bound descending, page
// ascending).  The cutoff is the Pk-th element of that order: a page is kept
// iff (key, page) is not below it, i.e. key > pk.key, or key == pk.key and
// page <= pk.page.
struct Pivot {
  uint32_t key;
  int page;
  int all;  // every candidate is kept
};

__device__ __forceinline__ bool kept(uint32_t key, int page, const Pivot& pv) {
  return pv.all || key > pv.key || (key == pv.key && page <= pv.page);
}

// The need-th element by exact bitwise search: the need-th largest key, then
// the page among that key's entries.  For very many equal-looking bounds;
// kept out of line.
__device__ __noinline__ Pivot select_pivot_bitwise(const float* vals, const int* ids, int id0, int M,
                                                  int need, int* s_scan) {
  const int tid = threadIdx.x;
  auto id_of = [&](int i) { return ids ? ids[i] : id0 + i; };
  uint32_t T = 0u;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    int cnt = 0;
    for (int i = tid; i < M; i += NT) cnt += order_key(vals[i]) >= cand;
    if (block_sum(cnt, s_scan) >= need) T = cand;
  }
  int gt = 0;
  for (int i = tid; i < M; i += NT) gt += order_key(vals[i]) > T;
  const int r = need - block_sum(gt, s_scan);   // >= 1
  int X = 0;                                   // the r-th smallest page with key T
  for (int bit = 14; bit >= 0; --bit) {
    const int cand = X | (1 << bit);
    int cnt = 0;
    for (int i = tid; i < M; i += NT) cnt += (order_key(vals[i]) == T) && (id_of(i) < cand);
    if (block_sum(cnt, s_scan) < r) X = cand;
  }
  Pivot pv;
  pv.all = 0;
  pv.key = T;
  pv.page = X;
  return pv;
}

// (bound order key, page) as one 64-bit value whose unsigned order is the
// selection order: larger bound first, then lower page.
__device__ __forceinline__ unsigned long long lex_key(uint32_t key, int page) {
  return (static_cast<unsigned long long>(key) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(page));
}

// The entry of rank nd - 1 (0-based, largest first) among n <= kRankMax
// distinct lexicographic keys lk[0..n): its key is counted against the
// others by NT / n_pow2 threads over slices and summed in shared memory
// (n <= 32: one warp, no block barrier before the result).  The winner is
// written to *win; every thread calls it and sees *win afterwards.
constexpr int kRankMax = 512;
__device__ void rank_lex(const unsigned long long* lk, int n, int nd, int* rk, unsigned long long* win) {
  const int tid = threadIdx.x;
  if (n <= 32) {
    if (tid < 32) {
      const unsigned long long ki = tid < n ? lk[tid] : 0ull;
      int r = 0;
      for (int j = 0; j < n; ++j) r += lk[j] > ki;
      if (tid < n && r == nd - 1) *win = ki;
    }
    __syncthreads();
    return;
  }
  int np2 = 64;
  while (np2 < n) np2 <<= 1;               // <= kRankMax
  const int parts = NT / np2;              // threads per entry
  if (tid < np2) rk[tid] = 0;
  __syncthreads();
  {
    const int i = tid % np2, part = tid / np2;
    if (i < n) {
      const unsigned long long ki = lk[i];
      const int j0 = part * n / parts, j1 = (part + 1) * n / parts;
      int r0 = 0, r1 = 0, r2 = 0, r3 = 0;
      int j = j0;
      for (; j + 3 < j1; j += 4) {
        r0 += lk[j] > ki;
        r1 += lk[j + 1] > ki;
        r2 += lk[j + 2] > ki;
        r3 += lk[j + 3] > ki;
      }
      for (; j < j1; ++j) r0 += lk[j] > ki;
      atomicAdd(&rk[i], (r0 + r1) + (r2 + r3));
    }
  }
  __syncthreads();
  if (tid < n && rk[tid] == nd - 1) *win = lk[tid];
  __syncthreads();
}

constexpr int kSubBins = 64;   // linear bins over a candidate set's value range

// The need-th element (1 <= need <= M) of entries i < M in the order (bound
// descending, page ascending); the bound of entry i is vals[i], its page
// ids[i] (or id0 + i when ids is null).  Pages are distinct and below 2^15.
// Up to kRankMax entries are ranked directly.  Larger sets are first cut
// down by linear bins over [min, max] of the bounds to the bin holding the
// need-th element (a bitwise search over all entries when very many bounds
// fall into one bin, e.g. equal bounds).  `scratch` holds at least
// kSubBins + 3 kRankMax ints.  Every thread must call it; every thread gets
// the same result.
__device__ Pivot select_pivot(const float* vals, const int* ids, int id0, int M, int need,
                              int* scratch, int* s_scan, int* s_misc, float* s_flt) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  auto id_of = [&](int i) { return ids ? ids[i] : id0 + i; };
  int* hist = scratch;                                                                 // [kSubBins]
  unsigned long long* lk = reinterpret_cast<unsigned long long*>(scratch + kSubBins);  // [kRankMax]
  int* rk = scratch + kSubBins + 2 * kRankMax;                                         // [kRankMax]
  __shared__ unsigned long long s_win;
  Pivot pv;
  pv.all = 0;
  if (M <= kRankMax) {
    for (int i = tid; i < M; i += NT) lk[i] = lex_key(order_key(vals[i]), id_of(i));
    __syncthreads();
    rank_lex(lk, M, need, rk, &s_win);
    pv.key = static_cast<uint32_t>(s_win >> 32);
    pv.page = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(s_win));
    __syncthreads();
    return pv;
  }
  float mn = INFINITY, mx = -INFINITY;
  for (int i = tid; i < M; i += NT) {
    mn = fminf(mn, vals[i]);
    mx = fmaxf(mx, vals[i]);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(FULL, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
  }
  if (lane == 0) {
    s_flt[2 * warp] = mn;
    s_flt[2 * warp + 1] = mx;
  }
  if (tid < kSubBins) hist[tid] = 0;
  if (tid == 0) s_misc[4] = 0;
  __syncthreads();
  mn = INFINITY;
  mx = -INFINITY;
#pragma unroll
  for (int w = 0; w < NWARPS; ++w) {
    mn = fminf(mn, s_flt[2 * w]);
    mx = fmaxf(mx, s_flt[2 * w + 1]);
  }
  const float range = mx - mn;
  const float inv = (range > 0.f && range <= FLT_MAX) ? static_cast<float>(kSubBins) / range : 0.f;
  // bin = round((u - mn) * inv) by one FMA (the 1.5 * 2^23 offset leaves the
  // rounded integer in the low mantissa bits); monotone in u, clamped.
  auto bucket = [&](float u) {
    const int bk = __float_as_int(fmaf(u - mn, inv, 12582912.f)) - 0x4B400000;
    return min(max(bk, 0), kSubBins - 1);
  };
  for (int i = tid; i < M; i += NT) atomicAdd(&hist[bucket(vals[i])], 1);
  __syncthreads();
  if (warp == 0) {   // from the top bin down: the bin holding the need-th element
    const int b0 = kSubBins - 1 - 2 * lane, b1 = b0 - 1;   // lane owns two bins, higher first
    const int h0 = hist[b0], h1 = hist[b1];
    int x = h0 + h1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(FULL, x, o);
      if (lane >= o) x += y;
    }
    const int before = x - h0 - h1;   // entries in higher bins than b0
    if (before < need && before + h0 >= need) {
      s_misc[2] = b0;
      s_misc[3] = before;
    } else if (before + h0 < need && before + h0 + h1 >= need) {
      s_misc[2] = b1;
      s_misc[3] = before + h0;
    }
  }
  __syncthreads();
  const int b2 = s_misc[2];
  const int need2 = need - s_misc[3];
  const int n2 = hist[b2];
  if (n2 <= kRankMax) {
    for (int i = tid; i < M; i += NT) {
      if (bucket(vals[i]) == b2) {
        const int slot = atomicAdd(&s_misc[4], 1);
        lk[slot] = lex_key(order_key(vals[i]), id_of(i));
      }
    }
    __syncthreads();
    rank_lex(lk, n2, need2, rk, &s_win);
    pv.key = static_cast<uint32_t>(s_win >> 32);
    pv.page = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(s_win));
    __syncthreads();
    return pv;
  }
  return select_pivot_bitwise(vals, ids, id0, M, need, s_scan);
}

// ------------------------------------------------------------ query prep

// x[r][d] . M[d][d] (both float32 in shared memory), in eight row groups:
// thread t forms, for every head h, the partial sums over rows
// [16 (t / 64), 16 (t / 64) + 16) of columns 2 (t % 64) and 2 (t % 64) + 1
// (packed FMAs).  M is read once per CTA, conflict-free; x by broadcast.
template <int RG>
__device__ __forceinline__ void product_partials(const float* x, const float* M, float2 (&acc)[RG]) {
  static_assert(NT == 8 * 64, "eight row groups of 64 column pairs");
  const int jp = threadIdx.x & 63, i0 = (threadIdx.x >> 6) * 16;
#pragma unroll
  for (int h = 0; h < RG; ++h) acc[h] = make_float2(0.f, 0.f);
#pragma unroll
  for (int ii = 0; ii < 16; ii += 4) {
    float2 m[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) m[e] = *reinterpret_cast<const float2*>(M + (i0 + ii + e) * kD + 2 * jp);
#pragma unroll
    for (int h = 0; h < RG; ++h) {
      const float4 xv = *reinterpret_cast<const float4*>(x + h * kD + i0 + ii);
      acc[h] = __ffma2_rn(m[0], make_float2(xv.x, xv.x), acc[h]);
      acc[h] = __ffma2_rn(m[1], make_float2(xv.y, xv.y), acc[h]);
      acc[h] = __ffma2_rn(m[2], make_float2(xv.z, xv.z), acc[h]);
      acc[h] = __ffma2_rn(m[3], make_float2(xv.w, xv.w), acc[h]);
    }
  }
}

// Stores thread t's partials at part[(t / 64) * RG + h][2 (t % 64) ..].
template <int RG>
__device__ __forceinline__ void store_partials(const float2 (&acc)[RG], float* part) {
#pragma unroll
  for (int h = 0; h < RG; ++h)
    *reinterpret_cast<float2*>(part + ((threadIdx.x >> 6) * RG + h) * kD + 2 * (threadIdx.x & 63)) = acc[h];
}

// Sum of the eight row-group partials of output oi = h * kD + j.
template <int RG>
__device__ __forceinline__ float product_sum(const float* part, int oi) {
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int rg = 0; rg < 8; rg += 2) {
    s0 += part[rg * RG * kD + oi];
    s1 += part[(rg + 1) * RG * kD + oi];
  }
  return s0 + s1;
}

// res[h * kD + j] = (x . M)[h][j] for the r query heads; M (64 KiB) is
// overwritten by the partial sums.  Every thread calls it.
template <int RG>
__device__ void query_product(const float* x, float* M, float* res) {
  float2 acc[RG];
  product_partials<RG>(x, M, acc);
  __syncthreads();                           // every thread has read M
  store_partials<RG>(acc, M);
  __syncthreads();
  for (int oi = threadIdx.x; oi < RG * kD; oi += NT) res[oi] = product_sum<RG>(M, oi);
  __syncthreads();
}

// ----------------------------------------------------- page bounds (Eq. 3)
//
// A warp scores 8 pages per task.  With HG heads per pass, LPP = 4 HG lanes
// share a page: lane j of the group holds dims [8 (j NCH + c), + 8) for its
// NCH = 4 / HG chunks c of the lower and the upper row (16 B each), so a
// page's bound is a sum over LPP lanes of per-lane partials.  The pair
// (l_d, u_d) times (min(q~_hd, 0), max(q~_hd, 0)) is one packed FMA, which is
// max(q~ l, q~ u) summed over the pair.  The chunk order is rotated per lane
// so that a quarter-warp's 16-B loads hit distinct banks.
template <int HG>
struct BoundsLayout {
  static constexpr int LPP = 4 * HG;            // lanes per page
  static constexpr int NCH = 4 / HG;            // 16-B chunks per row and lane
  static constexpr int PPS = 32 / LPP;          // pages per warp step
  static constexpr int STEPS = kTaskPages / PPS;  // == HG
  static constexpr int NV = STEPS * HG;         // partials per lane before reduction
};

// Butterfly reduce-scatter of NV values over groups of LPP lanes: afterwards
// v[0] holds the group sum of one value index (see the callers).
template <int NV, int O>
struct ReduceScatter {
  static __device__ __forceinline__ void run(float* v, int lane) {
    if constexpr (NV > 1) {
      constexpr int H = NV / 2;
      const bool up = (lane & O) != 0;
#pragma unroll
      for (int i = 0; i < H; ++i) {
        const float send = up ? v[i] : v[i + H];
        const float keep = up ? v[i + H] : v[i];
        v[i] = keep + __shfl_xor_sync(FULL, send, O);
      }
      if constexpr (O > 1) ReduceScatter<H, O / 2>::run(v, lane);
    } else {
      v[0] += __shfl_xor_sync(FULL, v[0], O);
      if constexpr (O > 1) ReduceScatter<1, O / 2>::run(v, lane);
    }
  }
};

// Loads this lane's (min(q~,0), max(q~,0)) pairs for heads [h0, h0 + HG).
template <int HG>
__device__ __forceinline__ void load_qpairs(const float* qt, int h0, float2 (&qp)[32], int lane) {
  using L = BoundsLayout<HG>;
  const int j = lane % L::LPP;
  const int rot = ((lane & 7) * L::NCH) >> 3;
#pragma unroll
  for (int i = 0; i < L::NCH; ++i) {
    const int c = (i + rot) % L::NCH;
    const int d0 = 8 * (j * L::NCH + c);
#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        const float v = qt[(h0 + h) * kD + d0 + e];
        qp[(i * 8 + e) * HG + h] = make_float2(fminf(v, 0.f), fmaxf(v, 0.f));
      }
  }
}

// Bounds of `np` (1..8) pages stored at `base` (shared address, 512 B each)
// for heads [h0, h0 + HG); returns, in the lanes with (lane & 3) == 0, the
// max over those heads for the task page task_page_of(lane).
template <int HG>
__device__ __forceinline__ float bounds_task(uint32_t base, int np, const float2 (&qp)[32], int lane) {
  using L = BoundsLayout<HG>;
  const int j = lane % L::LPP, p = lane / L::LPP;
  const int rot = ((lane & 7) * L::NCH) >> 3;
  float v[L::NV];
#pragma unroll
  for (int s = 0; s < L::STEPS; ++s) {
    const int tp = s * L::PPS + p;
    const uint32_t pg = base + static_cast<uint32_t>(tp < np ? tp : 0) * kPageBytes;
    float2 acc[HG];
#pragma unroll
    for (int h = 0; h < HG; ++h) acc[h] = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < L::NCH; ++i) {
      const int c = (i + rot) % L::NCH;
      const uint32_t off = 16u * static_cast<uint32_t>(j * L::NCH + c);
      const uint4 lo = lds128(pg + off);
      const uint4 hi = lds128(pg + 256u + off);
      const uint32_t wl[4] = {lo.x, lo.y, lo.z, lo.w};
      const uint32_t wh[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float l = (e & 1) ? bf_hi(wl[e >> 1]) : bf_lo(wl[e >> 1]);
        const float u = (e & 1) ? bf_hi(wh[e >> 1]) : bf_lo(wh[e >> 1]);
        const float2 lu = make_float2(l, u);
#pragma unroll
        for (int h = 0; h < HG; ++h) acc[h] = __ffma2_rn(lu, qp[(i * 8 + e) * HG + h], acc[h]);
      }
    }
#pragma unroll
    for (int h = 0; h < HG; ++h) v[s * HG + h] = acc[h].x + acc[h].y;
  }
  ReduceScatter<L::NV, L::LPP / 2>::run(v, lane);
  float u = v[0];
  if constexpr (HG == 4) {
    u = fmaxf(u, __shfl_xor_sync(FULL, u, 1));
    u = fmaxf(u, __shfl_xor_sync(FULL, u, 2));
  } else if constexpr (HG == 2) {
    u = fmaxf(u, __shfl_xor_sync(FULL, u, 2));
  }
  return u;
}

// The task page whose bound bounds_task<HG> leaves in `lane`.
template <int HG>
__device__ __forceinline__ int task_page_of(int lane) {
  if constexpr (HG == 4) return 2 * ((lane & 15) >> 2) + (lane >> 4);
  else if constexpr (HG == 2) return 4 * ((lane >> 2) & 1) + (lane >> 3);
  else return lane >> 2;
}

// ------------------------------------------------------------ attention

// Warp-level attention over groups of 8 selected tokens.  Lane l holds dims
// [4 l, 4 l + 4) of the queries (pre-scaled by scale * log2 e) and of its
// output accumulators.  Scores: per-lane partial dot products, reduced over
// the warp by a butterfly; the online softmax is float32 with exp2.
template <int HA>
struct AttnLayout {
  static constexpr int NV = 8 * HA;                       // (token, head) scores per group
  static constexpr int SHIFT = (NV == 32) ? 0 : (NV == 16) ? 1 : 2;  // lane = idx << SHIFT
};

template <int RG>
struct AttnState {
  static constexpr int HA = RG < 4 ? RG : 4;
  static constexpr int NPASS = RG / HA;
  float q[RG][4];
  float o[RG][4];
  float m[NPASS], l[NPASS];  // for head (lane >> SHIFT) % HA of each pass
};

template <int RG>
__device__ __forceinline__ void attend_group(AttnState<RG>& st, uint32_t kb, uint32_t vb, int nv,
                                             int lane) {
  constexpr int HA = AttnState<RG>::HA;
  constexpr int NV = AttnLayout<HA>::NV;
  constexpr int SH = AttnLayout<HA>::SHIFT;
  float kf[8][4];
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const uint2 w = lds64(kb + t * 256u + 8u * lane);
    kf[t][0] = bf_lo(w.x);
    kf[t][1] = bf_hi(w.x);
    kf[t][2] = bf_lo(w.y);
    kf[t][3] = bf_hi(w.y);
  }
  const int t_me = lane >> 2;   // token of this lane's score (NV = 8, 16 or 32)
#pragma unroll
  for (int ps = 0; ps < AttnState<RG>::NPASS; ++ps) {
    float v[NV];
#pragma unroll
    for (int t = 0; t < 8; ++t)
#pragma unroll
      for (int h = 0; h < HA; ++h) {
        const float* qh = st.q[ps * HA + h];
        float2 acc = __fmul2_rn(make_float2(kf[t][0], kf[t][1]), make_float2(qh[0], qh[1]));
        acc = __ffma2_rn(make_float2(kf[t][2], kf[t][3]), make_float2(qh[2], qh[3]), acc);
        v[t * HA + h] = acc.x + acc.y;
      }
    ReduceScatter<NV, 16>::run(v, lane);
    const float sc = t_me < nv ? v[0] : -INFINITY;
    float mx = sc;
    mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 16));
    const float m_new = fmaxf(st.m[ps], mx);     // finite: the group has a valid token
    const float alpha = exp2f(st.m[ps] - m_new); // 0 while m is -inf
    const float p = exp2f(sc - m_new);           // 0 for masked tokens
    float ps_sum = p;
    ps_sum += __shfl_xor_sync(FULL, ps_sum, 4);
    ps_sum += __shfl_xor_sync(FULL, ps_sum, 8);
    ps_sum += __shfl_xor_sync(FULL, ps_sum, 16);
    st.l[ps] = fmaf(st.l[ps], alpha, ps_sum);
    st.m[ps] = m_new;
#pragma unroll
    for (int h = 0; h < HA; ++h) {
      const float ah = __shfl_sync(FULL, alpha, h << SH);   // token 0, head h
#pragma unroll
      for (int e = 0; e < 4; ++e) st.o[ps * HA + h][e] *= ah;
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const uint2 w = lds64(vb + t * 256u + 8u * lane);
      const float2 v01 = make_float2(bf_lo(w.x), bf_hi(w.x));
      const float2 v23 = make_float2(bf_lo(w.y), bf_hi(w.y));
#pragma unroll
      for (int h = 0; h < HA; ++h) {
        const float pt = __shfl_sync(FULL, p, (t * HA + h) << SH);
        float* oh = st.o[ps * HA + h];
        float2 a01 = __ffma2_rn(v01, make_float2(pt, pt), make_float2(oh[0], oh[1]));
        float2 a23 = __ffma2_rn(v23, make_float2(pt, pt), make_float2(oh[2], oh[3]));
        oh[0] = a01.x;
        oh[1] = a01.y;
        oh[2] = a23.x;
        oh[3] = a23.y;
      }
    }
  }
}

// One warp: the merge weights of n partial softmax states of one head.
// State i has its running max at st[i * stride + d] and its sum at
// st[i * stride + d + 1].  Writes wgt[i] = 2^(m_i - M) (M the largest m_i;
// zero when every state is empty) and hdr = {M, sum_i wgt[i] l_i}.
template <bool GLOBAL>
__device__ __forceinline__ float state_ld(const float* p) {
  if constexpr (GLOBAL) return __ldcg(p);   // written by other CTAs: read at L2
  else return *p;
}

template <bool GLOBAL = false>
__device__ __forceinline__ void merge_weights(const float* st, int stride, int n, float* wgt, float* hdr) {
  const int lane = threadIdx.x & 31;
  float M = -INFINITY;
  for (int i = lane; i < n; i += 32) M = fmaxf(M, state_ld<GLOBAL>(st + i * stride + kD));
#pragma unroll
  for (int o2 = 16; o2 >= 1; o2 >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, o2));
  float L = 0.f;
  for (int i = lane; i < n; i += 32) {
    const float w = (M == -INFINITY) ? 0.f : exp2f(state_ld<GLOBAL>(st + i * stride + kD) - M);
    wgt[i] = w;
    L = fmaf(state_ld<GLOBAL>(st + i * stride + kD + 1), w, L);
  }
#pragma unroll
  for (int o2 = 16; o2 >= 1; o2 >>= 1) L += __shfl_xor_sync(FULL, L, o2);
  if (lane == 0) {
    hdr[0] = M;
    hdr[1] = L;
  }
}

// Attention of the group's r heads over `ns` tokens listed in sel[], then the
// CTA merge of the 16 warp states and the unit merge by the last CTA.
template <int RG>
__device__ void attend_and_finish(const DecodeArgs& a, int unit, int c, const int* sel, int ns,
                                  unsigned char* ring, uint32_t final_target, int* s_int) {
  using ST = AttnState<RG>;
  constexpr int HA = ST::HA;
  constexpr int SH = AttnLayout<HA>::SHIFT;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = unit / a.Hkv, g = unit % a.Hkv;
  const size_t unit_rows = static_cast<size_t>(unit) * a.n_cap;
  const uint16_t* Ku = a.K + unit_rows * kD;
  const uint16_t* Vu = a.V + unit_rows * kD;

  ST st;
  {
    const uint16_t* qg = a.q + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(g) * RG) * kD;
#pragma unroll
    for (int h = 0; h < RG; ++h) {
      const uint2 w = __ldg(reinterpret_cast<const uint2*>(qg + h * kD) + lane);
      st.q[h][0] = bf_lo(w.x) * a.scale_log2;
      st.q[h][1] = bf_hi(w.x) * a.scale_log2;
      st.q[h][2] = bf_lo(w.y) * a.scale_log2;
      st.q[h][3] = bf_hi(w.y) * a.scale_log2;
#pragma unroll
      for (int e = 0; e < 4; ++e) st.o[h][e] = 0.f;
    }
#pragma unroll
    for (int ps = 0; ps < ST::NPASS; ++ps) {
      st.m[ps] = -INFINITY;
      st.l[ps] = 0.f;
    }
  }

  // Per warp two 4-KiB buffers of [K rows 0-7 | V rows 0-7] (256 B each),
  // filled by cp.async: lane l copies 16-B column chunk l % 16 of rows
  // l / 16, + 2, ..., one commit group per token group (rows past the end
  // repeat a valid token, whose softmax weight is zero).
  unsigned char* wbuf = ring + warp * 8192;
  const int n_groups = (ns + 7) / 8;
  auto issue = [&](int gi, int buf) {
    if (gi < n_groups) {
      const uint32_t dst = smem_addr(wbuf + buf * 4096);
      const int ch = lane & 15;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = (lane >> 4) + 2 * i;            // 0-7: K row, 8-15: V row
        const int t = r & 7;
        const int n = sel[min(gi * 8 + t, ns - 1)];
        const uint16_t* src = (r < 8 ? Ku : Vu) + static_cast<size_t>(n) * kD + ch * 8;
        cp_async16(dst + r * 256 + ch * 16, src);
      }
    }
    cp_async_commit();
  };
  issue(warp, 0);
  issue(warp + NWARPS, 1);
  int it = 0;
  for (int gi = warp; gi < n_groups; gi += NWARPS, ++it) {
    const int buf = it & 1;
    cp_async_wait<1>();   // this lane's copies of group gi have landed
    __syncwarp();         // ... and every lane's
    const uint32_t kb = smem_addr(wbuf + buf * 4096);
    attend_group<RG>(st, kb, kb + 2048, min(8, ns - gi * 8), lane);
    __syncwarp();         // the buffer has been read
    issue(gi + 2 * NWARPS, buf);
  }
  cp_async_wait<0>();
  __syncthreads();        // the merge buffer below overlays the K / V buffers

  // merge the 16 warp states through shared memory: [warp][h][MS], the
  // d outputs then max and sum (rows padded to 16 B)
  constexpr int MS = kD + 4;
  float* mer = reinterpret_cast<float*>(ring);
#pragma unroll
  for (int h = 0; h < RG; ++h) {
    float* dst = mer + (warp * RG + h) * MS;
    *reinterpret_cast<float4*>(dst + 4 * lane) = make_float4(st.o[h][0], st.o[h][1], st.o[h][2], st.o[h][3]);
  }
#pragma unroll
  for (int ps = 0; ps < ST::NPASS; ++ps)
#pragma unroll
    for (int h = 0; h < HA; ++h)
      if (lane == (h << SH)) {
        float* dst = mer + (warp * RG + ps * HA + h) * MS;
        dst[kD] = st.m[ps];
        dst[kD + 1] = st.l[ps];
      }
  __syncthreads();

  constexpr int PS = part_stride(RG);
  float* part = a.wsPart + static_cast<size_t>(unit * kMaxCtasPerUnit + c) * PS;
  {
    float* wgt = mer + NWARPS * RG * MS;         // [RG][NWARPS]
    float* hdr = wgt + NWARPS * RG;              // [RG][2]: M, sum of weighted l
    if (warp < RG) merge_weights(mer + warp * MS, RG * MS, NWARPS, wgt + warp * NWARPS, hdr + 2 * warp);
    __syncthreads();
    for (int oi = tid; oi < RG * kD; oi += NT) {
      const int h = oi / kD, j = oi % kD;
      float O = 0.f;
#pragma unroll 4
      for (int w = 0; w < NWARPS; ++w) O = fmaf(mer[(w * RG + h) * MS + j], wgt[h * NWARPS + w], O);
      const float L = hdr[2 * h + 1];
      if (a.C == 1) {
        a.out[(static_cast<size_t>(b) * a.Hq + g * RG + h) * kD + j] = (L > 0.f) ? O / L : 0.f;
      } else {
        part[h * (kD + 2) + j] = O;
        if (j == 0) {
          part[h * (kD + 2) + kD] = hdr[2 * h];
          part[h * (kD + 2) + kD + 1] = L;
        }
      }
    }
  }

  // last CTA of the unit merges the C partial states and resets the counter
  uint32_t* ctr = a.counters + unit;
  __syncthreads();
  if (tid == 0) {
    const uint32_t old = atom_add_acq_rel(ctr, 1u);
    s_int[0] = (old == final_target - 1) ? 1 : 0;
    // this CTA's share of the step is done but for the final merge: the
    // next kernel on the stream may start launching (it waits for the
    // completion of this one before touching memory)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }
  __syncthreads();
  if (!s_int[0]) return;
  if (a.C > 1) {
    const float* parts = a.wsPart + static_cast<size_t>(unit * kMaxCtasPerUnit) * PS;
    float* wgt = mer;                  // [RG][C]
    float* hdr = wgt + a.C * RG;       // [RG][2]
    if (warp < RG) merge_weights<true>(parts + warp * (kD + 2), PS, a.C, wgt + warp * a.C, hdr + 2 * warp);
    __syncthreads();
    for (int oi = tid; oi < RG * kD; oi += NT) {
      const int h = oi / kD, j = oi % kD;
      float O = 0.f;
#pragma unroll 6
      for (int cc = 0; cc < a.C; ++cc) O = fmaf(__ldcg(parts + cc * PS + h * (kD + 2) + j), wgt[h * a.C + cc], O);
      const float L = hdr[2 * h + 1];
      a.out[(static_cast<size_t>(b) * a.Hq + g * RG + h) * kD + j] = (L > 0.f) ? O / L : 0.f;
    }
  }
  if (tid == 0) atomicExch(ctr, 0u);
}

// Thread 0 waits until the unit counter reaches `target` (acquire), then the
// CTA barrier releases everyone.  Returns false (HHR_ERR_TIMEOUT recorded)
// if the wait ran out.  Every thread of the CTA calls it.
__device__ bool unit_wait(const uint32_t* ctr, uint32_t target, const DecodeArgs& a, int* s_flag) {
  if (threadIdx.x == 0) {
    int ok = 1;
    const long long t0 = clock64();
    while (ld_acquire(ctr) < target) {
      if (static_cast<unsigned long long>(clock64() - t0) > a.spin_limit) {
        atomicExch(a.status, static_cast<uint32_t>(HHR_ERR_TIMEOUT));
        ok = 0;
        break;
      }
    }
    *s_flag = ok;
  }
  __syncthreads();
  return *s_flag != 0;
}

// ----------------------------------------------------------------------------
template <int RG, int WORDS, int MODE>
__global__ void __launch_bounds__(NT, 1) decode_kernel(const __grid_constant__ DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int BITS = WORDS * 32;
  constexpr int HG = RG < 4 ? RG : 4;           // heads per bounds pass
  constexpr int NPASS = RG / HG;
  __shared__ __align__(8) unsigned long long s_full[kSlots];
  __shared__ __align__(8) unsigned long long s_rwbar;
  __shared__ uint32_t s_slotcnt[kSlots];
  __shared__ uint32_t s_last[kSlots];           // last chunk (global count) issued into each slot
  __shared__ int s_scan[NWARPS + 1];
  __shared__ int s_scan1[NWARPS];
  __shared__ int s_misc[32];
  __shared__ float s_flt[2 * NWARPS];
  __shared__ int s_cum[kSample + 2];           // own bin counts, then their prefix
  __shared__ int s_fill[kSample + 1];
  __shared__ int s_task;                        // next scan task (dynamic assignment)
  __shared__ int s_cA[kMaxCtasPerUnit], s_cB[kMaxCtasPerUnit], s_cC[kMaxCtasPerUnit], s_cE[kMaxCtasPerUnit];
  __shared__ int s_dh[BITS + 2];                // distance histogram, then its prefix

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x % a.C;
  const DecodeSmem lay = decode_smem(RG, BITS, a.slice_pages, MODE);
  unsigned char* ring = smem + lay.ring;
  float* rw = reinterpret_cast<float*>(smem + lay.rw);
  float* sS = reinterpret_cast<float*>(smem + lay.sS);
  uint32_t* sE = reinterpret_cast<uint32_t*>(smem + lay.sE);
  float* sU = reinterpret_cast<float*>(smem + lay.sU);
  uint8_t* sBin = smem + lay.sBin;
  float* qt = reinterpret_cast<float*>(smem + lay.qt);
  float* qraw = reinterpret_cast<float*>(smem + lay.qraw);
  uint32_t* qc = reinterpret_cast<uint32_t*>(smem + lay.qc);
  const uint32_t ring_s = smem_addr(ring);
  const uint64_t pol_keep = policy_evict_last();
  const uint32_t rw_bar = smem_addr(&s_rwbar);
  if (tid == 0) {
    for (int s = 0; s < kSlots; ++s) mbar_init(smem_addr(&s_full[s]), 1u);
    mbar_init(rw_bar, 1u);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (tid < kSlots) {
    s_slotcnt[tid] = 0u;
    s_last[tid] = 0xFFFFFFFFu;
  }
  // Launched as a programmatic dependent of the previous kernel on the
  // stream: the set-up above touches only shared memory; wait here, before
  // any global memory access, until that kernel has completed and its
  // writes are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __syncthreads();
  uint32_t rw_seq = 0;     // phases of the R / W barrier used so far
  uint32_t chunk0 = 0;     // ring chunks used so far (slot = chunk % kSlots)

  for (int unit = blockIdx.x / a.C; unit < a.units; unit += a.grid_units) {
    const int b = unit / a.Hkv, g = unit % a.Hkv;
    uint32_t* ctr = a.counters + unit;

    if constexpr (MODE == kModeAttend) {
      const int n = min(max(a.nsel_in[unit], 0), a.k);
      const int s0 = static_cast<int>(static_cast<long long>(c) * n / a.C);
      const int s1 = static_cast<int>(static_cast<long long>(c + 1) * n / a.C);
      int* sel = reinterpret_cast<int*>(rw);
      const int32_t* src = a.tok_in + static_cast<size_t>(unit) * a.k;
      for (int i = s0 + tid; i < s1; i += NT) {
        const int t = src[i];
        sel[i - s0] = (t >= 0 && t < a.n_cap) ? t : 0;   // out-of-range indices are clamped
      }
      __syncthreads();
      attend_and_finish<RG>(a, unit, c, sel, s1 - s0, ring, static_cast<uint32_t>(a.C), s_misc);
      __syncthreads();
      continue;
    } else {
      const int NP = a.NP, Pk = a.Pk, S_ = a.page;
      const int pb = c * NP / a.C;            // c NP < 2^31: NP <= HHR_MAX_PAGES
      const int pe = (c + 1) * NP / a.C;
      const int n_own = pe - pb;
      const bool local = a.local != 0;
      const int n_smp = a.n_sample;                      // 0: own pages only (C == 1)
      const int n_sc = (n_smp + kChunkPages - 1) / kChunkPages;
      const int n_oc = (local && n_smp > 0) ? 0 : (n_own + kChunkPages - 1) / kChunkPages;
      const int n_chunks = n_sc + n_oc;
      const uint16_t* meta_u = a.meta + static_cast<size_t>(unit) * a.np_cap * 2 * kD;
      const uint16_t* qg = a.q + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(g) * RG) * kD;
      const float* Rg = a.R + static_cast<size_t>(g) * kD * kD;
      const float* Wg = a.W + static_cast<size_t>(g) * kD * BITS;
      // sampled mode: 8 blocks of 8 consecutive pages, block b starting at page b NP / 8
      auto smp_block = [&](int bl) { return bl * NP / 8; };
      // chunk k of this unit: the sample's chunks first, then the own pages'
      auto chunk_pages = [&](int k) {
        return k < n_sc ? min(kChunkPages, n_smp - k * kChunkPages)
                        : min(kChunkPages, n_own - (k - n_sc) * kChunkPages);
      };
      // one thread: fill ring slot of chunk k (its previous contents are no
      // longer read by any warp)
      auto issue_chunk = [&](int k) {
        const uint32_t gk = chunk0 + static_cast<uint32_t>(k);
        const uint32_t slot = gk % kSlots;
        const uint32_t bar = smem_addr(&s_full[slot]);
        const int np = chunk_pages(k);
        fence_proxy_async();
        mbar_expect_tx(bar, static_cast<uint32_t>(np) * kPageBytes);
        const uint32_t dst = ring_s + slot * kChunkBytes;
        if (k < n_sc && !local) {
          for (int bb = 0; bb < kChunkPages / 8; ++bb)
            bulk_g2s(dst + bb * 8 * kPageBytes, meta_u + static_cast<size_t>(smp_block(k * (kChunkPages / 8) + bb)) * 2 * kD,
                     8 * kPageBytes, bar);
        } else {
          const int p0 = k < n_sc ? k * kChunkPages : pb + (k - n_sc) * kChunkPages;
          bulk_g2s(dst, meta_u + static_cast<size_t>(p0) * 2 * kD, static_cast<uint32_t>(np) * kPageBytes, bar);
        }
        *reinterpret_cast<volatile uint32_t*>(&s_last[slot]) = gk;   // after expect_tx armed the phase
      };

      // thread 0, after a timed-out wait: record it and wait (bounded) for
      // every copy this CTA may still have in flight into shared memory
      auto drain = [&]() {
        atomicExch(a.status, static_cast<uint32_t>(HHR_ERR_TIMEOUT));
        for (int s2 = 0; s2 < kSlots; ++s2) {
          const uint32_t last = s_last[s2];
          if (last != 0xFFFFFFFFu) mbar_wait(smem_addr(&s_full[s2]), (last / kSlots) & 1u, a.spin_limit);
        }
        mbar_wait(rw_bar, rw_seq & 1u, a.spin_limit);
      };

      // ---------------------------------------------------------- phase 0
      // R by thread 0, which then waits for it; the ring by another warp
      // (a thread that issues many bulk copies is held back by the copy
      // engine's queue)
      if (tid == 0) {
        fence_proxy_async();
        mbar_expect_tx(rw_bar, kRWBytes);
        bulk_g2s_hint(smem_addr(rw), Rg, kRWBytes, rw_bar, pol_keep);
      }
      if (tid == 32)
        for (int k = 0; k < min(kSlots, n_chunks); ++k) issue_chunk(k);
      for (int i = tid; i < RG * kD; i += NT) qraw[i] = __uint_as_float(static_cast<uint32_t>(qg[i]) << 16);
      {
        const bool okr = (tid == 0) ? mbar_wait(rw_bar, rw_seq & 1u, a.spin_limit) : true;
        if (__syncthreads_or(!okr)) {
          if (tid == 0) drain();
          __syncthreads();
          return;
        }
        ++rw_seq;
      }
      if (tid == 0) s_task = NWARPS;     // tasks 0 .. NWARPS-1 go to warps 0 .. NWARPS-1
      query_product<RG>(qraw, rw, qt);   // q~ = q R (its barriers publish s_task too)
      if (tid == 0) {                     // W, first 128 columns
        fence_proxy_async();
        mbar_expect_tx(rw_bar, kRWBytes);
        if constexpr (BITS == kD) {
          bulk_g2s_hint(smem_addr(rw), Wg, kRWBytes, rw_bar, pol_keep);
        } else {
          for (int i = 0; i < kD; ++i)
            bulk_g2s_hint(smem_addr(rw + i * kD), Wg + static_cast<size_t>(i) * BITS, kD * 4, rw_bar, pol_keep);
        }
      }

      // ---------------------------------------------------------- phase 1
      int err = 0;
      {
        float2 qp[32];
        if constexpr (NPASS == 1) load_qpairs<HG>(qt, 0, qp, lane);
        const int n_tasks = n_chunks * kTasksPerChunk;
        // tasks in order, each warp taking the next one when it is free
        int t = warp;
        for (; t < n_tasks;) {
          const int k = t / kTasksPerChunk, jt = t % kTasksPerChunk;
          const uint32_t gk = chunk0 + static_cast<uint32_t>(k);
          const uint32_t slot = gk % kSlots;
          bool got = true;
          if (lane == 0) {
            // the slot's barrier phase belongs to chunk gk only once gk has
            // been issued into it (a parity wait on a later chunk would
            // otherwise see the previous phase): wait for that first
            const long long ts = clock64();
            while (*reinterpret_cast<volatile uint32_t*>(&s_last[slot]) != gk) {
              if (static_cast<unsigned long long>(clock64() - ts) > a.spin_limit) {
                got = false;
                break;
              }
            }
            if (got) got = mbar_wait(smem_addr(&s_full[slot]), (gk / kSlots) & 1u, a.spin_limit);
          }
          if (!__shfl_sync(FULL, got ? 1 : 0, 0)) {
            err = 1;
            break;
          }
          const int np = chunk_pages(k) - jt * kTaskPages;
          if (np > 0) {
            const uint32_t base = ring_s + slot * kChunkBytes + jt * kTaskPages * kPageBytes;
            float u;
            if constexpr (NPASS == 1) {
              u = bounds_task<HG>(base, min(np, kTaskPages), qp, lane);
            } else {
              load_qpairs<HG>(qt, 0, qp, lane);
              u = bounds_task<HG>(base, min(np, kTaskPages), qp, lane);
#pragma unroll
              for (int ps = 1; ps < NPASS; ++ps) {
                load_qpairs<HG>(qt, ps * HG, qp, lane);
                u = fmaxf(u, bounds_task<HG>(base, min(np, kTaskPages), qp, lane));
              }
            }
            const int tp = task_page_of<HG>(lane);
            if ((lane & 3) == 0 && tp < np) {
              const int i = (k < n_sc ? k : k - n_sc) * kChunkPages + jt * kTaskPages + tp;
              if (k < n_sc) sS[i] = u;
              else sU[i] = u;
            }
          }
          __syncwarp();
          int nxt = 0;
          if (lane == 0) {
            const uint32_t old = smem_atom_add_acq_rel(&s_slotcnt[slot], 1u);
            if (old == kTasksPerChunk - 1) {
              s_slotcnt[slot] = 0u;
              if (k + kSlots < n_chunks) issue_chunk(k + kSlots);
            }
            nxt = atomicAdd(&s_task, 1);
          }
          t = __shfl_sync(FULL, nxt, 0);
        }
      }
      chunk0 += static_cast<uint32_t>(n_chunks);
      if (__syncthreads_or(err)) {   // a ring copy never landed
        if (tid == 0) drain();
        __syncthreads();
        return;
      }

      // ---------------------------------------------------------- phase 2
      Pivot pv;
      pv.all = 0;
      pv.key = 0u;
      pv.page = 0;
      const float* ownU = (local && n_smp > 0) ? sS + pb : sU;
      if (!local) {
        // sample order keys, sorted descending (ties by index): the bin edges.
        // Entry i's rank is counted by NT / kSample threads over slices.
        static_assert(NT % kSample == 0, "sample ranking splits the comparisons evenly");
        uint32_t* sK = sE + kSample;   // keys, then ranks (the upper part of sE)
        int* sR = reinterpret_cast<int*>(sK + kSample);
        if (tid < kSample) {
          sK[tid] = order_key(sS[tid]);
          sR[tid] = 0;
        }
        for (int i = tid; i < kSample + 2; i += NT) s_cum[i] = 0;
        for (int i = tid; i < kSample + 1; i += NT) s_fill[i] = 0;
        __syncthreads();
        {
          constexpr int PARTS = NT / kSample, SL = kSample / PARTS;
          const int i = tid % kSample, j0 = (tid / kSample) * SL;
          const uint32_t ki = sK[i];
          int r = 0;
#pragma unroll
          for (int jj = 0; jj < SL; ++jj) {
            const uint32_t kj = sK[j0 + jj];
            r += static_cast<int>(kj > ki) | (static_cast<int>(kj == ki) & static_cast<int>(j0 + jj < i));
          }
          atomicAdd(&sR[i], r);
        }
        __syncthreads();
        if (tid < kSample) sE[sR[tid]] = sK[tid];
        __syncthreads();
      // own bins: bin(u) = number of edges above u
        for (int i = tid; i < n_own; i += NT) {
          const uint32_t ku = order_key(sU[i]);
          int lo = 0, hi = n_smp;
          while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (sE[mid] > ku) lo = mid + 1;
            else hi = mid;
          }
          sBin[i] = static_cast<uint8_t>(lo);
          atomicAdd(&s_cum[lo + 1], 1);
          if (a.dbg_U) a.dbg_U[static_cast<size_t>(unit) * a.NP + pb + i] = sU[i];
        }
        __syncthreads();
        if (warp == 0) {   // prefix over the kSample + 2 entries
          int run = 0;
          for (int base = 0; base < kSample + 2; base += 32) {
            int x = base + lane < kSample + 2 ? s_cum[base + lane] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const int y = __shfl_up_sync(FULL, x, o);
              if (lane >= o) x += y;
            }
            if (base + lane < kSample + 2) s_cum[base + lane] = run + x;
            run += __shfl_sync(FULL, x, 31);
          }
        }
        __syncthreads();
        {
          // publish: cumulative counts, and the own bounds ordered by bin,
          // stored centred on the expected cutoff bin
          int32_t* cum_g = a.wsCum + static_cast<size_t>(unit * kMaxCtasPerUnit + c) * kCumStride;
          for (int i = tid; i < kSample + 2; i += NT) cum_g[i] = s_cum[i];
          const int s = a.list_half;
          int2* list_g = a.wsList + static_cast<size_t>(unit) * a.list_stride + static_cast<size_t>(c) * 2 * s;
          const int cexp = s_cum[a.b_exp];
          for (int i = tid; i < n_own; i += NT) {
            const int bi = sBin[i];
            const int pos = s_cum[bi] + atomicAdd(&s_fill[bi], 1);
            list_g[s + pos - cexp] = make_int2(__float_as_int(sU[i]), pb + i);
          }
        }
      } else if (a.dbg_U) {
        for (int i = tid; i < n_own; i += NT) a.dbg_U[static_cast<size_t>(unit) * a.NP + pb + i] = ownU[i];
      }
      // unit barrier 1: arrive (the release covers what this CTA published
      // through the CTA barrier)
      __syncthreads();
      if (tid == 0) atom_add_acq_rel(ctr, 1u);
      if (!local) {
        // the codes of the pages likely to be kept into L2 (a hint only)
        const int b_spec = min(a.b_exp + 3, kSample);
        const size_t row_bytes = static_cast<size_t>(WORDS) * 4;
        const char* cbase = reinterpret_cast<const char*>(a.codes + static_cast<size_t>(unit) * a.n_cap * WORDS);
        for (int i = tid; i < n_own; i += NT) {
          if (sBin[i] <= b_spec) {
            const size_t b0 = static_cast<size_t>(pb + i) * S_ * row_bytes;
            const size_t b1 = min(static_cast<size_t>(pb + i + 1) * S_, static_cast<size_t>(a.n_valid)) * row_bytes;
            for (size_t off = b0 & ~static_cast<size_t>(127); off < b1; off += 128) prefetch_l2(cbase + off);
          }
        }
      }

      // query codes (Eq. 10 + sign) from W, 128 columns at a time
#pragma unroll 1
      for (int half = 0; half < BITS / kD; ++half) {
        const bool okw = (tid == 0) ? mbar_wait(rw_bar, rw_seq & 1u, a.spin_limit) : true;
        if (__syncthreads_or(!okw)) {
          if (tid == 0) drain();
          __syncthreads();
          return;
        }
        ++rw_seq;
        float* partw = reinterpret_cast<float*>(ring);   // [8][r][d]; the ring is free
        {
          float2 acc[RG];
          product_partials<RG>(qraw, rw, acc);
          store_partials<RG>(acc, partw);
        }
        __syncthreads();   // W read by every thread, the partials visible
        if (half + 1 < BITS / kD && tid == 0) {   // W columns 128-255 into the same buffer
          fence_proxy_async();
          mbar_expect_tx(rw_bar, kRWBytes);
          for (int i = 0; i < kD; ++i)
            bulk_g2s_hint(smem_addr(rw + i * kD), Wg + static_cast<size_t>(i) * BITS + kD, kD * 4, rw_bar, pol_keep);
        }
        for (int oi = tid; oi < RG * kD; oi += NT) {  // warp-uniform trip count
          const float z = product_sum<RG>(partw, oi);
          const uint32_t word = __ballot_sync(FULL, z > 0.f);
          const int h = oi / kD, t = oi % kD;
          if (lane == 0) qc[h * WORDS + half * (kD / 32) + t / 32] = word;
        }
        __syncthreads();
      }

      // ---------------------------------------------------------- phase 3
      const uint32_t t1 = static_cast<uint32_t>(a.C) + (a.test_extra_stage == 1 ? 1u : 0u);
      int my_off = 0;   // kept pages of the CTAs before this one
      if (Pk >= NP) {
        pv.all = 1;
        my_off = pb;
      } else if (local) {
        const float* allU = n_smp > 0 ? sS : sU;
        pv = select_pivot(allU, nullptr, 0, NP, Pk, reinterpret_cast<int*>(ring), s_scan, s_misc, s_flt);
        int cnt = 0;
        for (int p = tid; p < pb; p += NT) cnt += kept(order_key(allU[p]), p, pv);
        my_off = block_sum(cnt, s_scan);
      } else {
        if (!unit_wait(ctr, t1, a, s_misc)) return;
        const int C = a.C, s = a.list_half, win = a.win, W2 = 2 * win;
        constexpr int CS = kSample + 2, CSS = kCumStride;
        int* gCum = reinterpret_cast<int*>(ring);                                   // [C][CSS]
        int2* gWin = reinterpret_cast<int2*>(ring + align_up(sizeof(int) * C * CSS, 16));  // [C][2 win]
        int* gPart = reinterpret_cast<int*>(rw);                                    // [7][CS] (R/W is free)
        {
          // one round trip: every CTA's counts, and its list entries
          // [s - win, s + win) (those inside its area [0, 2 s))
          copy_rows_async(smem_addr(gCum),
                          reinterpret_cast<const char*>(a.wsCum + static_cast<size_t>(unit * kMaxCtasPerUnit) * kCumStride),
                          C, CSS / 4, sizeof(int) * kCumStride, sizeof(int) * CSS, 0, CSS / 4);
          const int c_lo = max(0, win - s) / 2, c_hi = min(W2, s + win) / 2;   // 16-B chunks = 2 entries
          copy_rows_async(smem_addr(gWin),
                          reinterpret_cast<const char*>(a.wsList + static_cast<size_t>(unit) * a.list_stride + (s - win)),
                          C, win, sizeof(int2) * 2 * s, sizeof(int2) * W2, c_lo, c_hi);
          cp_async_wait<0>();
        }
        __syncthreads();
        // partial bin totals: thread (part, b) sums rows part, part + 7, ...
        constexpr int PARTS = NT / CS;
        if (tid < PARTS * CS) {
          const int part = tid / CS, bb = tid - part * CS;
          int x0 = 0, x1 = 0;
          int cc = part;
          for (; cc + PARTS < C; cc += 2 * PARTS) {
            x0 += gCum[cc * CSS + bb];
            x1 += gCum[(cc + PARTS) * CSS + bb];
          }
          if (cc < C) x0 += gCum[cc * CSS + bb];
          gPart[part * CS + bb] = x0 + x1;
        }
        __syncthreads();
        // warp 0: tot[b] = entries of the unit in bins below b; the boundary
        // bin b* (tot[b*] < Pk <= tot[b* + 1]); per CTA its entries above b*
        // (s_cA), in b* (s_cB) and the offset of those among the candidates (s_cC)
        if (warp == 0) {
          constexpr int QB = (CS + 31) / 32;
          int tot[QB];
#pragma unroll
          for (int qq = 0; qq < QB; ++qq) {
            const int bb = lane + 32 * qq;
            int x = 0;
            if (bb < CS) {
#pragma unroll
              for (int part = 0; part < PARTS; ++part) x += gPart[part * CS + bb];
            }
            tot[qq] = x;
          }
          // tot is non-decreasing with tot[0] = 0 < Pk: b* = #{b : tot[b] < Pk} - 1
          int n_lt = 0;
#pragma unroll
          for (int qq = 0; qq < QB; ++qq) n_lt += __popc(__ballot_sync(FULL, lane + 32 * qq < CS && tot[qq] < Pk));
          const int bst = n_lt - 1;
          int tb = 0, tb1 = 0;
#pragma unroll
          for (int qq = 0; qq < QB; ++qq) {
            const int v = __shfl_sync(FULL, tot[qq], bst & 31);
            const int v1 = __shfl_sync(FULL, tot[qq], (bst + 1) & 31);
            if ((bst >> 5) == qq) tb = v;
            if (((bst + 1) >> 5) == qq) tb1 = v1;
          }
          int run = 0, outside = 0;
          for (int c0 = 0; c0 < C; c0 += 32) {
            const int cc = c0 + lane;
            int base = 0, cnt = 0, rel = 0;
            if (cc < C) {
              base = gCum[cc * CSS + bst];
              cnt = gCum[cc * CSS + bst + 1] - base;
              const int cexp = gCum[cc * CSS + a.b_exp];
              rel = base - cexp + win;   // first entry within the window row
              s_cA[cc] = base;
              s_cB[cc] = cnt;
              s_cE[cc] = cexp;
              // the window row holds entries [c_lo, c_hi) chunks: e in [2 c_lo, 2 c_hi)
              if (cnt > 0 && (rel < 2 * (max(0, win - s) / 2) || rel + cnt > 2 * (min(W2, s + win) / 2))) outside = 1;
            }
            int x = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const int y = __shfl_up_sync(FULL, x, o);
              if (lane >= o) x += y;
            }
            if (cc < C) s_cC[cc] = run + x - cnt;
            run += __shfl_sync(FULL, x, 31);
          }
          outside = __any_sync(FULL, outside);
          if (lane == 0) {
            s_misc[8] = bst;
            s_misc[5] = Pk - tb;    // need
            s_misc[6] = tb1 - tb;   // M
            s_misc[9] = outside;
          }
        }
        __syncthreads();
        const int need = s_misc[5];
        const int M = s_misc[6];
        const bool in_win = s_misc[9] == 0 && M <= (kRWBytes / 8);
        float* candU;
        int* candP;
        int* scratch;
        if (in_win) {
          // the boundary bin's entries, from the window rows, into the R/W buffer
          candU = rw;
          candP = reinterpret_cast<int*>(rw) + kRWBytes / 8;
          for (int cc = warp; cc < C; cc += NWARPS) {
            const int rel = s_cA[cc] - s_cE[cc] + win;
            for (int o = lane; o < s_cB[cc]; o += 32) {
              const int2 en = gWin[cc * W2 + rel + o];
              candU[s_cC[cc] + o] = __int_as_float(en.x);
              candP[s_cC[cc] + o] = en.y;
            }
          }
          __syncthreads();
          scratch = reinterpret_cast<int*>(ring);   // the window rows are dead
        } else {
          // some CTA's boundary entries lie outside the rows read: read the
          // boundary bin itself (a second round trip), into the ring
          candU = reinterpret_cast<float*>(ring);
          candP = reinterpret_cast<int*>(ring) + kRingBytes / 8;
          const int2* list_u = a.wsList + static_cast<size_t>(unit) * a.list_stride;
          for (int cc = 0; cc < C; ++cc) {
            const int first = s + s_cA[cc] - s_cE[cc];
            for (int o = tid; o < s_cB[cc]; o += NT) {
              const int2 en = __ldcg(list_u + static_cast<size_t>(cc) * 2 * s + first + o);
              candU[s_cC[cc] + o] = __int_as_float(en.x);
              candP[s_cC[cc] + o] = en.y;
            }
          }
          __syncthreads();
          scratch = reinterpret_cast<int*>(rw);
        }
        pv = select_pivot(candU, candP, 0, M, need, scratch, s_scan, s_misc, s_flt);
        // kept pages per CTA: all of its entries above the bin plus its
        // boundary entries that are not below the cutoff
        for (int cc = warp; cc < C; cc += NWARPS) {
          int cnt = 0;
          for (int o = lane; o < s_cB[cc]; o += 32) {
            const int i = s_cC[cc] + o;
            cnt += kept(order_key(candU[i]), candP[i], pv);
          }
#pragma unroll
          for (int o2 = 16; o2 >= 1; o2 >>= 1) cnt += __shfl_xor_sync(FULL, cnt, o2);
          if (lane == 0) s_cA[cc] += cnt;
        }
        __syncthreads();
        if (warp == 0) {
          int x = 0;
          for (int cc = lane; cc < c; cc += 32) x += s_cA[cc];
#pragma unroll
          for (int o2 = 16; o2 >= 1; o2 >>= 1) x += __shfl_xor_sync(FULL, x, o2);
          if (lane == 0) s_misc[10] = x;
        }
        __syncthreads();
        my_off = s_misc[10];
      }

      // own kept pages in ascending order -> my_pages; page_idx
      int* my_pages = reinterpret_cast<int*>(ring);                       // <= slice_pages
      uint16_t* tokD = reinterpret_cast<uint16_t*>(ring + align_up(sizeof(int) * a.slice_pages, 16));
      int nk;
      {
        // thread t takes own pages [t*span, (t+1)*span)
        const int span = (n_own + NT - 1) / NT;
        const int lo = min(n_own, tid * span), hi = min(n_own, lo + span);
        int cnt = 0;
        uint32_t mask = 0u;   // span <= 32 (n_own <= kMaxSlicePages < 32 NT)
        for (int i = lo; i < hi; ++i) {
          const bool kp = (local || pv.all) ? kept(order_key(ownU[i]), pb + i, pv)
                                            : (sBin[i] < s_misc[8] ||
                                               (sBin[i] == s_misc[8] && kept(order_key(ownU[i]), pb + i, pv)));
          if (kp) {
            mask |= 1u << (i - lo);
            ++cnt;
          }
        }
        int tot;
        int pos = block_excl_scan1(cnt, s_scan1, &tot);
        nk = tot;
        int32_t* pidx = a.page_idx + static_cast<size_t>(unit) * a.P;
        for (int i = lo; i < hi; ++i) {
          if ((mask >> (i - lo)) & 1u) {
            my_pages[pos] = pb + i;
            if (my_off + pos < a.P) pidx[my_off + pos] = pb + i;
            ++pos;
          }
        }
        if (c == 0)
          for (int i = Pk + tid; i < a.P; i += NT) pidx[i] = -1;
      }
      __syncthreads();

      // ---------------------------------------------------------- phase 4
      const int ntok = nk * S_;
      for (int i = tid; i < BITS + 2; i += NT) s_dh[i] = 0;
      uint32_t qcr[RG][WORDS];
#pragma unroll
      for (int h = 0; h < RG; ++h)
#pragma unroll
        for (int w = 0; w < WORDS; ++w) qcr[h][w] = qc[h * WORDS + w];
      __syncthreads();
      {
        const uint32_t* codes_u = a.codes + static_cast<size_t>(unit) * a.n_cap * WORDS;
        int32_t* dbgD = a.dbg_D ? a.dbg_D + static_cast<size_t>(unit) * a.P * S_ : nullptr;
        for (int i0 = warp * 32; i0 < ntok; i0 += NT) {
          const int i = i0 + lane;
          int D = 0xFFFF;
          if (i < ntok) {
            const int slot = i / S_, off = i - slot * S_;
            const long long n = static_cast<long long>(my_pages[slot]) * S_ + off;
            if (n < a.n_valid) {
              uint32_t kc[WORDS];
              const uint4* cp = reinterpret_cast<const uint4*>(codes_u + n * WORDS);
#pragma unroll
              for (int w4 = 0; w4 < WORDS / 4; ++w4) {
                const uint4 t = __ldcs(cp + w4);
                kc[w4 * 4 + 0] = t.x;
                kc[w4 * 4 + 1] = t.y;
                kc[w4 * 4 + 2] = t.z;
                kc[w4 * 4 + 3] = t.w;
              }
              int best = 1 << 20;
#pragma unroll
              for (int h = 0; h < RG; ++h) {
                int dist = 0;
#pragma unroll
                for (int w = 0; w < WORDS; ++w) dist += __popc(qcr[h][w] ^ kc[w]);
                best = min(best, dist);
              }
              D = best;
            }
            tokD[i] = static_cast<uint16_t>(D);
            if (dbgD && my_off + slot < a.P) dbgD[static_cast<size_t>(my_off + slot) * S_ + off] = (D == 0xFFFF) ? -1 : D;
          }
          const unsigned grp = __match_any_sync(FULL, D);
          if (D != 0xFFFF && lane == __ffs(grp) - 1) atomicAdd(&s_dh[D + 1], __popc(grp));
        }
        if (c == 0 && dbgD)
          for (int i = Pk * S_ + tid; i < a.P * S_; i += NT) dbgD[i] = -1;
      }
      __syncthreads();
      // prefix: s_dh[v] = own tokens with D < v, v = 0 .. BITS + 1
      if (warp == 0) {
        int run = 0;
        for (int base = 0; base < BITS + 2; base += 32) {
          int x = base + lane < BITS + 2 ? s_dh[base + lane] : 0;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(FULL, x, o);
            if (lane >= o) x += y;
          }
          if (base + lane < BITS + 2) s_dh[base + lane] = run + x;
          run += __shfl_sync(FULL, x, 31);
        }
      }
      __syncthreads();
      {
        int32_t* row = a.wsCumD + static_cast<size_t>(unit * kMaxCtasPerUnit + c) * a.cumD_stride;
        for (int i = tid; i < BITS + 2; i += NT) row[i] = s_dh[i];
      }
      // unit barrier 2 (the release by thread 0 covers the CTA's row through
      // the CTA barrier)
      __syncthreads();
      if (tid == 0) atom_add_acq_rel(ctr, 1u);
      const uint32_t t2 = 2u * static_cast<uint32_t>(a.C) + (a.test_extra_stage == 2 ? 1u : 0u);
      if (!unit_wait(ctr, t2, a, s_misc)) return;

      // ---------------------------------------------------------- phase 5
      constexpr int DS = BITS + 2, DSS = (BITS + 2 + 3) / 4 * 4;   // DSS == cumD_stride
      int* gD = reinterpret_cast<int*>(ring + align_up(sizeof(int) * a.slice_pages, 16) +
                                       align_up(sizeof(uint16_t) * a.slice_tokens, 16));   // [C][DSS]
      copy_rows_async(smem_addr(gD),
                      reinterpret_cast<const char*>(a.wsCumD + static_cast<size_t>(unit * kMaxCtasPerUnit) * DSS),
                      a.C, DSS / 4, sizeof(int) * DSS, sizeof(int) * DSS, 0, DSS / 4);
      cp_async_wait<0>();
      __syncthreads();
      // partial totals: thread (part, v) sums rows part, part + PD, ...
      constexpr int PD = NT / DS;
      int* dPart = reinterpret_cast<int*>(rw);   // [PD][DS] (R/W is free)
      if (tid < PD * DS) {
        const int part = tid / DS, v = tid - part * DS;
        int x0 = 0, x1 = 0;
        int cc = part;
        for (; cc + PD < a.C; cc += 2 * PD) {
          x0 += gD[cc * DSS + v];
          x1 += gD[(cc + PD) * DSS + v];
        }
        if (cc < a.C) x0 += gD[cc * DSS + v];
        dPart[part * DS + v] = x0 + x1;
      }
      __syncthreads();
      // warp 0: tot[v] = tokens of the unit with distance < v; k_eff; the
      // threshold T (tot[T] < k_eff <= tot[T + 1]); then, in CTA order, each
      // CTA's quota of ties at T and its output offset
      if (warp == 0) {
        constexpr int QV = (DS + 31) / 32;
        int tot[QV];
#pragma unroll
        for (int qq = 0; qq < QV; ++qq) {
          const int v = lane + 32 * qq;
          int x = 0;
          if (v < DS) {
#pragma unroll
            for (int part = 0; part < PD; ++part) x += dPart[part * DS + v];
          }
          tot[qq] = x;
        }
        const int total = __shfl_sync(FULL, tot[(DS - 1) / 32], (DS - 1) % 32);
        const int k_eff = min(a.k, total);
        int n_lt = 0;
#pragma unroll
        for (int qq = 0; qq < QV; ++qq) n_lt += __popc(__ballot_sync(FULL, lane + 32 * qq < DS && tot[qq] < k_eff));
        const int T = k_eff > 0 ? n_lt - 1 : -1;   // tot[0] = 0 < k_eff
        int tT = 0;
#pragma unroll
        for (int qq = 0; qq < QV; ++qq) {
          const int v = __shfl_sync(FULL, tot[qq], T & 31);
          if (T >= 0 && (T >> 5) == qq) tT = v;
        }
        if (lane == 0) {
          s_misc[11] = T;
          s_misc[15] = k_eff;
        }
        const int needT = T >= 0 ? k_eff - tT : 0;
        int pre_eq = 0, off = 0;
        for (int c0 = 0; c0 < a.C; c0 += 32) {
          const int cc = c0 + lane;
          const int below = (cc < a.C && T >= 0) ? gD[cc * DSS + T] : 0;
          const int eq = (cc < a.C && T >= 0) ? gD[cc * DSS + T + 1] - below : 0;
          int eq_in = eq;
#pragma unroll
          for (int o2 = 1; o2 < 32; o2 <<= 1) {
            const int y = __shfl_up_sync(FULL, eq_in, o2);
            if (lane >= o2) eq_in += y;
          }
          const int quota = max(0, min(needT - (pre_eq + eq_in - eq), eq));
          const int selc = below + quota;
          int sel_in = selc;
#pragma unroll
          for (int o2 = 1; o2 < 32; o2 <<= 1) {
            const int y = __shfl_up_sync(FULL, sel_in, o2);
            if (lane >= o2) sel_in += y;
          }
          if (cc == c) {
            s_misc[12] = off + sel_in - selc;
            s_misc[13] = quota;
            s_misc[14] = selc;
          }
          pre_eq += __shfl_sync(FULL, eq_in, 31);
          off += __shfl_sync(FULL, sel_in, 31);
        }
      }
      __syncthreads();
      const int T = s_misc[11], k_eff = s_misc[15];   // threshold distance (-1: nothing selected)
      const int tok_off = s_misc[12], my_quota = s_misc[13], my_sel = s_misc[14];
      int* sel = reinterpret_cast<int*>(rw);   // this CTA's selected tokens (ascending)
      {
        // one packed scan: (tokens below T) | (tokens at T) << 16
        const int span = (ntok + NT - 1) / NT;
        const int lo = min(ntok, tid * span), hi = min(ntok, lo + span);
        int lt = 0, eq = 0;
        for (int i = lo; i < hi; ++i) {
          const int D = tokD[i];
          lt += D < T;
          eq += D == T;
        }
        int tmp;
        const int pre = block_excl_scan1(lt | (eq << 16), s_scan1, &tmp);
        int lt_b = pre & 0xFFFF, eq_b = pre >> 16;
        int32_t* tout = a.tok_idx + static_cast<size_t>(unit) * a.k;
        for (int i = lo; i < hi; ++i) {
          const int D = tokD[i];
          int pos = -1;
          if (D < T) {
            pos = lt_b + min(eq_b, my_quota);
            ++lt_b;
          } else if (D == T) {
            if (eq_b < my_quota) pos = lt_b + eq_b;
            ++eq_b;
          }
          if (pos >= 0) {
            const int slot = i / S_;
            const int n = my_pages[slot] * S_ + (i - slot * S_);
            if (tok_off + pos < a.k) tout[tok_off + pos] = n;
            sel[pos] = n;
          }
        }
        if (c == 0) {
          if (tid == 0) a.n_sel[unit] = k_eff;
          for (int i = k_eff + tid; i < a.k; i += NT) tout[i] = -1;
        }
      }
      __syncthreads();

      if constexpr (MODE == kModeFused) {
        const uint32_t t3 = 3u * static_cast<uint32_t>(a.C);
        attend_and_finish<RG>(a, unit, c, sel, my_sel, ring, t3, s_misc);
      } else {
        if (tid == 0) {
          const uint32_t old = atom_add_acq_rel(ctr, 1u);
          if (old == 3u * a.C - 1u) atomicExch(ctr, 0u);
          asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        }
      }
      __syncthreads();
    }
  }
}

__global__ void wait_timeout_kernel(uint32_t* status, uint32_t* counter, unsigned long long spin) {
  if (threadIdx.x != 0) return;
  const long long t0 = clock64();
  while (ld_acquire(counter) < 1u) {
    if (static_cast<unsigned long long>(clock64() - t0) > spin) {
      atomicExch(status, static_cast<uint32_t>(HHR_ERR_TIMEOUT));
      return;
    }
    __nanosleep(64);
  }
}

template <int RG, int WORDS, int MODE>
cudaError_t launch_t(const DecodeArgs& a, size_t smem, cudaStream_t stream) {
  auto kern = decode_kernel<RG, WORDS, MODE>;
  static std::atomic<size_t> raised[kMaxDevices];
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), smem, raised);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.grid_units * a.C));
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  // programmatic dependent launch: the kernel's CTAs may become resident
  // while the previous kernel on the stream finishes (griddepcontrol.wait
  // at the kernel's start keeps the two steps' work ordered)
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int RG, int WORDS>
cudaError_t launch_mode(const DecodeArgs& a, int mode, size_t smem, cudaStream_t stream) {
  switch (mode) {
    case kModeSelect: return launch_t<RG, WORDS, kModeSelect>(a, smem, stream);
    case kModeFused: return launch_t<RG, WORDS, kModeFused>(a, smem, stream);
    case kModeAttend: return launch_t<RG, WORDS, kModeAttend>(a, smem, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <int RG>
cudaError_t launch_bits(const DecodeArgs& a, int bits, int mode, size_t smem, cudaStream_t stream) {
  switch (bits) {
    case 128: return launch_mode<RG, 4>(a, mode, smem, stream);
    case 256: return launch_mode<RG, 8>(a, mode, smem, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, int r, int bits, int mode, size_t smem_bytes,
                          cudaStream_t stream) {
  switch (r) {
    case 1: return launch_bits<1>(a, bits, mode, smem_bytes, stream);
    case 2: return launch_bits<2>(a, bits, mode, smem_bytes, stream);
    case 4: return launch_bits<4>(a, bits, mode, smem_bytes, stream);
    case 8: return launch_bits<8>(a, bits, mode, smem_bytes, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_wait_timeout(uint32_t* status, uint32_t* counter, unsigned long long spin,
                                cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(status, counter, spin);
  return cudaGetLastError();
}

}  // namespace hhr
