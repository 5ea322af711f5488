// Decode-time retrieval kernels for sm_100a.
//
// One (sequence, KV head) pair -- a "unit" -- is spread over C CTAs of a
// cooperative launch.  A fused step runs these phases per unit:
//
//   0  query prep      R arrives by one bulk copy; q~ = q R (Eq. 4) for the
//                      r query heads of the group, while every warp starts
//                      streaming its own run of page metadata into a
//                      lane-private shared-memory ring (cp.async, 16 B per
//                      lane and page)
//   1  page bounds     U_p = max_h sum_j max(q~_hj l_pj, q~_hj u_pj)  (Eq. 3)
//                      over this CTA's contiguous slice of pages, as a
//                      tensor-core product of 16-page tiles of the stored
//                      bounds with the exact bf16 terms of min(q~, 0) and
//                      max(q~, 0); then the query codes (Eq. 10, sign) from W
//      -- unit barrier 1 (U published in the workspace) --
//   2  page top-P      every CTA reads all U of its unit and finds the same
//                      P largest (ties to the lower page) with a 2048-bin
//                      histogram over [min U, max U] plus an exact ranking of
//                      the boundary bin
//   3  compaction      kept pages in ascending order; CTA c takes the c-th
//                      slice of them
//   4  Hamming         D_n = min_h popc(qcode_h xor code_n) (Eq. 2) for the
//                      tokens of the slice, one 16/32-B code load per token;
//                      a (b+1)-bin histogram of D is published
//      -- unit barrier 2 --
//   5  token top-k     the histograms of all CTAs give the threshold distance
//                      and each CTA's output offset; ties at the threshold go
//                      to the lower token index across CTAs
//   6  attention       each CTA attends over its own selected tokens in tiles
//                      of 16 per warp on the tensor cores: K/V rows staged by
//                      cp.async, online softmax in float32
//      -- last-arriving CTA merges the C partial softmax states --
//
// Variants chosen by hhr_dims.flags (compiled into a second instantiation;
// with every flag 0 their branches are compiled out): float32 page metadata
// (phase 1 on the CUDA cores, 1-KiB pages), GQA-sum distances (phase 4 sums
// over the group's heads; r*b + 1 histogram bins), and phase 1 on the CUDA
// cores for bf16 metadata (the comparison form of the tensor-core tiles).
// The attend-only launch also serves dense attention over every valid key
// (each CTA one contiguous key range, no token list).
//
// The kernel is launched as a programmatic dependent of the previous kernel
// on the stream; its set-up touches no global memory and may overlap that
// kernel's tail, and it waits for it before the first global access.  Inter-CTA waits
// spin on workspace counters with a clock64() limit; on expiry the kernel
// records HHR_ERR_TIMEOUT and returns.  The last CTA of a unit resets its
// counter, so the workspace is zero again after each call.

#include <cuda_bf16.h>

#include <cfloat>
#include <cstdint>
#include <type_traits>

#include "hhr_internal.cuh"

namespace hhr {
namespace {

constexpr int NT = kDecodeThreads;
constexpr int NWARPS = NT / 32;


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

// Arrival on a unit barrier: release (the CTA's prior writes, made visible to
// thread 0 by a CTA barrier, become visible before the count), no result.
__device__ __forceinline__ void red_add_release(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(d), "l"(gmem_src) : "memory");
}
// Copies 16 B when src_bytes is 16, writes 16 zero bytes when it is 0.
__device__ __forceinline__ void cp_async16_zfill(void* smem_dst, const void* gmem_src, uint32_t src_bytes) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(d), "l"(gmem_src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes) : "memory");
}

// 1-D bulk copy global -> shared on the TMA unit; completion is signalled on
// the mbarrier as transferred bytes.  Both addresses 16-B aligned, size a
// multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// The same copy with an L2 cache policy: evict-last for the small tensors
// every step re-reads (R, W).
__device__ __forceinline__ void bulk_g2s_keep(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
               :: "r"(dst), "l"(src), "r"(bytes), "r"(bar), "l"(pol) : "memory");
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

// Exclusive prefix sum over the CTA.  Every thread must call it.
__device__ int block_excl_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int w = lane < NWARPS ? s_warp[lane] : 0;
    int wx = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, wx, o);
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
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
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

__device__ __forceinline__ uint32_t order_key(float u) {
  const uint32_t x = __float_as_uint(u + 0.0f);  // -0 -> +0
  return (x & 0x80000000u) ? ~x : (x | 0x80000000u);
}

// Exact top-`Pk` of the NP bounds in sU, ties to the lower page index, as a
// bitmap: a 32-step bitwise search for the Pk-th largest order key, then a
// page-order scan for the ties.  Used only when very many bounds fall into
// one histogram bin (degenerate inputs), so it is kept out of line.
__device__ __noinline__ void exact_top_pages(const float* sU, int NP, int Pk, int* s_scan,
                                             uint32_t* sBits) {
  const int tid = threadIdx.x;
  uint32_t T = 0u;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    int cnt = 0;
    for (int p = tid; p < NP; p += NT) cnt += order_key(sU[p]) >= cand;
    if (block_sum(cnt, s_scan) >= Pk) T = cand;
  }
  int gt = 0;
  for (int p = tid; p < NP; p += NT) gt += order_key(sU[p]) > T;
  const int need_eq = Pk - block_sum(gt, s_scan);
  const int span = (NP + NT - 1) / NT;
  const int lo = tid * span, hi = min(NP, lo + span);
  int eq = 0;
  for (int p = lo; p < hi; ++p) eq += order_key(sU[p]) == T;
  int eqtot;
  int er = block_excl_scan(eq, s_scan, &eqtot);
  for (int p = lo; p < hi; ++p) {
    const uint32_t kk = order_key(sU[p]);
    bool keep = kk > T;
    if (kk == T) keep = (er++ < need_eq);
    if (keep) atomicOr(&sBits[p >> 5], 1u << (p & 31));
  }
}

// For a histogram of kBuckets bins and a count `need` >= 1 not above its
// total, finds the bin b* holding the need-th largest element (bins ordered
// by value) and the number of elements in bins above b*.  Thread t owns the
// four bins [4(NT-1-t), 4(NT-1-t) + 4), so a scan in thread order counts the
// elements in higher bins.  Every thread must call it; results in out[0..1].
__device__ void find_boundary(const int* hist, int need, int* s_warp, int* out) {
  static_assert(kBuckets == 4 * NT, "bin ownership assumes 4 bins per thread");
  const int base = 4 * (NT - 1 - static_cast<int>(threadIdx.x));
  const int c4 = hist[base] + hist[base + 1] + hist[base + 2] + hist[base + 3];
  int tot;
  int running = block_excl_scan(c4, s_warp, &tot);
  for (int bin = base + 3; bin >= base; --bin) {
    const int hcount = hist[bin];
    if (running < need && running + hcount >= need) {
      out[0] = bin;
      out[1] = running;
    }
    running += hcount;
  }
  __syncthreads();
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

// x[r][d] . M[d][d] (both float32 in shared memory), in eight row groups:
// thread t forms, for every head h, the partial sums over rows
// [16 (t / 64), 16 (t / 64) + 16) of columns 2 (t % 64) and 2 (t % 64) + 1
// with packed float32 FMAs.  M is read once per CTA, conflict-free; x by
// broadcast.
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

// ldmatrix: four (two) 8x8 b16 matrices; lane i supplies the row address of
// matrix i / 8, row i % 8 (lanes 0-15 for x2).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                              uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1) : "r"(addr) : "memory");
}

// d += A (16 x 16, row-major bf16) * B (16 x 8, column-major bf16), fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
               "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// v = hi + mid + lo exactly, each term a bf16 (v - hi and the next residual
// are exact in float32, and the last residual has at most 8 significant
// bits).  Stores the terms at column k of rows n0, n0 + 1, n0 + 2 of the
// [rows][256] bf16 operand whose 16-B chunks are swizzled by row & 7.
__device__ __forceinline__ void put_terms(uint16_t* qb, int n0, int k, float v) {
  float rest = v;
#pragma unroll
  for (int t = 0; t < 3; ++t) {
    const __nv_bfloat16 term = __float2bfloat16_rn(rest);
    rest -= __bfloat162float(term);
    const int n = n0 + t;
    qb[n * (2 * kD) + (((k >> 3) ^ (n & 7)) << 3) + (k & 7)] = __bfloat16_as_ushort(term);
  }
}

struct Smem {
  uint16_t* qb;    // bf16 terms of [min(q~, 0) ; max(q~, 0)], [8 nb][2 d], 16-B chunks swizzled
  float* qf;       // [r][d] queries (float), pre-scaled for attention
  float* qt;       // [r][d] q~ = q R (float), for float32 metadata
  uint32_t* qc;    // [r][w] query codes
  int* my_pages;   // kept pages of this CTA's slice
  uint16_t* tokD;  // distances of the slice's tokens
  int* sel;        // selected tokens of this CTA (ascending)
  unsigned char* scratch;
};

// One warp merges n partial softmax states of one head; lane l takes the V
// consecutive columns j0 + V l.  State i keeps its unnormalised outputs at
// o[i * stride + column], its running max (base-2 logits) at ml[i * stride]
// and its sum at ml[i * stride + 1]; an empty state has max -inf and sum 0.
// With M = max_i m_i and weights w_i = 2^(m_i - M) (all zero when every state
// is empty), res = sum_i w_i o_i over the lane's columns, and M and
// L = sum_i w_i l_i in every lane.  The first kLoads states' outputs are
// loaded at once (all in flight together; V = 4: 16-B loads, o, stride and
// j0 multiples of 4 floats), the rest one by one; n <= 64.  kL2: the states
// were written by other CTAs of this kernel, so they are read from L2.
template <int kLoads, bool kL2, int V>
__device__ __forceinline__ void merge_states(const float* o, const float* ml, int stride, int n, int j0,
                                             float (&res)[V], float& M, float& L) {
  static_assert(kLoads <= 32 && (V == 1 || V == 4), "lane i holds the weight of state i (and of 32 + i)");
  const int lane = threadIdx.x & 31;
  auto ld = [](const float* p) { return kL2 ? __ldcg(p) : *p; };
  auto ldv = [&](int i, float (&dst)[V]) {
    const float* p = o + i * stride + j0 + V * lane;
    if constexpr (V == 4) {
      const float4 t = kL2 ? __ldcg(reinterpret_cast<const float4*>(p)) : *reinterpret_cast<const float4*>(p);
      dst[0] = t.x;
      dst[1] = t.y;
      dst[2] = t.z;
      dst[3] = t.w;
    } else {
      dst[0] = ld(p);
    }
  };
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  if (lane < n) {
    m0 = ld(ml + lane * stride);
    l0 = ld(ml + lane * stride + 1);
  }
  if (lane + 32 < n) {
    m1 = ld(ml + (lane + 32) * stride);
    l1 = ld(ml + (lane + 32) * stride + 1);
  }
  float ov[kLoads][V];
#pragma unroll
  for (int i = 0; i < kLoads; ++i) {
    if (i < n) {
      ldv(i, ov[i]);
    } else {
#pragma unroll
      for (int v = 0; v < V; ++v) ov[i][v] = 0.f;
    }
  }
  float mx = fmaxf(m0, m1);
#pragma unroll
  for (int o2 = 16; o2 >= 1; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o2));
  const float w0 = (mx == -INFINITY) ? 0.f : exp2f(m0 - mx);
  const float w1 = (mx == -INFINITY) ? 0.f : exp2f(m1 - mx);
  float ls = fmaf(l0, w0, l1 * w1);
#pragma unroll
  for (int o2 = 16; o2 >= 1; o2 >>= 1) ls += __shfl_xor_sync(0xFFFFFFFFu, ls, o2);
  M = mx;
  L = ls;
#pragma unroll
  for (int v = 0; v < V; ++v) res[v] = 0.f;
#pragma unroll
  for (int i = 0; i < kLoads; ++i) {
    const float w = __shfl_sync(0xFFFFFFFFu, w0, i);
#pragma unroll
    for (int v = 0; v < V; ++v) res[v] = fmaf(ov[i][v], w, res[v]);
  }
  for (int i = kLoads; i < n; ++i) {   // warp-uniform trip count
    const float w = __shfl_sync(0xFFFFFFFFu, i < 32 ? w0 : w1, i & 31);
    float t[V];
    ldv(i, t);
#pragma unroll
    for (int v = 0; v < V; ++v) res[v] = fmaf(t[v], w, res[v]);
  }
}

// ----------------------------------------------------------------------------
// Phase 6: attention of the r heads over `cnt` tokens listed in sel[], then
// the per-unit merge.
//
// Warp w takes tiles of 16 selected tokens (tiles w, w + 16, ...).  Their K
// and V rows are staged in the warp's own 8 KB of shared memory (16-B chunk c
// of token row r at position c ^ (r & 7), so that ldmatrix is conflict-free)
// and both products run on the tensor cores with fp32 accumulation:
//   S = Q K^T   m16n8k16, rows = the r heads (bf16 queries, unscaled, so
//               the products are exact), columns = tokens;
//   O += P V    rows 0-7 = the bf16 value of each head's softmax weights,
//               rows 8-15 = the bf16 remainder, so P loses no precision.
// Online softmax in float32 (exp2 with the scale folded in).  The next
// tile's K is fetched during the softmax and P V, its V during the next Q K^T.
template <int RG, bool kDense = false>
__device__ void attend_and_finish(const DecodeArgs& a, int unit, int c, const int* sel, int cnt,
                                  const float* qf,
                                  unsigned char* scratch, uint32_t final_target, int* s_int,
                                  int dense0 = 0) {
  static_assert(RG <= 8, "the heads fill at most the upper 8 rows of an m16 tile");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g8 = lane >> 2, t4 = lane & 3;      // mma fragment: row (head), column pair
  const int lm = lane >> 3, lr = lane & 7;      // ldmatrix: matrix, row
  const int b = unit / a.Hkv, g = unit % a.Hkv;
  const size_t unit_rows = static_cast<size_t>(unit) * a.n_cap;
  const uint16_t* Ku = a.K + unit_rows * kD;
  const uint16_t* Vu = a.V + unit_rows * kD;

  unsigned char* kbuf = scratch + warp * 8192;
  unsigned char* vbuf = kbuf + 4096;
  const uint32_t kb_s = smem_addr(kbuf), vb_s = smem_addr(vbuf);
  const int n_tiles = (cnt + 15) / 16;
  // every lane: 8 of the tile's 256 16-B chunks of K (or V), one commit group;
  // rows past cnt are zero-filled
  auto issue = [&](const uint16_t* base, unsigned char* buf, int tile) {
    if (tile < n_tiles) {
      const int ch = lane & 15;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = (lane >> 4) + 2 * i;
        const int t = tile * 16 + r;
        const bool ok = t < cnt;
        // the token: sel[t], or dense0 + t without a list (dense attention)
        const int tok = kDense ? dense0 + t : (ok ? sel[t] : 0);
        const uint16_t* src = ok ? base + static_cast<size_t>(tok) * kD + ch * 8 : base;
        cp_async16_zfill(buf + r * 256 + ((ch ^ (r & 7)) << 4), src, ok ? 16u : 0u);
      }
    }
    cp_async_commit();
  };

  float o[kD / 8][4];
#pragma unroll
  for (int nt = 0; nt < kD / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;

  issue(Ku, kbuf, warp);
  issue(Vu, vbuf, warp);
  // The group's queries as the A tile of Q K^T in shared memory (above the
  // warps' K / V buffers): row h < r is head h, rows r..15 are zero; 16-B
  // chunk c of row h sits at c ^ (h & 7).  Fragments are read per k-step
  // with ldmatrix rather than held in registers.
  unsigned char* qtile = scratch + NWARPS * 8192;
  if (tid < 16 * 16) {
    const int h = tid >> 4, ch = tid & 15;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (h < RG) {
      if (qf) {   // the group's queries are already in shared memory as float (exact bf16 values)
        const float4 lo = *reinterpret_cast<const float4*>(qf + h * kD + ch * 8);
        const float4 hi = *reinterpret_cast<const float4*>(qf + h * kD + ch * 8 + 4);
        v.x = (__float_as_uint(lo.x) >> 16) | (__float_as_uint(lo.y) & 0xFFFF0000u);
        v.y = (__float_as_uint(lo.z) >> 16) | (__float_as_uint(lo.w) & 0xFFFF0000u);
        v.z = (__float_as_uint(hi.x) >> 16) | (__float_as_uint(hi.y) & 0xFFFF0000u);
        v.w = (__float_as_uint(hi.z) >> 16) | (__float_as_uint(hi.w) & 0xFFFF0000u);
      } else {
        v = __ldg(reinterpret_cast<const uint4*>(a.q + (static_cast<size_t>(b) * a.Hq + g * RG + h) * kD) + ch);
      }
    }
    *reinterpret_cast<uint4*>(qtile + h * 256 + ((ch ^ (h & 7)) << 4)) = v;
  }
  __syncthreads();   // (the first K / V tiles are already in flight)
  const uint32_t q_row = smem_addr(qtile) + ((lm & 1) * 8 + lr) * 256;
  for (int tile = warp; tile < n_tiles; tile += NWARPS) {
    cp_async_wait<1>();   // this lane's K chunks of the tile
    __syncwarp();         // ... and every lane's
    float sacc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll 2
    for (int ks = 0; ks < kD / 16; ++ks) {
      uint32_t b0, b1, b2, b3;
      uint32_t a0, a1, a2, a3;
      ldsm_x4(q_row + (static_cast<uint32_t>((2 * ks + (lm >> 1)) ^ lr) << 4), a0, a1, a2, a3);
      ldsm_x4(kb_s + ((lm >> 1) * 8 + lr) * 256 + (static_cast<uint32_t>((2 * ks + (lm & 1)) ^ lr) << 4),
              b0, b1, b2, b3);
      mma_bf16_16816(sacc[0], a0, a1, a2, a3, b0, b1);
      mma_bf16_16816(sacc[1], a0, a1, a2, a3, b2, b3);
    }
    __syncwarp();
    issue(Ku, kbuf, tile + NWARPS);

    // head g8's scores of tokens 2 t4, 2 t4 + 1, 8 + 2 t4, 9 + 2 t4
    const int valid = cnt - tile * 16;
    float sc[4] = {sacc[0][0], sacc[0][1], sacc[1][0], sacc[1][1]};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int tok = (e >> 1) * 8 + 2 * t4 + (e & 1);
      sc[e] = tok < valid ? sc[e] * a.scale_log2 : -INFINITY;
    }
    float mx = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
    const float m_new = fmaxf(m_run, mx);       // finite: the tile has a valid token
    const float alpha = exp2f(m_run - m_new);   // 0 while m_run is -inf
    float pr[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) pr[e] = exp2f(sc[e] - m_new);
    float ps = (pr[0] + pr[1]) + (pr[2] + pr[3]);
    ps += __shfl_xor_sync(0xFFFFFFFFu, ps, 1);
    ps += __shfl_xor_sync(0xFFFFFFFFu, ps, 2);
    l_run = fmaf(l_run, alpha, ps);
    m_run = m_new;
    uint32_t pa[4];
    {
      uint16_t hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat16 h16 = __float2bfloat16_rn(pr[e]);
        hi[e] = __bfloat16_as_ushort(h16);
        lo[e] = __bfloat16_as_ushort(__float2bfloat16_rn(pr[e] - __bfloat162float(h16)));
      }
      pa[0] = hi[0] | (static_cast<uint32_t>(hi[1]) << 16);   // row g8, tokens 2 t4, + 1
      pa[1] = lo[0] | (static_cast<uint32_t>(lo[1]) << 16);   // row g8 + 8
      pa[2] = hi[2] | (static_cast<uint32_t>(hi[3]) << 16);   // row g8, tokens 8 + 2 t4, + 1
      pa[3] = lo[2] | (static_cast<uint32_t>(lo[3]) << 16);
    }
#pragma unroll
    for (int nt = 0; nt < kD / 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[nt][e] *= alpha;

    cp_async_wait<1>();   // this lane's V chunks of the tile
    __syncwarp();
#pragma unroll
    for (int np = 0; np < kD / 16; ++np) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_trans(vb_s + ((lm & 1) * 8 + lr) * 256 + (static_cast<uint32_t>((2 * np + (lm >> 1)) ^ lr) << 4),
                    b0, b1, b2, b3);
      mma_bf16_16816(o[2 * np], pa[0], pa[1], pa[2], pa[3], b0, b1);
      mma_bf16_16816(o[2 * np + 1], pa[0], pa[1], pa[2], pa[3], b2, b3);
    }
    __syncwarp();
    issue(Vu, vbuf, tile + NWARPS);
  }
  cp_async_wait<0>();
  __syncthreads();   // the merge buffer below overlays the K / V tiles

  // merge the 16 warp states through shared memory: [warp][h][d + 2]
  float* mer = reinterpret_cast<float*>(scratch);
  if (g8 < RG) {
    float* dst = mer + (warp * RG + g8) * (kD + 2);
#pragma unroll
    for (int nt = 0; nt < kD / 8; ++nt) {
      dst[8 * nt + 2 * t4] = o[nt][0] + o[nt][2];
      dst[8 * nt + 2 * t4 + 1] = o[nt][1] + o[nt][3];
    }
    if (t4 == 0) {
      dst[kD] = m_run;
      dst[kD + 1] = l_run;
    }
  }
  __syncthreads();

  // the CTA's state: warp item = (head h, 32-column block) merges the 16
  // warp states of its columns.  Stored as [r][d] outputs, then (max, sum)
  // per head, so that each head's outputs are 16-B aligned.
  constexpr int PS = part_stride(RG);
  float* part = a.wsPart + static_cast<size_t>(unit * kMaxCtasPerUnit + c) * PS;
  for (int item = warp; item < RG * (kD / 32); item += NWARPS) {
    const int h = item / (kD / 32), j0 = (item % (kD / 32)) * 32;
    float M, L, O[1];
    merge_states<NWARPS, false, 1>(mer + h * (kD + 2), mer + h * (kD + 2) + kD, RG * (kD + 2), NWARPS, j0, O, M, L);
    if (a.C == 1) {
      a.out[(static_cast<size_t>(b) * a.Hq + g * RG + h) * kD + j0 + lane] = (L > 0.f) ? O[0] / L : 0.f;
    } else {
      part[h * kD + j0 + lane] = O[0];
      if (lane == 0) {
        part[RG * kD + 2 * h] = M;
        part[RG * kD + 2 * h + 1] = L;
      }
    }
  }

  // last CTA of the unit merges the C partial states and resets the counter
  __syncthreads();
  if (tid == 0) {
    const uint32_t old = atom_add_acq_rel(a.counters + unit, 1u);
    s_int[0] = (old == final_target - 1) ? 1 : 0;
    // this CTA's share of the step is done but for the final merge: the
    // next kernel on the stream may start launching (it waits for the
    // completion of this one before touching memory)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }
  __syncthreads();
  if (!s_int[0]) return;
  if (a.C > 1) {
    // the C partial states of the unit, straight from L2: one warp per
    // head, four columns a lane, the loads of up to 20 states all in flight
    // at once (16-B loads: many single-float loads in flight from one SM
    // take several L2 round trips)
    const float* parts = a.wsPart + static_cast<size_t>(unit * kMaxCtasPerUnit) * PS;
    for (int h = warp; h < RG; h += NWARPS) {
      float M, L, O[4];
      merge_states<20, true, 4>(parts + h * kD, parts + RG * kD + 2 * h, PS, a.C, 0, O, M, L);
      float* dst = a.out + (static_cast<size_t>(b) * a.Hq + g * RG + h) * kD + 4 * lane;
#pragma unroll
      for (int v = 0; v < 4; ++v) dst[v] = (L > 0.f) ? O[v] / L : 0.f;
    }
  }
  if (tid == 0) atomicExch(a.counters + unit, 0u);
}

// ----------------------------------------------------------------------------
// VAR: the variant flags (float32 metadata, GQA-sum, SIMT bounds) may be set;
// false compiles their branches out (every flag 0, the default readings).
template <int RG, int WORDS, int MODE, bool VAR>
__global__ void __launch_bounds__(NT, 1) decode_kernel(const __grid_constant__ DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_int[NWARPS + 16];
  __shared__ int s_scan1[NWARPS];
  __shared__ int s_aux[264];  // distance totals (<= 257 bins)
  __shared__ float s_flt[4];
  constexpr int BITS = WORDS * 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x % a.C;
  // the variant flags, compile-time false without VAR
  const bool meta_f32 = VAR && a.meta_f32, gqa_sum = VAR && a.gqa_sum, simt_bounds = VAR && a.simt_bounds;
  const int hbins = VAR ? a.hbins : BITS + 1;
  const DecodeSmem lay = decode_smem(a.NP, a.C, BITS, RG, a.slice_pages, a.slice_tokens, MODE, hbins);
  Smem S;
  S.qb = reinterpret_cast<uint16_t*>(smem + lay.qb);
  S.qf = reinterpret_cast<float*>(smem + lay.qf);
  S.qt = reinterpret_cast<float*>(smem + lay.qt);
  S.qc = reinterpret_cast<uint32_t*>(smem + lay.qc);
  S.my_pages = reinterpret_cast<int*>(smem + lay.my_pages);
  S.tokD = reinterpret_cast<uint16_t*>(smem + lay.tokD);
  S.sel = reinterpret_cast<int*>(smem + lay.sel);
  S.scratch = smem + lay.scratch;
  int* s_scan = s_int;              // NWARPS + 1 entries
  int* s_misc = s_int + NWARPS + 1; // scalars
  __shared__ __align__(8) unsigned long long s_rwbar;                       // W staging
  const uint32_t rw_addr = smem_addr(&s_rwbar);
  uint32_t rw_seq = 0;  // W phases used so far
  float* sRW = reinterpret_cast<float*>(S.scratch + NWARPS * kLaneSlots * 512);  // R / W staging
  // thread 0: one bulk copy of the d x d rotation of KV head g into sRW
  auto issue_r = [&](int g) {
    // the storage may last have been touched by generic-proxy accesses
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_expect_tx(rw_addr, kD * kD * sizeof(float));
    bulk_g2s_keep(smem_addr(sRW), a.R + static_cast<size_t>(g) * kD * kD, kD * kD * sizeof(float), rw_addr);
  };
  const int unit0 = blockIdx.x / a.C;
  // this CTA's page range and its warp's share of it (the same for every unit)
  const int pb = c * a.NP / a.C;      // c * NP < 2^20 (NP <= HHR_MAX_PAGES)
  const int pe = (c + 1) * a.NP / a.C;
  const int my_pages = pe - pb;
  const int wpb = pb + my_pages * warp / NWARPS;
  const int wpe = pb + my_pages * (warp + 1) / NWARPS;
  const int w_pages = wpe - wpb;
  if (tid == 0) {
    mbar_init(rw_addr, 1u);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if constexpr (MODE != kModeAttend) {
    // the B operand's unused columns (fourth term of each head, absent heads) stay zero
    for (int i = tid; i < 8 * ((RG * 4 + 7) / 8) * 2 * kD; i += NT) S.qb[i] = 0;
  }
  // Launched as a programmatic dependent of the previous kernel on the
  // stream: the set-up above touches no global memory and may overlap that
  // kernel's tail; from here on, its writes are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the first unit's R goes out before anything else: the query transform
  // waits on it
  if constexpr (MODE != kModeAttend)
    if (tid == 0 && unit0 < a.units) issue_r(unit0 % a.Hkv);
  __syncthreads();

  for (int unit = unit0; unit < a.units; unit += a.grid_units) {
    const int b = unit / a.Hkv, g = unit % a.Hkv;

    uint32_t* ctr = a.counters + unit;

    const uint16_t* qg = a.q + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(g) * RG) * kD;

    if constexpr (MODE == kModeAttend) {
      if (a.dense) {
        // dense attention over all n_valid keys: this CTA's contiguous
        // share, c * n / C .. (c + 1) * n / C (c * n < 2^26: n <= HHR_MAX_PAGES * 64)
        const int n = a.n_valid;
        const int s0 = c * n / a.C, s1 = (c + 1) * n / a.C;
        attend_and_finish<RG, true>(a, unit, c, nullptr, s1 - s0, nullptr, S.scratch, static_cast<uint32_t>(a.C),
                              s_misc, s0);
        __syncthreads();
        continue;
      }
      const int n = a.nsel_in[unit];
      const int s0 = c * n / a.C;         // c * n < 2^26 (n <= C * kMaxTokensPerCta)
      const int s1 = (c + 1) * n / a.C;
      const int32_t* src = a.tok_in + static_cast<size_t>(unit) * a.k;
#pragma unroll 8
      for (int i = s0 + tid; i < s1; i += NT) S.sel[i - s0] = src[i];
      __syncthreads();
      attend_and_finish<RG>(a, unit, c, S.sel, s1 - s0, nullptr, S.scratch, static_cast<uint32_t>(a.C), s_misc);
      __syncthreads();
      continue;
    } else {
      // ---------------------------------------------------------- phase 0
      // R reaches shared memory ahead of any metadata.  Every warp streams
      // its own run of pages into a lane-private ring: the first kLaneSlots
      // pages of each warp at once, the rest of the ring -- which shares its
      // storage with R -- as soon as q~ = q R is formed.  W follows by bulk
      // copy on an mbarrier once the ring has drained.
      const float* Wg = a.W + static_cast<size_t>(g) * kD * BITS;
      auto issue_w = [&](int half_w) {  // thread 0 only: 128 columns of W
        // the storage was last touched by generic-proxy copies and loads
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_expect_tx(rw_addr, kD * kD * sizeof(float));
        if constexpr (BITS == kD) {
          bulk_g2s_keep(smem_addr(sRW), Wg, kD * kD * sizeof(float), rw_addr);
        } else {
          for (int i = 0; i < kD; ++i)
            bulk_g2s_keep(smem_addr(sRW + i * kD), Wg + static_cast<size_t>(i) * BITS + half_w * kD,
                     kD * sizeof(float), rw_addr);
        }
      };
      // thread 0 waits for the next W phase; false (all threads) on timeout
      auto wait_rw = [&]() {
        const bool ok = (tid == 0) ? mbar_wait(rw_addr, rw_seq & 1u, a.spin_limit) : true;
        ++rw_seq;
        return !__syncthreads_or(!ok);
      };

      // This warp's pages [wpb, wpe).  Lane l only ever reads bytes
      // [16 l, 16 l + 16) of a page, so it copies exactly those bytes into its
      // own shared-memory slots with cp.async and waits on its own copies: no
      // barrier is involved.  Slot s of warp w is the 512 B at
      // (s * NWARPS + w) * 512: slots [0, kLaneSlots) lie below the R / W
      // buffer, slots [kLaneSlots, kRingSlots) inside it.
      constexpr int PPG = 8;                        // pages per ring group; an A tile is two groups
      constexpr int G0 = 2;                         // groups in flight while q~ is formed (all below R / W)
      constexpr int GR = kRingSlots / PPG;          // groups in flight afterwards
      static_assert(kLaneSlots % PPG == 0 && kRingSlots % PPG == 0 && G0 * PPG <= kLaneSlots,
                    "whole groups per ring; the groups issued before q~ stay below the R / W buffer");
      static_assert(GR == 3, "tile ti reads groups 2 ti, 2 ti + 1 and refills them with 2 ti + 3, 2 ti + 4");
      static_assert((kRingSlots - kLaneSlots) * NWARPS * 512 == kD * kD * sizeof(float),
                    "the upper ring slots fill the R / W buffer exactly");
      const int n_grp = (w_pages + PPG - 1) / PPG;
      // bf16 metadata: a page is 512 B (32 x 16 B), one slot.  Within a slot,
      // 16-B chunk c sits at position c ^ (s & 7), so that the same chunk of 8
      // consecutive slots covers all banks (ldmatrix below).
      // f32 metadata: a page is 1 KiB, two slots (lower bounds, upper
      // bounds), PPG / 2 pages per group; lane l keeps chunk l of each half at
      // position l (it alone reads it back).
      const size_t meta_row = static_cast<size_t>(unit) * a.np_cap + wpb;   // first page of the warp
      const uint4* wsrc = reinterpret_cast<const uint4*>(a.meta) + meta_row * (meta_f32 ? 64 : 32) + lane;
      uint4* ring = reinterpret_cast<uint4*>(S.scratch) + warp * 32;
      auto issue_group = [&](int gi) {  // every lane: its 16 B of each page half, one commit group
        if (!meta_f32) {
          if (gi < n_grp) {
#pragma unroll
            for (int pp = 0; pp < PPG; ++pp) {
              const int pg = gi * PPG + pp;
              const int s = pg % kRingSlots;
              if (pg < w_pages)
                cp_async16(ring + s * (NWARPS * 32) + (lane ^ (s & 7)), wsrc + static_cast<size_t>(pg) * 32);
            }
          }
        } else {
#pragma unroll
          for (int pp = 0; pp < PPG / 2; ++pp) {
            const int pg = gi * (PPG / 2) + pp;
            const int s = (2 * pg) % kRingSlots;
            if (pg < w_pages) {
              cp_async16(ring + s * (NWARPS * 32) + lane, wsrc + static_cast<size_t>(pg) * 64);
              cp_async16(ring + (s + 1) * (NWARPS * 32) + lane, wsrc + static_cast<size_t>(pg) * 64 + 32);
            }
          }
        }
        cp_async_commit();
      };

      // R alone first, one bulk copy (the first unit's went out at the
      // kernel's start): requested together with the metadata it would land
      // only with the whole first burst
      if (tid == 0 && unit != unit0) issue_r(g);
      // queries of the group, as float (raw) -- q~ is derived from these
      for (int i = tid; i < RG * kD; i += NT) S.qf[i] = __uint_as_float(static_cast<uint32_t>(qg[i]) << 16);
      if (!wait_rw()) {
        if (tid == 0) {
          atomicExch(a.status, static_cast<uint32_t>(HHR_ERR_TIMEOUT));
          mbar_wait(rw_addr, (rw_seq - 1) & 1u, a.spin_limit);   // the copy may still be in flight
        }
        __syncthreads();
        return;
      }
#pragma unroll
      for (int gi = 0; gi < G0; ++gi) issue_group(gi);
      {
        float2 acc[RG];
        product_partials<RG>(S.qf, sRW, acc);
        __syncthreads();                            // every thread has read R
        float* part = sRW;                          // [8][r][d] row-group sums, over R
        store_partials<RG>(acc, part);
        __syncthreads();
        for (int oi = tid; oi < RG * kD; oi += NT) {
          const float qt = product_sum<RG>(part, oi);
          const int h = oi / kD, j = oi % kD;
          S.qt[oi] = qt;
          put_terms(S.qb, 4 * h, j, fminf(qt, 0.f));
          put_terms(S.qb, 4 * h, kD + j, fmaxf(qt, 0.f));
        }
        __syncthreads();
      }
      // the upper ring slots now own the R / W storage
#pragma unroll
      for (int gi = G0; gi < GR; ++gi) issue_group(gi);

      // ---------------------------------------------------------- phase 1
      // Eq. 3 as a contraction: with b_h = [min(q~_h, 0) ; max(q~_h, 0)] and a
      // page's stored bounds [l ; u] (256 bf16), U_p = max_h [l ; u] . b_h.
      // Each warp multiplies tiles of 16 of its pages -- A fragments loaded
      // by ldmatrix straight from its ring -- by B = the exact bf16 terms of
      // the b_h (4 columns per head) on the tensor cores, fp32 accumulation.
      constexpr int NB = (RG * 4 + 7) / 8;          // n8 column blocks of B
      float* wsU_u = a.wsU + static_cast<size_t>(unit) * a.np_stride;
      float lmin = INFINITY, lmax = -INFINITY;
      const int n_tiles = (w_pages + 15) / 16;
      const int lm = lane >> 3, lr = lane & 7;      // ldmatrix: matrix, row
      const int g8 = lane >> 2, t4 = lane & 3;      // mma fragment: row, column pair
      const uint32_t ring_s = smem_addr(S.scratch) + warp * 512;
      const uint32_t qb_s = smem_addr(S.qb);
      if (meta_f32) {
        // Eq. 3 on float32 bounds, on the CUDA cores: lane l holds dimensions
        // 4 l .. 4 l + 3 of a page's lower and upper bounds, forms
        // sum_j min(q~_hj, 0) l_j + max(q~_hj, 0) u_j over them for every head,
        // and the warp sums the 32 lanes (the path is bound by the 1-KiB pages'
        // HBM traffic, not by this arithmetic).
        float qv[RG][4];
#pragma unroll
        for (int h = 0; h < RG; ++h) {
          const float4 t = *reinterpret_cast<const float4*>(S.qt + h * kD + 4 * lane);
          qv[h][0] = t.x;
          qv[h][1] = t.y;
          qv[h][2] = t.z;
          qv[h][3] = t.w;
        }
        const int n_grp32 = (w_pages + PPG / 2 - 1) / (PPG / 2);
        for (int gi = 0; gi < n_grp32; ++gi) {
          cp_async_wait<GR - 1>();   // this lane's chunks of group gi have landed
#pragma unroll 1
          for (int pp = 0; pp < PPG / 2; ++pp) {
            const int pl = gi * (PPG / 2) + pp;
            if (pl >= w_pages) break;   // warp-uniform
            const int sl = (2 * pl) % kRingSlots;
            const float4 lo = *reinterpret_cast<const float4*>(ring + sl * (NWARPS * 32) + lane);
            const float4 hi = *reinterpret_cast<const float4*>(ring + (sl + 1) * (NWARPS * 32) + lane);
            float u = -INFINITY;
#pragma unroll
            for (int h = 0; h < RG; ++h) {
              float t = fminf(qv[h][0], 0.f) * lo.x;
              t = fmaf(fmaxf(qv[h][0], 0.f), hi.x, t);
              t = fmaf(fminf(qv[h][1], 0.f), lo.y, t);
              t = fmaf(fmaxf(qv[h][1], 0.f), hi.y, t);
              t = fmaf(fminf(qv[h][2], 0.f), lo.z, t);
              t = fmaf(fmaxf(qv[h][2], 0.f), hi.z, t);
              t = fmaf(fminf(qv[h][3], 0.f), lo.w, t);
              t = fmaf(fmaxf(qv[h][3], 0.f), hi.w, t);
#pragma unroll
              for (int o2 = 16; o2 >= 1; o2 >>= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, o2);
              u = fmaxf(u, t);
            }
            if (lane == 0) {
              const int pg = wpb + pl;
              wsU_u[pg] = u;
              if (a.dbg_U) a.dbg_U[static_cast<size_t>(unit) * a.NP + pg] = u;
            }
            lmin = fminf(lmin, u);
            lmax = fmaxf(lmax, u);
          }
          issue_group(gi + GR);   // refill this lane's slots of group gi
        }
      } else if (simt_bounds) {
        // Eq. 3 on bf16 bounds on the CUDA cores (HHR_FLAG_SIMT_BOUNDS, the
        // comparison form of the tensor-core tiles below): lane l holds the 8
        // bf16 values of chunk l of a page -- dimensions 8 (l % 16) .. + 7 of
        // the lower row (l < 16) or of the upper row -- and the matching
        // min(q~, 0) or max(q~, 0) of every head; the warp sums the 32 lanes.
        const int j0 = 8 * (lane & 15);
        const bool upper = lane >= 16;
        float qs[RG][8];
#pragma unroll
        for (int h = 0; h < RG; ++h)
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float v = S.qt[h * kD + j0 + e];
            qs[h][e] = upper ? fmaxf(v, 0.f) : fminf(v, 0.f);
          }
        for (int gi = 0; gi < n_grp; ++gi) {
          cp_async_wait<GR - 1>();   // this lane's chunks of group gi have landed
#pragma unroll 1
          for (int pp = 0; pp < PPG; ++pp) {
            const int pl = gi * PPG + pp;
            if (pl >= w_pages) break;   // warp-uniform
            const int sl = pl % kRingSlots;
            const uint4 raw = ring[sl * (NWARPS * 32) + (lane ^ (sl & 7))];
            const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
            float x[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              x[2 * e] = __uint_as_float(wv[e] << 16);
              x[2 * e + 1] = __uint_as_float(wv[e] & 0xFFFF0000u);
            }
            float u = -INFINITY;
#pragma unroll
            for (int h = 0; h < RG; ++h) {
              float t = qs[h][0] * x[0];
#pragma unroll
              for (int e = 1; e < 8; ++e) t = fmaf(qs[h][e], x[e], t);
#pragma unroll
              for (int o2 = 16; o2 >= 1; o2 >>= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, o2);
              u = fmaxf(u, t);
            }
            if (lane == 0) {
              const int pg = wpb + pl;
              wsU_u[pg] = u;
              if (a.dbg_U) a.dbg_U[static_cast<size_t>(unit) * a.NP + pg] = u;
            }
            lmin = fminf(lmin, u);
            lmax = fmaxf(lmax, u);
          }
          issue_group(gi + GR);   // refill this lane's slots of group gi
        }
      } else {
        for (int ti = 0; ti < n_tiles; ++ti) {
          cp_async_wait<1>();   // this lane's groups 2 ti and 2 ti + 1 have landed
          __syncwarp();         // ... and every lane's
          // A row (lm & 1) * 8 + lr of the tile is page 16 ti + that row
          const uint32_t a_row = ring_s + (((2 * ti + (lm & 1)) % GR) * PPG + lr) * (NWARPS * 512);
          float acc[NB][4];
  #pragma unroll
          for (int nb = 0; nb < NB; ++nb)
  #pragma unroll
            for (int e = 0; e < 4; ++e) acc[nb][e] = 0.f;
  #pragma unroll 4
          for (int ks = 0; ks < 2 * kD / 16; ++ks) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(a_row + (static_cast<uint32_t>((2 * ks + (lm >> 1)) ^ lr) << 4), a0, a1, a2, a3);
  #pragma unroll
            for (int nb = 0; nb < NB; nb += 2) {
              if (nb + 1 < NB) {
                uint32_t b0, b1, b2, b3;
                const int n = (nb + (lm >> 1)) * 8 + lr;
                ldsm_x4(qb_s + n * 512 + (static_cast<uint32_t>((2 * ks + (lm & 1)) ^ lr) << 4), b0, b1, b2, b3);
                mma_bf16_16816(acc[nb], a0, a1, a2, a3, b0, b1);
                mma_bf16_16816(acc[nb + 1], a0, a1, a2, a3, b2, b3);
              } else {
                uint32_t b0, b1;
                ldsm_x2(qb_s + (nb * 8 + lr) * 512 + (static_cast<uint32_t>((2 * ks + (lm & 1)) ^ lr) << 4), b0, b1);
                mma_bf16_16816(acc[nb], a0, a1, a2, a3, b0, b1);
              }
            }
          }
          __syncwarp();
          issue_group(2 * ti + GR);       // refill the slots just read
          issue_group(2 * ti + GR + 1);
          // lane (g8, t4) holds columns 8 nb + 2 t4, + 1 (head 2 nb + t4 / 2)
          // of tile rows g8 and g8 + 8: add the terms, then take the max over
          // the heads
          float u0 = -INFINITY, u1 = -INFINITY;
  #pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            float s0 = acc[nb][0] + acc[nb][1];
            float s1 = acc[nb][2] + acc[nb][3];
            s0 += __shfl_xor_sync(0xFFFFFFFFu, s0, 1);
            s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, 1);
            if (2 * nb + (t4 >> 1) >= RG) {
              s0 = -INFINITY;
              s1 = -INFINITY;
            }
            u0 = fmaxf(u0, fmaxf(s0, __shfl_xor_sync(0xFFFFFFFFu, s0, 2)));
            u1 = fmaxf(u1, fmaxf(s1, __shfl_xor_sync(0xFFFFFFFFu, s1, 2)));
          }
          if (t4 == 0) {
  #pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
              const int pl = ti * 16 + g8 + 8 * hr;
              if (pl < w_pages) {
                const float u = hr ? u1 : u0;
                const int pg = wpb + pl;
                wsU_u[pg] = u;
                if (a.dbg_U) a.dbg_U[static_cast<size_t>(unit) * a.NP + pg] = u;
                lmin = fminf(lmin, u);
                lmax = fmaxf(lmax, u);
              }
            }
          }
        }
      }
      cp_async_wait<0>();
      // CTA min / max of its bounds
#pragma unroll
      for (int o2 = 16; o2 >= 1; o2 >>= 1) {
        lmin = fminf(lmin, __shfl_xor_sync(0xFFFFFFFFu, lmin, o2));
        lmax = fmaxf(lmax, __shfl_xor_sync(0xFFFFFFFFu, lmax, o2));
      }
      float* red = reinterpret_cast<float*>(s_aux);
      if (lane == 0) {
        red[warp] = lmin;
        red[NWARPS + warp] = lmax;
      }
      // every lane's ring copies have landed and been read: the R / W
      // storage is free for W
      __syncthreads();
      if (warp == 0) {
        float mn = lane < NWARPS ? red[lane] : INFINITY;
        float mx = lane < NWARPS ? red[NWARPS + lane] : -INFINITY;
#pragma unroll
        for (int o2 = NWARPS / 2; o2 >= 1; o2 >>= 1) {
          mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o2));
          mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o2));
        }
        if (lane == 0) {
          float* mm2 = a.wsMinMax + 2 * static_cast<size_t>(unit * kMaxCtasPerUnit + c);
          mm2[0] = mn;
          mm2[1] = mx;
        }
      }
      if (tid == 0) {
        issue_w(0);
        // unit barrier 1: arrive now (the release covers the CTA's U through
        // the CTA barrier above), wait after the query codes
        red_add_release(ctr, 1u);
      }
      // query codes (Eq. 10 + sign) from W in shared memory, 128 columns at
      // a time, while the other CTAs of the unit finish their bounds
      int w_done = 0;
      bool q_ok = true;
      while (w_done < BITS / kD) {
        q_ok = wait_rw();
        if (!q_ok) break;
        float* part = reinterpret_cast<float*>(S.scratch);  // [8][r][d], in the drained ring
        {
          float2 acc[RG];
          product_partials<RG>(S.qf, sRW, acc);
          store_partials<RG>(acc, part);
        }
        __syncthreads();                            // partial sums visible, this W half read
        if (w_done + 1 < BITS / kD && tid == 0) issue_w(w_done + 1);
        for (int oi = tid; oi < RG * kD; oi += NT) {  // warp-uniform trip count
          const float z = product_sum<RG>(part, oi);
          const uint32_t word = __ballot_sync(0xFFFFFFFFu, z > 0.f);
          const int h = oi / kD, t = oi % kD;
          if (lane == 0) S.qc[h * WORDS + w_done * (kD / 32) + t / 32] = word;
        }
        ++w_done;
        if (w_done < BITS / kD) __syncthreads();    // part is rewritten next
      }
      if (__syncthreads_or(!q_ok)) {
        if (tid == 0) {
          atomicExch(a.status, static_cast<uint32_t>(HHR_ERR_TIMEOUT));
          mbar_wait(rw_addr, (rw_seq - 1) & 1u, a.spin_limit);   // a copy may still be in flight
        }
        __syncthreads();
        return;
      }
      if (!unit_wait(ctr, static_cast<uint32_t>(a.C) + (a.test_extra_stage == 1 ? 1u : 0u), a, s_misc)) return;

      // ---------------------------------------------------------- phase 2
      const int NP = a.NP, Pk = a.Pk;
      float* sU = reinterpret_cast<float*>(S.scratch);
      int* sHist = reinterpret_cast<int*>(S.scratch + sizeof(float) * align_up(NP, 4));
      uint32_t* sBits = reinterpret_cast<uint32_t*>(sHist + kBuckets);
      const int nwords = (NP + 31) / 32;
      float* sCU = reinterpret_cast<float*>(sBits + align_up(nwords, 4));
      int* sCP = reinterpret_cast<int*>(sCU + kCandMax);
      float* sC2U = reinterpret_cast<float*>(sCP + kCandMax);
      int* sC2P = reinterpret_cast<int*>(sC2U + kCandMax);
      // all U of the unit, float4 per thread, kept in registers for the
      // histogram (the tail of a ragged NP goes straight to shared memory)
      constexpr int kU4 = (HHR_MAX_PAGES / 4 + NT - 1) / NT;
      const int n4 = NP / 4;
      float4 ureg[kU4];
      {
        const float4* src4 = reinterpret_cast<const float4*>(wsU_u);
#pragma unroll
        for (int u = 0; u < kU4; ++u) {
          const int i = tid + u * NT;
          ureg[u] = i < n4 ? __ldcg(src4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int p = n4 * 4 + tid; p < NP; p += NT) sU[p] = __ldcg(wsU_u + p);
      }
      for (int i = tid; i < kBuckets; i += NT) sHist[i] = 0;
      for (int i = tid; i < nwords; i += NT) sBits[i] = 0u;
      if (warp == 0) {
        const float* mm2 = a.wsMinMax + 2 * static_cast<size_t>(unit * kMaxCtasPerUnit);
        float mn = INFINITY, mx = -INFINITY;
        for (int i = lane; i < a.C; i += 32) {
          mn = fminf(mn, __ldcg(mm2 + 2 * i));
          mx = fmaxf(mx, __ldcg(mm2 + 2 * i + 1));
        }
#pragma unroll
        for (int o2 = 16; o2 >= 1; o2 >>= 1) {
          mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o2));
          mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o2));
        }
        if (lane == 0) {
          s_flt[0] = mn;
          s_flt[1] = mx;
        }
      }
      if (tid == 0) s_misc[2] = 0;
      __syncthreads();
#pragma unroll
      for (int u = 0; u < kU4; ++u) {
        const int i = tid + u * NT;
        if (i < n4) reinterpret_cast<float4*>(sU)[i] = ureg[u];
      }

      if (Pk >= NP) {
        for (int p0 = warp * 32; p0 < NP; p0 += NT) {
          const unsigned word = __ballot_sync(0xFFFFFFFFu, p0 + lane < NP);
          if (lane == 0) sBits[p0 >> 5] = word;
        }
      } else {
        const float gmin = s_flt[0];
        const float range = s_flt[1] - gmin;
        const float inv = (range > 0.f && range <= FLT_MAX) ? static_cast<float>(kBuckets) / range : 0.f;
        // bin = round((u - gmin) * inv) by one FMA: the 1.5 * 2^23 offset
        // leaves the rounded integer in the low mantissa bits.  Monotone in u,
        // and histogram and extraction use the same map, which is all the
        // selection needs; clamped for any input (NaN included).
        auto bucket = [&](float u) {
          const int bk = __float_as_int(fmaf(u - gmin, inv, 12582912.f)) - 0x4B400000;
          return min(max(bk, 0), kBuckets - 1);
        };
#pragma unroll
        for (int u = 0; u < kU4; ++u) {
          if (tid + u * NT < n4) {
            const int b0 = bucket(ureg[u].x), b1 = bucket(ureg[u].y);
            const int b2 = bucket(ureg[u].z), b3 = bucket(ureg[u].w);
            atomicAdd(&sHist[b0], 1);
            atomicAdd(&sHist[b1], 1);
            atomicAdd(&sHist[b2], 1);
            atomicAdd(&sHist[b3], 1);
          }
        }
        for (int p = n4 * 4 + tid; p < NP; p += NT) atomicAdd(&sHist[bucket(sU[p])], 1);
        __syncthreads();
        find_boundary(sHist, Pk, s_scan, &s_misc[3]);
        const int bstar = s_misc[3];
        const int need = Pk - s_misc[4];
        const int cntB = sHist[bstar];
        // four bitmap words per warp step (independent chains)
        if (cntB == need) {
          for (int p0 = warp * 32; p0 < NP; p0 += 4 * NT) {
            bool keep[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int p = p0 + u * NT + lane;
              keep[u] = p < NP && bucket(sU[p]) >= bstar;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int pw = p0 + u * NT;  // warp-uniform
              const unsigned word = __ballot_sync(0xFFFFFFFFu, keep[u]);
              if (lane == 0 && pw < NP) sBits[pw >> 5] = word;
            }
          }
        } else if (cntB <= kCandMax) {
          for (int p0 = warp * 32; p0 < NP; p0 += 4 * NT) {
            int bk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int p = p0 + u * NT + lane;
              bk[u] = p < NP ? bucket(sU[p]) : -1;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int pw = p0 + u * NT;  // warp-uniform
              const unsigned word = __ballot_sync(0xFFFFFFFFu, bk[u] > bstar);
              if (lane == 0 && pw < NP) sBits[pw >> 5] = word;
              if (bk[u] == bstar) {
                const int slot = atomicAdd(&s_misc[2], 1);
                sCU[slot] = sU[pw + lane];
                sCP[slot] = pw + lane;
              }
            }
          }
          __syncthreads();
          int nc = s_misc[2];
          int need2 = need;
          const float* fu = sCU;
          const int* fp = sCP;
          if (nc > kRankDirect) {
            // second level: linear bins over the boundary bin's own range
            float mn = INFINITY, mx = -INFINITY;
            for (int i = tid; i < nc; i += NT) {
              mn = fminf(mn, sCU[i]);
              mx = fmaxf(mx, sCU[i]);
            }
#pragma unroll
            for (int o2 = 16; o2 >= 1; o2 >>= 1) {
              mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o2));
              mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o2));
            }
            float* red2 = reinterpret_cast<float*>(sC2P + kCandMax);
            if (lane == 0) {
              red2[warp] = mn;
              red2[NWARPS + warp] = mx;
            }
            for (int i = tid; i < kBuckets; i += NT) sHist[i] = 0;
            if (tid == 0) s_misc[2] = 0;
            __syncthreads();
            float cmin = INFINITY, cmax = -INFINITY;
            for (int w2 = 0; w2 < NWARPS; ++w2) {
              cmin = fminf(cmin, red2[w2]);
              cmax = fmaxf(cmax, red2[NWARPS + w2]);
            }
            const float r2 = cmax - cmin;
            const float inv2 = (r2 > 0.f && r2 <= FLT_MAX) ? static_cast<float>(kBuckets) / r2 : 0.f;
            auto bucket2 = [&](float u) {
              const int bk = __float_as_int(fmaf(u - cmin, inv2, 12582912.f)) - 0x4B400000;
              return min(max(bk, 0), kBuckets - 1);
            };
            for (int i = tid; i < nc; i += NT) atomicAdd(&sHist[bucket2(sCU[i])], 1);
            __syncthreads();
            find_boundary(sHist, need, s_scan, &s_misc[5]);
            const int b2 = s_misc[5];
            need2 = need - s_misc[6];
            for (int i = tid; i < nc; i += NT) {
              const int bk = bucket2(sCU[i]);
              if (bk > b2) {
                atomicOr(&sBits[sCP[i] >> 5], 1u << (sCP[i] & 31));
              } else if (bk == b2) {
                const int slot = atomicAdd(&s_misc[2], 1);
                sC2U[slot] = sCU[i];
                sC2P[slot] = sCP[i];
              }
            }
            __syncthreads();
            nc = s_misc[2];
            fu = sC2U;
            fp = sC2P;
          }
          // exact ranking of the remaining boundary pages: larger bound first,
          // then lower page index
          for (int i = tid; i < nc; i += NT) {
            const float u = fu[i];
            const int pi = fp[i];
            int rank = 0;
#pragma unroll 8
            for (int j = 0; j < nc; ++j) {
              const float uj = fu[j];
              rank += (uj > u) || (uj == u && fp[j] < pi);
            }
            if (rank < need2) atomicOr(&sBits[pi >> 5], 1u << (pi & 31));
          }
        } else {
          // many equal-looking bounds: exact search for the Pk-th largest key
          exact_top_pages(sU, NP, Pk, s_scan, sBits);
        }
      }
      __syncthreads();
      {
        // the codes of the kept pages of this CTA's own page range into L2:
        // the compaction below hands them to some CTA's Hamming pass, whose
        // loads then hit L2 (a hint only; rows clamped to the codes buffer)
        const size_t row_bytes = static_cast<size_t>(WORDS) * 4;
        const char* cbase = reinterpret_cast<const char*>(a.codes + static_cast<size_t>(unit) * a.n_cap * WORDS);
        for (int p = pb + tid; p < pe; p += NT) {
          if ((sBits[p >> 5] >> (p & 31)) & 1u) {
            const size_t b0 = static_cast<size_t>(p) * a.page * row_bytes;
            const size_t b1 = min(static_cast<size_t>(p + 1) * a.page, static_cast<size_t>(a.n_cap)) * row_bytes;
            for (size_t off = b0 & ~static_cast<size_t>(127); off < b1; off += 128) prefetch_l2(cbase + off);
          }
        }
      }

      // ---------------------------------------------------------- phase 3
      const int ks = c * Pk / a.C;
      const int ke = (c + 1) * Pk / a.C;
      {
        // thread t owns bitmap words [t*wpt, (t+1)*wpt)
        const int wpt = (nwords + NT - 1) / NT;
        const int w0 = tid * wpt, w1 = min(nwords, w0 + wpt);
        int cnt = 0;
        for (int wi = w0; wi < w1; ++wi) cnt += __popc(sBits[wi]);
        int tot;
        int pos = block_excl_scan1(cnt, s_scan1, &tot);
        int32_t* pidx = a.page_idx + static_cast<size_t>(unit) * a.P;
        for (int wi = w0; wi < w1; ++wi) {
          uint32_t bits = sBits[wi];
          while (bits) {
            const int p = wi * 32 + __ffs(bits) - 1;
            bits &= bits - 1u;
            if (pos >= ks && pos < ke) S.my_pages[pos - ks] = p;
            if (c == 0) pidx[pos] = p;
            ++pos;
          }
        }
        if (c == 0)
          for (int i = Pk + tid; i < a.P; i += NT) pidx[i] = -1;
      }
      __syncthreads();

      // ---------------------------------------------------------- phase 4
      const int S_ = a.page;
      const int ntok = (ke - ks) * S_;
      const int HB = hbins;                            // distance bins: BITS + 1, or r BITS + 1 (GQA-sum)
      int* sHD = reinterpret_cast<int*>(S.scratch);  // [HB]
      for (int i = tid; i < HB; i += NT) sHD[i] = 0;
      uint32_t qc[RG][WORDS];
#pragma unroll
      for (int h = 0; h < RG; ++h)
#pragma unroll
        for (int w = 0; w < WORDS; ++w) qc[h][w] = S.qc[h * WORDS + w];
      __syncthreads();
      const uint32_t* codes_u = a.codes + static_cast<size_t>(unit) * a.n_cap * WORDS;
      int32_t* dbgD = a.dbg_D ? a.dbg_D + static_cast<size_t>(unit) * a.P * S_ : nullptr;
      // the token loop, specialised on the group aggregation
      auto hamming_pass = [&](auto sum_tag) {
        constexpr bool kSum = decltype(sum_tag)::value;
        for (int i0 = warp * 32; i0 < ntok; i0 += NT) {
          const int i = i0 + lane;
          int D = 0xFFFF;
          int slot = 0, off = 0;
          if (i < ntok) {
            slot = i / S_;
            off = i - slot * S_;
            const long long n = static_cast<long long>(S.my_pages[slot]) * S_ + off;
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
              int agg = kSum ? 0 : 1 << 20;   // Eq. 2 over the group: min, or sum (GQA-sum)
  #pragma unroll
              for (int h = 0; h < RG; ++h) {
                int dist = 0;
  #pragma unroll
                for (int w = 0; w < WORDS; ++w) dist += __popc(qc[h][w] ^ kc[w]);
                agg = kSum ? agg + dist : min(agg, dist);
              }
              D = agg;
            }
            S.tokD[i] = static_cast<uint16_t>(D);
            if (dbgD) dbgD[static_cast<size_t>(ks + slot) * S_ + off] = (D == 0xFFFF) ? -1 : D;
          }
          const unsigned grp = __match_any_sync(0xFFFFFFFFu, D);
          if (D != 0xFFFF && lane == __ffs(grp) - 1) atomicAdd(&sHD[D], __popc(grp));
        }
      };
      if (gqa_sum)
        hamming_pass(std::true_type{});
      else
        hamming_pass(std::false_type{});
      if (c == 0 && dbgD)
        for (int i = Pk * S_ + tid; i < a.P * S_; i += NT) dbgD[i] = -1;
      __syncthreads();
      {
        int32_t* hrow = a.wsHist + static_cast<size_t>(unit * kMaxCtasPerUnit + c) * HB;
        for (int i = tid; i < HB; i += NT) hrow[i] = sHD[i];
      }
      // unit barrier 2 (the release by thread 0 covers the CTA's histogram
      // row through the CTA barrier)
      __syncthreads();
      if (tid == 0) red_add_release(ctr, 1u);
      if (!unit_wait(ctr, 2u * static_cast<uint32_t>(a.C) + (a.test_extra_stage == 2 ? 1u : 0u), a, s_misc)) return;

      // ---------------------------------------------------------- phase 5
      int* sHA = reinterpret_cast<int*>(S.scratch);  // [C][HB]
      {
        // one batch of 16-B copies (a plain load/store loop would wait out an
        // L2 round trip per element, the compiler cannot reorder the global
        // loads past the shared stores).  The unit's area holds
        // kMaxCtasPerUnit rows of HB ints, so rounding the copy up to whole
        // 16-B chunks stays inside it.
        const char* hall = reinterpret_cast<const char*>(a.wsHist + static_cast<size_t>(unit * kMaxCtasPerUnit) * HB);
        const int chunks = (a.C * HB * 4 + 15) / 16;
        for (int i = tid; i < chunks; i += NT) cp_async16(reinterpret_cast<char*>(sHA) + 16 * i, hall + 16 * i);
        cp_async_commit();
        cp_async_wait<0>();
      }
      __syncthreads();
      // Every CTA row's exclusive prefix over the distances (warp per row:
      // lane l owns bins [VPL l, VPL l + VPL), bin HB empty, so that
      // pre[cc][HB] is the row's total) and the unit totals tot[v]; then
      // warp 0 alone finds the threshold distance T (the k_eff-th smallest),
      // how many tokens at T are still needed, and each CTA's tie quota and
      // output offset in CTA order.
      // VPLC: bins per lane known at compile time (the min distances, HB =
      // BITS + 1: loops unrolled, loads batched); 0: sized at run time
      // (GQA-sum, HB up to r BITS + 1)
      auto threshold = [&](auto vpl_tag) {
        constexpr int VPLC = decltype(vpl_tag)::value;
        const int HB = VPLC ? BITS + 1 : hbins;         // a compile-time constant with VPLC
        const int VPL = VPLC ? VPLC : (HB + 1 + 31) / 32;
        int* sPre = sHA + a.C * HB;                      // [C][HB + 1]
        int* sTot = sPre + a.C * (HB + 1);               // [HB]
        for (int cc = warp; cc < a.C; cc += NWARPS) {
          const int* row = sHA + cc * HB;
          const int v0 = lane * VPL;
          // compile-time bins: the lane's counts in registers, all loaded
          // before the first store (a store to sPre would otherwise order
          // every later load of row behind it)
          int hv[VPLC ? VPLC : 1];
          int loc = 0;
#pragma unroll
          for (int e = 0; e < (VPLC ? VPLC : VPL); ++e) {
            const int x = v0 + e < HB ? row[v0 + e] : 0;
            if (VPLC) hv[VPLC ? e : 0] = x;
            loc += x;
          }
          int incl = loc;
#pragma unroll
          for (int o2 = 1; o2 < 32; o2 <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o2);
            if (lane >= o2) incl += y;
          }
          int run = incl - loc;
#pragma unroll
          for (int e = 0; e < (VPLC ? VPLC : VPL); ++e) {
            const int v = v0 + e;
            if (v < HB) {
              sPre[cc * (HB + 1) + v] = run;
              run += VPLC ? hv[VPLC ? e : 0] : row[v];
            } else if (v == HB) {
              sPre[cc * (HB + 1) + HB] = run;   // the row's total
            }
          }
        }
        for (int v = tid; v < HB; v += NT) {
          int x = 0;
#pragma unroll 6
          for (int cc = 0; cc < a.C; ++cc) x += sHA[cc * HB + v];
          sTot[v] = x;
        }
        __syncthreads();
        if (warp == 0) {
          const int v0 = lane * VPL;
          int loc = 0;
#pragma unroll
          for (int e = 0; e < (VPLC ? VPLC : VPL); ++e)
            if (v0 + e < HB) loc += sTot[v0 + e];
          int incl = loc;
#pragma unroll
          for (int o2 = 1; o2 < 32; o2 <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o2);
            if (lane >= o2) incl += y;
          }
          const int total = __shfl_sync(0xFFFFFFFFu, incl, 31);
          const int k_eff = min(a.k, total);
          // the lane whose bins hold the k_eff-th smallest distance
          int T = -1, needT = 0;
          if (incl - loc < k_eff && incl >= k_eff) {
            int run = incl - loc;
#pragma unroll
            for (int e = 0; e < (VPLC ? VPLC : VPL); ++e) {
              const int v = v0 + e;
              const int xv = v < HB ? sTot[v] : 0;
              if (run < k_eff && run + xv >= k_eff) {
                T = v;
                needT = k_eff - run;
              }
              run += xv;
            }
          }
          const unsigned own = __ballot_sync(0xFFFFFFFFu, T >= 0);
          if (own) {
            const int src = __ffs(own) - 1;
            T = __shfl_sync(0xFFFFFFFFu, T, src);
            needT = __shfl_sync(0xFFFFFFFFu, needT, src);
          }
          int pre_eq = 0, off = 0;
          for (int c0 = 0; c0 < a.C; c0 += 32) {   // CTAs in order: tie quota and output offset
            const int cc = c0 + lane;
            int below = 0, eq = 0;
            if (cc < a.C && T >= 0) {
              below = sPre[cc * (HB + 1) + T];
              eq = sPre[cc * (HB + 1) + T + 1] - below;
            }
            int eq_in = eq;
#pragma unroll
            for (int o2 = 1; o2 < 32; o2 <<= 1) {
              const int y = __shfl_up_sync(0xFFFFFFFFu, eq_in, o2);
              if (lane >= o2) eq_in += y;
            }
            const int quota = max(0, min(needT - (pre_eq + eq_in - eq), eq));
            const int selc = below + quota;
            int sel_in = selc;
#pragma unroll
            for (int o2 = 1; o2 < 32; o2 <<= 1) {
              const int y = __shfl_up_sync(0xFFFFFFFFu, sel_in, o2);
              if (lane >= o2) sel_in += y;
            }
            if (cc == c) {
              s_misc[7] = off + sel_in - selc;
              s_misc[8] = quota;
              s_misc[9] = selc;
            }
            pre_eq += __shfl_sync(0xFFFFFFFFu, eq_in, 31);
            off += __shfl_sync(0xFFFFFFFFu, sel_in, 31);
          }
          if (lane == 0) {
            s_misc[5] = T;
            s_misc[6] = k_eff;
          }
        }
        __syncthreads();
      };
      if (gqa_sum)
        threshold(std::integral_constant<int, 0>{});
      else
        threshold(std::integral_constant<int, (BITS + 2 + 31) / 32>{});
      const int T = s_misc[5], k_eff = s_misc[6];
      const int my_off = s_misc[7], my_quota = s_misc[8], my_sel = s_misc[9];
      {
        // one packed scan: (tokens below T) | (tokens at T) << 16
        const int span = (ntok + NT - 1) / NT;
        const int lo = tid * span, hi = min(ntok, lo + span);
        int lt = 0, eq = 0;
        for (int i = lo; i < hi; ++i) {
          const int D = S.tokD[i];
          lt += D < T;
          eq += D == T;
        }
        int tmp;
        const int pre = block_excl_scan1(lt | (eq << 16), s_scan1, &tmp);
        int lt_b = pre & 0xFFFF, eq_b = pre >> 16;
        int32_t* tout = a.tok_idx + static_cast<size_t>(unit) * a.k;
        for (int i = lo; i < hi; ++i) {
          const int D = S.tokD[i];
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
            const int n = S.my_pages[slot] * S_ + (i - slot * S_);
            tout[my_off + pos] = n;
            S.sel[pos] = n;
          }
        }
        if (c == 0) {
          if (tid == 0) a.n_sel[unit] = k_eff;
          for (int i = k_eff + tid; i < a.k; i += NT) tout[i] = -1;
        }
      }
      __syncthreads();

      if constexpr (MODE == kModeFused) {
        attend_and_finish<RG>(a, unit, c, S.sel, my_sel, S.qf, S.scratch, 3u * static_cast<uint32_t>(a.C), s_misc);
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

template <int RG, int WORDS, int MODE, bool VAR>
cudaError_t launch_t(const DecodeArgs& a, size_t smem, cudaStream_t stream) {
  auto kern = decode_kernel<RG, WORDS, MODE, VAR>;
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
  const bool var = a.meta_f32 || a.gqa_sum || a.simt_bounds;
  switch (mode) {
    case kModeSelect:
      return var ? launch_t<RG, WORDS, kModeSelect, true>(a, smem, stream)
                 : launch_t<RG, WORDS, kModeSelect, false>(a, smem, stream);
    case kModeFused:
      return var ? launch_t<RG, WORDS, kModeFused, true>(a, smem, stream)
                 : launch_t<RG, WORDS, kModeFused, false>(a, smem, stream);
    case kModeAttend: return launch_t<RG, WORDS, kModeAttend, false>(a, smem, stream);
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

}  // namespace hhr
