// Key encoding for sm_100a on the 5th-generation tensor cores: rotation
// (Eq. 4), per-page extrema (definition under Eq. 3) and projection + sign
// (Eq. 10, Eq. 1) of "HHR: Hierarchical Hash Retrieval for Efficient LLM
// Generation".
//
// A CTA owns one KV head g and one 128-column output block of [R | W] and
// computes D = M^T K^T for tiles of 128 keys with tcgen05.mma (M = 128 output
// dimensions, N = 128 keys, K = 128 input dimensions), fp32 accumulation in
// tensor memory.  M^T stays in shared memory as three bf16 terms whose sum is
// the float32 weight exactly, so D carries float32 accuracy (the keys are
// bf16, so every product is exact).  With the output dimension on the TMEM
// lanes, an epilogue thread owns one output dimension across the tile's keys:
// a page's extrema are thread-local, a code word is one warp ballot per key.
//
// Warps: 0-3 epilogue (TMEM lanes 0-127), 4-7 producers (key tiles by
// cp.async into a 3-stage ring), 8 MMA issue (one elected thread) and TMEM
// allocation.  Every mbarrier wait is bounded; on expiry the kernel records
// HHR_ERR_TIMEOUT in a sticky word and leaves its loops.

#include <cuda_bf16.h>

#include <cstdint>

#include "hhr_internal.cuh"

namespace hhr {

__device__ uint32_t g_encode_err = 0;

namespace {

constexpr int kTileKeys = 128;                            // keys per tile (the MMA's N)
constexpr int kStages = 3;                                // key tiles in flight
constexpr int kTerms = 3;                                 // bf16 terms per float32 weight
constexpr int kOpBytes = 128 * kD * 2;                    // one [128 rows][128 k] bf16 operand
constexpr int kAtomBytes = 128 * 128;                     // 64 k of 128 rows (one swizzle atom column)
constexpr int kEpiWarps = 4, kProdWarps = 4;
constexpr int kMmaWarp = kEpiWarps + kProdWarps;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr uint32_t kAccCols = 128;                        // fp32 TMEM columns per accumulator
constexpr uint32_t kTmemCols = 2 * kAccCols;              // double-buffered
// kind::f16 instruction descriptor: D f32, A and B bf16, both K-major, N = 128, M = 128
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Byte offset of bf16 element (row r, k) in a [128 rows][128 k] operand laid
// out K-major with the 128-B swizzle: two 64-k atom columns of 16 KB, 8-row
// groups 1024 B apart, 16-B chunk c of row r at chunk position c ^ (r & 7).
__device__ __forceinline__ uint32_t sw128(int r, int k) {
  return static_cast<uint32_t>((k >> 6) * kAtomBytes + ((r >> 3) << 10) + ((r & 7) << 7) +
                               ((((k & 63) >> 3) ^ (r & 7)) << 4) + ((k & 7) << 1));
}

// Shared-memory matrix descriptor of such an operand (start address in 16-B
// units, leading offset 1, stride offset 1024 B between 8-row groups,
// descriptor version 1, 128-B swizzle).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
         (2ull << 61);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
               " selp.u32 %0, 1, 0, p;\n}" : "=r"(done) : "r"(bar), "r"(parity) : "memory");
  return done != 0;
}
// Waits for the completion of the phase with the given parity; false (and the
// sticky error set) once `limit` cycles have passed.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned long long limit) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  do {
    if (mbar_try(bar, parity)) return true;
  } while (static_cast<unsigned long long>(clock64() - t0) <= limit);
  atomicExch(&g_encode_err, static_cast<uint32_t>(HHR_ERR_TIMEOUT));
  return false;
}

// 16 B when src_bytes is 16, 16 zero bytes when it is 0.
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }
// Generic-proxy writes of this thread to shared memory become visible to the
// tensor cores' (async-proxy) reads.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t accumulate) {
  asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
               " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}"
               :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(kIdesc), "r"(accumulate) : "memory");
}
// Arrives on the mbarrier once every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" :: "r"(bar) : "memory");
}
// 32 consecutive fp32 columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
               "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
               "%30, %31}, [%32];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
                 "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
                 "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
                 "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
                 "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// v = hi + mid + lo exactly, each a bf16 (the residuals are exact in float32).
__device__ __forceinline__ void split3(float v, uint16_t& hi, uint16_t& mid, uint16_t& lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(h);
  const __nv_bfloat16 m = __float2bfloat16_rn(r1);
  const __nv_bfloat16 l = __float2bfloat16_rn(r1 - __bfloat162float(m));
  hi = __bfloat16_as_ushort(h);
  mid = __bfloat16_as_ushort(m);
  lo = __bfloat16_as_ushort(l);
}

// Stores the bounds of dimension j of one page at dst ([2][d]): bf16 rounded
// outward (the default), or float32 as computed (HHR_FLAG_META_F32).  MERGE:
// combined with the bounds already stored (keys encoded by an earlier call).
template <bool MERGE>
__device__ __forceinline__ void put_bounds(__nv_bfloat16* dst, int j, float mn, float mx) {
  __nv_bfloat16 lo = __float2bfloat16_rd(mn), hi = __float2bfloat16_ru(mx);
  if (MERGE) {
    lo = __hmin(lo, dst[j]);
    hi = __hmax(hi, dst[kD + j]);
  }
  dst[j] = lo;
  dst[kD + j] = hi;
}
template <bool MERGE>
__device__ __forceinline__ void put_bounds(float* dst, int j, float mn, float mx) {
  if (MERGE) {
    mn = fminf(mn, dst[j]);
    mx = fmaxf(mx, dst[kD + j]);
  }
  dst[j] = mn;
  dst[kD + j] = mx;
}

// Pages of S keys (a power of two, at most 64) over one chunk of 32 keys of a
// tile whose keys are all new (no masking, no merge): tree reductions with
// static register indices.  For S = 64 a page spans two chunks; its partial
// extrema are carried in mn / mx.
template <int S, typename MT>
__device__ __forceinline__ void full_chunk_extrema(const uint32_t (&v)[32], int ch, int key0,
                                                   MT* meta_u, int j, float& mn, float& mx) {
  constexpr int G = S < 32 ? S : 32;          // keys of one page inside this chunk
#pragma unroll
  for (int p0 = 0; p0 < 32; p0 += G) {
    float lo[G], hi[G];
#pragma unroll
    for (int i = 0; i < G; ++i) lo[i] = hi[i] = __uint_as_float(v[p0 + i]);
#pragma unroll
    for (int w = G / 2; w >= 1; w >>= 1)
#pragma unroll
      for (int i = 0; i < w; ++i) {
        lo[i] = fminf(lo[i], lo[i + w]);
        hi[i] = fmaxf(hi[i], hi[i + w]);
      }
    float pmn = lo[0], pmx = hi[0];
    if (S > 32) {
      pmn = fminf(pmn, mn);
      pmx = fmaxf(pmx, mx);
      mn = pmn;
      mx = pmx;
      if ((ch & 1) == 0) continue;             // the page continues in the next chunk
      mn = INFINITY;
      mx = -INFINITY;
    }
    const int first = key0 + ch * 32 + p0 - (S > 32 ? 32 : 0);
    put_bounds<false>(meta_u + static_cast<size_t>(first / S) * 2 * kD, j, pmn, pmx);
  }
}

// Running per-page extrema over 32 keys (columns ch * 32 .. + 31 of the
// tile) of output dimension j; a page's bounds are stored (put_bounds) when
// its last key has been seen.  MERGE: pages that start below n_begin are
// merged with the bounds already stored.
template <bool MERGE, typename MT>
__device__ __forceinline__ void page_extrema(const uint32_t (&v)[32], int ch, int key0, int S, int n_begin,
                                             int n_end, MT* meta_u, int j, float& mn, float& mx) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int col = ch * 32 + i, key = key0 + col;
    const float x = __uint_as_float(v[i]);
    if (key >= n_begin && key < n_end) {
      mn = fminf(mn, x);
      mx = fmaxf(mx, x);
    }
    if (((col + 1) & (S - 1)) == 0) {   // the page ends at this key
      if (mn <= mx) {
        const int first = key + 1 - S;
        MT* dstp = meta_u + static_cast<size_t>(first / S) * 2 * kD;
        if (MERGE && first < n_begin)    // keys [first, n_begin) were encoded before
          put_bounds<true>(dstp, j, mn, mx);
        else
          put_bounds<false>(dstp, j, mn, mx);
      }
      mn = INFINITY;
      mx = -INFINITY;
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) encode_kernel(const EncodeArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) unsigned long long bar_full[kStages], bar_empty[kStages];
  __shared__ __align__(8) unsigned long long bar_acc_full[2], bar_acc_empty[2];
  __shared__ uint32_t s_tmem;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // operands on a 1024-B boundary (the swizzle pattern repeats every 1024 B)
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;
  unsigned char* base = smem_raw + (base_s - raw_s);
  const uint32_t a_s = base_s;                              // [kTerms][kOpBytes]
  const uint32_t b_s = base_s + kTerms * kOpBytes;          // [kStages][kOpBytes]

  const int n_ob = 1 + a.bits / kD;
  const int g = blockIdx.y / n_ob, ob = blockIdx.y % n_ob;
  const int items = (a.units / a.Hkv) * a.n_tiles;          // (sequence, key tile) pairs of head g

  // A = M^T for M = R (ob 0) or W's columns [128 (ob - 1), 128 ob): row j,
  // input dimension k, as three bf16 terms
  {
    const float* M = ob == 0 ? a.R + static_cast<size_t>(g) * kD * kD
                             : a.W + static_cast<size_t>(g) * kD * a.bits + (ob - 1) * kD;
    const int ld = ob == 0 ? kD : a.bits;
    for (int w = tid; w < kD * (kD / 8); w += kThreads) {
      const int j = w % kD, kc = w / kD;                    // input dimensions 8 kc .. 8 kc + 7
      uint32_t t[kTerms][4];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        uint16_t h0, m0, l0, h1, m1, l1;
        split3(__ldg(M + static_cast<size_t>(kc * 8 + e) * ld + j), h0, m0, l0);
        split3(__ldg(M + static_cast<size_t>(kc * 8 + e + 1) * ld + j), h1, m1, l1);
        t[0][e >> 1] = h0 | (static_cast<uint32_t>(h1) << 16);
        t[1][e >> 1] = m0 | (static_cast<uint32_t>(m1) << 16);
        t[2][e >> 1] = l0 | (static_cast<uint32_t>(l1) << 16);
      }
      const uint32_t off = sw128(j, kc * 8);
#pragma unroll
      for (int tt = 0; tt < kTerms; ++tt)
        *reinterpret_cast<uint4*>(base + tt * kOpBytes + off) = make_uint4(t[tt][0], t[tt][1], t[tt][2], t[tt][3]);
    }
    fence_proxy_async();
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      // (the test hook makes the first stage wait for one arrival more than
      // the producers make: every role's wait then runs out and the kernel
      // leaves through its normal exit, with no MMA issued)
      mbar_init(smem_u32(&bar_full[s]), kProdWarps * 32 + (a.test_extra_arrival && s == 0 ? 1 : 0));
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(smem_u32(&bar_acc_full[x]), 1);
      mbar_init(smem_u32(&bar_acc_empty[x]), kEpiWarps * 32);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(&s_tmem)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp >= kEpiWarps && warp < kMmaWarp) {
    // ------------------------------------------------------------ producers
    const int pt = tid - kEpiWarps * 32;
    int lq = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x, ++lq) {
      const int s = lq % kStages;
      if (!mbar_wait(smem_u32(&bar_empty[s]), ((lq / kStages) & 1) ^ 1, a.spin_limit)) break;
      const int unit = (it / a.n_tiles) * a.Hkv + g;
      const int key0 = a.tile_begin + (it % a.n_tiles) * kTileKeys;
      const uint16_t* Ku = a.K + static_cast<size_t>(unit) * a.n_cap * kD;
      const uint32_t dst = b_s + s * kOpBytes;
#pragma unroll 4
      for (int u = 0; u < kTileKeys * 16 / (kProdWarps * 32); ++u) {
        const int q = pt + kProdWarps * 32 * u;
        const int r = q >> 4, cc = q & 15;                  // key row, 16-B chunk along k
        const int key = key0 + r;
        const bool ok = key >= a.n_begin && key < a.n_end;
        cp_async16_zfill(dst + sw128(r, cc * 8), ok ? Ku + static_cast<size_t>(key) * kD + cc * 8 : Ku,
                         ok ? 16u : 0u);
      }
      cp_async_commit();
      if (lq > 0) {   // the previous tile has landed: hand it to the tensor cores
        cp_async_wait<1>();
        fence_proxy_async();
        mbar_arrive(smem_u32(&bar_full[(lq - 1) % kStages]));
      }
    }
    cp_async_wait<0>();
    fence_proxy_async();
    if (lq > 0) mbar_arrive(smem_u32(&bar_full[(lq - 1) % kStages]));
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      int lq = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < items && ok; it += gridDim.x, ++lq) {
        const int s = lq % kStages, acc = lq & 1;
        ok = mbar_wait(smem_u32(&bar_acc_empty[acc]), ((lq >> 1) & 1) ^ 1, a.spin_limit);
        if (ok) ok = mbar_wait(smem_u32(&bar_full[s]), (lq / kStages) & 1, a.spin_limit);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * kAccCols;
#pragma unroll
        for (int tt = 0; tt < kTerms; ++tt)
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {
            const uint32_t koff = (ks >> 2) * kAtomBytes + (ks & 3) * 32;
            tc_mma(d, sw128_desc(a_s + tt * kOpBytes + koff), sw128_desc(b_s + s * kOpBytes + koff),
                   (tt | ks) != 0 ? 1u : 0u);
          }
        tc_commit(smem_u32(&bar_empty[s]));
        tc_commit(smem_u32(&bar_acc_full[acc]));
      }
      // every issued MMA has completed before TMEM is released
      if (lq > 0) mbar_wait(smem_u32(&bar_acc_full[(lq - 1) & 1]), ((lq - 1) >> 1) & 1, a.spin_limit);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int j = tid;                                      // output dimension = TMEM lane
    const int S = a.page;
    const int words = a.bits / 32;
    int lq = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x, ++lq) {
      const int acc = lq & 1;
      if (!mbar_wait(smem_u32(&bar_acc_full[acc]), (lq >> 1) & 1, a.spin_limit)) break;
      tc_fence_after();
      const int unit = (it / a.n_tiles) * a.Hkv + g;
      const int key0 = a.tile_begin + (it % a.n_tiles) * kTileKeys;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16) + acc * kAccCols;
      float mn = INFINITY, mx = -INFINITY;                  // running extrema of the current page
      uint32_t* codes_u = a.codes + static_cast<size_t>(unit) * a.n_cap * words;
#pragma unroll 1
      for (int ch = 0; ch < kTileKeys / 32; ++ch) {
        uint32_t v[32];
        tc_ld32(taddr + ch * 32, v);
        if (ob == 0) {
          // only a tile that starts below n_begin holds a page with keys
          // encoded by an earlier call (its bounds are merged, not replaced)
          auto extrema = [&](auto* meta_base) {
            auto* meta_u = meta_base + static_cast<size_t>(unit) * a.np_cap * 2 * kD;
            if (key0 >= a.n_begin && key0 + kTileKeys <= a.n_end) {
              switch (S) {
                case 1: full_chunk_extrema<1>(v, ch, key0, meta_u, j, mn, mx); break;
                case 2: full_chunk_extrema<2>(v, ch, key0, meta_u, j, mn, mx); break;
                case 4: full_chunk_extrema<4>(v, ch, key0, meta_u, j, mn, mx); break;
                case 8: full_chunk_extrema<8>(v, ch, key0, meta_u, j, mn, mx); break;
                case 16: full_chunk_extrema<16>(v, ch, key0, meta_u, j, mn, mx); break;
                case 32: full_chunk_extrema<32>(v, ch, key0, meta_u, j, mn, mx); break;
                default: full_chunk_extrema<64>(v, ch, key0, meta_u, j, mn, mx); break;
              }
            } else if (key0 < a.n_begin) {
              page_extrema<true>(v, ch, key0, S, a.n_begin, a.n_end, meta_u, j, mn, mx);
            } else {
              page_extrema<false>(v, ch, key0, S, a.n_begin, a.n_end, meta_u, j, mn, mx);
            }
          };
          if (a.meta_f32)
            extrema(static_cast<float*>(a.meta));
          else
            extrema(static_cast<__nv_bfloat16*>(a.meta));
        } else {
          uint32_t mine = 0u;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const uint32_t word = __ballot_sync(0xFFFFFFFFu, __uint_as_float(v[i]) > 0.f);
            if (lane == i) mine = word;
          }
          const int key = key0 + ch * 32 + lane;
          if (key >= a.n_begin && key < a.n_end)
            codes_u[static_cast<size_t>(key) * words + (ob - 1) * (kD / 32) + warp] = mine;
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_acc_empty[acc]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace

size_t encode_smem_bytes() { return static_cast<size_t>(kTerms + kStages) * kOpBytes + 1024; }

cudaError_t launch_encode(const EncodeArgs& a, int sms, cudaStream_t stream) {
  const size_t smem = encode_smem_bytes();
  static std::atomic<size_t> raised[kMaxDevices];
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(encode_kernel), smem, raised);
  if (e != cudaSuccess) return e;
  const int n_ob = 1 + a.bits / kD;
  const int groups = a.Hkv * n_ob;
  const int items = (a.units / a.Hkv) * a.n_tiles;
  int gx = sms / groups;
  if (gx < 1) gx = 1;
  if (gx > items) gx = items;
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(groups));
  encode_kernel<<<grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t encode_read_status(uint32_t* out, cudaStream_t stream) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_encode_err, sizeof(uint32_t), 0, cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  e = cudaMemcpyToSymbolAsync(g_encode_err, &zero, sizeof(uint32_t), 0, cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(stream);
}

}  // namespace hhr
