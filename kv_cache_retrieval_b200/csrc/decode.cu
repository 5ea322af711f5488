// Decode-time retrieval kernels for sm_100a.
//
// One (sequence, KV head) pair -- a "unit" -- is spread over C CTAs of a
// cooperative launch.  A fused step runs these phases per unit:
//
//   0  query prep      q~ = q R (Eq. 4) for the r query heads of the group
//   1  page bounds     U_p = max_h sum_j max(q~_hj l_pj, q~_hj u_pj)  (Eq. 3)
//                      over this CTA's contiguous slice of pages; metadata is
//                      streamed with 128-bit loads, one page (512 B) per warp
//                      load instruction, and the per-lane partial sums are
//                      folded with a butterfly reduce-scatter
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
//   6  attention       each CTA attends over its own selected tokens: K/V rows
//                      staged into shared memory with cp.async (16 B, L2 only),
//                      one half-warp per token, online softmax in float32
//      -- last-arriving CTA merges the C partial softmax states --
//
// Inter-CTA waits spin on workspace counters with a clock64() limit; on
// expiry the kernel records HHR_ERR_TIMEOUT and returns.  The last CTA of a
// unit resets its counter, so the workspace is zero again after each call.

#include <cuda_bf16.h>

#include <cfloat>
#include <cstdint>

#include "hhr_internal.cuh"

namespace hhr {
namespace {

constexpr int NT = kDecodeThreads;
constexpr int NWARPS = NT / 32;

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

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

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.cs.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }

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

__device__ int block_sum(int v, int* s_warp) {
  int total;
  block_excl_scan(v, s_warp, &total);
  return total;
}

// Unit barrier: every CTA of the unit adds one to the counter, then waits
// until it reaches `target`.  Returns false (and records HHR_ERR_TIMEOUT) if
// the wait ran out.  All threads of the CTA must call it.
__device__ bool unit_arrive_wait(uint32_t* ctr, uint32_t target, const DecodeArgs& a,
                                 int* s_flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atom_add_acq_rel(ctr, 1u);
    int ok = 1;
    const long long t0 = clock64();
    while (ld_acquire(ctr) < target) {
      if (static_cast<unsigned long long>(clock64() - t0) > a.spin_limit) {
        atomicExch(a.status, static_cast<uint32_t>(HHR_ERR_TIMEOUT));
        ok = 0;
        break;
      }
      __nanosleep(32);
    }
    __threadfence();
    *s_flag = ok;
  }
  __syncthreads();
  return *s_flag != 0;
}

// Butterfly reduce-scatter of NV per-lane partial sums over the 32 lanes.
// Afterwards v[0] of lane l holds the full sum of value index l >> (5 - log2 NV).
template <int NV>
__device__ __forceinline__ void reduce_scatter(float (&v)[NV], int lane) {
  constexpr int L = (NV >= 32) ? 5 : (NV >= 16) ? 4 : (NV >= 8) ? 3 : (NV >= 4) ? 2 : (NV >= 2) ? 1 : 0;
#pragma unroll
  for (int k = 0; k < L; ++k) {
    const int m = 16 >> k;
    const int h = NV >> (k + 1);
    const bool up = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float send = up ? v[i] : v[i + h];
      const float keep = up ? v[i + h] : v[i];
      v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, m);
    }
  }
#pragma unroll
  for (int k = L; k < 5; ++k) v[0] += __shfl_xor_sync(0xFFFFFFFFu, v[0], 16 >> k);
}

template <int NV>
struct Log2 {
  static constexpr int value = (NV >= 32) ? 5 : (NV >= 16) ? 4 : (NV >= 8) ? 3 : (NV >= 4) ? 2 : (NV >= 2) ? 1 : 0;
};

__device__ __forceinline__ uint32_t order_key(float u) {
  const uint32_t x = __float_as_uint(u + 0.0f);  // -0 -> +0
  return (x & 0x80000000u) ? ~x : (x | 0x80000000u);
}

struct Smem {
  float* qt;       // [r][d] rotated queries
  float* qf;       // [r][d] queries (float), pre-scaled for attention
  uint32_t* qc;    // [r][w] query codes
  int* my_pages;   // kept pages of this CTA's slice
  uint16_t* tokD;  // distances of the slice's tokens
  int* sel;        // selected tokens of this CTA (ascending)
  unsigned char* scratch;
};

// ----------------------------------------------------------------------------
// Phase 6: attention of the r heads over `cnt` tokens listed in sel[], then
// the per-unit merge.  sq: pre-scaled queries (scale * log2 e) [r][d].
template <int RG>
__device__ void attend_and_finish(const DecodeArgs& a, int unit, int c, const int* sel, int cnt,
                                  const float* sq, unsigned char* scratch, uint32_t final_target,
                                  int* s_int) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hf = lane >> 4, hl = lane & 15;
  const size_t unit_rows = static_cast<size_t>(unit) * a.n_cap;
  const uint16_t* Ku = a.K + unit_rows * kD;
  const uint16_t* Vu = a.V + unit_rows * kD;
  uint16_t* ring = reinterpret_cast<uint16_t*>(scratch);  // [stages][chunk][2][d]
  constexpr int STAGE_ELEMS = kAttnChunk * 2 * kD;

  const int n_stages = (cnt + kAttnChunk - 1) / kAttnChunk;
  auto issue = [&](int s) {
    if (s < n_stages) {
      const int tt = tid >> 4, part = tid & 15;  // token in stage, 16-B chunk of its row
      const int i = s * kAttnChunk + tt;
      if (i < cnt) {
        const size_t row = static_cast<size_t>(sel[i]) * kD;
        uint16_t* dst = ring + (s % kAttnStages) * STAGE_ELEMS + tt * 2 * kD;
        cp_async16(dst + part * 8, Ku + row + part * 8);
        cp_async16(dst + kD + part * 8, Vu + row + part * 8);
      }
    }
    cp_async_commit();
  };

  float q[RG][8];
#pragma unroll
  for (int h = 0; h < RG; ++h)
#pragma unroll
    for (int e = 0; e < 8; ++e) q[h][e] = sq[h * kD + hl * 8 + e];
  float m[RG], l[RG], o[RG][8];
#pragma unroll
  for (int h = 0; h < RG; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[h][e] = 0.f;
  }

#pragma unroll
  for (int s = 0; s < kAttnStages - 1; ++s) issue(s);
  for (int s = 0; s < n_stages; ++s) {
    cp_async_wait<kAttnStages - 2>();
    __syncthreads();
    issue(s + kAttnStages - 1);
    const int ti = warp * 2 + hf;
    const bool valid = s * kAttnChunk + ti < cnt;   // uniform within a half-warp
    const uint16_t* rowp = ring + (s % kAttnStages) * STAGE_ELEMS + ti * 2 * kD;
    uint4 kv = make_uint4(0u, 0u, 0u, 0u), vv = make_uint4(0u, 0u, 0u, 0u);
    if (valid) {
      kv = *reinterpret_cast<const uint4*>(rowp + hl * 8);
      vv = *reinterpret_cast<const uint4*>(rowp + kD + hl * 8);
    }
    const float kf[8] = {bf_lo(kv.x), bf_hi(kv.x), bf_lo(kv.y), bf_hi(kv.y),
                         bf_lo(kv.z), bf_hi(kv.z), bf_lo(kv.w), bf_hi(kv.w)};
    const float vf[8] = {bf_lo(vv.x), bf_hi(vv.x), bf_lo(vv.y), bf_hi(vv.y),
                         bf_lo(vv.z), bf_hi(vv.z), bf_lo(vv.w), bf_hi(vv.w)};
#pragma unroll
    for (int h = 0; h < RG; ++h) {
      float sdot = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) sdot = fmaf(q[h][e], kf[e], sdot);
      // butterfly over the 16 lanes of this half-warp: every lane ends with
      // the same (commutative) sum
      sdot += __shfl_xor_sync(0xFFFFFFFFu, sdot, 8);
      sdot += __shfl_xor_sync(0xFFFFFFFFu, sdot, 4);
      sdot += __shfl_xor_sync(0xFFFFFFFFu, sdot, 2);
      sdot += __shfl_xor_sync(0xFFFFFFFFu, sdot, 1);
      if (valid) {
        if (sdot > m[h]) {
          const float alpha = exp2f(m[h] - sdot);
          l[h] *= alpha;
#pragma unroll
          for (int e = 0; e < 8; ++e) o[h][e] *= alpha;
          m[h] = sdot;
        }
        const float p = exp2f(sdot - m[h]);
        l[h] += p;
#pragma unroll
        for (int e = 0; e < 8; ++e) o[h][e] = fmaf(p, vf[e], o[h][e]);
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // fold the two half-warps of each warp together, then merge the 16 warp
  // states through shared memory: [warp][h][d + 2]
#pragma unroll
  for (int h = 0; h < RG; ++h) {
    const float mo = __shfl_xor_sync(0xFFFFFFFFu, m[h], 16);
    const float lo = __shfl_xor_sync(0xFFFFFFFFu, l[h], 16);
    const float M = fmaxf(m[h], mo);
    const float wa = (M == -INFINITY) ? 0.f : exp2f(m[h] - M);
    const float wb = (M == -INFINITY) ? 0.f : exp2f(mo - M);
    l[h] = l[h] * wa + lo * wb;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float oo = __shfl_xor_sync(0xFFFFFFFFu, o[h][e], 16);
      o[h][e] = o[h][e] * wa + oo * wb;
    }
    m[h] = M;
  }
  float* mer = reinterpret_cast<float*>(scratch);
  if (hf == 0) {
#pragma unroll
    for (int h = 0; h < RG; ++h) {
      float* dst = mer + (warp * RG + h) * (kD + 2);
#pragma unroll
      for (int e = 0; e < 8; ++e) dst[hl * 8 + e] = o[h][e];
      if (hl == 0) {
        dst[kD] = m[h];
        dst[kD + 1] = l[h];
      }
    }
  }
  __syncthreads();

  const int b = unit / a.Hkv, g = unit % a.Hkv;
  float* part = a.wsPart + static_cast<size_t>(unit * kMaxCtasPerUnit + c) * RG * (kD + 2);
  for (int oi = tid; oi < RG * kD; oi += NT) {
    const int h = oi / kD, j = oi % kD;
    float M = -INFINITY;
    for (int w = 0; w < NWARPS; ++w) M = fmaxf(M, mer[(w * RG + h) * (kD + 2) + kD]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < NWARPS; ++w) {
        const float* src = mer + (w * RG + h) * (kD + 2);
        const float wgt = exp2f(src[kD] - M);
        L = fmaf(src[kD + 1], wgt, L);
        O = fmaf(src[j], wgt, O);
      }
    }
    if (a.C == 1) {
      a.out[(static_cast<size_t>(b) * a.Hq + g * RG + h) * kD + j] = (L > 0.f) ? O / L : 0.f;
    } else {
      part[h * (kD + 2) + j] = O;
      if (j == 0) {
        part[h * (kD + 2) + kD] = M;
        part[h * (kD + 2) + kD + 1] = L;
      }
    }
  }

  // last CTA of the unit merges the C partial states and resets the counter
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const uint32_t old = atom_add_acq_rel(a.counters + unit, 1u);
    s_int[0] = (old == final_target - 1) ? 1 : 0;
  }
  __syncthreads();
  if (!s_int[0]) return;
  __threadfence();
  if (a.C > 1) {
    const float* parts = a.wsPart + static_cast<size_t>(unit * kMaxCtasPerUnit) * RG * (kD + 2);
    for (int oi = tid; oi < RG * kD; oi += NT) {
      const int h = oi / kD, j = oi % kD;
      float M = -INFINITY;
      for (int cc = 0; cc < a.C; ++cc) M = fmaxf(M, __ldcg(parts + (cc * RG + h) * (kD + 2) + kD));
      float L = 0.f, O = 0.f;
      if (M != -INFINITY) {
        for (int cc = 0; cc < a.C; ++cc) {
          const float* src = parts + (cc * RG + h) * (kD + 2);
          const float wgt = exp2f(__ldcg(src + kD) - M);
          L = fmaf(__ldcg(src + kD + 1), wgt, L);
          O = fmaf(__ldcg(src + j), wgt, O);
        }
      }
      a.out[(static_cast<size_t>(b) * a.Hq + g * RG + h) * kD + j] = (L > 0.f) ? O / L : 0.f;
    }
  }
  if (tid == 0) atomicExch(a.counters + unit, 0u);
}

// ----------------------------------------------------------------------------
template <int RG, int WORDS, int MODE>
__global__ void __launch_bounds__(NT, 1) decode_kernel(const DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_int[NWARPS + 16];
  __shared__ int s_aux[2 * kMaxCtasPerUnit];
  __shared__ float s_flt[4];
  constexpr int BITS = WORDS * 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x % a.C;
  const DecodeSmem lay = decode_smem(a.NP, a.C, BITS, RG, a.slice_pages, a.slice_tokens, MODE);
  Smem S;
  S.qt = reinterpret_cast<float*>(smem + lay.qt);
  S.qf = reinterpret_cast<float*>(smem + lay.qf);
  S.qc = reinterpret_cast<uint32_t*>(smem + lay.qc);
  S.my_pages = reinterpret_cast<int*>(smem + lay.my_pages);
  S.tokD = reinterpret_cast<uint16_t*>(smem + lay.tokD);
  S.sel = reinterpret_cast<int*>(smem + lay.sel);
  S.scratch = smem + lay.scratch;
  int* s_scan = s_int;              // NWARPS + 1 entries
  int* s_misc = s_int + NWARPS + 1; // scalars

  for (int unit = blockIdx.x / a.C; unit < a.units; unit += a.grid_units) {
    const int b = unit / a.Hkv, g = unit % a.Hkv;
    uint32_t* ctr = a.counters + unit;

    // queries of the group, as float (raw) -- q~ is derived from these
    const uint16_t* qg = a.q + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(g) * RG) * kD;
    for (int i = tid; i < RG * kD; i += NT) S.qf[i] = __uint_as_float(static_cast<uint32_t>(qg[i]) << 16);
    __syncthreads();

    if constexpr (MODE == kModeAttend) {
      const int n = a.nsel_in[unit];
      const int s0 = static_cast<int>(static_cast<long long>(c) * n / a.C);
      const int s1 = static_cast<int>(static_cast<long long>(c + 1) * n / a.C);
      const int32_t* src = a.tok_in + static_cast<size_t>(unit) * a.k;
      for (int i = s0 + tid; i < s1; i += NT) S.sel[i - s0] = src[i];
      for (int i = tid; i < RG * kD; i += NT) S.qf[i] *= a.scale_log2;
      __syncthreads();
      attend_and_finish<RG>(a, unit, c, S.sel, s1 - s0, S.qf, S.scratch,
                            static_cast<uint32_t>(a.C), s_misc);
      __syncthreads();
      continue;
    } else {
      // ---------------------------------------------------------- phase 0
      const float* Rg = a.R + static_cast<size_t>(g) * kD * kD;
      for (int oi = tid; oi < RG * kD; oi += NT) {
        const int h = oi / kD, j = oi % kD;
        float acc = 0.f;
#pragma unroll 8
        for (int i = 0; i < kD; ++i) acc = fmaf(S.qf[h * kD + i], __ldg(Rg + i * kD + j), acc);
        S.qt[oi] = acc;
      }
      __syncthreads();

      // ---------------------------------------------------------- phase 1
      constexpr int PPI = (RG == 1) ? 8 : 16 / RG;  // pages per warp iteration
      constexpr int NV = PPI * RG;
      constexpr int LNV = Log2<NV>::value;
      constexpr int SH = 5 - LNV;                   // lanes sharing one value index
      const int half = lane >> 4, dl = (lane & 15) * 8;
      float qs[RG][8];
#pragma unroll
      for (int h = 0; h < RG; ++h)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float v = S.qt[h * kD + dl + e];
          qs[h][e] = half ? fmaxf(v, 0.f) : fminf(v, 0.f);
        }
      const long long pb = static_cast<long long>(c) * a.NP / a.C;
      const long long pe = static_cast<long long>(c + 1) * a.NP / a.C;
      const uint16_t* meta_u = a.meta + static_cast<size_t>(unit) * a.np_cap * 2 * kD;
      float* wsU_u = a.wsU + static_cast<size_t>(unit) * a.np_stride;
      float lmin = INFINITY, lmax = -INFINITY;
      for (long long p0 = pb + static_cast<long long>(warp) * PPI; p0 < pe;
           p0 += static_cast<long long>(NWARPS) * PPI) {
        uint4 x[PPI];
#pragma unroll
        for (int i = 0; i < PPI; ++i) {
          if (p0 + i < pe) x[i] = ld_stream16(meta_u + (p0 + i) * 2 * kD + lane * 8);
          else x[i] = make_uint4(0u, 0u, 0u, 0u);
        }
        float v[NV];
#pragma unroll
        for (int i = 0; i < PPI; ++i) {
          const float xf[8] = {bf_lo(x[i].x), bf_hi(x[i].x), bf_lo(x[i].y), bf_hi(x[i].y),
                               bf_lo(x[i].z), bf_hi(x[i].z), bf_lo(x[i].w), bf_hi(x[i].w)};
#pragma unroll
          for (int h = 0; h < RG; ++h) {
            float acc = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc = fmaf(qs[h][e], xf[e], acc);
            v[i * RG + h] = acc;
          }
        }
        reduce_scatter<NV>(v, lane);
        const int idx = lane >> SH;
        float u = v[0];
#pragma unroll
        for (int mm = 1; mm < RG; mm <<= 1) u = fmaxf(u, __shfl_xor_sync(0xFFFFFFFFu, u, mm << SH));
        const long long p = p0 + idx / RG;
        if ((idx % RG) == 0 && (lane & ((1 << SH) - 1)) == 0 && p < pe) {
          wsU_u[p] = u;
          if (a.dbg_U) a.dbg_U[static_cast<size_t>(unit) * a.NP + p] = u;
          lmin = fminf(lmin, u);
          lmax = fmaxf(lmax, u);
        }
      }
      // CTA min / max of its bounds
#pragma unroll
      for (int o2 = 16; o2 >= 1; o2 >>= 1) {
        lmin = fminf(lmin, __shfl_xor_sync(0xFFFFFFFFu, lmin, o2));
        lmax = fmaxf(lmax, __shfl_xor_sync(0xFFFFFFFFu, lmax, o2));
      }
      float* red = reinterpret_cast<float*>(S.scratch);
      if (lane == 0) {
        red[warp] = lmin;
        red[NWARPS + warp] = lmax;
      }
      __syncthreads();
      if (tid == 0) {
        float mn = INFINITY, mx = -INFINITY;
        for (int w = 0; w < NWARPS; ++w) {
          mn = fminf(mn, red[w]);
          mx = fmaxf(mx, red[NWARPS + w]);
        }
        float* mm2 = a.wsMinMax + 2 * static_cast<size_t>(unit * kMaxCtasPerUnit + c);
        mm2[0] = mn;
        mm2[1] = mx;
      }

      // unit barrier 1; the query codes are computed while waiting
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        atom_add_acq_rel(ctr, 1u);
      }
      {
        const float* Wg = a.W + static_cast<size_t>(g) * kD * BITS;
        for (int oi = tid; oi < RG * BITS; oi += NT) {  // warp-uniform trip count
          const int h = oi / BITS, t = oi % BITS;
          float acc = 0.f;
#pragma unroll 8
          for (int i = 0; i < kD; ++i) acc = fmaf(S.qf[h * kD + i], __ldg(Wg + i * BITS + t), acc);
          const uint32_t word = __ballot_sync(0xFFFFFFFFu, acc > 0.f);
          if (lane == 0) S.qc[h * WORDS + t / 32] = word;
        }
      }
      if (tid == 0) {
        int ok = 1;
        const long long t0 = clock64();
        while (ld_acquire(ctr) < static_cast<uint32_t>(a.C)) {
          if (static_cast<unsigned long long>(clock64() - t0) > a.spin_limit) {
            atomicExch(a.status, static_cast<uint32_t>(HHR_ERR_TIMEOUT));
            ok = 0;
            break;
          }
          __nanosleep(32);
        }
        __threadfence();
        s_misc[0] = ok;
      }
      __syncthreads();
      if (!s_misc[0]) return;

      // ---------------------------------------------------------- phase 2
      const int NP = a.NP, Pk = a.Pk;
      float* sU = reinterpret_cast<float*>(S.scratch);
      int* sHist = reinterpret_cast<int*>(S.scratch + sizeof(float) * align_up(NP, 4));
      uint32_t* sBits = reinterpret_cast<uint32_t*>(sHist + kBuckets);
      const int nwords = (NP + 31) / 32;
      float* sCU = reinterpret_cast<float*>(sBits + align_up(nwords, 4));
      int* sCP = reinterpret_cast<int*>(sCU + kCandMax);
      for (int p = tid; p < NP; p += NT) sU[p] = __ldcg(wsU_u + p);
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

      if (Pk >= NP) {
        for (int p0 = warp * 32; p0 < NP; p0 += NT) {
          const unsigned word = __ballot_sync(0xFFFFFFFFu, p0 + lane < NP);
          if (lane == 0) sBits[p0 >> 5] = word;
        }
      } else {
        const float gmin = s_flt[0];
        const float range = s_flt[1] - gmin;
        const float inv = (range > 0.f && range <= FLT_MAX) ? static_cast<float>(kBuckets) / range : 0.f;
        auto bucket = [&](float u) {
          const int bk = static_cast<int>((u - gmin) * inv);
          return bk < kBuckets - 1 ? bk : kBuckets - 1;
        };
        for (int p = tid; p < NP; p += NT) atomicAdd(&sHist[bucket(sU[p])], 1);
        __syncthreads();
        // thread t owns the four bins [4(NT-1-t), 4(NT-1-t)+4): a scan in
        // thread order counts the pages in higher bins
        static_assert(kBuckets == 4 * NT, "bin ownership assumes 4 bins per thread");
        const int base = 4 * (NT - 1 - tid);
        const int c4 = sHist[base] + sHist[base + 1] + sHist[base + 2] + sHist[base + 3];
        int tot;
        int running = block_excl_scan(c4, s_scan, &tot);
        for (int bin = base + 3; bin >= base; --bin) {
          const int hcount = sHist[bin];
          if (running < Pk && running + hcount >= Pk) {
            s_misc[3] = bin;
            s_misc[4] = running;
          }
          running += hcount;
        }
        __syncthreads();
        const int bstar = s_misc[3];
        const int need = Pk - s_misc[4];
        const int cntB = sHist[bstar];
        if (cntB == need) {
          for (int p0 = warp * 32; p0 < NP; p0 += NT) {
            const int p = p0 + lane;
            const unsigned word = __ballot_sync(0xFFFFFFFFu, p < NP && bucket(sU[p]) >= bstar);
            if (lane == 0) sBits[p0 >> 5] = word;
          }
        } else if (cntB <= kCandMax) {
          for (int p0 = warp * 32; p0 < NP; p0 += NT) {
            const int p = p0 + lane;
            const int bk = p < NP ? bucket(sU[p]) : -1;
            const unsigned word = __ballot_sync(0xFFFFFFFFu, bk > bstar);
            if (lane == 0) sBits[p0 >> 5] = word;
            if (bk == bstar) {
              const int slot = atomicAdd(&s_misc[2], 1);
              sCU[slot] = sU[p];
              sCP[slot] = p;
            }
          }
          __syncthreads();
          const int nc = s_misc[2];
          for (int i = tid; i < nc; i += NT) {
            const float u = sCU[i];
            const int pi = sCP[i];
            int rank = 0;
            for (int j = 0; j < nc; ++j) {
              const float uj = sCU[j];
              rank += (uj > u) || (uj == u && sCP[j] < pi);
            }
            if (rank < need) atomicOr(&sBits[pi >> 5], 1u << (pi & 31));
          }
        } else {
          // many equal-looking bounds: exact search for the Pk-th largest key
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
      }
      __syncthreads();

      // ---------------------------------------------------------- phase 3
      const int ks = static_cast<int>(static_cast<long long>(c) * Pk / a.C);
      const int ke = static_cast<int>(static_cast<long long>(c + 1) * Pk / a.C);
      {
        const int span = (NP + NT - 1) / NT;
        const int lo = tid * span, hi = min(NP, lo + span);
        int cnt = 0;
        for (int p = lo; p < hi; ++p) cnt += (sBits[p >> 5] >> (p & 31)) & 1u;
        int tot;
        int pos = block_excl_scan(cnt, s_scan, &tot);
        int32_t* pidx = a.page_idx + static_cast<size_t>(unit) * a.P;
        for (int p = lo; p < hi; ++p) {
          if ((sBits[p >> 5] >> (p & 31)) & 1u) {
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
      int* sHD = reinterpret_cast<int*>(S.scratch);  // [BITS + 1]
      for (int i = tid; i <= BITS; i += NT) sHD[i] = 0;
      uint32_t qc[RG][WORDS];
#pragma unroll
      for (int h = 0; h < RG; ++h)
#pragma unroll
        for (int w = 0; w < WORDS; ++w) qc[h][w] = S.qc[h * WORDS + w];
      __syncthreads();
      const uint32_t* codes_u = a.codes + static_cast<size_t>(unit) * a.n_cap * WORDS;
      int32_t* dbgD = a.dbg_D ? a.dbg_D + static_cast<size_t>(unit) * a.P * S_ : nullptr;
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
            int best = 1 << 20;
#pragma unroll
            for (int h = 0; h < RG; ++h) {
              int dist = 0;
#pragma unroll
              for (int w = 0; w < WORDS; ++w) dist += __popc(qc[h][w] ^ kc[w]);
              best = min(best, dist);
            }
            D = best;
          }
          S.tokD[i] = static_cast<uint16_t>(D);
          if (dbgD) dbgD[static_cast<size_t>(ks + slot) * S_ + off] = (D == 0xFFFF) ? -1 : D;
        }
        const unsigned grp = __match_any_sync(0xFFFFFFFFu, D);
        if (D != 0xFFFF && lane == __ffs(grp) - 1) atomicAdd(&sHD[D], __popc(grp));
      }
      if (c == 0 && dbgD)
        for (int i = Pk * S_ + tid; i < a.P * S_; i += NT) dbgD[i] = -1;
      __syncthreads();
      {
        int32_t* hrow = a.wsHist + static_cast<size_t>(unit * kMaxCtasPerUnit + c) * (BITS + 1);
        for (int i = tid; i <= BITS; i += NT) hrow[i] = sHD[i];
      }
      if (!unit_arrive_wait(ctr, 2u * a.C, a, &s_misc[0])) return;

      // ---------------------------------------------------------- phase 5
      int* sHA = reinterpret_cast<int*>(S.scratch);  // [C][BITS + 1]
      {
        const int32_t* hall = a.wsHist + static_cast<size_t>(unit * kMaxCtasPerUnit) * (BITS + 1);
        for (int i = tid; i < a.C * (BITS + 1); i += NT) sHA[i] = __ldcg(hall + i);
      }
      __syncthreads();
      int tv = 0;
      if (tid <= BITS)
        for (int cc = 0; cc < a.C; ++cc) tv += sHA[cc * (BITS + 1) + tid];
      int n_cand;
      const int cum = block_excl_scan(tv, s_scan, &n_cand);
      const int k_eff = min(a.k, n_cand);
      if (tid == 0) {
        s_misc[5] = -1;
        s_misc[6] = 0;
      }
      __syncthreads();
      if (tid <= BITS && tv > 0 && cum < k_eff && cum + tv >= k_eff) {
        s_misc[5] = tid;
        s_misc[6] = k_eff - cum;
      }
      __syncthreads();
      const int T = s_misc[5];
      const int needT = s_misc[6];
      int* sBelow = s_aux;
      int* sEq = s_aux + kMaxCtasPerUnit;
      if (tid < a.C) {
        int below = 0;
        for (int v = 0; v < T; ++v) below += sHA[tid * (BITS + 1) + v];
        sBelow[tid] = below;
        sEq[tid] = T >= 0 ? sHA[tid * (BITS + 1) + T] : 0;
      }
      __syncthreads();
      if (tid == 0) {
        int pre_eq = 0, off = 0;
        for (int cc = 0; cc < a.C; ++cc) {
          const int quota = max(0, min(needT - pre_eq, sEq[cc]));
          const int selc = sBelow[cc] + quota;
          if (cc == c) {
            s_misc[7] = off;
            s_misc[8] = quota;
            s_misc[9] = selc;
          }
          pre_eq += sEq[cc];
          off += selc;
        }
      }
      __syncthreads();
      const int my_off = s_misc[7], my_quota = s_misc[8], my_sel = s_misc[9];
      {
        const int span = (ntok + NT - 1) / NT;
        const int lo = tid * span, hi = min(ntok, lo + span);
        int eq = 0;
        for (int i = lo; i < hi; ++i) eq += S.tokD[i] == T;
        int tmp;
        const int eq_pre = block_excl_scan(eq, s_scan, &tmp);
        int er = eq_pre, cnt = 0;
        for (int i = lo; i < hi; ++i) {
          const int D = S.tokD[i];
          bool f = D < T;
          if (D == T) f = (er++ < my_quota);
          cnt += f;
        }
        int pos = block_excl_scan(cnt, s_scan, &tmp);
        er = eq_pre;
        int32_t* tout = a.tok_idx + static_cast<size_t>(unit) * a.k;
        for (int i = lo; i < hi; ++i) {
          const int D = S.tokD[i];
          bool f = D < T;
          if (D == T) f = (er++ < my_quota);
          if (f) {
            const int slot = i / S_;
            const int n = S.my_pages[slot] * S_ + (i - slot * S_);
            tout[my_off + pos] = n;
            S.sel[pos] = n;
            ++pos;
          }
        }
        if (c == 0) {
          if (tid == 0) a.n_sel[unit] = k_eff;
          for (int i = k_eff + tid; i < a.k; i += NT) tout[i] = -1;
        }
      }
      __syncthreads();

      if constexpr (MODE == kModeFused) {
        for (int i = tid; i < RG * kD; i += NT) S.qf[i] *= a.scale_log2;
        __syncthreads();
        attend_and_finish<RG>(a, unit, c, S.sel, my_sel, S.qf, S.scratch,
                              3u * static_cast<uint32_t>(a.C), s_misc);
      } else {
        if (tid == 0) {
          __threadfence();
          const uint32_t old = atom_add_acq_rel(ctr, 1u);
          if (old == 3u * a.C - 1u) atomicExch(ctr, 0u);
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
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.grid_units * a.C));
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
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
