// Key encoding for sm_100a: rotation (Eq. 4), per-page extrema (definition
// under Eq. 3) and projection + sign (Eq. 10, Eq. 1) of "HHR: Hierarchical
// Hash Retrieval for Efficient LLM Generation".
//
// One CTA encodes a tile of 64 consecutive keys of one (sequence, KV head).
// The tile is a [64 x 128] x [128 x 128] float32 product per pass (one pass
// for R, one per 128 columns of W), accumulated with fmaf in input-dimension
// order; each thread owns an 8 x 4 block of outputs.  The rotated tile is
// reduced per page to outward-rounded bf16 extrema, the projected tile is
// turned into code words with one warp ballot per 32 bits.

#include <cuda_bf16.h>

#include <cstdint>

#include "hhr_internal.cuh"

namespace hhr {
namespace {

constexpr int kTile = 64;      // keys per CTA
constexpr int kEncThreads = 256;
constexpr int kPadA = kTile + 4;   // transposed key tile row (floats)
constexpr int kPadB = kD + 4;      // operand / result row (floats)

struct EncSmem {
  float kt[kD][kPadA];      // keys, transposed: kt[i][row]
  float bm[kD][kPadB];      // R or a 128-column slice of W
  float res[kTile][kPadB];  // products of the current pass
};

__device__ __forceinline__ void load_operand(float (*bm)[kPadB], const float* src, int ld) {
  // 128 x 128 floats, row stride `ld` floats in global memory
#pragma unroll 16
  for (int idx = threadIdx.x; idx < kD * kD / 4; idx += kEncThreads) {
    const int i = idx / (kD / 4), j4 = idx % (kD / 4);
    const float4 v = __ldg(reinterpret_cast<const float4*>(src + static_cast<size_t>(i) * ld) + j4);
    *reinterpret_cast<float4*>(&bm[i][j4 * 4]) = v;
  }
}

__device__ __forceinline__ void tile_product(EncSmem& s) {
  const int rg = threadIdx.x >> 5;   // rows 8 rg .. 8 rg + 7 (warp-uniform)
  const int cg = threadIdx.x & 31;   // cols 4 cg .. 4 cg + 3
  float acc[8][4];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
#pragma unroll 4
  for (int i = 0; i < kD; ++i) {
    const float4 a0 = *reinterpret_cast<const float4*>(&s.kt[i][rg * 8]);
    const float4 a1 = *reinterpret_cast<const float4*>(&s.kt[i][rg * 8 + 4]);
    const float4 bv = *reinterpret_cast<const float4*>(&s.bm[i][cg * 4]);
    const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float bb[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(av[r], bb[c], acc[r][c]);
  }
#pragma unroll
  for (int r = 0; r < 8; ++r)
    *reinterpret_cast<float4*>(&s.res[rg * 8 + r][cg * 4]) =
        make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
}

__global__ void __launch_bounds__(kEncThreads, 1) encode_kernel(const EncodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  EncSmem& s = *reinterpret_cast<EncSmem*>(smem_raw);
  const int unit = blockIdx.y;
  const int g = unit % a.Hkv;
  const int t0 = a.tile_begin + blockIdx.x * kTile;  // first key of the tile
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const size_t unit_rows = static_cast<size_t>(unit) * a.n_cap;
  const uint16_t* Ku = a.K + unit_rows * kD;

  // key tile, transposed to [dim][row]; rows outside [n_begin, n_end) are 0
#pragma unroll 4
  for (int idx = threadIdx.x; idx < kTile * (kD / 8); idx += kEncThreads) {
    const int row = idx / (kD / 8), c8 = idx % (kD / 8);
    const int n = t0 + row;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (n >= a.n_begin && n < a.n_end) v = __ldg(reinterpret_cast<const uint4*>(Ku + static_cast<size_t>(n) * kD) + c8);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      s.kt[c8 * 8 + 2 * e][row] = __uint_as_float(w[e] << 16);
      s.kt[c8 * 8 + 2 * e + 1][row] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
  }
  load_operand(s.bm, a.R + static_cast<size_t>(g) * kD * kD, kD);
  __syncthreads();
  tile_product(s);
  __syncthreads();

  // per-page extrema of the rotated keys, rounded outward to bf16
  {
    const int S = a.page;
    const int pages = kTile / S;
    __nv_bfloat16* meta_u = reinterpret_cast<__nv_bfloat16*>(a.meta) + static_cast<size_t>(unit) * a.np_cap * 2 * kD;
    for (int idx = threadIdx.x; idx < pages * kD; idx += kEncThreads) {
      const int pl = idx / kD, j = idx % kD;
      const int n_page = t0 + pl * S;                 // first token of the page
      const int lo_n = max(n_page, a.n_begin);
      const int hi_n = min(n_page + S, a.n_end);
      if (lo_n >= hi_n) continue;                     // no new key in this page
      float mn = INFINITY, mx = -INFINITY;
      for (int n = lo_n; n < hi_n; ++n) {
        const float v = s.res[n - t0][j];
        mn = fminf(mn, v);
        mx = fmaxf(mx, v);
      }
      __nv_bfloat16 blo = __float2bfloat16_rd(mn);
      __nv_bfloat16 bhi = __float2bfloat16_ru(mx);
      const size_t page = static_cast<size_t>(n_page / S);
      __nv_bfloat16* dst = meta_u + page * 2 * kD;
      if (n_page < a.n_begin) {  // page already holds keys [n_page, n_begin)
        blo = __hmin(blo, dst[j]);
        bhi = __hmax(bhi, dst[kD + j]);
      }
      dst[j] = blo;
      dst[kD + j] = bhi;
    }
  }

  // projection + sign, 128 columns of W per pass
  const int words = a.bits / 32;
  uint32_t* codes_u = a.codes + unit_rows * words;
  for (int col0 = 0; col0 < a.bits; col0 += kD) {
    __syncthreads();
    load_operand(s.bm, a.W + static_cast<size_t>(g) * kD * a.bits + col0, a.bits);
    __syncthreads();
    tile_product(s);
    __syncthreads();
    // warp w packs rows w, w + 8, ...; lane = bit within a word
    for (int row = warp; row < kTile; row += kEncThreads / 32) {
      const int n = t0 + row;
      const bool live = n >= a.n_begin && n < a.n_end;   // warp-uniform
#pragma unroll
      for (int w4 = 0; w4 < kD / 32; ++w4) {
        const unsigned word = __ballot_sync(0xFFFFFFFFu, s.res[row][w4 * 32 + lane] > 0.f);
        if (live && lane == 0) codes_u[static_cast<size_t>(n) * words + col0 / 32 + w4] = word;
      }
    }
  }
}

}  // namespace

cudaError_t launch_encode(const EncodeArgs& a, cudaStream_t stream) {
  const size_t smem = sizeof(EncSmem);
  cudaError_t e = cudaFuncSetAttribute(encode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(a.n_tiles), static_cast<unsigned>(a.units));
  encode_kernel<<<grid, kEncThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace hhr
