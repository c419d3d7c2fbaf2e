// Shared-memory tile loaders for the linear-branch kernels.  Each thread
// issues a batch of independent 16-byte global loads before converting and
// storing any of them, so that many bytes are in flight per SM (these
// kernels are bound by HBM bandwidth).  Tiles are written in the 128-byte
// swizzled layout the UMMA descriptors expect: 64-column chunks of `rows`
// rows, 128 bytes per row.
#pragma once

#include <cuda_bf16.h>

#include "sla_ptx.cuh"

namespace sla {

__device__ __forceinline__ float phi_f(float x) { return x > 0.f ? x + 1.f : __expf(x); }
__device__ __forceinline__ float dphi_f(float x) { return x > 0.f ? 1.f : __expf(x); }

__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16(x0, x1);
  lo = pack_bf16(x0 - bf16_lo(hi), x1 - bf16_hi(hi));
}

// bf16 [rows x D] (row pitch D elements) -> swizzled tile; rows >= valid are 0.
template <int D, int kBatch = 8>
__device__ __forceinline__ void load_rows_sw(uint8_t* dst, int rows, const __nv_bfloat16* src,
                                             int valid_rows, int tid, int nthreads) {
  constexpr int kC = D / 8;
  const int total = rows * kC;
  for (int e0 = tid; e0 < total; e0 += nthreads * kBatch) {
    uint4 u[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int e = e0 + b * nthreads, r = e / kC, c8 = e % kC;
      u[b] = make_uint4(0, 0, 0, 0);
      if (e < total && r < valid_rows)
        u[b] = __ldg(reinterpret_cast<const uint4*>(src + size_t(r) * D + c8 * 8));
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int e = e0 + b * nthreads;
      if (e < total) st_sw128_unit(dst, rows, e / kC, (e % kC) * 8, u[b]);
    }
  }
}

// fp32 [rows x D] (row pitch D) -> bf16 hi and lo swizzled tiles (x = hi + lo).
template <int D, int kBatch = 4>
__device__ __forceinline__ void load_split_sw(uint8_t* hi_t, uint8_t* lo_t, int rows,
                                              const float* src, int valid_rows, int tid,
                                              int nthreads) {
  constexpr int kC = D / 8;
  const int total = rows * kC;
  for (int e0 = tid; e0 < total; e0 += nthreads * kBatch) {
    float4 a[kBatch], c[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int e = e0 + b * nthreads, r = e / kC, c8 = e % kC;
      a[b] = make_float4(0.f, 0.f, 0.f, 0.f);
      c[b] = a[b];
      if (e < total && r < valid_rows) {
        const float4* p = reinterpret_cast<const float4*>(src + size_t(r) * D + c8 * 8);
        a[b] = __ldg(p);
        c[b] = __ldg(p + 1);
      }
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int e = e0 + b * nthreads;
      if (e < total) {
        uint32_t h[4], l[4];
        split2(a[b].x, a[b].y, h[0], l[0]);
        split2(a[b].z, a[b].w, h[1], l[1]);
        split2(c[b].x, c[b].y, h[2], l[2]);
        split2(c[b].z, c[b].w, h[3], l[3]);
        st_sw128_unit(hi_t, rows, e / kC, (e % kC) * 8, make_uint4(h[0], h[1], h[2], h[3]));
        st_sw128_unit(lo_t, rows, e / kC, (e % kC) * 8, make_uint4(l[0], l[1], l[2], l[3]));
      }
    }
  }
}

// bf16 [rows x D] -> phi() as bf16 hi (and optionally lo) swizzled tiles.
template <int D, int kBatch = 8>
__device__ __forceinline__ void load_phi_sw(uint8_t* hi_t, uint8_t* lo_t, int rows,
                                            const __nv_bfloat16* src, int valid_rows, int tid,
                                            int nthreads) {
  constexpr int kC = D / 8;
  const int total = rows * kC;
  for (int e0 = tid; e0 < total; e0 += nthreads * kBatch) {
    uint4 u[kBatch];
    bool ok[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int e = e0 + b * nthreads, r = e / kC, c8 = e % kC;
      ok[b] = e < total && r < valid_rows;
      u[b] = make_uint4(0, 0, 0, 0);
      if (ok[b]) u[b] = __ldg(reinterpret_cast<const uint4*>(src + size_t(r) * D + c8 * 8));
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int e = e0 + b * nthreads;
      if (e < total) {
        const uint32_t w[4] = {u[b].x, u[b].y, u[b].z, u[b].w};
        uint32_t h[4], l[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float x0 = ok[b] ? phi_f(bf16_lo(w[i])) : 0.f;
          const float x1 = ok[b] ? phi_f(bf16_hi(w[i])) : 0.f;
          split2(x0, x1, h[i], l[i]);
        }
        st_sw128_unit(hi_t, rows, e / kC, (e % kC) * 8, make_uint4(h[0], h[1], h[2], h[3]));
        if (lo_t)
          st_sw128_unit(lo_t, rows, e / kC, (e % kC) * 8, make_uint4(l[0], l[1], l[2], l[3]));
      }
    }
  }
}

// Read one bf16 element of a swizzled tile (64-column chunks of `rows` rows).
__device__ __forceinline__ float ld_sw_bf16(const uint8_t* tile, int rows, int r, int c) {
  const uint8_t* p = tile + (c >> 6) * rows * 128 + sw128_offset(r, c & 63);
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
}

}  // namespace sla
