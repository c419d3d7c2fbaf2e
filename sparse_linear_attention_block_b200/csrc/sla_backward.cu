// Backward of SLA with the classes held fixed.
//
// SLA (arXiv 2509.24006), abstract: the fused kernel supports both forward
// and backward passes.  The pages give no backward formulas; these are the
// gradients of O = O_s + O_l W_proj as defined by the forward (classes are
// piecewise constant and carry no gradient):
//   sparse:  D_t = dO_t . O_s,t;  P = exp(S - LSE);  dV += P^T dO;
//            dP = dO V^T;  dS = P (dP - D);  dQ += scale dS K;  dK += scale dS^T Q
//   linear:  dO_l = dO W^T;  dnum = dO_l / den;  dden = -(dO_l . O_l) / den
//            A_i = phi(Q_i)^T dnum_i, a_i = phi(Q_i)^T dden_i   (per query block)
//            dh_j = sum_{i: j marginal in row i} A_i, dz_j alike   (aggregation GEMM)
//            dQ += (dnum H_i^T + dden Z_i) * phi'(Q)
//            dK += (V dh_j^T + dz_j) * phi'(K);  dV += phi(K) dh_j
//   W_proj:  dW = sum_t O_l,t^T dO_t
//
// Kernels (all tcgen05 for the contractions):
//   bwd_prep_kernel    per 128-token tile: D, dnum, dden; dW accumulated in TMEM
//                      across the tiles of a persistent CTA
//   bwd_summ_kernel    per 128-token tile: A_i (bf16 hi/lo planes) and a_i
//   bwd_sparse_kernel  per 128-key tile (key blocks 2q, 2q+1): walks the union of
//                      their critical query blocks (column CSR); dK, dV in TMEM,
//                      dQ^T per query block reduced into fp32 dQ with atomics
//   bwd_linear_kernel  per 128-token tile: the linear-branch dQ, dK, dV, added in place
#include <cuda_bf16.h>

#include "sla_internal.h"
#include "sla_ptx.cuh"

namespace sla {
namespace {

__device__ __forceinline__ float phi_f(float x) { return x > 0.f ? x + 1.f : __expf(x); }
__device__ __forceinline__ float dphi_f(float x) { return x > 0.f ? 1.f : __expf(x); }

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Load a [rows x D] bf16 row-major global tile into a 128B-swizzled tile
// (64-column chunks of `rows` rows), zero for rows >= valid_rows.
template <int D>
__device__ __forceinline__ void load_rows_sw(uint8_t* dst, int rows, const __nv_bfloat16* src,
                                             int valid_rows, int tid, int nthreads) {
  for (int e = tid; e < rows * (D / 8); e += nthreads) {
    const int r = e / (D / 8), c8 = e % (D / 8);
    uint4 u = make_uint4(0, 0, 0, 0);
    if (r < valid_rows) u = *reinterpret_cast<const uint4*>(src + size_t(r) * D + c8 * 8);
    st_sw128_unit(dst, rows, r, c8 * 8, u);
  }
}

// Load an fp32 [rows x D] global matrix into bf16 hi/lo 128B-swizzled tiles
// (64-column chunks of `rows` rows); rows >= valid_rows are zero.
template <int D>
__device__ __forceinline__ void load_split_sw(uint8_t* hi_t, uint8_t* lo_t, int rows,
                                              const float* src, int valid_rows, int tid,
                                              int nthreads) {
  for (int e = tid; e < rows * (D / 8); e += nthreads) {
    const int r = e / (D / 8), c8 = e % (D / 8);
    float x[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (r < valid_rows) {
      const float4 u0 = *reinterpret_cast<const float4*>(src + size_t(r) * D + c8 * 8);
      const float4 u1 = *reinterpret_cast<const float4*>(src + size_t(r) * D + c8 * 8 + 4);
      x[0] = u0.x; x[1] = u0.y; x[2] = u0.z; x[3] = u0.w;
      x[4] = u1.x; x[5] = u1.y; x[6] = u1.z; x[7] = u1.w;
    }
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      h[i] = pack_bf16(x[2 * i], x[2 * i + 1]);
      l[i] = pack_bf16(x[2 * i] - bf16_lo(h[i]), x[2 * i + 1] - bf16_hi(h[i]));
    }
    st_sw128_unit(hi_t, rows, r, c8 * 8, make_uint4(h[0], h[1], h[2], h[3]));
    st_sw128_unit(lo_t, rows, r, c8 * 8, make_uint4(l[0], l[1], l[2], l[3]));
  }
}

// ============================================================================ bwd_prep
// Persistent over 128-token tiles (query blocks 2p, 2p+1); 128 threads, one
// row each; thread 0 issues the MMAs.  Per tile:
//   G = dO W^T, NUM_h = phi(Q) (H_h,hi + H_h,lo)           (tcgen05)
//   O_l = NUM / den, D = dO . O_s, dnum = G / den, dden = -(G . O_l) / den
//   dW += (O_l,hi + O_l,lo)^T dO  accumulated in TMEM over the CTA's tiles
constexpr int kTile32 = 128 * 128 * 2;  // 128 rows x 2 chunks (D = 64 padded)

template <int D>
__global__ void __launch_bounds__(128, 1) bwd_prep_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ d_o,
    const __nv_bfloat16* __restrict__ w_proj, const float* __restrict__ o_s,
    const float* __restrict__ den, const float* __restrict__ h_agg, float* __restrict__ dvec,
    float* __restrict__ dnum, float* __restrict__ dden, float* __restrict__ dw, int N, int T,
    int BH, int* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = base;                  // phi(Q)                      [t][a]
  uint8_t* sDO = sA + kTile32;         // dO                          [t][c]
  uint8_t* sW = sDO + kTile32;         // W_proj                      [a][c]
  uint8_t* sHh = sW + kTile32;         // H hi [a][c], later O_l hi   [t][a]
  uint8_t* sHl = sHh + kTile32;        // H lo [a][c], later O_l lo   [t][a]
  __shared__ uint64_t bar[3];
  __shared__ uint32_t tmem_base;
  const int t = threadIdx.x, warp = t / 32, half = t >> 6;
  const int P = (T + 1) / 2, ntiles = P * BH;
  constexpr uint32_t kCols = 4 * D;  // G | NUM0 | NUM1 | dW
  if (warp == 0) tmem_alloc(&tmem_base, kCols);
  if (t == 0) {
    for (int b = 0; b < 3; ++b) mbar_init(&bar[b], 1);
    fence_barrier_init();
  }
  load_rows_sw<D>(sW, D, w_proj, D, t, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const uint32_t lane_base = uint32_t(warp * 32) << 16;
  int it = 0;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int bh = tile / P, p = tile % P;
    const int blk = 2 * p + half;
    const bool row_ok = blk < T;
    const size_t tok = size_t(p) * 128 + t;
    const size_t rowoff = (size_t(bh) * N + tok) * D;
    bool ok = true;
    load_rows_sw<D>(sDO, 128, d_o + (size_t(bh) * N + size_t(p) * 128) * D,
                    min(128, N - p * 128), t, 128);
    for (int c8 = 0; c8 < D / 8; ++c8) {
      uint4 u = make_uint4(0, 0, 0, 0);
      if (row_ok) u = *reinterpret_cast<const uint4*>(q + rowoff + c8 * 8);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      uint32_t pw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) pw[e] = pack_bf16(phi_f(bf16_lo(w[e])), phi_f(bf16_hi(w[e])));
      st_sw128_unit(sA, 128, t, c8 * 8, make_uint4(pw[0], pw[1], pw[2], pw[3]));
    }
    for (int m = 0; m < 2; ++m) {
      const int b2 = 2 * p + m;
      load_split_sw<D>(sHh, sHl, D, h_agg + (size_t(bh) * T + (b2 < T ? b2 : 0)) * D * D,
                       b2 < T ? D : 0, t, 128);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (t == 0) {
        constexpr uint32_t id_g = idesc_bf16(128, D, 0, 0);
        constexpr uint32_t id_n = idesc_bf16(128, D, 0, 1);
        if (m == 0) {
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_ss(tmem, desc_kmajor(smem_u32(sDO), 128, ks), desc_kmajor(smem_u32(sW), D, ks),
                   id_g, ks > 0);
        }
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          mma_ss(tmem + (1 + m) * D, desc_kmajor(smem_u32(sA), 128, ks),
                 desc_mnmajor(smem_u32(sHh), D, ks), id_n, ks > 0);
          mma_ss(tmem + (1 + m) * D, desc_kmajor(smem_u32(sA), 128, ks),
                 desc_mnmajor(smem_u32(sHl), D, ks), id_n, 1);
        }
        mma_commit(&bar[m]);
      }
      ok = mbar_wait(&bar[m], it & 1, err, nullptr) && ok;
      tc_fence_after();
    }
    // per row: O_l, D, dnum, dden
    const float dn = row_ok ? den[size_t(bh) * N + tok] : 0.f;
    const float inv = dn > 0.f ? 1.0f / dn : 0.f;
    float gdot = 0.f, dsum = 0.f;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 16) {
      float g[16], nm[16];
      tmem_ld16(tmem + lane_base + c0, g);
      tmem_ld16(tmem + lane_base + (1 + half) * D + c0, nm);
      tmem_ld_wait();
      uint32_t ol_hi[8], ol_lo[8];
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        const float o0 = nm[e] * inv, o1 = nm[e + 1] * inv;
        gdot = fmaf(g[e], o0, fmaf(g[e + 1], o1, gdot));
        ol_hi[e / 2] = pack_bf16(o0, o1);
        ol_lo[e / 2] = pack_bf16(o0 - bf16_lo(ol_hi[e / 2]), o1 - bf16_hi(ol_hi[e / 2]));
      }
      if (row_ok) {
        const float* osr = o_s + rowoff + c0;
        const __nv_bfloat16* dor = d_o + rowoff + c0;
        float* dnr = dnum + rowoff + c0;
#pragma unroll
        for (int e = 0; e < 16; e += 8) {
          const uint4 u = *reinterpret_cast<const uint4*>(dor + e);
          const float4 s0 = *reinterpret_cast<const float4*>(osr + e);
          const float4 s1 = *reinterpret_cast<const float4*>(osr + e + 4);
          dsum = fmaf(bf16_lo(u.x), s0.x, fmaf(bf16_hi(u.x), s0.y, dsum));
          dsum = fmaf(bf16_lo(u.y), s0.z, fmaf(bf16_hi(u.y), s0.w, dsum));
          dsum = fmaf(bf16_lo(u.z), s1.x, fmaf(bf16_hi(u.z), s1.y, dsum));
          dsum = fmaf(bf16_lo(u.w), s1.z, fmaf(bf16_hi(u.w), s1.w, dsum));
          *reinterpret_cast<float4*>(dnr + e) =
              make_float4(g[e] * inv, g[e + 1] * inv, g[e + 2] * inv, g[e + 3] * inv);
          *reinterpret_cast<float4*>(dnr + e + 4) =
              make_float4(g[e + 4] * inv, g[e + 5] * inv, g[e + 6] * inv, g[e + 7] * inv);
        }
      }
      st_sw128_unit(sHh, 128, t, c0, make_uint4(ol_hi[0], ol_hi[1], ol_hi[2], ol_hi[3]));
      st_sw128_unit(sHh, 128, t, c0 + 8, make_uint4(ol_hi[4], ol_hi[5], ol_hi[6], ol_hi[7]));
      st_sw128_unit(sHl, 128, t, c0, make_uint4(ol_lo[0], ol_lo[1], ol_lo[2], ol_lo[3]));
      st_sw128_unit(sHl, 128, t, c0 + 8, make_uint4(ol_lo[4], ol_lo[5], ol_lo[6], ol_lo[7]));
    }
    if (row_ok) {
      dvec[size_t(bh) * N + tok] = dsum;
      dden[size_t(bh) * N + tok] = dn > 0.f ? -gdot * inv : 0.f;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (t == 0) {
      constexpr uint32_t id_w = idesc_bf16(128, D, 1, 1);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        mma_ss(tmem + 3 * D, desc_mnmajor(smem_u32(sHh), 128, ks),
               desc_mnmajor(smem_u32(sDO), 128, ks), id_w, (it | ks) != 0);
        mma_ss(tmem + 3 * D, desc_mnmajor(smem_u32(sHl), 128, ks),
               desc_mnmajor(smem_u32(sDO), 128, ks), id_w, 1);
      }
      mma_commit(&bar[2]);
    }
    ok = mbar_wait(&bar[2], it & 1, err, nullptr) && ok;
    tc_fence_after();
    const int failed = __syncthreads_or(!ok);  // CTA-uniform exit on a timed-out wait
    tc_fence_after();
    if (failed) break;
  }
  // flush this CTA's share of dW
  if (it > 0 && warp * 32 < D) {
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      float v[32];
      tmem_ld32(tmem + lane_base + 3 * D + c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) atomicAdd(dw + size_t(t) * D + c0 + e, v[e]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free(tmem, kCols);
}

// ============================================================================ bwd_summ
// Per 128-token tile: A_h = phi(Q_h)^T dnum_h for the two query blocks
// (M = feature a, N = c, K = the block's 64 tokens; hi*hi + hi*lo + lo*hi),
// written as bf16 hi/lo planes, and a_h = sum_t phi(Q_t) dden_t (fp32).
template <int D>
__global__ void __launch_bounds__(128, 1) bwd_summ_kernel(
    const __nv_bfloat16* __restrict__ q, const float* __restrict__ dnum,
    const float* __restrict__ dden, __nv_bfloat16* __restrict__ summ_hi,
    __nv_bfloat16* __restrict__ summ_lo, float* __restrict__ zsum, int N, int T, int* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQh = base;                 // phi(Q) hi [t][a]
  uint8_t* sQl = sQh + kTile32;        // phi(Q) lo
  uint8_t* sNh = sQl + kTile32;        // dnum hi   [t][c]
  uint8_t* sNl = sNh + kTile32;        // dnum lo
  __shared__ float sDd[128];
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base;
  const int p = blockIdx.x, bh = blockIdx.y, t = threadIdx.x, warp = t / 32, half = t >> 6;
  const bool row_ok = 2 * p + half < T;
  const size_t tok = size_t(p) * 128 + t;
  const size_t rowoff = (size_t(bh) * N + tok) * D;
  if (warp == 0) tmem_alloc(&tmem_base, 2 * D);
  if (t == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  for (int c8 = 0; c8 < D / 8; ++c8) {
    uint4 u = make_uint4(0, 0, 0, 0);
    if (row_ok) u = *reinterpret_cast<const uint4*>(q + rowoff + c8 * 8);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a = row_ok ? phi_f(bf16_lo(w[e])) : 0.f, b = row_ok ? phi_f(bf16_hi(w[e])) : 0.f;
      h[e] = pack_bf16(a, b);
      l[e] = pack_bf16(a - bf16_lo(h[e]), b - bf16_hi(h[e]));
    }
    st_sw128_unit(sQh, 128, t, c8 * 8, make_uint4(h[0], h[1], h[2], h[3]));
    st_sw128_unit(sQl, 128, t, c8 * 8, make_uint4(l[0], l[1], l[2], l[3]));
  }
  load_split_sw<D>(sNh, sNl, 128, dnum + (size_t(bh) * N + size_t(p) * 128) * D,
                   min(128, N - p * 128), t, 128);
  sDd[t] = row_ok ? dden[size_t(bh) * N + tok] : 0.f;
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  if (t == 0) {
    constexpr uint32_t id = idesc_bf16(128, D, 1, 1);
    for (int m = 0; m < 2; ++m) {
      const uint32_t o = m * 8192;  // the block's 64 token rows inside each chunk
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t qh = desc_mnmajor(smem_u32(sQh) + o, 128, ks);
        const uint64_t ql = desc_mnmajor(smem_u32(sQl) + o, 128, ks);
        const uint64_t nh = desc_mnmajor(smem_u32(sNh) + o, 128, ks);
        const uint64_t nl = desc_mnmajor(smem_u32(sNl) + o, 128, ks);
        mma_ss(tmem + m * D, qh, nh, id, ks > 0);
        mma_ss(tmem + m * D, qh, nl, id, 1);
        mma_ss(tmem + m * D, ql, nh, id, 1);
      }
    }
    mma_commit(&bar);
  }
  const bool ok = mbar_wait(&bar, 0, err, nullptr);
  tc_fence_after();
  if (warp * 32 < D) {
    const int a = t;
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
#pragma unroll 1
    for (int m = 0; m < 2; ++m) {
      const int b2 = 2 * p + m;
      const size_t o = ((size_t(bh) * T + (b2 < T ? b2 : 0)) * D + a) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + lane_base + m * D + c0, v);
        tmem_ld_wait();
        if (b2 < T && ok) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint32_t h[4], l[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              h[i] = pack_bf16(v[e + 2 * i], v[e + 2 * i + 1]);
              l[i] = pack_bf16(v[e + 2 * i] - bf16_lo(h[i]), v[e + 2 * i + 1] - bf16_hi(h[i]));
            }
            *reinterpret_cast<uint4*>(summ_hi + o + c0 + e) = make_uint4(h[0], h[1], h[2], h[3]);
            *reinterpret_cast<uint4*>(summ_lo + o + c0 + e) = make_uint4(l[0], l[1], l[2], l[3]);
          }
        }
      }
      if (b2 < T) {
        float acc = 0.f;
        for (int r = 0; r < 64; ++r) {
          const int row = m * 64 + r;
          const uint32_t so = (a >> 6) * 128 * 128 + sw128_offset(row, a & 63);
          const float ph = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sQh + so));
          const float pl = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sQl + so));
          acc = fmaf(ph + pl, sDd[row], acc);
        }
        zsum[(size_t(bh) * T + b2) * D + a] = acc;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free(tmem, 2 * D);
}

// ============================================================================ bwd_sparse
constexpr int kBStages = 2;

template <int D>
struct BwdSmem {
  static constexpr int kKV = 128 * D * 2;        // K or V tile (128 keys)
  static constexpr int kQ = 64 * D * 2;          // Q_i or dO_i tile (64 queries)
  static constexpr int kStage = 2 * kQ + 2 * 256;  // Q, dO, LSE, D
  static constexpr int kDS = 128 * 128;          // dS^T bf16 [128 keys][64 q]
  static constexpr int kTiles = 2 * kKV + kBStages * kStage + kDS;
  static size_t total(int T) { return 1024 + kTiles + size_t(2 * T) * 3 + 16; }
};

template <int D>
__global__ void __launch_bounds__(192, 1) bwd_sparse_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
    const float* __restrict__ lse, const float* __restrict__ dvec,
    const int32_t* __restrict__ col_ptr, const int32_t* __restrict__ col_idx, int N, int T,
    int n_crit, float scale_log2, float scale, float* __restrict__ dq, float* __restrict__ dk,
    float* __restrict__ dv, int* err) {
  using L = BwdSmem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sK = base;
  uint8_t* sV = sK + L::kKV;
  uint8_t* sStage = sV + L::kKV;
  uint8_t* sDS = sStage + kBStages * L::kStage;
  uint16_t* ulist = reinterpret_cast<uint16_t*>(sDS + L::kDS);
  uint8_t* uflag = reinterpret_cast<uint8_t*>(ulist + 2 * T);

  __shared__ uint64_t kv_full, st_full[kBStages], st_empty[kBStages], s_full, p_full, m_done,
      fin;
  __shared__ uint32_t tmem_base;
  __shared__ int n_union, abort_flag;
  const int qp = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x / 32, lane = lane_id();
  const int kb0 = 2 * qp, kb1 = 2 * qp + 1;
  const bool has1 = kb1 < T;
  constexpr uint32_t kST = 0, kDPT = 64, kDQT = 128, kDV = 192, kDK = 192 + D;

  if (warp == 0) tmem_alloc(&tmem_base, 512);
  if (threadIdx.x == 32) {
    mbar_init(&kv_full, 1);
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 1);
    }
    mbar_init(&s_full, 1);
    mbar_init(&p_full, 128);
    mbar_init(&m_done, 1);
    mbar_init(&fin, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x == 128) {
    // union of the critical query blocks of key blocks 2q and 2q+1
    const int32_t* cp = col_ptr + size_t(bh) * (T + 1);
    const int32_t* ci = col_idx + size_t(bh) * T * n_crit;
    int a = cp[kb0], ae = cp[kb0 + 1];
    int b = has1 ? cp[kb1] : 0, be = has1 ? cp[kb1 + 1] : 0;
    const int cap = T * n_crit;
    if (a < 0 || ae > cap || a > ae || b < 0 || be > cap || b > be) {
      set_error(err, SLA_ERR_DEVICE);
      a = ae = b = be = 0;
    }
    int n = 0;
    while (a < ae || b < be) {
      const int x = a < ae ? ci[a] : 0x7FFFFFFF;
      const int y = b < be ? ci[b] : 0x7FFFFFFF;
      int i, f;
      if (x == y) { i = x; f = 3; ++a; ++b; }
      else if (x < y) { i = x; f = 1; ++a; }
      else { i = y; f = 2; ++b; }
      if (i < 0 || i >= T || n >= 2 * T) { set_error(err, SLA_ERR_DEVICE); continue; }
      ulist[n] = uint16_t(i);
      uflag[n] = uint8_t(f);
      ++n;
    }
    n_union = n;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const int nU = n_union;

  if (warp == 4) {
    if (lane == 0 && nU > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(&kv_full, 2 * L::kKV);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(sK + c * 128 * 128, &kv_full, &tm_k, c * 64, qp * 128, bh);
        tma_load_3d(sV + c * 128 * 128, &kv_full, &tm_v, c * 64, qp * 128, bh);
      }
      int issued = 0;
      for (int n = 0; n < nU; ++n) {
        const int s = n % kBStages;
        if (n >= kBStages &&
            !mbar_wait(&st_empty[s], ((n / kBStages) + 1) & 1, err, &abort_flag))
          break;
        uint8_t* st = sStage + s * L::kStage;
        const int i = ulist[n];
        mbar_arrive_expect_tx(&st_full[s], L::kStage);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(st + c * 64 * 128, &st_full[s], &tm_q, c * 64, i * 64, bh);
          tma_load_3d(st + L::kQ + c * 64 * 128, &st_full[s], &tm_do, c * 64, i * 64, bh);
        }
        bulk_load(st + 2 * L::kQ, lse + size_t(bh) * N + size_t(i) * 64, 256, &st_full[s]);
        bulk_load(st + 2 * L::kQ + 256, dvec + size_t(bh) * N + size_t(i) * 64, 256,
                  &st_full[s]);
        ++issued;
      }
      if (abort_flag) {
        mbar_wait(&kv_full, 0, nullptr, nullptr);
        for (int n = (issued > kBStages ? issued - kBStages : 0); n < issued; ++n)
          mbar_wait(&st_full[n % kBStages], (n / kBStages) & 1, nullptr, nullptr);
      }
    }
  } else if (warp == 5) {
    if (lane == 0 && nU > 0) {
      constexpr uint32_t id_s = idesc_bf16(128, 64, 0, 0);   // S^T, dP^T
      constexpr uint32_t id_g = idesc_bf16(128, D, 0, 1);    // dV, dK (A from TMEM)
      constexpr uint32_t id_q = idesc_bf16(128, 64, 1, 1);   // dQ^T = K^T dS^T
      bool ok = mbar_wait(&kv_full, 0, err, &abort_flag);
      const uint32_t k0 = smem_u32(sK), v0 = smem_u32(sV), ds0 = smem_u32(sDS);
      for (int n = 0; ok && n < nU; ++n) {
        const int s = n % kBStages;
        if (!(ok = mbar_wait(&st_full[s], (n / kBStages) & 1, err, &abort_flag))) break;
        tc_fence_after();
        const uint32_t q0 = smem_u32(sStage + s * L::kStage), do0 = q0 + L::kQ;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          mma_ss(tmem + kST, desc_kmajor(k0, 128, ks), desc_kmajor(q0, 64, ks), id_s, ks > 0);
          mma_ss(tmem + kDPT, desc_kmajor(v0, 128, ks), desc_kmajor(do0, 64, ks), id_s, ks > 0);
        }
        mma_commit(&s_full);
        if (!(ok = mbar_wait(&p_full, n & 1, err, &abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          mma_ts(tmem + kDV, tmem + kST + ks * 8, desc_mnmajor(do0, 64, ks), id_g, (n | ks) != 0);
          mma_ts(tmem + kDK, tmem + kDPT + ks * 8, desc_mnmajor(q0, 64, ks), id_g, (n | ks) != 0);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss(tmem + kDQT, desc_mnmajor(k0, 128, ks), desc_mnmajor(ds0, 128, ks), id_q, ks > 0);
        mma_commit(&m_done);
        mma_commit(&st_empty[s]);
      }
      mma_commit(&fin);
      mbar_wait(&fin, 0, nullptr, nullptr);
    }
  } else {
    const int r = threadIdx.x;  // key row == TMEM lane
    const int half = r >> 6;
    const bool key_ok = (half == 0) || has1;
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    bool ok = true;
    for (int n = 0; n < nU; ++n) {
      const int s = n % kBStages;
      const int i = ulist[n];
      const float* sl = reinterpret_cast<const float*>(sStage + s * L::kStage + 2 * L::kQ);
      const float* sd = sl + 64;
      if (!(ok = mbar_wait(&s_full, n & 1, err, &abort_flag))) break;
      tc_fence_after();
      float st[64], dp[64];
      tmem_ld32(tmem + lane_base + kST, reinterpret_cast<float(&)[32]>(st[0]));
      tmem_ld32(tmem + lane_base + kST + 32, reinterpret_cast<float(&)[32]>(st[32]));
      tmem_ld32(tmem + lane_base + kDPT, reinterpret_cast<float(&)[32]>(dp[0]));
      tmem_ld32(tmem + lane_base + kDPT + 32, reinterpret_cast<float(&)[32]>(dp[32]));
      tmem_ld_wait();
      const bool member = key_ok && ((uflag[n] >> half) & 1);
#pragma unroll
      for (int e = 0; e < 64; ++e) {
        const float pr = member ? exp2f(fmaf(st[e], scale_log2, -sl[e] * 1.4426950408889634f))
                                : 0.f;
        st[e] = pr;
        dp[e] = pr * (dp[e] - sd[e]);
      }
      uint32_t pk[16];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(st[32 * h2 + 2 * e], st[32 * h2 + 2 * e + 1]);
        tmem_st16(tmem + lane_base + kST + 16 * h2, pk);
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(dp[32 * h2 + 2 * e], dp[32 * h2 + 2 * e + 1]);
        tmem_st16(tmem + lane_base + kDPT + 16 * h2, pk);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          st_sw128_unit(sDS, 128, r, 32 * h2 + 8 * u,
                        make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]));
      }
      fence_proxy_async_smem();
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full);
      if (!(ok = mbar_wait(&m_done, n & 1, err, &abort_flag))) break;
      tc_fence_after();
      // dQ_i^T rows (lane = feature a) reduced into dQ
      if (warp * 32 < D) {
        float* dst = dq + (size_t(bh) * N + size_t(i) * 64) * D + r;
#pragma unroll 1
        for (int c0 = 0; c0 < 64; c0 += 32) {
          float v[32];
          tmem_ld32(tmem + lane_base + kDQT + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) atomicAdd(dst + size_t(c0 + e) * D, v[e] * scale);
        }
      }
    }
    // dK, dV of this tile's keys
    const size_t key = size_t(qp) * 128 + r;
    float* dkr = dk + (size_t(bh) * N + key) * D;
    float* dvr = dv + (size_t(bh) * N + key) * D;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      float a[32], b[32];
      if (nU > 0) {
        tmem_ld32(tmem + lane_base + kDK + c0, a);
        tmem_ld32(tmem + lane_base + kDV + c0, b);
        tmem_ld_wait();
      }
      if (key_ok) {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const bool h = nU > 0 && ok;
          *reinterpret_cast<float4*>(dkr + c0 + e) =
              h ? make_float4(a[e] * scale, a[e + 1] * scale, a[e + 2] * scale, a[e + 3] * scale)
                : make_float4(0.f, 0.f, 0.f, 0.f);
          *reinterpret_cast<float4*>(dvr + c0 + e) =
              h ? make_float4(b[e], b[e + 1], b[e + 2], b[e + 3]) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free(tmem, 512);
}

// ============================================================================ bwd_linear
// Per 128-token tile (blocks 2p, 2p+1 as query blocks and as key blocks);
// 128 threads, one row each; thread 0 issues the MMAs; the two halves' H
// (resp. dh) pass through one shared-memory slot in turn.
//   phase 1: dQ += ((dnum_hi + dnum_lo) (H_hi + H_lo)^T + dden Z) * phi'(Q)
//   phase 2: dK += (V (dh_hi + dh_lo)^T + dz) * phi'(K)
//            dV += (phi(K)_hi + phi(K)_lo) (dh_hi + dh_lo)
// (products drop the lo*lo term).
template <int D>
__global__ void __launch_bounds__(128, 1) bwd_linear_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const float* __restrict__ h_agg,
    const float* __restrict__ z_agg, const float* __restrict__ dh,
    const float* __restrict__ dz, const float* __restrict__ dnum, const float* __restrict__ dden,
    float* __restrict__ dq, float* __restrict__ dk, float* __restrict__ dv, int N, int T,
    int* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* s0 = base;             // phase 1: dnum hi | phase 2: V        [t][c]
  uint8_t* s1 = s0 + kTile32;     // phase 1: dnum lo | phase 2: phi(K) hi [t][a]
  uint8_t* s2 = s1 + kTile32;     //                    phase 2: phi(K) lo [t][a]
  uint8_t* sMh = s2 + kTile32;    // H / dh hi [a][c]
  uint8_t* sMl = sMh + kTile32;   // H / dh lo [a][c]
  __shared__ float sZ[2][D];
  __shared__ uint64_t bar[4];
  __shared__ uint32_t tmem_base;
  const int p = blockIdx.x, bh = blockIdx.y, t = threadIdx.x, warp = t / 32, half = t >> 6;
  const bool row_ok = 2 * p + half < T;
  const size_t tok = size_t(p) * 128 + t;
  const size_t rowoff = (size_t(bh) * N + tok) * D;
  const uint32_t lane_base = uint32_t(warp * 32) << 16;
  constexpr uint32_t kCols = 4 * D;
  if (warp == 0) tmem_alloc(&tmem_base, kCols);
  if (t == 0) {
    for (int b = 0; b < 4; ++b) mbar_init(&bar[b], 1);
    fence_barrier_init();
  }
  // ---------------- phase 1: dQ
  load_split_sw<D>(s0, s1, 128, dnum + (size_t(bh) * N + size_t(p) * 128) * D,
                   min(128, N - p * 128), t, 128);
  for (int e = t; e < 2 * D; e += 128) {
    const int b2 = 2 * p + e / D;
    sZ[e / D][e % D] = b2 < T ? z_agg[(size_t(bh) * T + b2) * D + e % D] : 0.f;
  }
  bool ok = true;
  for (int m = 0; m < 2; ++m) {
    const int b2 = 2 * p + m;
    load_split_sw<D>(sMh, sMl, D, h_agg + (size_t(bh) * T + (b2 < T ? b2 : 0)) * D * D,
                     b2 < T ? D : 0, t, 128);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (t == 0) {
      constexpr uint32_t id = idesc_bf16(128, D, 0, 0);
      const uint32_t hh = smem_u32(sMh), hl = smem_u32(sMl);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint64_t ah = desc_kmajor(smem_u32(s0), 128, ks);
        const uint64_t al = desc_kmajor(smem_u32(s1), 128, ks);
        mma_ss(tmem_base + m * D, ah, desc_kmajor(hh, D, ks), id, ks > 0);
        mma_ss(tmem_base + m * D, ah, desc_kmajor(hl, D, ks), id, 1);
        mma_ss(tmem_base + m * D, al, desc_kmajor(hh, D, ks), id, 1);
      }
      mma_commit(&bar[m]);
    }
    ok = mbar_wait(&bar[m], 0, err, nullptr) && ok;
    tc_fence_after();
  }
  const uint32_t tmem = tmem_base;
  {
    const float ddn = row_ok ? dden[size_t(bh) * N + tok] : 0.f;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 16) {
      float g[16];
      tmem_ld16(tmem + lane_base + half * D + c0, g);
      tmem_ld_wait();
      if (row_ok && ok) {
        const uint4 u0 = *reinterpret_cast<const uint4*>(q + rowoff + c0);
        const uint4 u1 = *reinterpret_cast<const uint4*>(q + rowoff + c0 + 8);
        const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
        float* dst = dq + rowoff + c0;
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          float4 cur = *reinterpret_cast<float4*>(dst + e);
          cur.x += (g[e] + ddn * sZ[half][c0 + e]) * dphi_f(bf16_lo(w[e / 2]));
          cur.y += (g[e + 1] + ddn * sZ[half][c0 + e + 1]) * dphi_f(bf16_hi(w[e / 2]));
          cur.z += (g[e + 2] + ddn * sZ[half][c0 + e + 2]) * dphi_f(bf16_lo(w[e / 2 + 1]));
          cur.w += (g[e + 3] + ddn * sZ[half][c0 + e + 3]) * dphi_f(bf16_hi(w[e / 2 + 1]));
          *reinterpret_cast<float4*>(dst + e) = cur;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // ---------------- phase 2: dK, dV
  for (int e = t; e < 2 * D; e += 128) {
    const int b2 = 2 * p + e / D;
    sZ[e / D][e % D] = b2 < T ? dz[(size_t(bh) * T + b2) * D + e % D] : 0.f;
  }
  for (int c8 = 0; c8 < D / 8; ++c8) {
    uint4 uv = make_uint4(0, 0, 0, 0), uk = uv;
    if (row_ok) {
      uv = *reinterpret_cast<const uint4*>(v + rowoff + c8 * 8);
      uk = *reinterpret_cast<const uint4*>(k + rowoff + c8 * 8);
    }
    st_sw128_unit(s0, 128, t, c8 * 8, uv);
    const uint32_t w[4] = {uk.x, uk.y, uk.z, uk.w};
    uint32_t h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a = phi_f(bf16_lo(w[e])), b = phi_f(bf16_hi(w[e]));
      h[e] = pack_bf16(a, b);
      l[e] = pack_bf16(a - bf16_lo(h[e]), b - bf16_hi(h[e]));
    }
    st_sw128_unit(s1, 128, t, c8 * 8, make_uint4(h[0], h[1], h[2], h[3]));
    st_sw128_unit(s2, 128, t, c8 * 8, make_uint4(l[0], l[1], l[2], l[3]));
  }
  for (int m = 0; m < 2; ++m) {
    const int b2 = 2 * p + m;
    load_split_sw<D>(sMh, sMl, D, dh + (size_t(bh) * T + (b2 < T ? b2 : 0)) * D * D,
                     b2 < T ? D : 0, t, 128);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (t == 0) {
      constexpr uint32_t id_k = idesc_bf16(128, D, 0, 0);
      constexpr uint32_t id_v = idesc_bf16(128, D, 0, 1);
      const uint32_t hh = smem_u32(sMh), hl = smem_u32(sMl);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint64_t av = desc_kmajor(smem_u32(s0), 128, ks);
        const uint64_t kh = desc_kmajor(smem_u32(s1), 128, ks);
        const uint64_t kl = desc_kmajor(smem_u32(s2), 128, ks);
        mma_ss(tmem + m * D, av, desc_kmajor(hh, D, ks), id_k, ks > 0);
        mma_ss(tmem + m * D, av, desc_kmajor(hl, D, ks), id_k, 1);
        mma_ss(tmem + (2 + m) * D, kh, desc_mnmajor(hh, D, ks), id_v, ks > 0);
        mma_ss(tmem + (2 + m) * D, kh, desc_mnmajor(hl, D, ks), id_v, 1);
        mma_ss(tmem + (2 + m) * D, kl, desc_mnmajor(hh, D, ks), id_v, 1);
      }
      mma_commit(&bar[2 + m]);
    }
    ok = mbar_wait(&bar[2 + m], 0, err, nullptr) && ok;
    tc_fence_after();
  }
#pragma unroll 1
  for (int c0 = 0; c0 < D; c0 += 16) {
    float gk[16], gv[16];
    tmem_ld16(tmem + lane_base + half * D + c0, gk);
    tmem_ld16(tmem + lane_base + (2 + half) * D + c0, gv);
    tmem_ld_wait();
    if (row_ok && ok) {
      const uint4 u0 = *reinterpret_cast<const uint4*>(k + rowoff + c0);
      const uint4 u1 = *reinterpret_cast<const uint4*>(k + rowoff + c0 + 8);
      const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
      float* dkd = dk + rowoff + c0;
      float* dvd = dv + rowoff + c0;
#pragma unroll
      for (int e = 0; e < 16; e += 4) {
        float4 ck = *reinterpret_cast<float4*>(dkd + e);
        float4 cv = *reinterpret_cast<float4*>(dvd + e);
        ck.x += (gk[e] + sZ[half][c0 + e]) * dphi_f(bf16_lo(w[e / 2]));
        ck.y += (gk[e + 1] + sZ[half][c0 + e + 1]) * dphi_f(bf16_hi(w[e / 2]));
        ck.z += (gk[e + 2] + sZ[half][c0 + e + 2]) * dphi_f(bf16_lo(w[e / 2 + 1]));
        ck.w += (gk[e + 3] + sZ[half][c0 + e + 3]) * dphi_f(bf16_hi(w[e / 2 + 1]));
        cv.x += gv[e];
        cv.y += gv[e + 1];
        cv.z += gv[e + 2];
        cv.w += gv[e + 3];
        *reinterpret_cast<float4*>(dkd + e) = ck;
        *reinterpret_cast<float4*>(dvd + e) = cv;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free(tmem, kCols);
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
}

}  // namespace

cudaError_t launch_bwd_prep(const Problem& p, const void* q, const void* d_o, const void* w_proj,
                            const float* o_s, const float* den, const float* h_agg, float* dvec,
                            float* dnum, float* dden, float* dw, int num_sms, int* err,
                            cudaStream_t s) {
  const int tiles = ((p.T + 1) / 2) * p.BH;
  const int grid = tiles < num_sms ? tiles : num_sms;
  const size_t smem = 1024 + 5 * kTile32;
  cudaError_t e;
  if (p.d == 128) {
    if ((e = set_smem(bwd_prep_kernel<128>, smem)) != cudaSuccess) return e;
    bwd_prep_kernel<128><<<grid, 128, smem, s>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)d_o, (const __nv_bfloat16*)w_proj, o_s,
        den, h_agg, dvec, dnum, dden, dw, p.N, p.T, p.BH, err);
  } else {
    if ((e = set_smem(bwd_prep_kernel<64>, smem)) != cudaSuccess) return e;
    bwd_prep_kernel<64><<<grid, 128, smem, s>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)d_o, (const __nv_bfloat16*)w_proj, o_s,
        den, h_agg, dvec, dnum, dden, dw, p.N, p.T, p.BH, err);
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_summ(const Problem& p, const void* q, const float* dnum,
                            const float* dden, __nv_bfloat16* summ_hi, __nv_bfloat16* summ_lo,
                            float* zsum, int* err, cudaStream_t s) {
  dim3 grid((p.T + 1) / 2, p.BH);
  const size_t smem = 1024 + 4 * kTile32;
  cudaError_t e;
  if (p.d == 128) {
    if ((e = set_smem(bwd_summ_kernel<128>, smem)) != cudaSuccess) return e;
    bwd_summ_kernel<128><<<grid, 128, smem, s>>>((const __nv_bfloat16*)q, dnum, dden, summ_hi,
                                                 summ_lo, zsum, p.N, p.T, err);
  } else {
    if ((e = set_smem(bwd_summ_kernel<64>, smem)) != cudaSuccess) return e;
    bwd_summ_kernel<64><<<grid, 128, smem, s>>>((const __nv_bfloat16*)q, dnum, dden, summ_hi,
                                                summ_lo, zsum, p.N, p.T, err);
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_sparse(const Problem& p, const void* q, const void* k, const void* v,
                              const void* d_o, const float* lse, const float* dvec,
                              const int32_t* col_ptr, const int32_t* col_idx, float* dq,
                              float* dk, float* dv, int* err, cudaStream_t s) {
  CUtensorMap tq, tk, tv, tdo;
  if (!make_tmap_bhnd(&tq, q, p.BH, p.N, p.d, 64)) return cudaErrorInvalidValue;
  if (!make_tmap_bhnd(&tk, k, p.BH, p.N, p.d, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bhnd(&tv, v, p.BH, p.N, p.d, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bhnd(&tdo, d_o, p.BH, p.N, p.d, 64)) return cudaErrorInvalidValue;
  dim3 grid((p.T + 1) / 2, p.BH);
  cudaError_t e;
#define SLA_BWD(DD)                                                                           \
  {                                                                                           \
    const size_t smem = BwdSmem<DD>::total(p.T);                                              \
    e = set_smem(bwd_sparse_kernel<DD>, smem);                                                \
    if (e != cudaSuccess) return e;                                                           \
    bwd_sparse_kernel<DD><<<grid, 192, smem, s>>>(tq, tk, tv, tdo, lse, dvec, col_ptr,        \
                                                  col_idx, p.N, p.T, p.n_crit, p.scale_log2,   \
                                                  p.scale, dq, dk, dv, err);                  \
  }
  if (p.d == 128) {
    SLA_BWD(128)
  } else {
    SLA_BWD(64)
  }
#undef SLA_BWD
  return cudaGetLastError();
}

cudaError_t launch_bwd_linear(const Problem& p, const void* q, const void* k, const void* v,
                              const float* h_agg, const float* z_agg, const float* dh,
                              const float* dz, const float* dnum, const float* dden, float* dq,
                              float* dk, float* dv, int* err, cudaStream_t s) {
  dim3 grid((p.T + 1) / 2, p.BH);
  const size_t smem = 1024 + 5 * kTile32;
  cudaError_t e;
  if (p.d == 128) {
    if ((e = set_smem(bwd_linear_kernel<128>, smem)) != cudaSuccess) return e;
    bwd_linear_kernel<128><<<grid, 128, smem, s>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, h_agg, z_agg,
        dh, dz, dnum, dden, dq, dk, dv, p.N, p.T, err);
  } else {
    if ((e = set_smem(bwd_linear_kernel<64>, smem)) != cudaSuccess) return e;
    bwd_linear_kernel<64><<<grid, 128, smem, s>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, h_agg, z_agg,
        dh, dz, dnum, dden, dq, dk, dv, p.N, p.T, err);
  }
  return cudaGetLastError();
}

}  // namespace sla
