// Backward of SLA's linear branch and W_proj, classes held fixed.
//
// SLA (arXiv 2509.24006), abstract: the fused kernel supports both forward
// and backward passes.  The pages give no backward formulas; these are the
// gradients of O = O_s + O_l W_proj as defined by the forward (classes are
// piecewise constant and carry no gradient):
//   dO_l = dO W^T;  dnum = dO_l / den;  dden = -(dO_l . O_l) / den
//   A_i = phi(Q_i)^T dnum_i, a_i = phi(Q_i)^T dden_i        (per query block)
//   dh_j = sum_{i: j marginal in row i} A_i, dz_j alike     (aggregation GEMM)
//   dQ += (dnum H_i^T + dden Z_i) * phi'(Q)
//   dK += (V dh_j^T + dz_j) * phi'(K);  dV += phi(K) dh_j
//   dW = sum_t O_l,t^T dO_t;  and D_t = dO_t . O_s,t for the sparse branch.
// The sparse-branch gradients are in sla_sparse_bwd.cu.
//
// Kernels (tcgen05 for the contractions, split-bf16 precision as in the
// forward's linear branch; 256 threads: thread t owns tile row t % 128 and
// column half t / 128):
//   bwd_prep_kernel    persistent over 128-token tiles: D, dnum, dden; dW
//                      accumulated in TMEM across the CTA's tiles
//   bwd_summ_kernel    per 128-token tile: (A_i | a_i) as bf16 hi/lo planes
//   bwd_linear_kernel  per 128-token tile: the linear-branch dQ, dK, dV, added
//                      in place to the sparse-branch gradients
#include <cuda_bf16.h>

#include "sla_internal.h"
#include "sla_ptx.cuh"
#include "sla_tile.cuh"

namespace sla {
namespace {

constexpr int kTile32 = 128 * 128 * 2;  // 128 rows x 2 chunks (D = 64 padded)

// ============================================================================ bwd_prep
template <int D>
__global__ void __launch_bounds__(256, 1) bwd_prep_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ d_o,
    const __nv_bfloat16* __restrict__ w_proj, const float* __restrict__ o_s,
    const float* __restrict__ den, const __nv_bfloat16* __restrict__ hz_hi,
    const __nv_bfloat16* __restrict__ hz_lo, float* __restrict__ dvec,
    float* __restrict__ dnum, float* __restrict__ dden, float* __restrict__ dw, int N, int T,
    int BH, int* err) {
  constexpr int W = D * D + D, DH = D / 2;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = align_smem_1024(smem_raw);
  uint8_t* sA = base;                  // phi(Q)                      [t][a]
  uint8_t* sDO = sA + kTile32;         // dO                          [t][c]
  uint8_t* sW = sDO + kTile32;         // W_proj                      [a][c]
  uint8_t* sHh = sW + kTile32;         // H hi [a][c], later O_l hi   [t][a]
  uint8_t* sHl = sHh + kTile32;        // H lo [a][c], later O_l lo   [t][a]
  __shared__ float sRed[2][2][128];
  __shared__ uint64_t bar[3];
  __shared__ uint32_t tmem_base;
  const int t = threadIdx.x, warp = t / 32, r = t & 127, ch = t >> 7, half = r >> 6;
  const int P = (T + 1) / 2, ntiles = P * BH;
  const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
  constexpr uint32_t kCols = 4 * D;  // G | NUM0 | NUM1 | dW
  if (warp == 0) tmem_alloc(&tmem_base, kCols);
  if (t == 0) {
    for (int b = 0; b < 3; ++b) mbar_init(&bar[b], 1);
    fence_barrier_init();
  }
  load_rows_sw<D>(sW, D, w_proj, D, t, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  int it = 0;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int bh = tile / P, p = tile % P;
    const bool row_ok = 2 * p + half < T;
    const int valid_rows = (2 * p + 1 < T) ? 128 : 64;
    const size_t tok = size_t(p) * 128 + r;
    const size_t rowoff = (size_t(bh) * N + tok) * D;
    const size_t tile_off = (size_t(bh) * N + size_t(p) * 128) * D;
    bool ok = true;
    load_rows_sw<D>(sDO, 128, d_o + tile_off, valid_rows, t, 256);
    load_phi_sw<D>(sA, nullptr, 128, q + tile_off, valid_rows, t, 256);
    for (int m = 0; m < 2; ++m) {
      const int b2 = 2 * p + m;
      const size_t hrow = (size_t(bh) * T + (b2 < T ? b2 : 0)) * W;
      load_rows_sw<D>(sHh, D, hz_hi + hrow, b2 < T ? D : 0, t, 256);
      load_rows_sw<D>(sHl, D, hz_lo + hrow, b2 < T ? D : 0, t, 256);
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
    // per row (this thread's column half): O_l, D, dnum, dden
    const float dn = row_ok ? den[size_t(bh) * N + tok] : 0.f;
    const float inv = dn > 0.f ? 1.0f / dn : 0.f;
    float gdot = 0.f, dsum = 0.f;
#pragma unroll 1
    for (int c0 = ch * DH; c0 < (ch + 1) * DH; c0 += 16) {
      float g[16], nm[16];
      tmem_ld16(tmem + lane_base + c0, g);
      tmem_ld16(tmem + lane_base + (1 + half) * D + c0, nm);
      float4 s4[4];
      uint4 d2[2];
      if (row_ok) {
#pragma unroll
        for (int u = 0; u < 4; ++u) s4[u] = __ldg(reinterpret_cast<const float4*>(o_s + rowoff + c0) + u);
#pragma unroll
        for (int u = 0; u < 2; ++u) d2[u] = __ldg(reinterpret_cast<const uint4*>(d_o + rowoff + c0) + u);
      }
      tmem_ld_wait();
      uint32_t ol_hi[8], ol_lo[8];
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        const float o0 = nm[e] * inv, o1 = nm[e + 1] * inv;
        gdot = fmaf(g[e], o0, fmaf(g[e + 1], o1, gdot));
        split2(o0, o1, ol_hi[e / 2], ol_lo[e / 2]);
      }
      if (row_ok) {
        const float* sv = reinterpret_cast<const float*>(s4);
        const uint32_t dw4[8] = {d2[0].x, d2[0].y, d2[0].z, d2[0].w, d2[1].x, d2[1].y, d2[1].z, d2[1].w};
#pragma unroll
        for (int e = 0; e < 8; ++e)
          dsum = fmaf(bf16_lo(dw4[e]), sv[2 * e], fmaf(bf16_hi(dw4[e]), sv[2 * e + 1], dsum));
        float* dnr = dnum + rowoff + c0;
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          *reinterpret_cast<float4*>(dnr + e) =
              make_float4(g[e] * inv, g[e + 1] * inv, g[e + 2] * inv, g[e + 3] * inv);
      }
      st_sw128_unit(sHh, 128, r, c0, make_uint4(ol_hi[0], ol_hi[1], ol_hi[2], ol_hi[3]));
      st_sw128_unit(sHh, 128, r, c0 + 8, make_uint4(ol_hi[4], ol_hi[5], ol_hi[6], ol_hi[7]));
      st_sw128_unit(sHl, 128, r, c0, make_uint4(ol_lo[0], ol_lo[1], ol_lo[2], ol_lo[3]));
      st_sw128_unit(sHl, 128, r, c0 + 8, make_uint4(ol_lo[4], ol_lo[5], ol_lo[6], ol_lo[7]));
    }
    sRed[0][ch][r] = gdot;
    sRed[1][ch][r] = dsum;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (ch == 0 && row_ok) {
      dvec[size_t(bh) * N + tok] = sRed[1][0][r] + sRed[1][1][r];
      dden[size_t(bh) * N + tok] = dn > 0.f ? -(sRed[0][0][r] + sRed[0][1][r]) * inv : 0.f;
    }
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
  // flush this CTA's share of dW (lane = row a of dW, this thread's column half)
  if (it > 0 && (warp & 3) * 32 < D) {
#pragma unroll 1
    for (int c0 = ch * DH; c0 < (ch + 1) * DH; c0 += 32) {
      float v[32];
      tmem_ld32(tmem + lane_base + 3 * D + c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) atomicAdd(dw + size_t(r) * D + c0 + e, v[e]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free(tmem, kCols);
}

// ============================================================================ bwd_summ
// Per 128-token tile: A_h = phi(Q_h)^T dnum_h for the two query blocks
// (M = feature a, N = c, K = the block's 64 tokens; hi*hi + hi*lo + lo*hi)
// and a_h = sum_t phi(Q_t) dden_t, written as bf16 hi/lo summary rows.
template <int D>
__global__ void __launch_bounds__(256, 1) bwd_summ_kernel(
    const __nv_bfloat16* __restrict__ q, const float* __restrict__ dnum,
    const float* __restrict__ dden, __nv_bfloat16* __restrict__ summ_hi,
    __nv_bfloat16* __restrict__ summ_lo, int N, int T, int* err) {
  constexpr int W = D * D + D, DH = D / 2;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = align_smem_1024(smem_raw);
  uint8_t* sQh = base;                 // phi(Q) hi [t][a]
  uint8_t* sQl = sQh + kTile32;        // phi(Q) lo
  uint8_t* sNh = sQl + kTile32;        // dnum hi   [t][c]
  uint8_t* sNl = sNh + kTile32;        // dnum lo
  __shared__ float sDd[128];
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base;
  const int p = blockIdx.x, bh = blockIdx.y, t = threadIdx.x, warp = t / 32;
  const int r = t & 127, ch = t >> 7;
  const int valid_rows = (2 * p + 1 < T) ? 128 : 64;
  const size_t tile_off = (size_t(bh) * N + size_t(p) * 128) * D;
  if (warp == 0) tmem_alloc(&tmem_base, 2 * D);
  if (t == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  load_phi_sw<D>(sQh, sQl, 128, q + tile_off, valid_rows, t, 256);
  load_split_sw<D>(sNh, sNl, 128, dnum + tile_off, valid_rows, t, 256);
  if (t < 128) sDd[t] = t < valid_rows ? dden[size_t(bh) * N + size_t(p) * 128 + t] : 0.f;
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
  // a_m (m = this thread's column half), fp32 from phi hi + lo, while the MMAs run
  const int m_a = ch;
  if (r < D && 2 * p + m_a < T) {
    float acc = 0.f;
    for (int rr = 0; rr < 64; ++rr) {
      const int row = m_a * 64 + rr;
      acc = fmaf(ld_sw_bf16(sQh, 128, row, r) + ld_sw_bf16(sQl, 128, row, r), sDd[row], acc);
    }
    const size_t o = (size_t(bh) * T + 2 * p + m_a) * W + D * D + r;
    const __nv_bfloat16 h = __float2bfloat16(acc);
    summ_hi[o] = h;
    summ_lo[o] = __float2bfloat16(acc - __bfloat162float(h));
  }
  const bool ok = mbar_wait(&bar, 0, err, nullptr);
  tc_fence_after();
  if ((warp & 3) * 32 < D) {
    const int a = r;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
#pragma unroll 1
    for (int m = 0; m < 2; ++m) {
      const int b2 = 2 * p + m;
      const size_t o = (size_t(bh) * T + (b2 < T ? b2 : 0)) * W + size_t(a) * D;
#pragma unroll 1
      for (int c0 = ch * DH; c0 < (ch + 1) * DH; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + lane_base + m * D + c0, v);
        tmem_ld_wait();
        if (b2 < T && ok) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint32_t h[4], l[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) split2(v[e + 2 * i], v[e + 2 * i + 1], h[i], l[i]);
            *reinterpret_cast<uint4*>(summ_hi + o + c0 + e) = make_uint4(h[0], h[1], h[2], h[3]);
            *reinterpret_cast<uint4*>(summ_lo + o + c0 + e) = make_uint4(l[0], l[1], l[2], l[3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free(tmem, 2 * D);
}

// ============================================================================ bwd_linear
// Per 128-token tile (blocks 2p, 2p+1 as query blocks and as key blocks); the
// two halves' H (resp. dh) pass through one shared-memory slot in turn.
//   phase 1: dQ += ((dnum_hi + dnum_lo) (H_hi + H_lo)^T + dden Z) * phi'(Q)
//   phase 2: dK += (V (dh_hi + dh_lo)^T + dz) * phi'(K)
//            dV += (phi(K)_hi + phi(K)_lo) (dh_hi + dh_lo)
// (products drop the lo*lo term).
template <int D>
__global__ void __launch_bounds__(256, 1) bwd_linear_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ hz_hi,
    const __nv_bfloat16* __restrict__ hz_lo, const __nv_bfloat16* __restrict__ dh_hi,
    const __nv_bfloat16* __restrict__ dh_lo, const float* __restrict__ dnum,
    const float* __restrict__ dden, float* __restrict__ dq, float* __restrict__ dk,
    float* __restrict__ dv, int N, int T, int* err) {
  constexpr int W = D * D + D, DH = D / 2;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = align_smem_1024(smem_raw);
  uint8_t* s0 = base;             // phase 1: dnum hi | phase 2: V         [t][c]
  uint8_t* s1 = s0 + kTile32;     // phase 1: dnum lo | phase 2: phi(K) hi [t][a]
  uint8_t* s2 = s1 + kTile32;     //                    phase 2: phi(K) lo [t][a]
  uint8_t* sMh = s2 + kTile32;    // H / dh hi [a][c]
  uint8_t* sMl = sMh + kTile32;   // H / dh lo [a][c]
  __shared__ float sZ[2][D];
  __shared__ uint64_t bar[4];
  __shared__ uint32_t tmem_base;
  const int p = blockIdx.x, bh = blockIdx.y, t = threadIdx.x, warp = t / 32;
  const int r = t & 127, ch = t >> 7, half = r >> 6;
  const bool row_ok = 2 * p + half < T;
  const int valid_rows = (2 * p + 1 < T) ? 128 : 64;
  const size_t tok = size_t(p) * 128 + r;
  const size_t rowoff = (size_t(bh) * N + tok) * D;
  const size_t tile_off = (size_t(bh) * N + size_t(p) * 128) * D;
  const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
  constexpr uint32_t kCols = 4 * D;
  if (warp == 0) tmem_alloc(&tmem_base, kCols);
  if (t == 0) {
    for (int b = 0; b < 4; ++b) mbar_init(&bar[b], 1);
    fence_barrier_init();
  }
  // ---------------- phase 1: dQ
  load_split_sw<D>(s0, s1, 128, dnum + tile_off, valid_rows, t, 256);
  for (int e = t; e < 2 * D; e += 256) {
    const int b2 = 2 * p + e / D;
    const size_t zo = (size_t(bh) * T + b2) * W + D * D + e % D;
    sZ[e / D][e % D] =
        b2 < T ? __bfloat162float(hz_hi[zo]) + __bfloat162float(hz_lo[zo]) : 0.f;
  }
  bool ok = true;
  for (int m = 0; m < 2; ++m) {
    const int b2 = 2 * p + m;
    const size_t hrow = (size_t(bh) * T + (b2 < T ? b2 : 0)) * W;
    load_rows_sw<D>(sMh, D, hz_hi + hrow, b2 < T ? D : 0, t, 256);
    load_rows_sw<D>(sMl, D, hz_lo + hrow, b2 < T ? D : 0, t, 256);
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
    for (int c0 = ch * DH; c0 < (ch + 1) * DH; c0 += 16) {
      float g[16];
      tmem_ld16(tmem + lane_base + half * D + c0, g);
      float4 cur[4];
      uint4 u[2];
      if (row_ok) {
#pragma unroll
        for (int i = 0; i < 4; ++i) cur[i] = reinterpret_cast<const float4*>(dq + rowoff + c0)[i];
#pragma unroll
        for (int i = 0; i < 2; ++i) u[i] = __ldg(reinterpret_cast<const uint4*>(q + rowoff + c0) + i);
      }
      tmem_ld_wait();
      if (row_ok && ok) {
        float* cv = reinterpret_cast<float*>(cur);
        const uint32_t w[8] = {u[0].x, u[0].y, u[0].z, u[0].w, u[1].x, u[1].y, u[1].z, u[1].w};
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          cv[e] += (g[e] + ddn * sZ[half][c0 + e]) * dphi_f(bf16_lo(w[e / 2]));
          cv[e + 1] += (g[e + 1] + ddn * sZ[half][c0 + e + 1]) * dphi_f(bf16_hi(w[e / 2]));
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) reinterpret_cast<float4*>(dq + rowoff + c0)[i] = cur[i];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // ---------------- phase 2: dK, dV
  for (int e = t; e < 2 * D; e += 256) {
    const int b2 = 2 * p + e / D;
    const size_t zo = (size_t(bh) * T + b2) * W + D * D + e % D;
    sZ[e / D][e % D] =
        b2 < T ? __bfloat162float(dh_hi[zo]) + __bfloat162float(dh_lo[zo]) : 0.f;
  }
  load_rows_sw<D>(s0, 128, v + tile_off, valid_rows, t, 256);
  load_phi_sw<D>(s1, s2, 128, k + tile_off, valid_rows, t, 256);
  for (int m = 0; m < 2; ++m) {
    const int b2 = 2 * p + m;
    const size_t hrow = (size_t(bh) * T + (b2 < T ? b2 : 0)) * W;
    load_rows_sw<D>(sMh, D, dh_hi + hrow, b2 < T ? D : 0, t, 256);
    load_rows_sw<D>(sMl, D, dh_lo + hrow, b2 < T ? D : 0, t, 256);
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
  for (int c0 = ch * DH; c0 < (ch + 1) * DH; c0 += 16) {
    float gk[16], gv[16];
    tmem_ld16(tmem + lane_base + half * D + c0, gk);
    tmem_ld16(tmem + lane_base + (2 + half) * D + c0, gv);
    float4 ck[4], cv[4];
    uint4 u[2];
    if (row_ok) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        ck[i] = reinterpret_cast<const float4*>(dk + rowoff + c0)[i];
        cv[i] = reinterpret_cast<const float4*>(dv + rowoff + c0)[i];
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) u[i] = __ldg(reinterpret_cast<const uint4*>(k + rowoff + c0) + i);
    }
    tmem_ld_wait();
    if (row_ok && ok) {
      float* kk = reinterpret_cast<float*>(ck);
      float* vv = reinterpret_cast<float*>(cv);
      const uint32_t w[8] = {u[0].x, u[0].y, u[0].z, u[0].w, u[1].x, u[1].y, u[1].z, u[1].w};
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        kk[e] += (gk[e] + sZ[half][c0 + e]) * dphi_f(bf16_lo(w[e / 2]));
        kk[e + 1] += (gk[e + 1] + sZ[half][c0 + e + 1]) * dphi_f(bf16_hi(w[e / 2]));
        vv[e] += gv[e];
        vv[e + 1] += gv[e + 1];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        reinterpret_cast<float4*>(dk + rowoff + c0)[i] = ck[i];
        reinterpret_cast<float4*>(dv + rowoff + c0)[i] = cv[i];
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
                            const float* o_s, const float* den, const __nv_bfloat16* hz_hi,
                            const __nv_bfloat16* hz_lo, float* dvec,
                            float* dnum, float* dden, float* dw, int num_sms, int* err,
                            cudaStream_t s) {
  const int tiles = ((p.T + 1) / 2) * p.BH;
  const int grid = tiles < num_sms ? tiles : num_sms;
  const size_t smem = 1024 + 5 * kTile32;
  cudaError_t e;
  if (p.d == 128) {
    if ((e = set_smem(bwd_prep_kernel<128>, smem)) != cudaSuccess) return e;
    bwd_prep_kernel<128><<<grid, 256, smem, s>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)d_o, (const __nv_bfloat16*)w_proj, o_s,
        den, hz_hi, hz_lo, dvec, dnum, dden, dw, p.N, p.T, p.BH, err);
  } else {
    if ((e = set_smem(bwd_prep_kernel<64>, smem)) != cudaSuccess) return e;
    bwd_prep_kernel<64><<<grid, 256, smem, s>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)d_o, (const __nv_bfloat16*)w_proj, o_s,
        den, hz_hi, hz_lo, dvec, dnum, dden, dw, p.N, p.T, p.BH, err);
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_summ(const Problem& p, const void* q, const float* dnum,
                            const float* dden, __nv_bfloat16* summ_hi, __nv_bfloat16* summ_lo,
                            int* err, cudaStream_t s) {
  dim3 grid((p.T + 1) / 2, p.BH);
  const size_t smem = 1024 + 4 * kTile32;
  cudaError_t e;
  if (p.d == 128) {
    if ((e = set_smem(bwd_summ_kernel<128>, smem)) != cudaSuccess) return e;
    bwd_summ_kernel<128><<<grid, 256, smem, s>>>((const __nv_bfloat16*)q, dnum, dden, summ_hi,
                                                 summ_lo, p.N, p.T, err);
  } else {
    if ((e = set_smem(bwd_summ_kernel<64>, smem)) != cudaSuccess) return e;
    bwd_summ_kernel<64><<<grid, 256, smem, s>>>((const __nv_bfloat16*)q, dnum, dden, summ_hi,
                                                summ_lo, p.N, p.T, err);
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_linear(const Problem& p, const void* q, const void* k, const void* v,
                              const __nv_bfloat16* hz_hi, const __nv_bfloat16* hz_lo,
                              const __nv_bfloat16* dh_hi, const __nv_bfloat16* dh_lo,
                              const float* dnum,
                              const float* dden, float* dq, float* dk, float* dv, int* err,
                              cudaStream_t s) {
  dim3 grid((p.T + 1) / 2, p.BH);
  const size_t smem = 1024 + 5 * kTile32;
  cudaError_t e;
  if (p.d == 128) {
    if ((e = set_smem(bwd_linear_kernel<128>, smem)) != cudaSuccess) return e;
    bwd_linear_kernel<128><<<grid, 256, smem, s>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, hz_hi, hz_lo,
        dh_hi, dh_lo,
        dnum, dden, dq, dk, dv, p.N, p.T, err);
  } else {
    if ((e = set_smem(bwd_linear_kernel<64>, smem)) != cudaSuccess) return e;
    bwd_linear_kernel<64><<<grid, 256, smem, s>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, hz_hi, hz_lo,
        dh_hi, dh_lo,
        dnum, dden, dq, dk, dv, p.N, p.T, err);
  }
  return cudaGetLastError();
}

}  // namespace sla
