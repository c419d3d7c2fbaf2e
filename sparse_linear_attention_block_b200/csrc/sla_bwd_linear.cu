// Backward of SLA's linear branch and of W_proj, classes held fixed.
//
// SLA (arXiv 2509.24006), abstract: the fused kernel supports both forward
// and backward passes.  The pages give no backward formulas; these are the
// gradients of O = O_s + O_l W_proj as the forward defines it (classes are
// piecewise constant and carry no gradient):
//   G = dO W^T;  dnum = G / den;  dden = -(G . O_l) / den;  D_t = dO_t . O_s,t
//   dW = sum_t O_l,t^T dO_t
//   A_i = phi(Q_i)^T dnum_i,  a_i = phi(Q_i)^T dden_i        (per query block)
//   dQ  = (dnum H_i^T + dden Z_i^T) * phi'(Q)                 (linear share)
//   dh_j, dz_j = sums of A_i, a_i over the rows i with j marginal (a GEMM)
//   dK += (V dh_j^T + dz_j) * phi'(K);  dV += phi(K) dh_j
// with phi = elu + 1, so phi'(x) = min(phi(x), 1).
//
// Both kernels put features on TMEM lanes and the block's 64 tokens on TMEM
// columns (every product has M = 128; d = 64 pads with zeros), take H_i and
// dh_j as bf16 hi/lo planes by TMA, and keep the forward's split-bf16
// precision (hi*hi + hi*lo + lo*hi where a value is fp32).
//   bwd_q_kernel  persistent, one CTA (two warpgroups, one per half of the
//                 block's tokens) per SM, per query block: D_t, dden,
//                 A_i | a_i (summary rows for the transposed aggregation),
//                 dQ's linear share (written; the sparse branch adds to it),
//                 dW accumulated in TMEM across the CTA's blocks
//   bwd_k_kernel  persistent, per key block: dK, dV linear shares added to
//                 the sparse branch's values, inputs double-buffered; two
//                 warpgroups, one per half of the block's tokens, in the
//                 read-modify-write of dK, dV
#include <cuda_bf16.h>

#include "sla_internal.h"
#include "sla_ptx.cuh"
#include "sla_tile.cuh"

namespace sla {
namespace {

// Warp reduce-scatter: v[j] summed over the 32 lanes lands in lane j
// (31 shuffles for 32 values).
__device__ __forceinline__ float warp_reduce_scatter32(float (&v)[32]) {
  const int lane = int(lane_id());
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) {
    const bool up = (lane & m) != 0;
#pragma unroll
    for (int j = 0; j < m; ++j) {
      const float send = up ? v[j] : v[j + m];
      const float keep = up ? v[j + m] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, m);
    }
  }
  return v[0];
}

// Element (row, col) of a bf16 K-major swizzled tile (64-column chunks of `rows` rows).
__device__ __forceinline__ float tile_at(const uint8_t* tile, int rows, int row, int col) {
  return ld_sw_bf16(tile, rows, row, col);
}

constexpr int kQH = 32768;  // one H plane tile: 2 chunks x 128 rows x 128 B
constexpr int kQT = 16384;  // a [64 t][128] or [128][64 t] bf16 tile
// bwd_q shared memory: H hi/lo, dO, phi hi/lo, dnum^T hi/lo, A_i staging
constexpr int kBqSmem = 1024 + 2 * kQH + kQT + 2 * kQT + 2 * kQT + 2 * kQT;

template <int D>
__global__ void __launch_bounds__(256, 1) bwd_q_kernel(
    const __grid_constant__ CUtensorMap tm_hh, const __grid_constant__ CUtensorMap tm_hl,
    const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_ah,
    const __grid_constant__ CUtensorMap tm_al, const __nv_bfloat16* __restrict__ q,
    const __nv_bfloat16* __restrict__ d_o, const __nv_bfloat16* __restrict__ w_proj,
    const float* __restrict__ o_s, const float* __restrict__ den,
    const __nv_bfloat16* __restrict__ hz_hi, const __nv_bfloat16* __restrict__ hz_lo,
    float* __restrict__ dvec, float* __restrict__ dq, __nv_bfloat16* __restrict__ summ_hi,
    __nv_bfloat16* __restrict__ summ_lo, float* __restrict__ dw, float gate, float gate_slope,
    float* __restrict__ d_gate, int N, int T, int nblk, int* err) {
  constexpr int W = D * D + D;
  constexpr int kU = D / 8;
  constexpr int kRowsPerPass = 256 / kU;
  constexpr int kPass = 64 / kRowsPerPass;
  constexpr int DH = D / 2;  // A_i columns per warpgroup
  // TMEM columns: W (packed A), dW, G^T, NUM^T -> O_l^T (packed), dQ^T, A_i
  constexpr uint32_t kW = 0, kDW = 64, kG = 192, kNum = 256, kDq = 320, kA = 384;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = align_smem_1024(smem_raw);
  uint8_t* sHh = base;
  uint8_t* sHl = sHh + kQH;
  uint8_t* sDO = sHl + kQH;   // dO [64 t][c'] K-major (TMA)
  uint8_t* sPh = sDO + kQT;   // phi(Q) hi [64 t][a] K-major
  uint8_t* sPl = sPh + kQT;
  uint8_t* sNh = sPl + kQT;   // dnum^T hi [c][64 t]
  uint8_t* sNl = sNh + kQT;
  // A_i leaves as 64-column hi/lo tiles written by TMA stores: columns [0, 64)
  // staged in the dnum^T tiles (free once the block's products are done),
  // columns [64, 128) in sAx
  uint8_t* sAx = sNl + kQT;
  __shared__ float sZ[D];
  __shared__ float sInv[64], sDd[64];
  __shared__ float sRed[2][4][64];  // per-warp partial sums: G . O_l and dO . O_s
  __shared__ uint64_t bar_in, bar_c1, bar_c2;
  __shared__ uint32_t tmem_base;
  // warpgroup g owns tokens [32g, 32g+32) of each block (TMEM columns), and
  // its thread f = t % 128 owns feature f (TMEM lane)
  const int t = threadIdx.x, warp = t / 32, lane = int(lane_id());
  const int g = t >> 7, f = t & 127, wq = warp & 3;
  const bool lane_ok = wq * 32 < D;
  const uint32_t lane_base = uint32_t(wq * 32) << 16;
  const int t0 = 32 * g;  // first token of this warpgroup
  auto tok_of = [&](int blk) { return size_t(blk / T) * N + size_t(blk % T) * 64; };

  if (warp == 0) tmem_alloc(&tmem_base, 512);
  if (t == 0) {
    mbar_init(&bar_in, 1);
    mbar_init(&bar_c1, 1);
    mbar_init(&bar_c2, 1);
    fence_barrier_init();
  }
  if (D == 64) {  // zero the feature padding of the H and phi tiles
    for (int e = t; e < (kQH - 8192) / 16; e += 256) {
      reinterpret_cast<uint4*>(sHh + 8192)[e] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(sHl + 8192)[e] = make_uint4(0, 0, 0, 0);
    }
    for (int e = t; e < 8192 / 16; e += 256) {
      reinterpret_cast<uint4*>(sPh + 8192)[e] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(sPl + 8192)[e] = make_uint4(0, 0, 0, 0);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  auto request_in = [&](int blk) {  // one thread: H_i (both planes) and dO of block blk
    mbar_arrive_expect_tx(&bar_in, 2 * D * D * 2 + 64 * D * 2);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d(sHh + c * 16384, &bar_in, &tm_hh, c * 64, 0, blk);
      tma_load_3d(sHl + c * 16384, &bar_in, &tm_hl, c * 64, 0, blk);
      tma_load_3d(sDO + c * 8192, &bar_in, &tm_do, c * 64, (blk % T) * 64, blk / T);
    }
  };
  if (t == 0) {
    tma_prefetch_desc(&tm_hh);
    tma_prefetch_desc(&tm_hl);
    tma_prefetch_desc(&tm_do);
    request_in(blockIdx.x);
  }
  // W into TMEM as the A operand of G^T = W dO^T: lane c holds row c of W;
  // warpgroup g writes the columns of W's half g
  if (lane_ok) {
    const uint4* wr = reinterpret_cast<const uint4*>(w_proj + size_t(f) * D);
#pragma unroll
    for (int c0 = g * DH; c0 < (g + 1) * DH; c0 += 32) {
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint4 x = __ldg(wr + c0 / 8 + e);
        pk[4 * e] = x.x;
        pk[4 * e + 1] = x.y;
        pk[4 * e + 2] = x.z;
        pk[4 * e + 3] = x.w;
      }
      tmem_st16(tmem + lane_base + kW + c0 / 2, pk);
    }
  }
  tmem_st_wait();
  const int u = t % kU, r0 = t / kU;
  uint4 qv[kPass];
  float os[32];  // O_s[t0 + j][f] of the block about to be processed
  auto load_in = [&](int blk) {  // Q (phi input) and this thread's O_s column
    const size_t tk = tok_of(blk);
#pragma unroll
    for (int b = 0; b < kPass; ++b)
      qv[b] = __ldg(reinterpret_cast<const uint4*>(q + (tk + r0 + b * kRowsPerPass) * D) + u);
    if (lane_ok) {
#pragma unroll
      for (int j = 0; j < 32; ++j) os[j] = __ldg(o_s + (tk + t0 + j) * D + f);
    }
  };
  auto load_zd = [&](int blk) {  // Z_i (hi + lo) and 1 / den of block blk
    if (t < D)
      sZ[t] = __bfloat162float(hz_hi[size_t(blk) * W + D * D + t]) +
              __bfloat162float(hz_lo[size_t(blk) * W + D * D + t]);
    if (t >= 128 && t < 192) {
      const float dn = den[tok_of(blk) + (t - 128)];
      sInv[t - 128] = dn > 0.f ? 1.0f / dn : 0.f;
    }
  };
  load_in(blockIdx.x);
  load_zd(blockIdx.x);
  bool ok = true;
  float gate_acc = 0.f;  // sum over this CTA's tokens of G . O_l (threads < 64)
  int k = 0;
  for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x, ++k) {
    const size_t tok0 = tok_of(blk);
    const int nxt = blk + int(gridDim.x);
    if (t == 0 && nxt < nblk) {  // the next block's Q, dO, O_s rows and H, Z into L2 meanwhile
      bulk_prefetch_l2(q + tok_of(nxt) * D, 64 * D * 2);
      bulk_prefetch_l2(d_o + tok_of(nxt) * D, 64 * D * 2);
      bulk_prefetch_l2(o_s + tok_of(nxt) * D, 64 * D * 4);
      bulk_prefetch_l2(hz_hi + size_t(nxt) * W, W * 2);
      bulk_prefetch_l2(hz_lo + size_t(nxt) * W, W * 2);
    }
    // ---- phi(Q) as hi/lo K-major tiles [64 t][a]
#pragma unroll
    for (int b = 0; b < kPass; ++b) {
      const int rr = r0 + b * kRowsPerPass;
      const uint32_t w4[4] = {qv[b].x, qv[b].y, qv[b].z, qv[b].w};
      uint32_t h[4], l[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) split2(phi_f(bf16_lo(w4[e])), phi_f(bf16_hi(w4[e])), h[e], l[e]);
      st_sw128_unit(sPh, 64, rr, 8 * u, make_uint4(h[0], h[1], h[2], h[3]));
      st_sw128_unit(sPl, 64, rr, 8 * u, make_uint4(l[0], l[1], l[2], l[3]));
    }
    fence_proxy_async_smem();
    if (t == 0) bulk_wait_read_all();  // the previous A_i stores have left the dnum tiles
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ---- G^T = W dO^T (A = W from TMEM); NUM^T = (H_hi + H_lo)^T phi_hi^T
    if (t == 0) {
      ok = mbar_wait(&bar_in, k & 1, err, nullptr);
      if (ok) {
        tc_fence_after();
        constexpr uint32_t id_g = idesc_bf16(128, 64, 0, 0);
        constexpr uint32_t id_n = idesc_bf16(128, 64, 1, 0);
        const uint64_t bdo = desc_kmajor_base(smem_u32(sDO));
        const uint64_t ah = desc_mnmajor_base(smem_u32(sHh), 128);
        const uint64_t al = desc_mnmajor_base(smem_u32(sHl), 128);
        const uint64_t bp = desc_kmajor_base(smem_u32(sPh));
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_ts(tmem + kG, tmem + kW + ks * 8, desc_advance(bdo, kmajor_step_bytes(64, ks)), id_g,
                 ks > 0);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t bk = desc_advance(bp, kmajor_step_bytes(64, ks));
          mma_ss(tmem + kNum, desc_advance(ah, mnmajor_step_bytes(ks)), bk, id_n, ks > 0);
          mma_ss(tmem + kNum, desc_advance(al, mnmajor_step_bytes(ks)), bk, id_n, 1);
        }
      } else {
        mbar_wait(&bar_in, k & 1, nullptr, nullptr);  // let an in-flight copy land
      }
      mma_commit(&bar_c1);
    }
    // ---- D_t = dO_t . O_s,t while the products run (this warpgroup's 32 tokens)
    if (lane_ok) {
      const bool in_ok = mbar_wait(&bar_in, k & 1, err, nullptr);
#pragma unroll
      for (int j = 0; j < 32; ++j) os[j] *= in_ok ? tile_at(sDO, 64, t0 + j, f) : 0.f;
      sRed[1][wq][t0 + lane] = warp_reduce_scatter32(os);
    }
    ok = mbar_wait(&bar_c1, k & 1, err, nullptr) && ok;
    tc_fence_after();
    if (__syncthreads_or(!ok)) break;  // CTA-uniform exit; no copy is in flight
    // ---- O_l = NUM / den (back into TMEM, packed, as dW's A operand), dnum^T tiles,
    //      per-token partial sums of G . O_l
    float nm[32], gv[32];
    if (lane_ok) {
      tmem_ld32(tmem + lane_base + kNum + t0, nm);
      tmem_ld32(tmem + lane_base + kG + t0, gv);
      tmem_ld_wait();
    }
    tc_fence_before();
    __syncthreads();  // every NUM^T column read before the packed O_l overwrites them
    tc_fence_after();
    if (lane_ok) {
      uint32_t dnh[16], dnl[16], ph[16], pl[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float i0 = sInv[t0 + j], i1 = sInv[t0 + j + 1];
        const float o0 = nm[j] * i0, o1 = nm[j + 1] * i1;
        split2(o0, o1, ph[j / 2], pl[j / 2]);
        split2(gv[j] * (gate * i0), gv[j + 1] * (gate * i1), dnh[j / 2], dnl[j / 2]);
        gv[j] *= o0;
        gv[j + 1] *= o1;
      }
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        st_sw128_unit(sNh, 128, f, t0 + 8 * q4,
                      make_uint4(dnh[4 * q4], dnh[4 * q4 + 1], dnh[4 * q4 + 2], dnh[4 * q4 + 3]));
        st_sw128_unit(sNl, 128, f, t0 + 8 * q4,
                      make_uint4(dnl[4 * q4], dnl[4 * q4 + 1], dnl[4 * q4 + 2], dnl[4 * q4 + 3]));
      }
      tmem_st16(tmem + lane_base + kNum + 16 * g, ph);
      tmem_st16(tmem + lane_base + kNum + 32 + 16 * g, pl);
      sRed[0][wq][t0 + lane] = warp_reduce_scatter32(gv);
      tmem_st_wait();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (t < 64) {  // per token: dden, D
      float gs = 0.f, ds = 0.f;
#pragma unroll
      for (int w = 0; w < D / 32; ++w) {
        gs += sRed[0][w][t];
        ds += sRed[1][w][t];
      }
      sDd[t] = -gate * gs * sInv[t];
      dvec[tok0 + t] = ds;
      gate_acc += gs;
    }
    __syncthreads();
    tc_fence_after();
    // ---- dW += O_l^T dO;  dQ^T = H dnum^T (split products);  A_i = phi^T dnum
    if (t == 0) {
      constexpr uint32_t id_w = idesc_bf16(128, D, 0, 1);
      constexpr uint32_t id_q = idesc_bf16(128, 64, 0, 1);
      constexpr uint32_t id_a = idesc_bf16(128, D, 1, 0);
      const uint64_t bdo = desc_mnmajor_base(smem_u32(sDO), 64);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_ts(tmem + kDW, tmem + kNum + ks * 8, desc_advance(bdo, mnmajor_step_bytes(ks)), id_w,
               (k | ks) != 0);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_ts(tmem + kDW, tmem + kNum + 32 + ks * 8, desc_advance(bdo, mnmajor_step_bytes(ks)),
               id_w, 1);
      const uint64_t ahk = desc_kmajor_base(smem_u32(sHh)), alk = desc_kmajor_base(smem_u32(sHl));
      const uint64_t bnh = desc_mnmajor_base(smem_u32(sNh), 128);
      const uint64_t bnl = desc_mnmajor_base(smem_u32(sNl), 128);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t ao = kmajor_step_bytes(128, ks), bo = mnmajor_step_bytes(ks);
        mma_ss(tmem + kDq, desc_advance(ahk, ao), desc_advance(bnh, bo), id_q, ks > 0);
        mma_ss(tmem + kDq, desc_advance(alk, ao), desc_advance(bnh, bo), id_q, 1);
        mma_ss(tmem + kDq, desc_advance(ahk, ao), desc_advance(bnl, bo), id_q, 1);
      }
      const uint64_t aph = desc_mnmajor_base(smem_u32(sPh), 64);
      const uint64_t apl = desc_mnmajor_base(smem_u32(sPl), 64);
      const uint64_t bkh = desc_kmajor_base(smem_u32(sNh)), bkl = desc_kmajor_base(smem_u32(sNl));
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint32_t ao = mnmajor_step_bytes(ks), bo = kmajor_step_bytes(128, ks);
        mma_ss(tmem + kA, desc_advance(aph, ao), desc_advance(bkh, bo), id_a, ks > 0);
        mma_ss(tmem + kA, desc_advance(aph, ao), desc_advance(bkl, bo), id_a, 1);
        mma_ss(tmem + kA, desc_advance(apl, ao), desc_advance(bkh, bo), id_a, 1);
      }
      mma_commit(&bar_c2);
    }
    // ---- a_i = phi(Q_i)^T dden (fp32 from phi hi + lo): each warpgroup sums
    //      its 32 tokens, warpgroup 0 adds the halves and writes the Z part
    float ai = 0.f;
    if (f < D) {
#pragma unroll 8
      for (int j = 0; j < 32; ++j)
        ai = fmaf(tile_at(sPh, 64, t0 + j, f) + tile_at(sPl, 64, t0 + j, f), sDd[t0 + j], ai);
      if (g == 1) (&sRed[0][0][0])[f] = ai;  // sRed[0] (256 floats) is free again
    }
    __syncthreads();
    if (g == 0 && f < D) {
      ai += (&sRed[0][0][0])[f];
      const __nv_bfloat16 h = __float2bfloat16_rn(ai);
      summ_hi[size_t(blk) * W + D * D + f] = h;
      summ_lo[size_t(blk) * W + D * D + f] = __float2bfloat16_rn(ai - __bfloat162float(h));
    }
    ok = mbar_wait(&bar_c2, k & 1, err, nullptr);
    tc_fence_after();
    if (__syncthreads_or(!ok)) break;
    if (t == 0 && nxt < nblk) request_in(nxt);  // H, dO tiles are free again
    if (nxt < nblk) load_in(nxt);
    if (lane_ok) {
      // ---- dQ's linear share (lane = feature a, this warpgroup's tokens), written
      const float za = sZ[f];
      float v[32];
      tmem_ld32(tmem + lane_base + kDq + t0, v);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float dph = fminf(tile_at(sPh, 64, t0 + j, f) + tile_at(sPl, 64, t0 + j, f), 1.0f);
        dq[(tok0 + t0 + j) * D + f] = fmaf(sDd[t0 + j], za, v[j]) * dph;
      }
      // A_i, row a of the summary (hi/lo planes), this warpgroup's column half,
      // into the swizzled staging tiles
#pragma unroll 1
      for (int c0 = g * DH; c0 < (g + 1) * DH; c0 += 32) {
        tmem_ld32(tmem + lane_base + kA + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint32_t hh[4], ll[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) split2(v[e + 2 * m], v[e + 2 * m + 1], hh[m], ll[m]);
          const int c = c0 + e;
          uint8_t* sth = c < 64 ? sNh : sAx;
          uint8_t* stl = c < 64 ? sNl : sAx + kQT;
          st_sw128_unit(sth, D, f, c & 63, make_uint4(hh[0], hh[1], hh[2], hh[3]));
          st_sw128_unit(stl, D, f, c & 63, make_uint4(ll[0], ll[1], ll[2], ll[3]));
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();  // sZ, sDd, the phi tiles and TMEM dQ^T / A_i are free
    tc_fence_after();
    if (t == 0) {
#pragma unroll
      for (int ch = 0; ch < D / 64; ++ch) {
        tma_store_3d(&tm_ah, ch == 0 ? sNh : sAx, ch * 64, 0, blk);
        tma_store_3d(&tm_al, ch == 0 ? sNl : sAx + kQT, ch * 64, 0, blk);
      }
      bulk_commit();
    }
    if (nxt < nblk) load_zd(nxt);
  }
  if (t == 0) bulk_wait_all();
  // this CTA's share of dW (lane = row c of dW, this warpgroup's column half)
  if (ok && k > 0 && lane_ok) {
#pragma unroll 1
    for (int c0 = g * DH; c0 < (g + 1) * DH; c0 += 32) {
      float v[32];
      tmem_ld32(tmem + lane_base + kDW + c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) atomicAdd(dw + size_t(f) * D + c0 + e, v[e] * gate);
    }
  }
  // d gamma += g (1 - g) * sum of G . O_l (the linear branch's share of
  // sum O . dO before the gate), one reduction per warp
  if (d_gate && ok && t < 64) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) gate_acc += __shfl_xor_sync(0xffffffffu, gate_acc, m);
    if (lane == 0) atomicAdd(d_gate, gate_slope * gate_acc);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free(tmem, 512);
}

// ============================================================================ bwd_k
// Per key block j (64 keys), lane = feature:
//   dK^T = (dh_hi + dh_lo) V^T            (M = a, N = 64 keys, K = c)
//   dV^T = dh^T phi(K)^T (split products)  (M = c, N = 64 keys, K = a)
//   dk[t][a] += (dK^T[a][t] + dz_a) * phi'(k[t][a]);  dv[t][c] += dV^T[c][t]
// Stage n % 2 holds block n's dh tiles and V; TMEM buffer n % 2 its products,
// so block n's products run while block n-1's sums are added to dk, dv
// (warpgroup h: tokens 32h..32h+31, its thread f: feature f).
constexpr int kBkStage = 2 * kQH + kQT;                 // dh hi, dh lo, V
constexpr int kBkSmem = 1024 + 2 * kBkStage + 2 * kQT;  // + phi(K) hi/lo

template <int D>
__global__ void __launch_bounds__(256, 1) bwd_k_kernel(
    const __grid_constant__ CUtensorMap tm_dh, const __grid_constant__ CUtensorMap tm_dl,
    const __grid_constant__ CUtensorMap tm_v, const __nv_bfloat16* __restrict__ kin,
    const __nv_bfloat16* __restrict__ dh_hi, const __nv_bfloat16* __restrict__ dh_lo,
    float* __restrict__ dk, float* __restrict__ dv, int N, int T, int nv, int nblk, int* err) {
  constexpr int W = D * D + D;
  constexpr int kU = D / 8;
  constexpr int kRowsPerPass = 256 / kU;
  constexpr int kPass = 64 / kRowsPerPass;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = align_smem_1024(smem_raw);
  uint8_t* sPh = base + 2 * kBkStage;  // phi(K) hi [64 t][a]
  uint8_t* sPl = sPh + kQT;
  __shared__ uint64_t full[2], done[2];
  __shared__ uint32_t tmem_base;
  const int t = threadIdx.x, warp = t / 32;
  const int f = t & 127, th = t >> 7;  // feature (TMEM lane), token half
  const bool lane_ok = (warp & 3) * 32 < D;
  const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
  auto tok_of = [&](int blk) { return size_t(blk / T) * N + size_t(blk % T) * 64; };
  auto blk_of = [&](int n) { return int(blockIdx.x) + n * int(gridDim.x); };
  const int nloc = nblk > int(blockIdx.x) ? (nblk - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;

  if (warp == 0) tmem_alloc(&tmem_base, 256);
  if (t == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&full[b], 1);
      mbar_init(&done[b], 1);
    }
    fence_barrier_init();
  }
  if (D == 64) {  // zero the feature padding of the dh and phi tiles
    for (int st = 0; st < 2; ++st) {
      uint8_t* sg = base + st * kBkStage;
      for (int e = t; e < (kQH - 8192) / 16; e += 256) {
        reinterpret_cast<uint4*>(sg + 8192)[e] = make_uint4(0, 0, 0, 0);
        reinterpret_cast<uint4*>(sg + kQH + 8192)[e] = make_uint4(0, 0, 0, 0);
      }
    }
    for (int e = t; e < 8192 / 16; e += 256) {
      reinterpret_cast<uint4*>(sPh + 8192)[e] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(sPl + 8192)[e] = make_uint4(0, 0, 0, 0);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  int requested = 0, consumed = 0;  // thread 0's count of stage copies issued / waited for
  auto request = [&](int n) {       // one thread: block n's dh tiles and V into stage n % 2
    uint8_t* sg = base + (n & 1) * kBkStage;
    const int blk = blk_of(n);
    mbar_arrive_expect_tx(&full[n & 1], 2 * D * D * 2 + 64 * D * 2);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d(sg + c * 16384, &full[n & 1], &tm_dh, c * 64, 0, blk);
      tma_load_3d(sg + kQH + c * 16384, &full[n & 1], &tm_dl, c * 64, 0, blk);
      tma_load_3d(sg + 2 * kQH + c * 8192, &full[n & 1], &tm_v, c * 64, (blk % T) * 64, blk / T);
    }
    ++requested;
  };
  if (t == 0) {
    tma_prefetch_desc(&tm_dh);
    tma_prefetch_desc(&tm_dl);
    tma_prefetch_desc(&tm_v);
    for (int n = 0; n < 2 && n < nloc; ++n) request(n);
  }
  const int u = t % kU, r0 = t / kU;
  uint4 kv[kPass];
  auto load_k = [&](int n) {
    const size_t tk = tok_of(blk_of(n));
#pragma unroll
    for (int b = 0; b < kPass; ++b)
      kv[b] = __ldg(reinterpret_cast<const uint4*>(kin + (tk + r0 + b * kRowsPerPass) * D) + u);
  };
  // block n's sums (TMEM buffer n % 2) added into dk, dv; lane = feature,
  // this warpgroup's 32 tokens
  auto epilogue = [&](int n, bool write) {
    if (!lane_ok) return;
    const int blk = blk_of(n);
    const size_t tk = tok_of(blk);
    const uint32_t acc = tmem + lane_base + uint32_t(n & 1) * 128;
    const float dz = __bfloat162float(dh_hi[size_t(blk) * W + D * D + f]) +
                     __bfloat162float(dh_lo[size_t(blk) * W + D * D + f]);
    {
      const int q32 = 32 * th;
      // 96 independent loads per thread in flight
      float ck[32], cv[32], kk[32], gk[32], gv[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const size_t idx = (tk + q32 + j) * D + f;
        ck[j] = dk[idx];
        cv[j] = dv[idx];
        kk[j] = __bfloat162float(kin[idx]);
      }
      tmem_ld32(acc + q32, gk);
      tmem_ld32(acc + 64 + q32, gv);
      tmem_ld_wait();
      if (write) {
        // keys of this block that exist (key padding; all 32 except in a
        // sequence's partial last block, where padded keys keep dK = dV = 0)
        const int lim = nv - ((blk % T) * 64 + q32);
        if (lim >= 32) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const size_t idx = (tk + q32 + j) * D + f;
            dk[idx] = fmaf(gk[j] + dz, dphi_f(kk[j]), ck[j]);
            dv[idx] = cv[j] + gv[j];
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (j >= lim) break;
            const size_t idx = (tk + q32 + j) * D + f;
            dk[idx] = fmaf(gk[j] + dz, dphi_f(kk[j]), ck[j]);
            dv[idx] = cv[j] + gv[j];
          }
        }
      }
    }
  };
  bool ok = true;
  int last_commit = -1;
  if (nloc > 0) load_k(0);
  for (int n = 0; n < nloc; ++n) {
    const int b = n & 1;
    if (t == 0) {  // into L2 meanwhile: the dK, dV rows of block n (added to in the next
                   // iteration) and the K rows of block n+1 (prefetching dh two blocks
                   // ahead as well measured slower)
      const size_t tk = tok_of(blk_of(n));
      bulk_prefetch_l2(dk + tk * D, 64 * D * 4);
      bulk_prefetch_l2(dv + tk * D, 64 * D * 4);
      if (n + 1 < nloc) bulk_prefetch_l2(kin + tok_of(blk_of(n + 1)) * D, 64 * D * 2);
    }
    if (n > 0) {  // block n-1's products done: the phi tiles and stage (n-1) % 2 are free
      ok = mbar_wait(&done[(n - 1) & 1], ((n - 1) >> 1) & 1, err, nullptr);
      tc_fence_after();
      if (__syncthreads_or(!ok)) break;
      if (t == 0 && n + 1 < nloc) request(n + 1);
    }
    // phi(K) as hi/lo K-major tiles [64 t][a]
#pragma unroll
    for (int p = 0; p < kPass; ++p) {
      const int rr = r0 + p * kRowsPerPass;
      const uint32_t w4[4] = {kv[p].x, kv[p].y, kv[p].z, kv[p].w};
      uint32_t h[4], l[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) split2(phi_f(bf16_lo(w4[e])), phi_f(bf16_hi(w4[e])), h[e], l[e]);
      st_sw128_unit(sPh, 64, rr, 8 * u, make_uint4(h[0], h[1], h[2], h[3]));
      st_sw128_unit(sPl, 64, rr, 8 * u, make_uint4(l[0], l[1], l[2], l[3]));
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (t == 0) {
      ok = mbar_wait(&full[b], (n >> 1) & 1, err, nullptr);
      if (ok) {
        ++consumed;
        tc_fence_after();
        uint8_t* sg = base + b * kBkStage;
        const uint32_t kDk = tmem + uint32_t(b) * 128, kDv = kDk + 64;
        constexpr uint32_t id_k = idesc_bf16(128, 64, 0, 0);
        constexpr uint32_t id_v = idesc_bf16(128, 64, 1, 0);
        const uint64_t ahk = desc_kmajor_base(smem_u32(sg));
        const uint64_t alk = desc_kmajor_base(smem_u32(sg + kQH));
        const uint64_t bv = desc_kmajor_base(smem_u32(sg + 2 * kQH));
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t ao = kmajor_step_bytes(128, ks), bo = kmajor_step_bytes(64, ks);
          mma_ss(kDk, desc_advance(ahk, ao), desc_advance(bv, bo), id_k, ks > 0);
          mma_ss(kDk, desc_advance(alk, ao), desc_advance(bv, bo), id_k, 1);
        }
        const uint64_t ahm = desc_mnmajor_base(smem_u32(sg), 128);
        const uint64_t alm = desc_mnmajor_base(smem_u32(sg + kQH), 128);
        const uint64_t bph = desc_kmajor_base(smem_u32(sPh)), bpl = desc_kmajor_base(smem_u32(sPl));
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t ao = mnmajor_step_bytes(ks), bo = kmajor_step_bytes(64, ks);
          mma_ss(kDv, desc_advance(ahm, ao), desc_advance(bph, bo), id_v, ks > 0);
          mma_ss(kDv, desc_advance(alm, ao), desc_advance(bph, bo), id_v, 1);
          mma_ss(kDv, desc_advance(ahm, ao), desc_advance(bpl, bo), id_v, 1);
        }
      }
      mma_commit(&done[b]);  // arrives even when nothing was issued
      last_commit = n;
    }
    if (n + 1 < nloc) load_k(n + 1);
    if (n > 0) epilogue(n - 1, true);
    tc_fence_before();
    if (__syncthreads_or(!ok)) break;  // TMEM buffer (n-1) % 2 is free again
    tc_fence_after();
  }
  if (ok && nloc > 0) {
    ok = mbar_wait(&done[(nloc - 1) & 1], ((nloc - 1) >> 1) & 1, err, nullptr);
    tc_fence_after();
    ok = !__syncthreads_or(!ok);
    if (ok) epilogue(nloc - 1, true);
  }
  if (!ok && t == 0) {  // drain copies and products still in flight before exit
    for (int m = consumed; m < requested; ++m)
      mbar_wait(&full[m & 1], (m >> 1) & 1, nullptr, nullptr);
    if (last_commit >= 0) mbar_wait(&done[last_commit & 1], (last_commit >> 1) & 1, nullptr, nullptr);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free(tmem, 256);
}

// D_t = dO_t . O_s,t alone (the linear branch dropped): one warp per token.
template <int D>
__global__ void __launch_bounds__(256) dvec_kernel(const __nv_bfloat16* __restrict__ d_o,
                                                   const float* __restrict__ o_s,
                                                   float* __restrict__ dvec, size_t ntok) {
  const size_t tk = blockIdx.x * size_t(8) + threadIdx.x / 32;
  if (tk >= ntok) return;
  const int lane = int(lane_id());
  float acc = 0.f;
#pragma unroll
  for (int c = lane * 2; c < D; c += 64) {
    const float2 o2 = __ldg(reinterpret_cast<const float2*>(o_s + tk * D + c));
    const __nv_bfloat162 g2 = *reinterpret_cast<const __nv_bfloat162*>(d_o + tk * D + c);
    acc = fmaf(__low2float(g2), o2.x, fmaf(__high2float(g2), o2.y, acc));
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
  if (lane == 0) dvec[tk] = acc;
}

}  // namespace

cudaError_t launch_dvec(const Problem& p, const void* d_o, const float* o_s, float* dvec,
                        cudaStream_t s) {
  const size_t ntok = size_t(p.BH) * p.N;
  const unsigned grid = unsigned((ntok + 7) / 8);
  if (p.d == 128)
    dvec_kernel<128><<<grid, 256, 0, s>>>((const __nv_bfloat16*)d_o, o_s, dvec, ntok);
  else
    dvec_kernel<64><<<grid, 256, 0, s>>>((const __nv_bfloat16*)d_o, o_s, dvec, ntok);
  return cudaGetLastError();
}

cudaError_t launch_bwd_q(const Problem& p, const void* q, const void* d_o, const void* w_proj,
                         const float* o_s, const float* den, const __nv_bfloat16* hz_hi,
                         const __nv_bfloat16* hz_lo, float* dvec, float* dq,
                         __nv_bfloat16* summ_hi, __nv_bfloat16* summ_lo, float* dw, float gate,
                         float* d_gate, int num_sms, int* err, cudaStream_t s) {
  const float slope = gate * (1.0f - gate);
  CUtensorMap th, tl, tdo, tah, tal;
  if (!make_tmap_summary(&th, hz_hi, p.BH * p.T, p.d)) return cudaErrorInvalidValue;
  if (!make_tmap_summary(&tl, hz_lo, p.BH * p.T, p.d)) return cudaErrorInvalidValue;
  if (!make_tmap_summary(&tah, summ_hi, p.BH * p.T, p.d)) return cudaErrorInvalidValue;
  if (!make_tmap_summary(&tal, summ_lo, p.BH * p.T, p.d)) return cudaErrorInvalidValue;
  if (!make_tmap_bhnd(&tdo, d_o, p.BH, p.N, p.d, 64)) return cudaErrorInvalidValue;
  const int nblk = p.BH * p.T;
  const int grid = nblk < num_sms ? nblk : num_sms;
  cudaError_t e;
  if (p.d == 128) {
    e = cudaFuncSetAttribute(bwd_q_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kBqSmem);
    if (e != cudaSuccess) return e;
    bwd_q_kernel<128><<<grid, 256, kBqSmem, s>>>(
        th, tl, tdo, tah, tal, (const __nv_bfloat16*)q, (const __nv_bfloat16*)d_o,
        (const __nv_bfloat16*)w_proj, o_s, den, hz_hi, hz_lo, dvec, dq, summ_hi, summ_lo, dw, gate,
        slope, d_gate, p.N, p.T, nblk, err);
  } else {
    e = cudaFuncSetAttribute(bwd_q_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kBqSmem);
    if (e != cudaSuccess) return e;
    bwd_q_kernel<64><<<grid, 256, kBqSmem, s>>>(
        th, tl, tdo, tah, tal, (const __nv_bfloat16*)q, (const __nv_bfloat16*)d_o,
        (const __nv_bfloat16*)w_proj, o_s, den, hz_hi, hz_lo, dvec, dq, summ_hi, summ_lo, dw, gate,
        slope, d_gate, p.N, p.T, nblk, err);
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_k(const Problem& p, const void* k, const void* v,
                         const __nv_bfloat16* dh_hi, const __nv_bfloat16* dh_lo, float* dk,
                         float* dv, int num_sms, int* err, cudaStream_t s) {
  CUtensorMap th, tl, tv;
  if (!make_tmap_summary(&th, dh_hi, p.BH * p.T, p.d)) return cudaErrorInvalidValue;
  if (!make_tmap_summary(&tl, dh_lo, p.BH * p.T, p.d)) return cudaErrorInvalidValue;
  if (!make_tmap_bhnd(&tv, v, p.BH, p.N, p.d, 64)) return cudaErrorInvalidValue;
  const int nblk = p.BH * p.T;
  const int grid = nblk < num_sms ? nblk : num_sms;
  cudaError_t e;
  if (p.d == 128) {
    e = cudaFuncSetAttribute(bwd_k_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kBkSmem);
    if (e != cudaSuccess) return e;
    bwd_k_kernel<128><<<grid, 256, kBkSmem, s>>>(th, tl, tv, (const __nv_bfloat16*)k, dh_hi, dh_lo,
                                                 dk, dv, p.N, p.T, p.nv, nblk, err);
  } else {
    e = cudaFuncSetAttribute(bwd_k_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kBkSmem);
    if (e != cudaSuccess) return e;
    bwd_k_kernel<64><<<grid, 256, kBkSmem, s>>>(th, tl, tv, (const __nv_bfloat16*)k, dh_hi, dh_lo,
                                                dk, dv, p.N, p.T, p.nv, nblk, err);
  }
  return cudaGetLastError();
}

}  // namespace sla
