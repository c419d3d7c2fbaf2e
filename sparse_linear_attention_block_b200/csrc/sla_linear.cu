// Linear-attention branch of SLA for marginal pairs.
//
// SLA (arXiv 2509.24006), abstract / framework step 3: marginal attention
// weights get O(N) linear attention.  Reading used here: feature map
// phi = elu + 1, per key block h_j = phi(K_j)^T V_j and z_j = sum phi(K_j),
// per query block H_i = sum of h_j over its marginal key blocks (Z_i alike),
// O_l = phi(Q) H_i / (phi(Q) . Z_i), and O = O_s + O_l W_proj.
//
// Precision.  The gradient through phi(Q) involves H_i - O_l Z_i, a
// difference of nearly equal terms, so the linear branch keeps ~16 mantissa
// bits: fp32 values x are carried as a bf16 pair x = hi + lo and products use
// hi*hi + hi*lo + lo*hi (the 0/1 marginal matrix is exact in bf16, so the
// aggregation needs only M*h_hi + M*h_lo).  Accumulation is fp32 in TMEM.
//
// Layout.  A per-block summary row is the d x d matrix followed by the
// d-vector: (h_j | z_j), (H_i | Z_i); one GEMM aggregates both.
//
// Kernels:
//   summaries_kernel   (h_j | z_j) as bf16 hi/lo planes (tcgen05)      HBM-bound
//   agg_gemm_kernel    C = M * (B_hi + B_lo), M the 0/1 matrix, C as hi/lo  tensor/HBM
// (the combination O = O_s + (phi(Q) H_i / den) W_proj is in sla_fwd_linear.cu)
#include <cuda_bf16.h>

#include <algorithm>

#include "sla_internal.h"
#include "sla_ptx.cuh"
#include "sla_tile.cuh"

namespace sla {
namespace {

// ------------------------------------------------------------------ summaries
// One CTA per (key block j, head); 128 threads.  phi(K_j)^T (M = feature a,
// K = token; as hi and lo bf16 tiles) and V_j (N = c) are written MN-major
// into swizzled shared memory; h_j = phi_hi^T V + phi_lo^T V by tcgen05
// (M=128, N=D, K=64; for D = 64 the M dimension is zero-padded to 128).
// h_j's hi and lo planes leave through the (then free) phi tiles as swizzled
// 64-column halves written by TMA stores, one contiguous 16 KB box each.
template <int D>
__global__ void __launch_bounds__(128) summaries_kernel(const __grid_constant__ CUtensorMap tm_hi,
                                                        const __grid_constant__ CUtensorMap tm_lo,
                                                        const __nv_bfloat16* __restrict__ k,
                                                        const __nv_bfloat16* __restrict__ v,
                                                        __nv_bfloat16* __restrict__ summ_hi,
                                                        __nv_bfloat16* __restrict__ summ_lo,
                                                        int N, int T, int nv, int* err) {
  constexpr int kChunks = D / 8;
  constexpr int kGroups = 128 / kChunks;
  constexpr int kRowsPer = kBlock / kGroups;
  constexpr int W = D * D + D;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = align_smem_1024(smem_raw);
  uint8_t* sPhiH = base;           // 2 chunks x 64 rows x 128 B = 16 KB (M padded to 128)
  uint8_t* sPhiL = base + 16384;   // same for the lo part
  uint8_t* sV = base + 32768;      // D/64 chunks x 8 KB
  float* zred = reinterpret_cast<float*>(sV + (D / 64) * 8192);  // [kGroups][D]
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base;
  const int j = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const int warp = t / 32;
  if (warp == 0) tmem_alloc(&tmem_base, 128);
  if (t == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  if (D == 64) {  // zero the padding chunks (features 64..127)
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int e = t; e < 8192 / 16; e += 128) {
      reinterpret_cast<uint4*>(sPhiH + 8192)[e] = z;
      reinterpret_cast<uint4*>(sPhiL + 8192)[e] = z;
    }
  }
  const int c8 = t % kChunks, g = t / kChunks;
  const size_t off = (size_t(bh) * N + size_t(j) * kBlock) * D;
  const int valid = min(kBlock, nv - j * kBlock);  // keys of this block that exist
  uint4 uk[kRowsPer], uv[kRowsPer];
#pragma unroll
  for (int i = 0; i < kRowsPer; ++i) {
    const int row = g + i * kGroups;
    uk[i] = __ldg(reinterpret_cast<const uint4*>(k + off + size_t(row) * D + c8 * 8));
    uv[i] = __ldg(reinterpret_cast<const uint4*>(v + off + size_t(row) * D + c8 * 8));
  }
  float zacc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (valid < kBlock) {  // a sequence's partial last block: padded keys contribute nothing
#pragma unroll
    for (int i = 0; i < kRowsPer; ++i)
      if (g + i * kGroups >= valid) uk[i] = uv[i] = make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < kRowsPer; ++i) {
    const int row = g + i * kGroups;
    const bool rv = valid == kBlock || row < valid;
    const uint32_t w[4] = {uk[i].x, uk[i].y, uk[i].z, uk[i].w};
    uint32_t ph[4], pl[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a = rv ? phi_f(bf16_lo(w[e])) : 0.f, b = rv ? phi_f(bf16_hi(w[e])) : 0.f;
      zacc[2 * e] += a;
      zacc[2 * e + 1] += b;
      split2(a, b, ph[e], pl[e]);
    }
    st_sw128_unit(sPhiH, 64, row, c8 * 8, make_uint4(ph[0], ph[1], ph[2], ph[3]));
    st_sw128_unit(sPhiL, 64, row, c8 * 8, make_uint4(pl[0], pl[1], pl[2], pl[3]));
    st_sw128_unit(sV, 64, row, c8 * 8, uv[i]);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) zred[g * D + c8 * 8 + e] = zacc[e];
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  if (t == 0) {
    constexpr uint32_t idesc = idesc_bf16(128, D, 1, 1);
    const uint32_t ah = smem_u32(sPhiH), al = smem_u32(sPhiL), b0 = smem_u32(sV);
#pragma unroll
    for (int ks = 0; ks < kBlock / 16; ++ks) {
      mma_ss(tmem, desc_mnmajor(ah, 64, ks), desc_mnmajor(b0, 64, ks), idesc, ks > 0);
      mma_ss(tmem, desc_mnmajor(al, 64, ks), desc_mnmajor(b0, 64, ks), idesc, 1);
    }
    mma_commit(&bar);
  }
  const size_t rowbase = (size_t(bh) * T + j) * W;
  if (t < D / 2) {  // z_j (fp32 sum) -> hi/lo at column d*d
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int gg = 0; gg < kGroups; ++gg) {
      s0 += zred[gg * D + 2 * t];
      s1 += zred[gg * D + 2 * t + 1];
    }
    uint32_t h, l;
    split2(s0, s1, h, l);
    reinterpret_cast<uint32_t*>(summ_hi + rowbase + D * D)[t] = h;
    reinterpret_cast<uint32_t*>(summ_lo + rowbase + D * D)[t] = l;
  }
  const bool ok = mbar_wait(&bar, 0, err, nullptr);
  tc_fence_after();
  // the products have read the phi tiles: they now stage h_j's output halves
#pragma unroll 1
  for (int c0 = 0; c0 < D; c0 += 64) {
    if (c0 > 0) {  // the previous half's stores have read the staging tiles
      if (t == 0) bulk_wait_read_all();
      __syncthreads();
    }
    if (ok && warp * 32 < D) {
      const int a = warp * 32 + lane_id();
      float vals[2][32];
      tmem_ld32(tmem_addr(tmem, warp * 32, c0), vals[0]);
      tmem_ld32(tmem_addr(tmem, warp * 32, c0 + 32), vals[1]);
      tmem_ld_wait();
#pragma unroll
      for (int q8 = 0; q8 < 8; ++q8) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          split2(vals[q8 >> 2][(q8 & 3) * 8 + 2 * e], vals[q8 >> 2][(q8 & 3) * 8 + 2 * e + 1],
                 hi[e], lo[e]);
        st_sw128_unit(sPhiH, D, a, q8 * 8, make_uint4(hi[0], hi[1], hi[2], hi[3]));
        st_sw128_unit(sPhiL, D, a, q8 * 8, make_uint4(lo[0], lo[1], lo[2], lo[3]));
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (t == 0 && ok) {
      tma_store_3d(&tm_hi, sPhiH, c0, 0, bh * T + j);
      tma_store_3d(&tm_lo, sPhiL, c0, 0, bh * T + j);
      bulk_commit();
    }
  }
  if (t == 0) bulk_wait_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free(tmem, 128);
}

// ------------------------------------------------------------------ aggregation GEMM
// C[bh][i][n] = sum_k A[bh][i][k] * (Bhi + Blo)[bh][k][n] with A the bf16 0/1
// marginal matrix [Tp x Tp] (K-major), B the per-block summary rows [T x W]
// as bf16 hi/lo planes (MN-major); C (fp32 in TMEM) is written back as bf16
// hi/lo planes [T x W] (C = hi + lo), the operand format of its consumers.
// Persistent and warp-specialised: a work tile is 256 rows (two 128-row
// M tiles) x 128 columns of one head; tiles of the same column slice are
// adjacent in the schedule, so the second M half finds its B slice in L2.
// Warp 0 = TMA producer over a 3-stage ring (K in steps of 64), warp 1 =
// MMA issuer into one of two TMEM accumulator buffers (256 columns each),
// warps 2-5 = epilogue of the previous tile while the next one is multiplied:
// TMEM -> hi/lo bf16 -> a swizzled 128 x 64 staging tile per plane -> TMA
// stores (whole 128-byte lines instead of one 16-byte piece per row).
constexpr int kAggBN = 128, kAggBK = 64, kAggStages = 3, kAggMT = 2;
constexpr int kAggA = 128 * kAggBK * 2;        // 16 KB per 128-row tile
constexpr int kAggB = kAggBK * kAggBN * 2;     // 16 KB per plane
constexpr int kAggStageBytes = kAggMT * kAggA + 2 * kAggB;
constexpr int kAggOut = 128 * 64 * 2;          // staging tile: 128 rows x 64 columns
constexpr int kAggEpiWarps = 4;
constexpr int kAggThreads = 64 + 32 * kAggEpiWarps;

__global__ void __launch_bounds__(kAggThreads, 1) agg_gemm_kernel(
    const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_bh,
    const __grid_constant__ CUtensorMap tm_bl, const __grid_constant__ CUtensorMap tm_oh,
    const __grid_constant__ CUtensorMap tm_ol, int T, int Tp, int NN, int BH, int* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = align_smem_1024(smem_raw);
  uint8_t* sOut = base + kAggStages * kAggStageBytes;  // hi then lo staging tile
  __shared__ uint64_t full[kAggStages], empty[kAggStages], acc_full[2], acc_empty[2], fin, esync;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int warp = threadIdx.x / 32;
  const int nk = Tp / kAggBK;
  const int nmg = (Tp / 128 + kAggMT - 1) / kAggMT;  // 256-row groups
  const int nnt = (NN + kAggBN - 1) / kAggBN;         // 128-column slices
  const int ntiles = BH * nnt * nmg;
  const int nloc = ntiles > int(blockIdx.x) ? (ntiles - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
  auto tile_of = [&](int n, int& mg, int& nt, int& bh) {
    const int t = int(blockIdx.x) + n * int(gridDim.x);
    mg = t % nmg;
    nt = (t / nmg) % nnt;
    bh = t / (nmg * nnt);
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < kAggStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kAggEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init(&fin, 1);
    mbar_init(&esync, 32 * kAggEpiWarps);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(&tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  int it = 0;  // K steps issued (producer) or consumed (MMA issuer)

  if (warp == 0 && lane_id() == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_bh);
    tma_prefetch_desc(&tm_bl);
    bool ok = true;
    for (int n = 0; n < nloc && ok; ++n) {
      int mg, nt, bh;
      tile_of(n, mg, nt, bh);
      const int nmt = min(kAggMT, Tp / 128 - mg * kAggMT);
      for (int kt = 0; kt < nk; ++kt, ++it) {
        const int s = it % kAggStages;
        if (it >= kAggStages &&
            !mbar_wait(&empty[s], ((it / kAggStages) + 1) & 1, err, &abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* sa = base + s * kAggStageBytes;
        uint8_t* sb = sa + kAggMT * kAggA;
        mbar_arrive_expect_tx(&full[s], nmt * kAggA + 2 * kAggB);
        for (int m = 0; m < nmt; ++m)
          tma_load_3d(sa + m * kAggA, &full[s], &tm_a, kt * kAggBK, (mg * kAggMT + m) * 128, bh);
        for (int c = 0; c < 2; ++c) {
          tma_load_3d(sb + c * 8192, &full[s], &tm_bh, nt * kAggBN + c * 64, kt * kAggBK, bh);
          tma_load_3d(sb + kAggB + c * 8192, &full[s], &tm_bl, nt * kAggBN + c * 64,
                      kt * kAggBK, bh);
        }
      }
    }
  } else if (warp == 1 && lane_id() == 0) {
    constexpr uint32_t idesc = idesc_bf16(128, kAggBN, 0, 1);
    bool ok = true;
    for (int n = 0; n < nloc && ok; ++n) {
      int mg, nt, bh;
      tile_of(n, mg, nt, bh);
      const int nmt = min(kAggMT, Tp / 128 - mg * kAggMT);
      const int buf = n & 1;
      if (n >= 2 && !mbar_wait(&acc_empty[buf], ((n >> 1) + 1) & 1, err, &abort_flag)) break;
      tc_fence_after();
      const uint32_t acc = tmem + uint32_t(buf) * (kAggMT * kAggBN);
      for (int kt = 0; kt < nk; ++kt, ++it) {
        const int s = it % kAggStages;
        if (!mbar_wait(&full[s], (it / kAggStages) & 1, err, &abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(base + s * kAggStageBytes);
        const uint64_t bhd = desc_mnmajor_base(sa + kAggMT * kAggA, kAggBK);
        const uint64_t bld = desc_mnmajor_base(sa + kAggMT * kAggA + kAggB, kAggBK);
        for (int m = 0; m < nmt; ++m) {
          const uint64_t ad = desc_kmajor_base(sa + m * kAggA);
#pragma unroll
          for (int ks = 0; ks < kAggBK / 16; ++ks) {
            const uint64_t av = desc_advance(ad, kmajor_step_bytes(128, ks));
            mma_ss(acc + m * kAggBN, av, desc_advance(bhd, mnmajor_step_bytes(ks)), idesc,
                   (kt | ks) != 0);
            mma_ss(acc + m * kAggBN, av, desc_advance(bld, mnmajor_step_bytes(ks)), idesc, 1);
          }
        }
        mma_commit(&empty[s]);
      }
      if (ok) mma_commit(&acc_full[buf]);
    }
    // every product issued has finished before TMEM is released
    mma_commit(&fin);
    mbar_wait(&fin, 0, nullptr, nullptr);
  } else if (warp >= 2) {
    const int q = warp % 4;  // the TMEM lane quadrant this warp may access
    const int r = q * 32 + lane_id();  // row of the 128-row M tile == TMEM lane
    const bool leader = warp == 2 && lane_id() == 0;
    uint32_t ephase = 0;
    // barrier of the epilogue warps with a bounded wait
    auto epi_sync = [&]() -> bool {
      mbar_arrive(&esync);
      const bool okw = mbar_wait(&esync, ephase & 1, err, &abort_flag);
      ++ephase;
      return okw;
    };
    bool ok = true;
    for (int n = 0; n < nloc && ok; ++n) {
      int mg, nt, bh;
      tile_of(n, mg, nt, bh);
      const int nmt = min(kAggMT, Tp / 128 - mg * kAggMT);
      const int buf = n & 1;
      if (!mbar_wait(&acc_full[buf], (n >> 1) & 1, err, &abort_flag)) break;
      tc_fence_after();
      for (int m = 0; m < nmt && ok; ++m) {
#pragma unroll 1
        for (int cbase = 0; cbase < kAggBN; cbase += 64) {
          const uint32_t col = buf * (kAggMT * kAggBN) + m * kAggBN + cbase;
          float vals[2][32];
          tmem_ld32(tmem_addr(tmem, q * 32, col), vals[0]);
          tmem_ld32(tmem_addr(tmem, q * 32, col + 32), vals[1]);
          tmem_ld_wait();
          // the staging tiles are free once the previous stores have read them
          if (leader) bulk_wait_read_all();
          if (!(ok = epi_sync())) break;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            uint32_t h[4], l[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              split2(vals[u >> 2][(u & 3) * 8 + 2 * e], vals[u >> 2][(u & 3) * 8 + 2 * e + 1], h[e],
                     l[e]);
            st_sw128_unit(sOut, 128, r, u * 8, make_uint4(h[0], h[1], h[2], h[3]));
            st_sw128_unit(sOut + kAggOut, 128, r, u * 8, make_uint4(l[0], l[1], l[2], l[3]));
          }
          fence_proxy_async_smem();
          if (!(ok = epi_sync())) break;
          if (leader) {  // rows past T and columns past NN are clipped by the store
            const int x = nt * kAggBN + cbase, y = (mg * kAggMT + m) * 128;
            tma_store_3d(&tm_oh, sOut, x, y, bh);
            tma_store_3d(&tm_ol, sOut + kAggOut, x, y, bh);
            bulk_commit();
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane_id() == 0) mbar_arrive(&acc_empty[buf]);
    }
    if (leader) bulk_wait_all();
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (abort_flag && warp == 0 && lane_id() == 0)  // copies still in flight land first
    for (int j = (it > kAggStages ? it - kAggStages : 0); j < it; ++j)
      mbar_wait(&full[j % kAggStages], (j / kAggStages) & 1, nullptr, nullptr);
  __syncwarp();
  if (warp == 0) tmem_free(tmem, 512);
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
}

}  // namespace

cudaError_t launch_summaries(const Problem& p, const void* k, const void* v,
                             __nv_bfloat16* summ_hi, __nv_bfloat16* summ_lo, int* err,
                             cudaStream_t s) {
  dim3 grid(p.T, p.BH);
  const int groups = 128 / (p.d / 8);
  const size_t smem = 1024 + 32768 + (p.d / 64) * 8192 + sizeof(float) * groups * p.d;
  CUtensorMap th, tl;
  if (!make_tmap_summary(&th, summ_hi, p.BH * p.T, p.d)) return cudaErrorInvalidValue;
  if (!make_tmap_summary(&tl, summ_lo, p.BH * p.T, p.d)) return cudaErrorInvalidValue;
  cudaError_t e;
  if (p.d == 128) {
    if ((e = set_smem(summaries_kernel<128>, smem)) != cudaSuccess) return e;
    summaries_kernel<128><<<grid, 128, smem, s>>>(th, tl, (const __nv_bfloat16*)k,
                                                  (const __nv_bfloat16*)v, summ_hi, summ_lo,
                                                  p.N, p.T, p.nv, err);
  } else {
    if ((e = set_smem(summaries_kernel<64>, smem)) != cudaSuccess) return e;
    summaries_kernel<64><<<grid, 128, smem, s>>>(th, tl, (const __nv_bfloat16*)k,
                                                 (const __nv_bfloat16*)v, summ_hi, summ_lo, p.N,
                                                 p.T, p.nv, err);
  }
  return cudaGetLastError();
}

cudaError_t launch_aggregate(const Problem& p, const __nv_bfloat16* mmat,
                             const __nv_bfloat16* summ_hi, const __nv_bfloat16* summ_lo,
                             __nv_bfloat16* out_hi, __nv_bfloat16* out_lo, int* err,
                             cudaStream_t s) {
  const int NN = summary_width(p.d);
  CUtensorMap ta, tbh, tbl;
  if (!make_tmap_3d(&ta, mmat, p.Tp, p.Tp, p.BH, 64, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_3d(&tbh, summ_hi, NN, p.T, p.BH, 64, 64)) return cudaErrorInvalidValue;
  if (!make_tmap_3d(&tbl, summ_lo, NN, p.T, p.BH, 64, 64)) return cudaErrorInvalidValue;
  CUtensorMap toh, tol;
  if (!make_tmap_3d(&toh, out_hi, NN, p.T, p.BH, 64, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_3d(&tol, out_lo, NN, p.T, p.BH, 64, 128)) return cudaErrorInvalidValue;
  const size_t smem = 1024 + kAggStages * kAggStageBytes + 2 * kAggOut;
  cudaError_t e = set_smem(agg_gemm_kernel, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cudaErrorUnknown;
  const int ntiles = p.BH * ((NN + kAggBN - 1) / kAggBN) * ((p.Tp / 128 + kAggMT - 1) / kAggMT);
  agg_gemm_kernel<<<std::min(ntiles, sms), kAggThreads, smem, s>>>(ta, tbh, tbl, toh, tol, p.T,
                                                                  p.Tp, NN, p.BH, err);
  return cudaGetLastError();
}

}  // namespace sla
