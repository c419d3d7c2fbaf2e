// Sparse branch of the SLA backward: gradients of the critical-pair softmax
// attention with the classes held fixed.
//
// SLA (arXiv 2509.24006), abstract: the kernel supports forward and backward
// passes.  Standard softmax-attention gradients restricted to critical pairs
// (u over the tokens of the critical key blocks of t's query block):
//   P_tu = exp(scale Q_t.K_u - LSE_t),  D_t = dO_t . O_s,t
//   dV_u += P_tu dO_t,  dS_tu = P_tu (dO_t.V_u - D_t)
//   dQ_t += scale dS_tu K_u,  dK_u += scale dS_tu Q_t
//
// Design (sm_100a).  One CTA owns 128 keys = key blocks 2q, 2q+1 and walks the
// sorted union of their critical query blocks (column CSR).  Per query block
// i (64 queries): S^T = K Q_i^T and dP^T = V dO_i^T (tcgen05, M = 128 keys),
// P^T and dS^T back to TMEM (bf16) for dV += P^T dO_i and dK += dS^T Q_i (A
// from TMEM), and dQ_i^T = K^T dS^T (dS^T via shared memory).  Warp roles:
//   warps 0-3 / 4-7  two compute warpgroups taking alternate query blocks, so
//                    one computes P, dS while the other drains its dQ;
//   warp 8           TMA producer: K, V once; Q_i, dO_i, LSE_i, D_i per stage;
//   warp 9           single-thread tcgen05 issuer.
// The warpgroup returns the stage to the producer as soon as the MMAs of its
// query block are done, reads dQ_i^T from TMEM into registers (freeing the
// buffer for the next S^T) and adds it into fp32 dQ with coalesced
// fire-and-forget reductions.
// TMEM (512 columns): per buffer b in {0,1}: S^T at 128b (later dQ^T), dP^T at
// 128b + 64; dV at 256, dK at 256 + d.
#include <cuda_bf16.h>

#include "sla_internal.h"
#include "sla_ptx.cuh"
#include "sla_union.cuh"

namespace sla {
namespace {

constexpr int kNSt = 3;  // Q/dO stages

template <int D>
struct SbSmem {
  static constexpr int kKV = 128 * D * 2;       // K or V tile (128 keys)
  static constexpr int kQ = 64 * D * 2;         // Q_i or dO_i tile (64 queries)
  static constexpr int kStage = 2 * kQ + 1024;  // Q, dO, LSE[64], D[64] (1024-aligned)
  static constexpr int kDS = 128 * 64 * 2;      // dS^T bf16 [128 keys][64 q], per warpgroup
  static constexpr int kTiles = 2 * kKV + kNSt * kStage + 2 * kDS;
  static size_t total(int T) { return 1024 + kTiles + size_t(2 * T) * 3 + 16; }
};

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 16-byte fire-and-forget fp32 reduction into global memory
__device__ __forceinline__ void red_add_v4(float* dst, float4 v) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(v.x), "f"(v.y),
               "f"(v.z), "f"(v.w)
               : "memory");
}

template <int D>
__global__ void __launch_bounds__(320, 1) bwd_sparse_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
    const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
    const float* __restrict__ lse, const float* __restrict__ dvec,
    const int32_t* __restrict__ col_ptr, const int32_t* __restrict__ col_idx,
    const int32_t* __restrict__ order, int N, int T,
    int n_crit, int nv, float scale_log2, float scale, float* __restrict__ dq, float* __restrict__ dk,
    float* __restrict__ dv, int* err) {
  using L = SbSmem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = align_smem_1024(smem_raw);
  uint8_t* sK = base;
  uint8_t* sV = sK + L::kKV;
  uint8_t* sSt = sV + L::kKV;
  uint8_t* sDS = sSt + kNSt * L::kStage;
  uint16_t* ulist = reinterpret_cast<uint16_t*>(sDS + 2 * L::kDS);
  uint8_t* uflag = reinterpret_cast<uint8_t*>(ulist + 2 * T);

  __shared__ uint64_t kv_full, st_full[kNSt], st_empty[kNSt], s_full[2], p_full[2], m_done[2],
      tfree[2], wsync[2], fin;
  __shared__ uint32_t tmem_base;
  __shared__ int n_union, abort_flag;
  // this CTA's tile: key-block pair qp of head bh, taken in the order given
  // (heads in sequence, each head's longest column lists first)
  const int npairs = (T + 1) / 2;
  const int item = order[blockIdx.x];
  const int qp = item % npairs, bh = item / npairs;
  const int warp = threadIdx.x / 32, lane = lane_id();
  const int kb0 = 2 * qp, kb1 = 2 * qp + 1;
  const bool has1 = kb1 < T;
  constexpr uint32_t kDV = 256, kDK = 256 + D;

  if (warp == 0) tmem_alloc(&tmem_base, 512);
  if (threadIdx.x == 32) {
    mbar_init(&kv_full, 1);
    for (int s = 0; s < kNSt; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 128);
      mbar_init(&m_done[b], 1);
      mbar_init(&tfree[b], 128);
      mbar_init(&wsync[b], 128);
    }
    mbar_init(&fin, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 8) {
    // union of the critical query blocks of key blocks 2q and 2q+1; flag bit h
    // = query block critical for key block 2q+h (bitmap scratch in the still
    // idle stage buffers)
    const int32_t* cp = col_ptr + size_t(bh) * (T + 1);
    const int32_t* ci = col_idx + size_t(bh) * T * n_crit;
    int a = cp[kb0], ae = cp[kb0 + 1];
    int b = has1 ? cp[kb1] : 0, be = has1 ? cp[kb1 + 1] : 0;
    const int cap = T * n_crit;
    if (a < 0 || ae > cap || a > ae || b < 0 || be > cap || b > be || ae - a > T || be - b > T) {
      if (lane == 0) set_error(err, SLA_ERR_DEVICE);
      a = ae = b = be = 0;
    }
    const int n = warp_union(ci + a, ae - a, ci + b, be - b, T, reinterpret_cast<uint32_t*>(sSt),
                             ulist, uflag, err);
    if (lane == 0) n_union = n;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const int nU = n_union;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && nU > 0) {
      fence_proxy_async_smem();  // the union's scratch used these buffers generically
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
        const int s = n % kNSt;
        if (n >= kNSt && !mbar_wait(&st_empty[s], ((n / kNSt) + 1) & 1, err, &abort_flag)) break;
        uint8_t* st = sSt + s * L::kStage;
        const int i = ulist[n];
        mbar_arrive_expect_tx(&st_full[s], 2 * L::kQ + 512);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(st + c * 64 * 128, &st_full[s], &tm_q, c * 64, i * 64, bh);
          tma_load_3d(st + L::kQ + c * 64 * 128, &st_full[s], &tm_do, c * 64, i * 64, bh);
        }
        bulk_load(st + 2 * L::kQ, lse + size_t(bh) * N + size_t(i) * 64, 256, &st_full[s]);
        bulk_load(st + 2 * L::kQ + 256, dvec + size_t(bh) * N + size_t(i) * 64, 256, &st_full[s]);
        ++issued;
      }
      if (abort_flag) {
        mbar_wait(&kv_full, 0, nullptr, nullptr);
        for (int n = (issued > kNSt ? issued - kNSt : 0); n < issued; ++n)
          mbar_wait(&st_full[n % kNSt], (n / kNSt) & 1, nullptr, nullptr);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nU > 0) {
      constexpr uint32_t id_s = idesc_bf16(128, 64, 0, 0);  // S^T, dP^T
      constexpr uint32_t id_g = idesc_bf16(128, D, 0, 1);   // dV, dK (A from TMEM)
      constexpr uint32_t id_q = idesc_bf16(128, 64, 1, 1);  // dQ^T = K^T dS^T
      bool ok = mbar_wait(&kv_full, 0, err, &abort_flag);
      const uint64_t kd_k = desc_kmajor_base(smem_u32(sK)), vd_k = desc_kmajor_base(smem_u32(sV));
      const uint64_t kd_mn = desc_mnmajor_base(smem_u32(sK), 128);
      // Two in-order streams, issued whichever is ready first:
      //   S(n):  S^T_n, dP^T_n into buffer n&1 (needs stage n loaded and, for
      //          n >= 2, dQ^T_{n-2} drained from that buffer; at most one
      //          S ahead of the G stream, so every barrier stays within a phase)
      //   G(n):  dV, dK += ...; dQ^T_n (needs P_n, dS_n from the warpgroup)
      int ns = 0, ng = 0;
      uint64_t t_last = globaltimer_ns();
      while (ok && ng < nU) {
        bool progressed = false;
        if (ns < nU && ns <= ng + 1 && mbar_test(&st_full[ns % kNSt], (ns / kNSt) & 1) &&
            (ns < 2 || mbar_test(&tfree[ns & 1], ((ns >> 1) - 1) & 1))) {
          tc_fence_after();
          const uint32_t q0 = smem_u32(sSt + (ns % kNSt) * L::kStage), do0 = q0 + L::kQ;
          const uint32_t st_t = tmem + (ns & 1) * 128, dp_t = st_t + 64;
          const uint64_t qd = desc_kmajor_base(q0), dod = desc_kmajor_base(do0);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            mma_ss(st_t, desc_advance(kd_k, kmajor_step_bytes(128, ks)),
                   desc_advance(qd, kmajor_step_bytes(64, ks)), id_s, ks > 0);
            mma_ss(dp_t, desc_advance(vd_k, kmajor_step_bytes(128, ks)),
                   desc_advance(dod, kmajor_step_bytes(64, ks)), id_s, ks > 0);
          }
          mma_commit(&s_full[ns & 1]);
          ++ns;
          progressed = true;
        }
        if (ng < ns && mbar_test(&p_full[ng & 1], (ng >> 1) & 1)) {
          tc_fence_after();
          const int b = ng & 1;
          const uint32_t q0 = smem_u32(sSt + (ng % kNSt) * L::kStage), do0 = q0 + L::kQ;
          const uint32_t st_t = tmem + b * 128, dp_t = st_t + 64;
          const uint64_t qd = desc_mnmajor_base(q0, 64), dod = desc_mnmajor_base(do0, 64);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            mma_ts(tmem + kDV, st_t + ks * 8, desc_advance(dod, mnmajor_step_bytes(ks)), id_g,
                   (ng | ks) != 0);
            mma_ts(tmem + kDK, dp_t + ks * 8, desc_advance(qd, mnmajor_step_bytes(ks)), id_g,
                   (ng | ks) != 0);
          }
          const uint64_t dsd = desc_mnmajor_base(smem_u32(sDS + b * L::kDS), 128);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)  // dQ^T overwrites S^T (its P was consumed by dV above)
            mma_ss(st_t, desc_advance(kd_mn, mnmajor_step_bytes(ks)),
                   desc_advance(dsd, mnmajor_step_bytes(ks)), id_q, ks > 0);
          mma_commit(&m_done[b]);
          ++ng;
          progressed = true;
        }
        if (progressed) {
          t_last = globaltimer_ns();
        } else if (abort_flag) {
          ok = false;
        } else if (globaltimer_ns() - t_last > kWaitLimitNs) {
          set_error(err, SLA_ERR_TIMEOUT);
          abort_flag = 1;
          ok = false;
        }
      }
      mma_commit(&fin);
      mbar_wait(&fin, 0, nullptr, nullptr);
    }
  } else {
    // ------------------------------------------------------------ compute warpgroups
    const int wg = warp >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;  // key row == TMEM lane
    const int half = r >> 6;
    const bool key_ok = (half == 0) || has1;  // the key block exists
    // a padded key (key padding) gets no weight; its dK, dV rows stay 0
    const bool key_valid = key_ok && qp * 128 + r < nv;
    const uint32_t lane_base = uint32_t(wq * 32) << 16;
    uint8_t* ds_tile = sDS + wg * L::kDS;
    bool ok = true;
    uint32_t wphase = 0;
    // warpgroup barrier with a bounded wait (a thread that gave up cannot
    // leave the other 127 stuck, as a named barrier would)
    auto wg_sync = [&]() -> bool {
      mbar_arrive(&wsync[wg]);
      const bool r = mbar_wait(&wsync[wg], wphase & 1, err, &abort_flag);
      ++wphase;
      return r;
    };
    for (int n = wg; n < nU; n += 2) {
      const int s = n % kNSt;
      uint8_t* st = sSt + s * L::kStage;
      const float* sl = reinterpret_cast<const float*>(st + 2 * L::kQ);
      const float* sd = sl + 64;
      const int i = ulist[n];
      if (!(ok = mbar_wait(&s_full[wg], (n >> 1) & 1, err, &abort_flag))) break;
      tc_fence_after();
      // (a padded query row of this block has LSE = +inf, so its P is 0)
      const bool member = key_valid && ((uflag[n] >> half) & 1);
      const uint32_t st_t = tmem + lane_base + wg * 128, dp_t = st_t + 64;
#pragma unroll
      for (int c0 = 0; c0 < 64; c0 += 32) {
        float sv[32], dpv[32];
        tmem_ld32(st_t + c0, sv);
        tmem_ld32(dp_t + c0, dpv);
        tmem_ld_wait();
        uint32_t pk[16], dk16[16];
        // LSE and D of these 32 queries, as 16-byte broadcast loads
        float lv[32], dv4[32];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          *reinterpret_cast<float4*>(&lv[e]) = *reinterpret_cast<const float4*>(sl + c0 + e);
          *reinterpret_cast<float4*>(&dv4[e]) = *reinterpret_cast<const float4*>(sd + c0 + e);
        }

#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float p0 = 0.f, p1 = 0.f;
          if (member) {
            p0 = exp2f(fmaf(sv[e], scale_log2, -lv[e] * 1.4426950408889634f));
            p1 = exp2f(fmaf(sv[e + 1], scale_log2, -lv[e + 1] * 1.4426950408889634f));
          }
          pk[e / 2] = pack_bf16(p0, p1);
          dk16[e / 2] = pack_bf16(p0 * (dpv[e] - dv4[e]), p1 * (dpv[e + 1] - dv4[e + 1]));
        }
        tmem_st16(st_t + c0 / 2, pk);
        tmem_st16(dp_t + c0 / 2, dk16);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          st_sw128_unit(ds_tile, 128, r, c0 + 8 * u,
                        make_uint4(dk16[4 * u], dk16[4 * u + 1], dk16[4 * u + 2], dk16[4 * u + 3]));
      }
      fence_proxy_async_smem();
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[wg]);
      if (!(ok = mbar_wait(&m_done[wg], (n >> 1) & 1, err, &abort_flag))) break;
      tc_fence_after();
      // The MMAs are done with Q_i, dO_i and this warpgroup read LSE_i, D_i:
      // hand the stage back to the producer before draining dQ.
      if (wq == 0 && lane == 0) mbar_arrive(&st_empty[s]);
      // dQ_i^T (lane = feature a, 64 query columns) added into dQ with
      // fire-and-forget fp32 reductions.
      float v[64];
      if (wq * 32 < D) {
        tmem_ld32(st_t, reinterpret_cast<float(&)[32]>(v[0]));
        tmem_ld32(st_t + 32, reinterpret_cast<float(&)[32]>(v[32]));
        tmem_ld_wait();
      }
      tc_fence_before();
      mbar_arrive(&tfree[wg]);  // the buffer is free once dQ^T is in registers
      // Transpose through this warpgroup's dS^T tile (its MMA is done and the
      // tile is not written again before this warpgroup's next query block),
      // 32 queries at a time, then add 16-byte vectors into dQ.
      float* stg = reinterpret_cast<float*>(ds_tile);
      float* gdq = dq + (size_t(bh) * N + size_t(i) * 64) * D;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (ok) {
          if (wq * 32 < D) {
#pragma unroll
            for (int e = 0; e < 32; ++e) stg[e * D + r] = v[32 * h + e] * scale;
          }
          ok = wg_sync();
        }
        if (ok) {
          const float4* s4 = reinterpret_cast<const float4*>(stg);
#pragma unroll
          for (int idx = r; idx < 32 * D / 4; idx += 128) {
            const int qq = idx / (D / 4), a4 = idx % (D / 4);
            red_add_v4(gdq + size_t(32 * h + qq) * D + a4 * 4, s4[idx]);
          }
          ok = wg_sync();
        }
      }
      if (!ok) break;
    }
    // dK (warpgroup 0) and dV (warpgroup 1) of this tile's keys: fp32 rows
    // staged as 128-byte swizzled 32-column tiles (in the K/V tiles for dV, the
    // stage buffers for dK: every product has finished with them) and written
    // by TMA stores; rows past N (a missing second key block) are clipped.
    if (nU > 0) {
      ok = mbar_wait(&fin, 0, err, &abort_flag) && ok;
      tc_fence_after();
    }
    uint8_t* stg_out = wg == 0 ? sSt : sK;
    const uint32_t acc = tmem + lane_base + (wg == 0 ? kDK : kDV);
    const float mul = wg == 0 ? scale : 1.0f;
    const bool h = nU > 0 && ok;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      float a[32];
      if (nU > 0) {
        tmem_ld32(acc + c0, a);
        tmem_ld_wait();
      }
      uint8_t* tile = stg_out + (c0 / 32) * (128 * 128);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        *reinterpret_cast<float4*>(tile + r * 128 + ((u ^ (r & 7)) * 16)) =
            h ? make_float4(a[4 * u] * mul, a[4 * u + 1] * mul, a[4 * u + 2] * mul,
                            a[4 * u + 3] * mul)
              : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    fence_proxy_async_smem();
    const bool synced = wg_sync();
    if (wq == 0 && lane == 0 && synced) {
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32)
        tma_store_3d(wg == 0 ? &tm_dk : &tm_dv, stg_out + (c0 / 32) * (128 * 128), c0, qp * 128,
                     bh);
      bulk_commit();
      bulk_wait_all();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free(tmem, 512);
}

}  // namespace

namespace {

// ------------------------------------------------------------------ tile order
// One CTA per head: a counting sort of the head's key-block pairs by the summed
// length of their two column lists (an upper bound of the pair's union, the
// tile's work), longest first.  Heads stay in sequence, so the tiles running
// at any time share one head's Q and dO in L2, and every head's tiles end
// with its shortest ones.  Pairs of equal length keep no particular order.
constexpr int kOrderThreads = 1024;

__global__ void __launch_bounds__(kOrderThreads) pair_order_kernel(
    const int32_t* __restrict__ col_ptr, int32_t* __restrict__ order, int T) {
  extern __shared__ int cnt[];  // [2T + 1] buckets, bucket b = 2T - length
  __shared__ int part[kOrderThreads];
  const int npairs = (T + 1) / 2, nb = 2 * T + 1, t = threadIdx.x, bh = blockIdx.x;
  const int32_t* cp = col_ptr + size_t(bh) * (T + 1);
  auto length = [&](int qp) {
    const int j0 = 2 * qp, j1 = 2 * qp + 1;
    int len = cp[j0 + 1] - cp[j0];
    if (j1 < T) len += cp[j1 + 1] - cp[j1];
    return min(max(len, 0), 2 * T);
  };
  for (int b = t; b < nb; b += kOrderThreads) cnt[b] = 0;
  __syncthreads();
  for (int qp = t; qp < npairs; qp += kOrderThreads) atomicAdd(&cnt[2 * T - length(qp)], 1);
  __syncthreads();
  // exclusive scan of the buckets: thread t owns a contiguous run of them
  const int per = (nb + kOrderThreads - 1) / kOrderThreads;
  const int b0 = min(nb, t * per), b1 = min(nb, b0 + per);
  int sum = 0;
  for (int b = b0; b < b1; ++b) sum += cnt[b];
  part[t] = sum;
  __syncthreads();
  for (int o = 1; o < kOrderThreads; o <<= 1) {  // inclusive scan of the run sums
    const int v = t >= o ? part[t - o] : 0;
    __syncthreads();
    part[t] += v;
    __syncthreads();
  }
  int run = part[t] - sum;
  for (int b = b0; b < b1; ++b) {
    const int c = cnt[b];
    cnt[b] = run;
    run += c;
  }
  __syncthreads();
  int32_t* out = order + size_t(bh) * npairs;
  for (int qp = t; qp < npairs; qp += kOrderThreads)
    out[atomicAdd(&cnt[2 * T - length(qp)], 1)] = bh * npairs + qp;
}

}  // namespace

cudaError_t launch_pair_order(const Problem& p, const int32_t* col_ptr, int32_t* order,
                              cudaStream_t s) {
  const size_t smem = sizeof(int) * size_t(2 * p.T + 1);
  cudaError_t e = cudaFuncSetAttribute(pair_order_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  pair_order_kernel<<<p.BH, kOrderThreads, smem, s>>>(col_ptr, order, p.T);
  return cudaGetLastError();
}

cudaError_t launch_bwd_sparse(const Problem& p, const void* q, const void* k, const void* v,
                              const void* d_o, const float* lse, const float* dvec,
                              const int32_t* col_ptr, const int32_t* col_idx,
                              const int32_t* order, float* dq, float* dk, float* dv, int* err,
                              cudaStream_t s) {
  CUtensorMap tq, tk, tv, tdo, tdk, tdv;
  if (!make_tmap_f32_bhnd(&tdk, dk, p.BH, p.N, p.d, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_f32_bhnd(&tdv, dv, p.BH, p.N, p.d, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bhnd(&tq, q, p.BH, p.N, p.d, 64)) return cudaErrorInvalidValue;
  if (!make_tmap_bhnd(&tk, k, p.BH, p.N, p.d, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bhnd(&tv, v, p.BH, p.N, p.d, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bhnd(&tdo, d_o, p.BH, p.N, p.d, 64)) return cudaErrorInvalidValue;
  dim3 grid(((p.T + 1) / 2) * p.BH);
  cudaError_t e;
  if (p.d == 128) {
    const size_t smem = SbSmem<128>::total(p.T);
    e = cudaFuncSetAttribute(bwd_sparse_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem));
    if (e != cudaSuccess) return e;
    bwd_sparse_kernel<128><<<grid, 320, smem, s>>>(tq, tk, tv, tdo, tdk, tdv, lse, dvec, col_ptr,
                                                   col_idx, order,
                                                   p.N, p.T, p.n_crit, p.nv, p.scale_log2, p.scale, dq,
                                                   dk, dv, err);
  } else {
    const size_t smem = SbSmem<64>::total(p.T);
    e = cudaFuncSetAttribute(bwd_sparse_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem));
    if (e != cudaSuccess) return e;
    bwd_sparse_kernel<64><<<grid, 320, smem, s>>>(tq, tk, tv, tdo, tdk, tdv, lse, dvec, col_ptr,
                                                  col_idx, order,
                                                  p.N, p.T, p.n_crit, p.nv, p.scale_log2, p.scale, dq,
                                                  dk, dv, err);
  }
  return cudaGetLastError();
}

}  // namespace sla
