// Sparse branch of the SLA forward: exact softmax attention restricted to the
// critical (query block, key block) pairs.
//
// SLA (arXiv 2509.24006), abstract / framework step 2: critical weights get
// full O(N^2)-class attention; negligible ones are skipped (step 4).  For a
// query token t of block i with critical key blocks C(i):
//   O_s,t = sum_{u in C(i)} softmax_u(scale Q_t.K_u) V_u,  LSE_t = log sum exp,
// and O_s,t = 0, LSE_t = -inf when C(i) is empty.
//
// Design (sm_100a).  One CTA owns a 128-row tile = query blocks 2p and 2p+1
// (tcgen05's natural M = 128), and walks the sorted union of their critical
// key-block lists; rows whose block does not have a given key block critical
// get probability 0 for it (that work is executed but not counted as
// executed-block FLOPs).  Warp roles:
//   warps 0-3  softmax: one query row per thread, S from TMEM, P back to
//              TMEM (bf16, aliasing S), lazy rescaling of O in TMEM
//   warp 4     TMA producer: Q tile once; K_j tiles into a 2-slot ring whose
//              slot is freed as soon as S_n = Q K_n^T has been computed, V_j
//              into a 3-slot ring freed by P_n V_n (separate rings keep the K
//              copies off the softmax -> P V -> S chain; the third V slot
//              gives a V copy two iterations to land)
//   warp 5     MMA issuer (one thread): S_n into one of two TMEM buffers,
//              O += P_n V_n with P read from TMEM
// TMEM: S buffers at columns [0,64) and [64,128), O at [128, 128+D).
// Shared memory: Q, the K and V slots, the union list and the barriers, all in
// the dynamic region (no static shared memory, so that two CTAs fit on an SM
// with the third V slot; the region starts 1024-byte aligned, which is
// checked).
#include <cuda_bf16.h>

#include "sla_internal.h"
#include "sla_ptx.cuh"
#include "sla_union.cuh"

namespace sla {
namespace {

constexpr int kStages = 2;   // K slots
constexpr int kVStages = 3;  // V slots
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct FwdBars {
  uint64_t q_full, k_full[kStages], k_empty[kStages], v_full[kVStages], v_empty[kVStages],
      s_full[2], p_full[2], o_done, mma_done, osync;
  uint32_t tmem_base;
  int n_union, abort_flag;
};

template <int D>
struct FwdSmem {
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kKVBytes = 64 * D * 2;  // one K or V tile
  static constexpr int kTiles = kQBytes + (kStages + kVStages) * kKVBytes;  // K slots, then V slots
  // then the union list (2*n_crit uint16 block indices, then 2*n_crit flag
  // bytes) and the barriers
  __host__ __device__ static size_t bars(int n_crit) {
    return kTiles + (size_t(2 * n_crit) * 3 + 15) / 16 * 16;
  }
  static size_t total(int n_crit) { return bars(n_crit) + sizeof(FwdBars); }
};

template <int D>
__global__ void __launch_bounds__(192, 2) fwd_sparse_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_os,
    const int32_t* __restrict__ crit_idx, int N, int T, int n_crit, int nv, float scale_log2,
    float* __restrict__ lse, int* err) {
  using L = FwdSmem<D>;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  // the swizzled tiles need 1024-byte alignment: the kernel has no static
  // shared memory, so the dynamic region starts at the CTA's window; if it
  // does not, nothing is done and the launch reports an error
  if ((smem_u32(smem_raw) & 1023u) != 0u) {
    if (threadIdx.x == 0) set_error(err, SLA_ERR_DEVICE);
    return;
  }
  uint8_t* base = smem_raw;
  uint8_t* sQ = base;
  uint8_t* sKV = base + L::kQBytes;
  uint16_t* ulist = reinterpret_cast<uint16_t*>(base + L::kTiles);
  uint8_t* uflag = base + L::kTiles + 2 * (2 * n_crit);
  FwdBars& bb = *reinterpret_cast<FwdBars*>(base + L::bars(n_crit));
  uint64_t &q_full = bb.q_full, &o_done = bb.o_done, &mma_done = bb.mma_done, &osync = bb.osync;
  uint64_t *k_full = bb.k_full, *k_empty = bb.k_empty, *v_full = bb.v_full,
           *v_empty = bb.v_empty, *s_full = bb.s_full, *p_full = bb.p_full;
  uint32_t& tmem_base = bb.tmem_base;
  int &n_union = bb.n_union, &abort_flag = bb.abort_flag;

  const int p = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x / 32, lane = lane_id();
  const int blk0 = 2 * p, blk1 = 2 * p + 1;
  const bool has1 = blk1 < T;

  if (warp == 0) tmem_alloc(&tmem_base, 256);
  if (threadIdx.x == 32) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 128);
    }
    mbar_init(&o_done, 1);
    mbar_init(&mma_done, 1);
    mbar_init(&osync, 128);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 4) {
    // sorted union of the two rows' critical lists (bitmap scratch in the
    // still idle K/V slots); flag bit h = member of row 2p+h
    const int32_t* l0 = crit_idx + (size_t(bh) * T + blk0) * n_crit;  // row 2p+1 follows
    const int n = warp_union(l0, n_crit, l0 + n_crit, has1 ? n_crit : 0, T,
                             reinterpret_cast<uint32_t*>(sKV), ulist, uflag, err);
    if (lane == 0) n_union = n;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const int nU = n_union;
  const uint32_t tm_o = tmem + 128;

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    // (sla_debug_inject's SLA_INJECT_WITHHOLD_LOADS: issue none of the copies,
    // so that every wait on them runs out with nothing in flight)
    const bool withhold = (err[kInjectWordOffset / 4] & SLA_INJECT_WITHHOLD_LOADS) != 0;
    if (lane == 0 && nU > 0 && !withhold) {
      fence_proxy_async_smem();  // the union's scratch used these buffers generically
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(&q_full, L::kQBytes);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) tma_load_3d(sQ + c * 128 * 128, &q_full, &tm_q, c * 64, p * 128, bh);
      // K_n needs S_{n-2} done, V_n needs P_{n-3} V_{n-3} done; the pipe
      // completes S_0, S_1, PV_0, S_2, PV_1, S_3, ... so requests go out in
      // that order: K_0 V_0 K_1 V_1 V_2 K_2 K_3, then V_m K_{m+1} for m >= 3.
      int nk = 0, nv = 0;  // K and V copies issued
      auto load_k = [&](int n) -> bool {
        const int s = n % kStages;
        if (n >= kStages && !mbar_wait(&k_empty[s], ((n / kStages) + 1) & 1, err, &abort_flag))
          return false;
        uint8_t* sk = sKV + s * L::kKVBytes;
        mbar_arrive_expect_tx(&k_full[s], L::kKVBytes);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sk + c * 64 * 128, &k_full[s], &tm_k, c * 64, int(ulist[n]) * kBlock, bh);
        ++nk;
        return true;
      };
      auto load_v = [&](int n) -> bool {
        const int s = n % kVStages;
        if (n >= kVStages && !mbar_wait(&v_empty[s], ((n / kVStages) + 1) & 1, err, &abort_flag))
          return false;
        uint8_t* sv = sKV + (kStages + s) * L::kKVBytes;
        mbar_arrive_expect_tx(&v_full[s], L::kKVBytes);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sv + c * 64 * 128, &v_full[s], &tm_v, c * 64, int(ulist[n]) * kBlock, bh);
        ++nv;
        return true;
      };
      bool go = true;
      for (int n = 0; go && n < 2 && n < nU; ++n) go = load_k(n) && load_v(n);
      if (go && 2 < nU) go = load_v(2);
      for (int n = 2; go && n < 4 && n < nU; ++n) go = load_k(n);
      for (int m = 3; go && m < nU; ++m) {
        go = load_v(m);
        if (go && m + 1 >= 4 && m + 1 < nU) go = load_k(m + 1);
      }
      if (abort_flag) {
        // let copies already in flight land before the CTA exits
        mbar_wait(&q_full, 0, nullptr, nullptr);
        for (int n = (nk > kStages ? nk - kStages : 0); n < nk; ++n)
          mbar_wait(&k_full[n % kStages], (n / kStages) & 1, nullptr, nullptr);
        for (int n = (nv > kVStages ? nv - kVStages : 0); n < nv; ++n)
          mbar_wait(&v_full[n % kVStages], (n / kVStages) & 1, nullptr, nullptr);
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && nU > 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 64, 0, 0);
      constexpr uint32_t idesc_o = idesc_bf16(128, D, 0, 1);
      const uint64_t qd = desc_kmajor_base(smem_u32(sQ));
      bool ok = mbar_wait(&q_full, 0, err, &abort_flag);
      auto issue_s = [&](int n) -> bool {
        const int s = n % kStages;
        if (!mbar_wait(&k_full[s], (n / kStages) & 1, err, &abort_flag)) return false;
        tc_fence_after();
        const uint64_t kd = desc_kmajor_base(smem_u32(sKV + s * L::kKVBytes));
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_ss(tmem + (n & 1) * 64, desc_advance(qd, kmajor_step_bytes(128, ks)),
                 desc_advance(kd, kmajor_step_bytes(64, ks)), idesc_s, ks > 0);
        mma_commit(&s_full[n & 1]);
        mma_commit(&k_empty[s]);
        return true;
      };
      auto issue_pv = [&](int n) -> bool {
        const int s = n % kVStages;
        if (!mbar_wait(&p_full[n & 1], (n >> 1) & 1, err, &abort_flag) ||
            !mbar_wait(&v_full[s], (n / kVStages) & 1, err, &abort_flag))
          return false;
        tc_fence_after();
        const uint64_t vd = desc_mnmajor_base(smem_u32(sKV + (kStages + s) * L::kKVBytes), 64);
        const uint32_t pt = tmem + (n & 1) * 64;  // P aliases the first 32 columns of S
#pragma unroll
        for (int ks = 0; ks < kBlock / 16; ++ks)
          mma_ts(tm_o, pt + ks * 8, desc_advance(vd, mnmajor_step_bytes(ks)), idesc_o, (n | ks) != 0);
        mma_commit(&o_done);
        mma_commit(&v_empty[s]);
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && nU > 1) ok = issue_s(1);
      for (int n = 0; ok && n < nU; ++n) {
        ok = issue_pv(n);
        if (ok && n + 2 < nU) ok = issue_s(n + 2);
      }
      mma_commit(&mma_done);
      mbar_wait(&mma_done, 0, nullptr, nullptr);
    }
  } else {
    // ---------------------------------------------------------------- softmax warps 0-3
    const int r = threadIdx.x;  // tile row == TMEM lane
    const int half = r >> 6;
    const int blk = blk0 + half;
    const bool row_ok = blk < T;
    // a padded query row (key padding) attends to nothing: O_s = 0, LSE = +inf
    const bool q_valid = size_t(p) * 128 + r < size_t(nv);
    const int last_keys = nv - (T - 1) * kBlock;  // valid keys of block T-1
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int n = 0; n < nU; ++n) {
      const uint32_t sb = tmem + lane_base + (n & 1) * 64;
      ok = mbar_wait(&s_full[n & 1], (n >> 1) & 1, err, &abort_flag);
      if (!ok) break;
      tc_fence_after();
      float sv[64];
      tmem_ld32(sb, reinterpret_cast<float(&)[32]>(sv[0]));
      tmem_ld32(sb + 32, reinterpret_cast<float(&)[32]>(sv[32]));
      tmem_ld_wait();
      const bool member = row_ok && q_valid && ((uflag[n] >> half) & 1);
      float alpha = 1.f;
      if (member) {
        if (int(ulist[n]) == T - 1 && last_keys < kBlock) {  // padded keys: no weight
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (e >= last_keys) sv[e] = -INFINITY;
        }
        float mx = -INFINITY;  // the scale is positive: max of the raw scores, then scaled
#pragma unroll
        for (int e = 0; e < 64; ++e) mx = fmaxf(mx, sv[e]);
        mx *= scale_log2;
        if (mx > m_run + kRescaleThreshold || m_run == -INFINITY) {
          alpha = exp2f(m_run - mx);  // 0 when m_run == -inf
          l_run *= alpha;
          m_run = mx;
        }
        float sum = 0.f;
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          sv[e] = exp2f(fmaf(sv[e], scale_log2, -m_run));
          sum += sv[e];
        }
        l_run += sum;
      } else {
#pragma unroll
        for (int e = 0; e < 64; ++e) sv[e] = 0.f;
      }
      {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(sv[2 * e], sv[2 * e + 1]);
        tmem_st16(sb, pk);
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(sv[32 + 2 * e], sv[32 + 2 * e + 1]);
        tmem_st16(sb + 16, pk);
      }
      // O must not be rescaled before the previous P V has landed
      if (n > 0) {
        ok = mbar_wait(&o_done, (n - 1) & 1, err, &abort_flag);
        if (!ok) break;
        tc_fence_after();
      }
      if (__any_sync(0xFFFFFFFFu, alpha != 1.f) && n > 0) {
        const uint32_t ob = tm_o + lane_base;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 16) {
          float ov[16];
          tmem_ld16(ob + c0, ov);
          tmem_ld_wait();
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) w[e] = __float_as_uint(ov[e] * alpha);
          tmem_st16(ob + c0, w);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[n & 1]);
    }
    // ---------------------------------------------------------------- epilogue
    if (ok && nU > 0) {
      ok = mbar_wait(&o_done, (nU - 1) & 1, err, &abort_flag);
      tc_fence_after();
    }
    // O_s rows staged as 128-byte swizzled 32-column fp32 tiles in the Q and
    // K/V buffers (every product has finished with them) and written by TMA
    // stores; rows past N (a missing second block) are clipped by the store
    const size_t tok = size_t(p) * 128 + r;
    const bool have = ok && nU > 0 && l_run > 0.f;
    const float inv = have ? 1.0f / l_run : 0.f;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      float ov[32];
      if (nU > 0) {
        tmem_ld32(tm_o + lane_base + c0, ov);
        tmem_ld_wait();
      }
      uint8_t* tile = base + (c0 / 32) * (128 * 128);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        *reinterpret_cast<float4*>(tile + r * 128 + ((u ^ (r & 7)) * 16)) =
            have ? make_float4(ov[4 * u] * inv, ov[4 * u + 1] * inv, ov[4 * u + 2] * inv,
                               ov[4 * u + 3] * inv)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    fence_proxy_async_smem();
    mbar_arrive(&osync);
    if (mbar_wait(&osync, 0, err, &abort_flag) && r == 0) {
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32)
        tma_store_3d(&tm_os, base + (c0 / 32) * (128 * 128), c0, p * 128, bh);
      bulk_commit();
      bulk_wait_all();
    }
    if (row_ok)
      lse[size_t(bh) * N + tok] =
          have ? (m_run + __log2f(l_run)) * 0.69314718055994530942f
               : (q_valid ? -INFINITY : INFINITY);  // +inf: a padded row, P = 0 everywhere
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free(tmem, 256);
}

}  // namespace

cudaError_t launch_fwd_sparse(const Problem& p, const void* q, const void* k, const void* v,
                              const int32_t* crit_idx, float* o_s, float* lse, int* err,
                              cudaStream_t s) {
  CUtensorMap tq, tk, tv, tos;
  if (!make_tmap_f32_bhnd(&tos, o_s, p.BH, p.N, p.d, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bhnd(&tq, q, p.BH, p.N, p.d, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bhnd(&tk, k, p.BH, p.N, p.d, 64)) return cudaErrorInvalidValue;
  if (!make_tmap_bhnd(&tv, v, p.BH, p.N, p.d, 64)) return cudaErrorInvalidValue;
  dim3 grid((p.T + 1) / 2, p.BH);
  cudaError_t e;
  if (p.d == 128) {
    const int smem = int(FwdSmem<128>::total(p.n_crit));
    e = cudaFuncSetAttribute(fwd_sparse_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem);
    if (e != cudaSuccess) return e;
    fwd_sparse_kernel<128><<<grid, 192, smem, s>>>(tq, tk, tv, tos, crit_idx, p.N, p.T, p.n_crit,
                                                   p.nv, p.scale_log2, lse, err);
  } else {
    const int smem = int(FwdSmem<64>::total(p.n_crit));
    e = cudaFuncSetAttribute(fwd_sparse_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem);
    if (e != cudaSuccess) return e;
    fwd_sparse_kernel<64><<<grid, 192, smem, s>>>(tq, tk, tv, tos, crit_idx, p.N, p.T, p.n_crit,
                                                  p.nv, p.scale_log2, lse, err);
  }
  return cudaGetLastError();
}

}  // namespace sla
