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
// Design (sm_100a).  A tile is 128 keys = key blocks 2q, 2q+1; its work is the
// sorted union of their critical query blocks (column CSR), one query block
// (64 queries) per iteration.  The kernel is persistent: one CTA per SM walks
// tiles in the order given (heads in sequence, longest unions first), with one
// iteration counter g that runs on across tiles, so that the stage ring, the
// TMEM chunks and the two compute warpgroups keep their rhythm at a tile
// boundary.  Per iteration g (query block i):
//   S^T = K Q_i^T, dP^T = V dO_i^T       (tcgen05, M = 128 keys, N = 64)
//   P^T = exp2(log2(e) (scale S^T - LSE_i)) -> TMEM over S^T,
//   dS^T = P^T (dP^T - D_i) -> TMEM over S^T and shared memory
//                                        (both compute warpgroups, 32 query
//                                        columns each; LSE_i, D_i come with
//                                        the stage)
//   dV += P^T dO_i, dK += dS^T Q_i       (A = P^T, dS^T from TMEM)
//   dQ_i^T = K^T dS^T                    (M = d, N = 64)
//   dQ_i += scale dQ_i^T^T               (fp32 bulk reductions, TMA engine)
// TMEM: dV at column 256, dK at 256 + d; four 64-column chunks at 0..255
// rotate through S^T(g) -> dQ^T(g) in chunk g % 4 and dP^T(g) in chunk
// (g + 1) % 4, so a chunk's life is S^T(g), dQ^T(g), dP^T(g + 3), S^T(g + 4).
// P^T(g) (bf16, two per column) of queries 32w..32w+31 lies over the first 16
// of those queries' own S^T columns, 32w..32w+15 of the chunk, and dS^T(g)
// over the next 16, 32w+16..32w+31.
// The S groups (S^T, dP^T) and the G groups (dV, dK, dQ^T) come from two
// issuing threads and interleave in the tensor pipe: S(g + 1) needs only the
// warpgroups' load of dP^T(g) and the drain of dQ^T(g - 2); G(g) needs P^T(g),
// dS^T(g), computed while S(g + 1) runs.  Both warpgroups work on every
// iteration, each on half of its query columns, so that the chain from S(g)
// to G(g) is as short as the compute allows.
// Warp roles (512 threads; registers rebalanced with setmaxnreg):
//   warps 0-3 / 4-7  compute warpgroups (query columns 0-31 / 32-63 of every
//                    g): P^T, dS^T, and the tile's dK (warpgroup 0) / dV (1)
//                    epilogue  [168 registers]
//   warps 8-11       dQ warpgroup: dQ^T out of TMEM, transposed into a shared
//                    fp32 tile of 32 query rows, added into dQ by one bulk
//                    reduction of the TMA engine per half (the rows of a query
//                    block are contiguous in dQ), so that neither the compute
//                    warps nor the mbarrier traffic queue behind 8192 scalar
//                    reductions per iteration  [96]
//   warp 12          TMA producer: K, V per tile; Q_i, dO_i, LSE_i and D_i of
//                    query block i per iteration into a 3-stage ring  [80]
//   warps 13 / 14    single-thread tcgen05 issuers of the S and the G groups
//                    (warp 15 idle)  [80]
#include <cuda_bf16.h>

#include "sla_internal.h"
#include "sla_ptx.cuh"
#include "sla_union.cuh"

namespace sla {
namespace {

constexpr int kNSt = 3;  // Q/dO stages
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct SbSmem {
  static constexpr int kKV = 128 * D * 2;       // K or V tile (128 keys)
  static constexpr int kQ = 64 * D * 2;         // Q_i or dO_i tile (64 queries)
  static constexpr int kLD = 1024;              // LSE_i, D_i (64 fp32 each; 1024-byte pitch)
  static constexpr int kStage = 2 * kQ + kLD;   // Q, dO, LSE_i, D_i
  static constexpr int kStageBytes = 2 * kQ + 512;  // what a stage's copies bring
  static constexpr int kDS = 128 * 64 * 2;      // dS^T bf16 [128 keys][64 queries]
  static constexpr int kStg = 32 * D * 4;       // fp32 dQ rows of 32 queries
  static constexpr int kTotal = 1024 + 2 * kKV + kNSt * kStage + 2 * kDS + kStg;
};

// The waits of this kernel poll with test_wait instead of a suspending
// try_wait (measured faster here: the waiting warps resume without a
// wake-up delay); the same time limit and abort flag as mbar_wait.
__device__ __forceinline__ bool wait_spin(uint64_t* bar, uint32_t phase, int* err,
                                          volatile int* abort_flag) {
  if (mbar_test(bar, phase)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_test(bar, phase)) return true;
    if (abort_flag && *abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      set_error(err, SLA_ERR_TIMEOUT);
      if (abort_flag) *abort_flag = 1;
      return false;
    }
  }
}

// At most one committed bulk group of this thread is still reading shared memory.
__device__ __forceinline__ void bulk_wait_read_le1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// dst[0 .. bytes/4) += src[...] (fp32), by the TMA engine, in the bulk async
// group of the issuing thread; both addresses 16-byte aligned, bytes a multiple
// of 16
__device__ __forceinline__ void bulk_reduce_add_f32(float* dst, const float* src, uint32_t bytes) {
  asm volatile(
      "cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst),
      "r"(smem_u32(src)), "r"(bytes)
      : "memory");
}

// A tile: key-block pair qp of head bh, its union length, where its union list
// starts (the pair's slot in the column CSR); valid = false ends the walk.
struct Tile {
  int bh, qp, n, valid;
  long long slot;
};

__device__ __forceinline__ Tile tile_at(const int32_t* order, const int32_t* ulen,
                                        const int32_t* col_ptr, int idx, int n_tiles, int T,
                                        int n_crit) {
  Tile t{0, 0, 0, 0, 0};
  if (idx >= n_tiles) return t;
  const int npairs = (T + 1) / 2;
  const int item = order[idx];
  t.qp = item % npairs;
  t.bh = item / npairs;
  t.n = ulen[item];
  t.slot = (long long)t.bh * T * n_crit + col_ptr[size_t(t.bh) * (T + 1) + 2 * t.qp];
  t.valid = 1;
  return t;
}

template <int D>
__global__ void __launch_bounds__(512, 1) bwd_sparse_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
    const float* __restrict__ lse, const float* __restrict__ dvec, const int32_t* __restrict__ col_ptr,
    const uint16_t* __restrict__ ulist,
    const uint8_t* __restrict__ uflag, const int32_t* __restrict__ ulen,
    const int32_t* __restrict__ order, int* __restrict__ sched, int n_tiles, int N, int T,
    int n_crit, int nv, float scale, float* __restrict__ dq,
    float* __restrict__ dk, float* __restrict__ dv, int* err) {
  using L = SbSmem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = align_smem_1024(smem_raw);
  uint8_t* sK = base;
  uint8_t* sV = sK + L::kKV;
  uint8_t* sSt = sV + L::kKV;
  uint8_t* sDS = sSt + kNSt * L::kStage;  // two buffers, for even and odd iterations
  float* sStg = reinterpret_cast<float*>(sDS + 2 * L::kDS);  // dQ staging for bulk reductions

  __shared__ uint64_t kv_full, tile_done, acc_free, st_full[kNSt], st_empty[kNSt], s_full[2],
      ld_done[2], p_full[2], m_done[4], dq_free[4], tq_full[2], tq_empty[2], fin;
  __shared__ Tile tq[2];  // the tile walk, published by the producer
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int warp = threadIdx.x / 32, lane = lane_id();
  constexpr uint32_t kDV = 256, kDK = 256 + D;

  if (warp == 0) tmem_alloc(&tmem_base, 512);
  if (threadIdx.x == 32) {
    mbar_init(&kv_full, 1);
    mbar_init(&tile_done, 1);
    mbar_init(&acc_free, 256);
    for (int s = 0; s < kNSt; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&ld_done[b], 256);
      mbar_init(&p_full[b], 256);
      mbar_init(&m_done[b], 1);
      mbar_init(&m_done[b + 2], 1);
      mbar_init(&dq_free[b], 128);
      mbar_init(&dq_free[b + 2], 128);
      mbar_init(&tq_full[b], 1);
      mbar_init(&tq_empty[b], 2 + 3 * 128);  // the two issuers and three warpgroups
    }
    mbar_init(&fin, 2);  // one commit from each issuer
    abort_flag = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  // The m-th tile of this CTA, as published by the producer (consumers only).
  auto next_tile = [&](long m, Tile* t) -> bool {
    if (!wait_spin(&tq_full[m & 1], uint32_t(m >> 1) & 1, err, &abort_flag)) return false;
    *t = tq[m & 1];
    mbar_arrive(&tq_empty[m & 1]);
    return t->valid != 0;
  };

  // registers: launched with 128 per thread (65536 in all); the compute
  // warpgroups take 168, the dQ warpgroup 96 and the last warpgroup 80
  // (2 x 168 + 96 + 80 = 512 per thread slot of a warpgroup = 65536 / 128)
  // (each warpgroup executes its one setmaxnreg at the top of its branch)
  if (warp >= 12) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 80;" ::: "memory");
   if (warp == 12 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      long g = 0;       // iterations issued before the current tile
      int tw = 0;       // tiles with work so far
      long issued = 0;  // stage loads issued
      bool kv_pending = false, ok = true;
      // tiles are taken from a counter shared by all CTAs, in the order given
      auto fetch = [&]() -> Tile {
        return tile_at(order, ulen, col_ptr, atomicAdd(sched, 1), n_tiles, T, n_crit);
      };
      auto publish = [&](long m, const Tile& t) -> bool {
        if (m >= 2 && !wait_spin(&tq_empty[m & 1], uint32_t((m >> 1) - 1) & 1, err, &abort_flag))
          return false;
        tq[m & 1] = t;
        mbar_arrive(&tq_full[m & 1]);
        return true;
      };
      // two tiles of look-ahead: the next tile is published while the
      // current one starts, the one after it is fetched once the current
      // tile's loads are out (the counter and the tile's lookups take a few
      // round trips to global memory)
      Tile cur = fetch();
      Tile after = cur.valid ? fetch() : cur;
      ok = publish(0, cur);
      for (long m = 0; ok && cur.valid; ++m) {
        const Tile t = cur;
        cur = after;
        if (!(ok = publish(m + 1, cur))) break;
        if (t.n <= 0) {
          after = cur.valid ? fetch() : cur;
          continue;
        }
        if (cur.valid && cur.n > 0) {  // the next tile's K/V into L2 meanwhile
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_prefetch_l2_3d(&tm_k, c * 64, cur.qp * 128, cur.bh);
            tma_prefetch_l2_3d(&tm_v, c * 64, cur.qp * 128, cur.bh);
          }
        }
        auto load_stage = [&](int k) -> bool {
          const long gg = g + k;
          const int s = int(gg % kNSt);
          if (gg >= kNSt &&
              !wait_spin(&st_empty[s], uint32_t((gg / kNSt) + 1) & 1, err, &abort_flag))
            return false;
          uint8_t* st = sSt + s * L::kStage;
          const int i = ulist[t.slot + k];
          if (k + kNSt < t.n) {  // this tile's Q, dO three iterations ahead into L2
            const int ia = ulist[t.slot + k + kNSt];
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
              tma_prefetch_l2_3d(&tm_q, c * 64, ia * 64, t.bh);
              tma_prefetch_l2_3d(&tm_do, c * 64, ia * 64, t.bh);
            }
          }
          mbar_arrive_expect_tx(&st_full[s], L::kStageBytes);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_3d(st + c * 64 * 128, &st_full[s], &tm_q, c * 64, i * 64, t.bh);
            tma_load_3d(st + L::kQ + c * 64 * 128, &st_full[s], &tm_do, c * 64, i * 64, t.bh);
          }
          const size_t row0 = size_t(t.bh) * N + size_t(i) * 64;
          bulk_load(st + 2 * L::kQ, lse + row0, 256, &st_full[s]);
          bulk_load(st + 2 * L::kQ + 256, dvec + row0, 256, &st_full[s]);
          ++issued;
          return true;
        };
        // stages of the first iterations need only earlier iterations' stages
        // back, not the end of the previous tile: issue them before its K/V wait
        const int early = t.n < kNSt - 1 ? t.n : kNSt - 1;
        for (int k = 0; ok && k < early; ++k) ok = load_stage(k);
        if (ok && tw > 0) ok = wait_spin(&tile_done, uint32_t(tw - 1) & 1, err, &abort_flag);
        if (!ok) break;
        // every product of the previous tile is done: K, V may be replaced
        mbar_arrive_expect_tx(&kv_full, 2 * L::kKV);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(sK + c * 128 * 128, &kv_full, &tm_k, c * 64, t.qp * 128, t.bh);
          tma_load_3d(sV + c * 128 * 128, &kv_full, &tm_v, c * 64, t.qp * 128, t.bh);
        }
        kv_pending = true;
        for (int k = early; ok && k < t.n; ++k) ok = load_stage(k);
        after = cur.valid ? fetch() : cur;
        g += t.n;
        ++tw;
      }
      if (abort_flag) {
        // let copies already in flight land before the CTA exits
        if (kv_pending) wait_spin(&kv_full, uint32_t(tw - 1) & 1, nullptr, nullptr);
        for (long n = (issued > kNSt ? issued - kNSt : 0); n < issued; ++n)
          wait_spin(&st_full[n % kNSt], uint32_t(n / kNSt) & 1, nullptr, nullptr);
      }
    }
   } else if ((warp == 13 || warp == 14) && lane == 0) {
    // ------------------------------------------------------------ MMA issuers
    // Two threads feed the tensor pipe: warp 13 the S groups, warp 14 the G
    // groups.  The pipe takes only a few instructions ahead of execution, so a
    // single issuer that checks barriers between groups leaves it idle for
    // every check; with two, one stream's checks overlap the other's
    // products.  The two streams touch different TMEM chunks (the chunk
    // rotation above), so only the barriers order them; each commit tracks its
    // own thread's products.
    {
      constexpr uint32_t id_s = idesc_bf16(128, 64, 0, 0);  // S^T, dP^T
      constexpr uint32_t id_g = idesc_bf16(128, D, 0, 1);   // dV (A from TMEM), dK
      constexpr uint32_t id_q = idesc_bf16(128, 64, 1, 1);  // dQ^T = K^T dS^T
      const uint64_t kd_k = desc_kmajor_base(smem_u32(sK)), vd_k = desc_kmajor_base(smem_u32(sV));
      const uint64_t kd_mn = desc_mnmajor_base(smem_u32(sK), 128);
      const bool s_stream = warp == 13;
      long g = 0;
      int tw = 0;
      bool ok = true;
      // S(gg): S^T into chunk gg % 4, dP^T into chunk (gg + 1) % 4, once the
      // stage is loaded, dP^T(gg - 1) is out of its chunk and dQ^T(gg - 3) is
      // drained
      auto issue_s = [&](long gg) -> bool {
        const int s = int(gg % kNSt);
        if (!wait_spin(&st_full[s], uint32_t(gg / kNSt) & 1, err, &abort_flag)) return false;
        if (gg >= 1 &&
            !wait_spin(&ld_done[(gg - 1) & 1], uint32_t((gg - 1) >> 1) & 1, err, &abort_flag))
          return false;
        if (gg >= 3 &&
            !wait_spin(&dq_free[(gg - 3) & 3], uint32_t((gg - 3) >> 2) & 1, err, &abort_flag))
          return false;
        tc_fence_after();
        const uint32_t q0 = smem_u32(sSt + s * L::kStage), do0 = q0 + L::kQ;
        const uint32_t cs = tmem + uint32_t(gg & 3) * 64, cp = tmem + uint32_t((gg + 1) & 3) * 64;
        const uint64_t qd = desc_kmajor_base(q0), dod = desc_kmajor_base(do0);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          mma_ss(cs, desc_advance(kd_k, kmajor_step_bytes(128, ks)),
                 desc_advance(qd, kmajor_step_bytes(64, ks)), id_s, ks > 0);
          mma_ss(cp, desc_advance(vd_k, kmajor_step_bytes(128, ks)),
                 desc_advance(dod, kmajor_step_bytes(64, ks)), id_s, ks > 0);
        }
        mma_commit(&s_full[gg & 1]);
        return true;
      };
      // G(gg): dV += P^T dO_i, dK += dS^T Q_i (both A operands in chunk gg % 4:
      // queries 16k..16k+15 of P^T at column 8 (k & 1) + 32 (k >> 1), of dS^T 16
      // columns further), then dQ^T
      // over the same chunk (one thread's products run in order: dV has read
      // P^T by then).  G(gg) follows S(gg) through p_full, so the commit after
      // dV and dK frees the stage for the producer.
      auto issue_g = [&](long gg, bool first, bool last) -> bool {
        if (!wait_spin(&p_full[gg & 1], uint32_t(gg >> 1) & 1, err, &abort_flag)) return false;
        if (first && tw > 0 &&
            !wait_spin(&acc_free, uint32_t(tw - 1) & 1, err, &abort_flag))
          return false;
        tc_fence_after();
        const int s = int(gg % kNSt);
        const uint32_t q0 = smem_u32(sSt + s * L::kStage), do0 = q0 + L::kQ;
        const uint64_t qmn = desc_mnmajor_base(q0, 64), domn = desc_mnmajor_base(do0, 64);
        const uint32_t cs = tmem + uint32_t(gg & 3) * 64;
        const uint32_t ds0 = smem_u32(sDS + (gg & 1) * L::kDS);
        const uint64_t dsd_mn = desc_mnmajor_base(ds0, 128);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t acc = (!first || ks > 0) ? 1u : 0u;
          const uint32_t pa = cs + (ks & 1) * 8 + (ks >> 1) * 32;
          mma_ts(tmem + kDV, pa, desc_advance(domn, mnmajor_step_bytes(ks)), id_g, acc);
          mma_ts(tmem + kDK, pa + 16, desc_advance(qmn, mnmajor_step_bytes(ks)), id_g, acc);
        }
        mma_commit(&st_empty[s]);  // the last products that read the stage
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss(cs, desc_advance(kd_mn, mnmajor_step_bytes(ks)),
                 desc_advance(dsd_mn, mnmajor_step_bytes(ks)), id_q, ks > 0);
        mma_commit(&m_done[gg & 3]);
        if (last) mma_commit(&tile_done);
        return true;
      };
      Tile t;
      for (long m = 0; ok && (ok = next_tile(m, &t)); ++m) {
        if (t.n <= 0) continue;
        if (s_stream) {
          if (!(ok = wait_spin(&kv_full, uint32_t(tw) & 1, err, &abort_flag))) break;
          for (int k = 0; ok && k < t.n; ++k) ok = issue_s(g + k);
        } else {
          for (int k = 0; ok && k < t.n; ++k) ok = issue_g(g + k, k == 0, k == t.n - 1);
        }
        g += t.n;
        ++tw;
      }
      mma_commit(&fin);
      mbar_wait(&fin, 0, nullptr, nullptr);
    }
   }
  } else if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 96;" ::: "memory");
    // ------------------------------------------------------------ dQ warpgroup
    // dQ_i^T (lane = feature, 64 query columns) of every iteration, in four
    // quarters of 16 queries: each is written transposed into one of two
    // staging buffers [16][d] (a warp's stores for one query cover 32
    // consecutive features) and added into the 16 contiguous dQ rows by one
    // bulk reduction issued by thread 256; the reduction of one quarter reads
    // its buffer while the next quarter is written into the other.
    // The warpgroup synchronizes with hardware named barrier 1.  Every thread
    // runs the same sequence of them: the trip counts come from the shared
    // tile queue, and each wait's outcome is made common to the warpgroup with
    // bar.red.and before anything depends on it, so no thread can be left at
    // a barrier that another has skipped.
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_base = uint32_t(wq * 32) << 16;
    const bool leader = threadIdx.x == 256;
    auto wg_bar = [] { named_bar_sync(1, 128); };
    auto wg_all = [](bool p) -> bool { return named_bar_and(1, 128, p); };
    float* stg[2] = {sStg, sStg + 16 * D};
    long g = 0;
    bool ok = true;
    Tile t;
    for (long m = 0; ok; ++m) {
      const bool got = next_tile(m, &t);
      if (!wg_all(got)) break;
      for (int k = 0; k < t.n; ++k) {
        const long gg = g + k;
        const int i = ulist[t.slot + k];
        float* gdq = dq + (size_t(t.bh) * N + size_t(i) * 64) * D;
        const uint32_t cs = tmem + lane_base + uint32_t(gg & 3) * 64;
        const bool w = wait_spin(&m_done[gg & 3], uint32_t(gg >> 2) & 1, err, &abort_flag);
        if (!(ok = wg_all(w))) break;
        tc_fence_after();
        float v[64];
        if (wq * 32 < D) {
          tmem_ld32(cs, reinterpret_cast<float(&)[32]>(v[0]));
          tmem_ld32(cs + 32, reinterpret_cast<float(&)[32]>(v[32]));
          tmem_ld_wait();
        }
        tc_fence_before();
        mbar_arrive(&dq_free[gg & 3]);
#pragma unroll
        for (int qt = 0; qt < 4; ++qt) {
          float* buf = stg[qt & 1];
          if (leader) bulk_wait_read_le1();  // the reduction that read this buffer is done with it
          wg_bar();
          if (r < D) {
#pragma unroll
            for (int c = 0; c < 16; ++c) buf[c * D + r] = v[16 * qt + c] * scale;
          }
          fence_proxy_async_smem();
          wg_bar();
          if (leader) {
            bulk_reduce_add_f32(gdq + size_t(16 * qt) * D, buf, 16 * D * 4);
            bulk_commit();
          }
        }
      }
      g += t.n > 0 ? t.n : 0;
    }
    if (leader) bulk_wait_all();
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 168;" ::: "memory");
    // ------------------------------------------------------------ compute warpgroups
    const int wg = warp >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;  // key row == TMEM lane (dQ^T: feature row)
    const int half = r >> 6;
    const uint32_t lane_base = uint32_t(wq * 32) << 16;
    long g = 0;
    int tw = 0;
    bool ok = true;
    Tile t;
    for (long m = 0; ok && (ok = next_tile(m, &t)); ++m) {
      const bool key_ok = (half == 0) || (2 * t.qp + 1 < T);  // the key block exists
      const int key = t.qp * 128 + r;
      // a padded key (key padding) gets no weight; its dK, dV rows stay 0
      const bool key_valid = key_ok && key < nv;
      float* out_row = (wg == 0 ? dk : dv) + (size_t(t.bh) * N + key) * D;
      if (t.n <= 0) {
        if (key_ok) {
#pragma unroll 4
          for (int c = 0; c < D; c += 4)
            *reinterpret_cast<float4*>(out_row + c) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        continue;
      }
      for (int k = 0; k < t.n; ++k) {
        const long gg = g + k;
        const int fl = uflag[t.slot + k];
        // this warpgroup's 32 query columns of the S^T and dP^T chunks
        const uint32_t cs = tmem + lane_base + uint32_t(gg & 3) * 64 + 32 * wg;
        const uint32_t cp = tmem + lane_base + uint32_t((gg + 1) & 3) * 64 + 32 * wg;
        // (each wait's outcome is made common to the warp: the TMEM loads and
        // stores that follow are warp-collective)
        // (the stage's LSE_i, D_i, read below, landed before S(gg) was issued:
        // its issuer waited for the stage's copies, and this wait is ordered
        // before the reads)
        ok = __all_sync(0xFFFFFFFFu, wait_spin(&s_full[gg & 1], uint32_t(gg >> 1) & 1, err, &abort_flag));
        if (!ok) break;
        tc_fence_after();
        // (a padded query row of this block has LSE = +inf, so its P is 0)
        const bool member = key_valid && ((fl >> half) & 1);
        uint32_t pk[16], dsk[16];
        // dP^T first: its chunk is the next S^T's, so it is handed back as soon
        // as it is in registers; then S^T (P^T and dS^T go back over S^T)
        float dpa[32], sv[32];
        tmem_ld32(cp, dpa);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&ld_done[gg & 1]);
        tmem_ld32(cs, sv);
        tmem_ld_wait();
        // LSE, D of this warpgroup's 32 queries, from the iteration's stage (the
        // stage is released only after G(gg), which waits for this thread's p_full)
        const float* ld = reinterpret_cast<const float*>(sSt + (gg % kNSt) * L::kStage + 2 * L::kQ) +
                          32 * wg;
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(ld + e);
          const float4 d4 = *reinterpret_cast<const float4*>(ld + 64 + e);
          const float lq[4] = {l4.x, l4.y, l4.z, l4.w}, dq4[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
          for (int m = 0; m < 4; m += 2) {
            float p0 = 0.f, p1 = 0.f;
            if (member) {
              p0 = exp2f(kLog2e * fmaf(sv[e + m], scale, -lq[m]));
              p1 = exp2f(kLog2e * fmaf(sv[e + m + 1], scale, -lq[m + 1]));
            }
            pk[(e + m) / 2] = pack_bf16(p0, p1);
            dsk[(e + m) / 2] = pack_bf16(p0 * (dpa[e + m] - dq4[m]), p1 * (dpa[e + m + 1] - dq4[m + 1]));
          }
        }
        tmem_st16(cs, pk);
        tmem_st16(cs + 16, dsk);
        // dS^T into this iteration's buffer once its last reader, G(gg - 2), is done
        if (gg >= 2) {
          ok = __all_sync(0xFFFFFFFFu, wait_spin(&m_done[(gg - 2) & 3], uint32_t((gg - 2) >> 2) & 1,
                                                 err, &abort_flag));
          if (!ok) break;
        }
        uint8_t* ds_tile = sDS + (gg & 1) * L::kDS;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          st_sw128_unit(ds_tile, 128, r, 32 * wg + 8 * u,
                        make_uint4(dsk[4 * u], dsk[4 * u + 1], dsk[4 * u + 2], dsk[4 * u + 3]));
        fence_proxy_async_smem();
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[gg & 1]);
      }
      if (!ok) break;
      // the tile's dK (warpgroup 0) / dV (warpgroup 1) rows, straight from TMEM
      ok = __all_sync(0xFFFFFFFFu, wait_spin(&tile_done, uint32_t(tw) & 1, err, &abort_flag));
      if (!ok) break;
      tc_fence_after();
      const uint32_t acc = tmem + lane_base + (wg == 0 ? kDK : kDV);
      const float mul = wg == 0 ? scale : 1.0f;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        float a[32];
        tmem_ld32(acc + c0, a);
        tmem_ld_wait();
        if (key_ok) {
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4*>(out_row + c0 + c) =
                make_float4(a[c] * mul, a[c + 1] * mul, a[c + 2] * mul, a[c + 3] * mul);
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_free);  // the accumulators may be overwritten by the next tile
      g += t.n;
      ++tw;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free(tmem, 512);
}

// ------------------------------------------------------------------ tile unions
// One warp per key-block pair: the sorted union of the critical query blocks of
// key blocks 2q and 2q+1 (column CSR), written into the pair's slot of the CSR
// (its two lists' entries, which the union never outnumbers), with flag bit h
// = query block critical for key block 2q+h, and the union's length.
constexpr int kUnionWarps = 8;

__global__ void __launch_bounds__(kUnionWarps * 32) pair_union_kernel(
    const int32_t* __restrict__ col_ptr, const int32_t* __restrict__ col_idx, int BH, int T,
    int n_crit, uint16_t* __restrict__ ulist, uint8_t* __restrict__ uflag,
    int32_t* __restrict__ ulen, int* err) {
  extern __shared__ uint32_t ubits[];  // [kUnionWarps][2 * ceil(T/32)]
  const int npairs = (T + 1) / 2;
  const int w = threadIdx.x / 32, lane = lane_id();
  const int item = blockIdx.x * kUnionWarps + w;
  if (item >= BH * npairs) return;
  const int bh = item / npairs, qp = item % npairs;
  const int kb0 = 2 * qp, kb1 = 2 * qp + 1;
  const bool has1 = kb1 < T;
  const int32_t* cp = col_ptr + size_t(bh) * (T + 1);
  const int32_t* ci = col_idx + size_t(bh) * T * n_crit;
  int a = cp[kb0], ae = cp[kb0 + 1];
  int b = has1 ? cp[kb1] : ae, be = has1 ? cp[kb1 + 1] : ae;
  const int cap = T * n_crit;
  if (a < 0 || ae > cap || a > ae || b != ae || be > cap || b > be || ae - a > T || be - b > T) {
    if (lane == 0) set_error(err, SLA_ERR_DEVICE);
    if (lane == 0) ulen[item] = 0;
    return;
  }
  const size_t slot = size_t(bh) * T * n_crit + a;
  const int n = warp_union(ci + a, ae - a, ci + b, be - b, T,
                           ubits + w * 2 * ((T + 31) / 32), ulist + slot, uflag + slot, err);
  if (lane == 0) ulen[item] = n;
}

// ------------------------------------------------------------------ tile order
// One CTA: a counting sort of all key-block pairs by the key
//   head + kStagger * (1 - length / longest length),
// ascending.  Heads come in sequence, so the tiles running at any time share
// the Q and dO of a few heads in L2, and within the window of kStagger heads
// the longest unions (the tiles' work) start first, so that no long tile of
// the last heads starts near the end of the walk.  Pairs in one bucket keep no
// particular order.
constexpr int kOrderThreads = 1024;
constexpr int kOrderBuckets = 8192;
constexpr float kStagger = 4.0f;

__global__ void __launch_bounds__(kOrderThreads) pair_order_kernel(
    const int32_t* __restrict__ ulen, int32_t* __restrict__ order, int* __restrict__ sched,
    int n_items, int npairs, int BH) {
  __shared__ int cnt[kOrderBuckets];
  __shared__ int part[kOrderThreads];
  __shared__ int longest;
  const int t = threadIdx.x;
  if (t == 0) longest = 1;
  for (int b = t; b < kOrderBuckets; b += kOrderThreads) cnt[b] = 0;
  __syncthreads();
  int mx = 1;
  for (int i = t; i < n_items; i += kOrderThreads) mx = max(mx, ulen[i]);
  atomicMax(&longest, mx);
  __syncthreads();
  const float inv_len = 1.0f / float(longest);
  const float per = float(kOrderBuckets) / (float(BH) + kStagger);
  auto bucket = [&](int i) {
    const float len = float(min(max(ulen[i], 0), longest));
    const int b = int((float(i / npairs) + kStagger * (1.0f - len * inv_len)) * per);
    return min(max(b, 0), kOrderBuckets - 1);
  };
  for (int i = t; i < n_items; i += kOrderThreads) atomicAdd(&cnt[bucket(i)], 1);
  __syncthreads();
  // exclusive scan of the buckets: thread t owns a contiguous run of them
  constexpr int kPer = kOrderBuckets / kOrderThreads;
  const int b0 = t * kPer;
  int sum = 0;
#pragma unroll
  for (int b = 0; b < kPer; ++b) sum += cnt[b0 + b];
  part[t] = sum;
  __syncthreads();
  for (int o = 1; o < kOrderThreads; o <<= 1) {  // inclusive scan of the run sums
    const int v = t >= o ? part[t - o] : 0;
    __syncthreads();
    part[t] += v;
    __syncthreads();
  }
  int run = part[t] - sum;
#pragma unroll
  for (int b = 0; b < kPer; ++b) {
    const int c = cnt[b0 + b];
    cnt[b0 + b] = run;
    run += c;
  }
  __syncthreads();
  for (int i = t; i < n_items; i += kOrderThreads) order[atomicAdd(&cnt[bucket(i)], 1)] = i;
  if (t == 0) *sched = 0;  // the sparse backward's tile counter
}

}  // namespace

cudaError_t launch_pair_order(const Problem& p, const int32_t* col_ptr, const int32_t* col_idx,
                              uint16_t* ulist, uint8_t* uflag, int32_t* ulen, int32_t* order,
                              int* sched, int* err, cudaStream_t s) {
  const int npairs = (p.T + 1) / 2;
  const size_t ubytes = sizeof(uint32_t) * kUnionWarps * 2 * size_t((p.T + 31) / 32);
  const int ublocks = (p.BH * npairs + kUnionWarps - 1) / kUnionWarps;
  pair_union_kernel<<<ublocks, kUnionWarps * 32, ubytes, s>>>(col_ptr, col_idx, p.BH, p.T,
                                                              p.n_crit, ulist, uflag, ulen, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  pair_order_kernel<<<1, kOrderThreads, 0, s>>>(ulen, order, sched, p.BH * npairs, npairs, p.BH);
  return cudaGetLastError();
}

cudaError_t launch_bwd_sparse(const Problem& p, const void* q, const void* k, const void* v,
                              const void* d_o, const float* lse, const float* dvec,
                              const int32_t* col_ptr, const uint16_t* ulist, const uint8_t* uflag,
                              const int32_t* ulen, const int32_t* order, int* sched, float* dq,
                              float* dk, float* dv, int num_sms, int* err, cudaStream_t s) {
  // LSE_i and D_i go to shared memory by bulk copies: 16-byte aligned rows
  if ((reinterpret_cast<uintptr_t>(lse) | reinterpret_cast<uintptr_t>(dvec)) % 16 != 0)
    return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv, tdo;
  if (!make_tmap_bhnd(&tq, q, p.BH, p.N, p.d, 64)) return cudaErrorInvalidValue;
  if (!make_tmap_bhnd(&tk, k, p.BH, p.N, p.d, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bhnd(&tv, v, p.BH, p.N, p.d, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bhnd(&tdo, d_o, p.BH, p.N, p.d, 64)) return cudaErrorInvalidValue;
  const int n_tiles = ((p.T + 1) / 2) * p.BH;
  dim3 grid(std::min(n_tiles, std::max(num_sms, 1)));
  cudaError_t e;
  if (p.d == 128) {
    constexpr size_t smem = SbSmem<128>::kTotal;
    e = cudaFuncSetAttribute(bwd_sparse_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem));
    if (e != cudaSuccess) return e;
    bwd_sparse_kernel<128><<<grid, 512, smem, s>>>(tq, tk, tv, tdo, lse, dvec, col_ptr, ulist,
                                                   uflag, ulen, order, sched, n_tiles, p.N, p.T,
                                                   p.n_crit, p.nv, p.scale, dq, dk,
                                                   dv, err);
  } else {
    constexpr size_t smem = SbSmem<64>::kTotal;
    e = cudaFuncSetAttribute(bwd_sparse_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem));
    if (e != cudaSuccess) return e;
    bwd_sparse_kernel<64><<<grid, 512, smem, s>>>(tq, tk, tv, tdo, lse, dvec, col_ptr, ulist,
                                                  uflag, ulen, order, sched, n_tiles, p.N, p.T, p.n_crit,
                                                  p.nv, p.scale, dq, dk, dv, err);
  }
  return cudaGetLastError();
}

}  // namespace sla
