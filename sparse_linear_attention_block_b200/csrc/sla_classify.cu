// Classification of (query block, key block) pairs.
//
// SLA (arXiv 2509.24006), abstract / framework step 1: attention weights are
// sorted into critical, marginal and negligible groups.  The pages do not say
// how; this file implements the reading used throughout the library:
// block mean-pooled Q and K, pooled logits s_ij = mean(Q_i).mean(K_j)*scale,
// and per row an exact selection of the n_crit largest and n_negl smallest
// logits, ties broken toward the lower key-block index.  Ranking logits is
// equivalent to ranking the row softmax of the pooled scores.
#include <cuda_bf16.h>

#include <algorithm>

#include "sla_internal.h"
#include "sla_ptx.cuh"

namespace sla {
namespace {

// ------------------------------------------------------------------ pooling
// One CTA per (block j, head bh); 128 threads.  Each thread sums a 16-byte
// column chunk over a subset of the 64 rows, then the partial sums are
// combined through shared memory.  HBM-bound: reads Q and K once.
template <int D>
__global__ void __launch_bounds__(128) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k,
                                                   float* __restrict__ qbar,
                                                   float* __restrict__ kbar, int N, int T,
                                                   int nv) {
  constexpr int kChunks = D / 8;          // 16-byte chunks per row
  constexpr int kGroups = 128 / kChunks;  // row groups
  constexpr int kRowsPer = kBlock / kGroups;
  __shared__ float red[2][kGroups][D];
  const int j = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const int c8 = t % kChunks, g = t / kChunks;
  const size_t base = (size_t(bh) * N + size_t(j) * kBlock) * D;
  const int valid = min(kBlock, nv - j * kBlock);  // tokens of this block that exist
#pragma unroll
  for (int which = 0; which < 2; ++which) {
    const __nv_bfloat16* src = (which == 0 ? q : k) + base;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < kRowsPer; ++i) {
      const int row = g + i * kGroups;
      if (row >= valid) continue;
      const uint4 u = *reinterpret_cast<const uint4*>(src + size_t(row) * D + c8 * 8);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += bf16_lo(w[e]);
        acc[2 * e + 1] += bf16_hi(w[e]);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[which][g][c8 * 8 + e] = acc[e];
  }
  __syncthreads();
  for (int c = t; c < 2 * D; c += 128) {
    const int which = c / D, col = c % D;
    float s = 0.f;
#pragma unroll
    for (int gg = 0; gg < kGroups; ++gg) s += red[which][gg][col];
    float* dst = (which == 0 ? qbar : kbar) + (size_t(bh) * T + j) * D;
    dst[col] = s / float(valid);
  }
}

// ------------------------------------------------------------------ classify
// Order-preserving map of a float to uint32 (-0 canonicalised to +0).
__device__ __forceinline__ uint32_t ordered_bits(float x) {
  uint32_t b = __float_as_uint(x);
  if (b == 0x80000000u) b = 0;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Selection thresholds.  For the order (score desc, index asc) a threshold
// is the n-th element's ordered score v and index jt: an element is at or
// before it iff its ordered score is > v, or == v with index <= jt.  For the
// reverse order (score asc, index desc) v holds the complemented score and the
// index test is >= jt.
struct Threshold {
  uint32_t v;
  int jt;
};

// The n-th element of a row of `len` scores (smem, len <= 32 * KPL) in the
// order (score desc, index asc), or with `flip` in the reverse order (score
// asc, index desc), found by one warp.  The row is held in registers as
// order-preserving 32-bit keys (complemented when flipped; element j in lane
// j % 32, slot j / 32; slots past len hold 0, below every key).  A bracket
// [a, b) of key values with #(key >= a) >= n > #(key >= b) is narrowed by a
// safeguarded interpolation search (the pivot from the two counts; a plain
// halving whenever an interpolation step did not halve the bracket), each step
// one count by warp sums, until it holds one key value or at most 32 elements.
// Then either the need-th equal key in index order is taken, or the bracket's
// elements are compacted one per lane (through 64 words of shared scratch)
// and ranked against each other by shuffles.  Exact for any input without NaN.
template <int KPL>
__device__ Threshold select_side(const float* row, int len, int n, bool flip,
                                 uint32_t* scratch) {
  constexpr uint32_t kAll = 0xFFFFFFFFu;
  const int lane = lane_id();
  uint32_t key[KPL];
  uint32_t kmin = ~0u, kmax = 0u;
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const int j = 32 * e + lane;
    uint32_t k = 0u;
    if (j < len) {
      k = ordered_bits(row[j]);
      if (flip) k = ~k;
      kmin = min(kmin, k);
    }
    key[e] = k;
    kmax = max(kmax, k);
  }
  uint32_t a = __reduce_min_sync(kAll, kmin);
  uint32_t b = __reduce_max_sync(kAll, kmax) + 1u;  // keys never reach 0xFFFFFFFF
  int ca = len, cb = 0;
  bool halve = false;
  while (b - a > 1u && ca - cb > 32) {
    const uint32_t w = b - a;
    uint32_t p = halve ? a + w / 2u
                       : a + 1u + uint32_t((uint64_t(w - 1u) * uint32_t(ca - n)) /
                                           uint32_t(ca - cb));
    p = min(max(p, a + 1u), b - 1u);
    int c = 0;
#pragma unroll
    for (int e = 0; e < KPL; ++e) c += key[e] >= p;
    c = __reduce_add_sync(kAll, c);
    if (c >= n) {
      a = p;
      ca = c;
    } else {
      b = p;
      cb = c;
    }
    halve = !halve && uint64_t(b - a) * 2u > uint64_t(w);
  }
  const int need = n - cb;  // rank of the answer inside the bracket (1-based)
  Threshold th{a, -1};
  if (b - a == 1u) {  // one key value: the need-th equal element in index order
    int seen = 0;
#pragma unroll
    for (int s = 0; s < KPL; ++s) {
      const int e = flip ? KPL - 1 - s : s;
      uint32_t m = __ballot_sync(kAll, key[e] == a);  // a zero slot never equals a
      const int cnt = __popc(m);
      if (th.jt < 0 && seen + cnt >= need) {
        for (int r = need - seen; r > 1; --r) m &= flip ? ~(1u << (31 - __clz(m))) : m - 1u;
        th.jt = 32 * e + (flip ? 31 - __clz(m) : __ffs(int(m)) - 1);
      }
      seen += cnt;
    }
    return th;
  }
  // at most 32 elements in [a, b): one per lane, then ranks by shuffles
  int base = 0;
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const bool in = key[e] >= a && key[e] < b;
    const uint32_t m = __ballot_sync(kAll, in);
    if (in) {
      const int pos = base + __popc(m & ((1u << lane) - 1u));
      scratch[pos] = key[e];
      scratch[32 + pos] = uint32_t(32 * e + lane);
    }
    base += __popc(m);
  }
  __syncwarp();
  const int cnt = ca - cb;
  const uint32_t mk = lane < cnt ? scratch[lane] : 0u;
  const int mj = lane < cnt ? int(scratch[32 + lane]) : 0;
  int rank = 0;
  for (int l = 0; l < cnt; ++l) {
    const uint32_t ok = __shfl_sync(kAll, mk, l);
    const int oj = __shfl_sync(kAll, mj, l);
    rank += ok > mk || (ok == mk && (flip ? oj > mj : oj < mj));
  }
  const uint32_t hit = __ballot_sync(kAll, lane < cnt && rank == need - 1);
  const int src = __ffs(int(hit)) - 1;
  th.v = __shfl_sync(kAll, mk, src);
  th.jt = __shfl_sync(kAll, mj, src);
  __syncwarp();  // scratch may be reused by the next selection
  return th;
}

__device__ __forceinline__ bool before_or_at(uint32_t o, int j, Threshold t, bool flip) {
  if (flip) o = ~o;
  return o > t.v || (o == t.v && (flip ? j >= t.jt : j <= t.jt));
}

constexpr int kRowsPerCta = 8;  // one warp per query-block row
constexpr int kKTile = 32;      // coarse keys staged per step (hierarchical selection)

// Scores of the flat classifier: a CTA's 8 rows against key tiles of 128,
// staged 32 features at a time through a cp.async double buffer (the next
// chunk is in flight while the current one is multiplied).  Thread (rg, kq)
// of the 4 x 64 grid holds the 2 x 2 block rows {2rg, 2rg+1} x keys
// {kq, kq + 64}: per 4 features it reads 2 query and 2 key float4s (each a
// conflict-free wavefront across the warp, thanks to the padded rows) for 16
// FMAs.  The small staging buffers keep two or three CTAs on an SM.
constexpr int kSKeys = 128;      // keys per score tile
constexpr int kSChunk = 32;      // features staged per step
constexpr int kSStride = kSChunk + 4;
constexpr int kSBuf = kSKeys * kSStride;  // floats per staging buffer

// 16-byte global -> shared copy; src_bytes = 0 writes zeros (out-of-range key)
__device__ __forceinline__ void cp_async16(float* dst, const float* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// One CTA per 8 rows of one head.  When `logits_in` is null the pooled logits
// are computed from qbar/kbar (fp32), otherwise read from it.  KPL: row
// scores per lane in the selection (T <= 32 * KPL).
template <int D, int KPL>
__global__ void __launch_bounds__(256) classify_kernel(
    const float* __restrict__ qbar, const float* __restrict__ kbar,
    const float* __restrict__ logits_in, float* __restrict__ logits_out,
    int8_t* __restrict__ cls, int32_t* __restrict__ crit_idx, uint32_t* __restrict__ marg_bits,
    int T, int n_crit, int n_negl, float scale) {
  extern __shared__ __align__(16) float smem[];
  constexpr int kQStride = D + 4;
  constexpr int kChunks = D / kSChunk;
  float* srow = smem;                                // [8][T]
  float* sq = srow + kRowsPerCta * T;                // [8][D+4]
  float* sk = sq + kRowsPerCta * kQStride;           // 2 x [128][32+4], then 8 x 64 words
  const int bh = blockIdx.y, warp = threadIdx.x / 32, lane = lane_id();
  const int i = blockIdx.x * kRowsPerCta + warp;
  const bool row_ok = i < T;
  float* row = srow + warp * T;

  if (logits_in == nullptr) {
    for (int e = threadIdx.x; e < kRowsPerCta * D / 4; e += blockDim.x) {
      const int r = e / (D / 4), a4 = e % (D / 4), ii = blockIdx.x * kRowsPerCta + r;
      const float4 x = ii < T ? reinterpret_cast<const float4*>(qbar + (size_t(bh) * T + ii) * D)[a4]
                              : make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(sq + r * kQStride + 4 * a4) = x;
    }
    const int rg = lane >> 3, kq = warp * 8 + (lane & 7);
    const float* kb = kbar + size_t(bh) * T * D;
    const int nsteps = (T + kSKeys - 1) / kSKeys * kChunks;
    // step st = (key tile st / kChunks, feature chunk st % kChunks) into buffer st & 1
    auto stage = [&](int st) {
      float* dst = sk + (st & 1) * kSBuf;
      const int j0 = (st / kChunks) * kSKeys, c0 = (st % kChunks) * kSChunk;
#pragma unroll
      for (int x = 0; x < kSKeys * kSChunk / 4 / 256; ++x) {
        const int e = threadIdx.x + 256 * x;
        const int key = e / (kSChunk / 4), a4 = e % (kSChunk / 4), jj = j0 + key;
        const bool in = jj < T;
        cp_async16(dst + key * kSStride + 4 * a4, in ? kb + size_t(jj) * D + c0 + 4 * a4 : kb,
                   in ? 16 : 0);
      }
      cp_async_commit();
    };
    stage(0);
    float acc[2][2];
    for (int st = 0; st < nsteps; ++st) {
      if (st + 1 < nsteps) {
        stage(st + 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();  // step st landed for every thread's copies
      const int chunk = st % kChunks, j0 = (st / kChunks) * kSKeys;
      if (chunk == 0) {
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int j = 0; j < 2; ++j) acc[r][j] = 0.f;
      }
      const float* kbuf = sk + (st & 1) * kSBuf;
      const float* q0 = sq + (2 * rg) * kQStride + chunk * kSChunk;
      const float* q1 = q0 + kQStride;
#pragma unroll
      for (int a = 0; a < kSChunk; a += 4) {
        const float4 x0 = *reinterpret_cast<const float4*>(q0 + a);
        const float4 x1 = *reinterpret_cast<const float4*>(q1 + a);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float4 y = *reinterpret_cast<const float4*>(kbuf + (kq + 64 * j) * kSStride + a);
          acc[0][j] = fmaf(x0.x, y.x, acc[0][j]); acc[0][j] = fmaf(x0.y, y.y, acc[0][j]);
          acc[0][j] = fmaf(x0.z, y.z, acc[0][j]); acc[0][j] = fmaf(x0.w, y.w, acc[0][j]);
          acc[1][j] = fmaf(x1.x, y.x, acc[1][j]); acc[1][j] = fmaf(x1.y, y.y, acc[1][j]);
          acc[1][j] = fmaf(x1.z, y.z, acc[1][j]); acc[1][j] = fmaf(x1.w, y.w, acc[1][j]);
        }
      }
      if (chunk == kChunks - 1) {
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int jj = j0 + kq + 64 * j;
            if (jj < T) srow[(2 * rg + r) * T + jj] = acc[r][j] * scale;
          }
      }
      __syncthreads();  // buffer st & 1 may be refilled by step st + 2
    }
    __syncthreads();  // every row complete
    if (row_ok && logits_out) {
      for (int j = lane; j < T; j += 32) logits_out[(size_t(bh) * T + i) * T + j] = row[j];
    }
  } else {
    if (row_ok)
      for (int j = lane; j < T; j += 32) row[j] = logits_in[(size_t(bh) * T + i) * T + j];
    __syncwarp();
  }
  if (!row_ok) return;

  uint32_t* scratch = reinterpret_cast<uint32_t*>(sk + 2 * kSBuf) + warp * 64;
  const Threshold th = n_crit > 0 ? select_side<KPL>(row, T, n_crit, false, scratch)
                                  : Threshold{0, -1};
  const Threshold tl = n_negl > 0 ? select_side<KPL>(row, T, n_negl, true, scratch)
                                  : Threshold{0, -1};
  const size_t rbase = size_t(bh) * T + i;
  int8_t* crow = cls + rbase * T;
  int32_t* idx = crit_idx + rbase * n_crit;
  const int words = (T + 31) / 32;
  uint32_t* mrow = marg_bits + rbase * words;
  int written = 0;
  for (int j0 = 0; j0 < words * 32; j0 += 32) {
    const int j = j0 + lane;
    int c = 0;
    bool in = j < T;
    if (in) {
      const uint32_t o = ordered_bits(row[j]);
      if (n_crit > 0 && before_or_at(o, j, th, false)) c = 1;
      else if (n_negl > 0 && before_or_at(o, j, tl, true)) c = -1;
      crow[j] = int8_t(c);
    }
    const uint32_t crit_mask = __ballot_sync(0xFFFFFFFFu, in && c == 1);
    const uint32_t marg_mask = __ballot_sync(0xFFFFFFFFu, in && c == 0);
    if (in && c == 1) {
      const int pos = written + __popc(crit_mask & ((1u << lane) - 1u));
      if (pos < n_crit) idx[pos] = j;
    }
    written += __popc(crit_mask);
    if (lane == 0) mrow[j0 / 32] = marg_mask;
  }
}

// ------------------------------------------------------------------ hierarchical selection
// "Trainable Log-linear Sparse Attention for Efficient Diffusion Transformers"
// (abstract): top-K is taken on a coarse level first and the next level only
// looks inside the indices it kept.  Here the coarse level is super-blocks of
// G consecutive key blocks with mean key Kc_J; per query-block row its first
// c_hi super-blocks (coarse score desc, J asc) hold the critical candidates and
// its last c_lo the negligible ones.  The host routes the case in which the
// two lists could meet (c_hi + c_lo > TG) to the flat kernel above, so here
// the lists are disjoint and each holds enough blocks for its count.

// Kc_J = mean of the block means of super-block J (the last may be partial).
// One CTA per (J, head), one thread per feature.
__global__ void coarse_keys_kernel(const float* __restrict__ kbar, float* __restrict__ kc,
                                   int T, int TG, int G, int D) {
  const int J = blockIdx.x, bh = blockIdx.y, a = threadIdx.x;
  if (a >= D) return;
  const int j0 = J * G, j1 = min(T, j0 + G);
  const float* src = kbar + (size_t(bh) * T) * D + a;
  float s = 0.f;
  for (int j = j0; j < j1; ++j) s += src[size_t(j) * D];
  kc[(size_t(bh) * TG + J) * D + a] = s / float(j1 - j0);
}

struct HierArgs {
  const float* qbar;       // [BH,T,D]   (null with fine_in)
  const float* kbar;       // [BH,T,D]
  const float* kc;         // [BH,TG,D]
  const float* fine_in;    // [BH,T,T]   caller scores, or null
  const float* coarse_in;  // [BH,T,TG]  caller coarse scores, or null
  float* fine_out;         // [BH,T,T]   candidate entries only, or null
  float* coarse_out;       // [BH,T,TG]  or null
  int8_t* cls;
  int32_t* crit_idx;
  uint32_t* marg_bits;
  int* err;
  int T, TG, G, c_hi, c_lo, cap_hi, cap_lo, n_crit, n_negl, rows, BH;
  float scale;
  size_t smem;
};

// Per-warp shared scratch, in floats / words.
__host__ __device__ inline int hier_warp_words(int T, int TG, int cap_hi, int cap_lo, int c_hi,
                                               int c_lo) {
  const int W = (T + 31) / 32;
  return TG + cap_hi + cap_lo + c_hi + c_lo + 2 * W + 64;
}

// Block index of candidate position p of a list of super-blocks (ascending).
__device__ __forceinline__ int cand_block(const int* list, int p, int G) {
  return list[p / G] * G + p % G;
}

// Fine scores of nb candidate positions into out[]: four candidates per step,
// eight lanes per candidate, each lane a contiguous D/8-feature slice of the
// pooled query (registers) against the same slice of the pooled key (L2).
template <int D>
__device__ void fine_scores(const float* qrow, const float* kbar_h, const int* list, int nb,
                            int G, float scale, float* out, float* fine_out_row) {
  constexpr int kPer = D / 8;  // features per lane
  const int lane = lane_id(), sub = lane & 7, grp = lane >> 3;
  float qv[kPer];
#pragma unroll
  for (int e = 0; e < kPer; e += 4) {
    const float4 x = *reinterpret_cast<const float4*>(qrow + sub * kPer + e);
    qv[e] = x.x; qv[e + 1] = x.y; qv[e + 2] = x.z; qv[e + 3] = x.w;
  }
  for (int p0 = 0; p0 < nb; p0 += 4) {
    const int p = p0 + grp;
    float acc = 0.f;
    int j = 0;
    if (p < nb) {
      j = cand_block(list, p, G);
      const float4* kr = reinterpret_cast<const float4*>(kbar_h + size_t(j) * D + sub * kPer);
#pragma unroll
      for (int e = 0; e < kPer / 4; ++e) {
        const float4 y = __ldg(kr + e);
        acc = fmaf(qv[4 * e], y.x, acc);
        acc = fmaf(qv[4 * e + 1], y.y, acc);
        acc = fmaf(qv[4 * e + 2], y.z, acc);
        acc = fmaf(qv[4 * e + 3], y.w, acc);
      }
    }
    acc += __shfl_xor_sync(0xFFFFFFFFu, acc, 1);
    acc += __shfl_xor_sync(0xFFFFFFFFu, acc, 2);
    acc += __shfl_xor_sync(0xFFFFFFFFu, acc, 4);
    if (p < nb && sub == 0) {
      const float v = acc * scale;
      out[p] = v;
      if (fine_out_row) fine_out_row[j] = v;
    }
  }
}

// Candidate positions of one list whose ordered score is at or before the
// threshold, as bits by block index.
__device__ __forceinline__ void mark_selected(const float* cand, const int* list, int nb, int G,
                                              Threshold t, bool flip, uint32_t* bits) {
  for (int p = lane_id(); p < nb; p += 32) {
    if (before_or_at(ordered_bits(cand[p]), p, t, flip)) {
      const int j = cand_block(list, p, G);
      atomicOr(&bits[j >> 5], 1u << (j & 31));
    }
  }
}

// One warp per query-block row, `rows` rows per CTA (blockDim = 32 * rows).
// KPL: entries per lane in the selections (TG, cap_hi, cap_lo <= 32 * KPL).
template <int D, int KPL>
__global__ void __launch_bounds__(256) hier_classify_kernel(const HierArgs a) {
  extern __shared__ __align__(16) float smem[];
  constexpr int kStride = D + 4;
  const int T = a.T, TG = a.TG, G = a.G, rows = a.rows;
  const bool compute = a.fine_in == nullptr;
  float* sq = smem;                                  // [rows][D]
  float* sk = sq + rows * D;                         // [32][D+4]
  float* wbase = compute ? sk + kKTile * kStride : smem;
  const int bh = blockIdx.y, warp = threadIdx.x / 32, lane = lane_id();
  const int i = blockIdx.x * rows + warp;
  const bool row_ok = i < T;
  const int W = (T + 31) / 32;
  float* crow = wbase + size_t(warp) * hier_warp_words(T, TG, a.cap_hi, a.cap_lo, a.c_hi, a.c_lo);
  float* cand = crow + TG;                           // [cap_hi] then [cap_lo]
  int* list_hi = reinterpret_cast<int*>(cand + a.cap_hi + a.cap_lo);
  int* list_lo = list_hi + a.c_hi;
  uint32_t* bits_c = reinterpret_cast<uint32_t*>(list_lo + a.c_lo);
  uint32_t* bits_n = bits_c + W;
  uint32_t* scratch = bits_n + W;  // 64 words for the selections

  // ---- coarse scores sc_iJ (all warps take part in the staging)
  if (a.coarse_in == nullptr) {
    for (int e = threadIdx.x; e < rows * D; e += blockDim.x) {
      const int r = e / D, f = e % D, ii = blockIdx.x * rows + r;
      sq[e] = ii < T ? a.qbar[(size_t(bh) * T + ii) * D + f] : 0.f;
    }
    for (int J0 = 0; J0 < TG; J0 += kKTile) {
      __syncthreads();
      for (int e = threadIdx.x; e < kKTile * D; e += blockDim.x) {
        const int r = e / D, f = e % D, JJ = J0 + r;
        sk[r * kStride + f] = JJ < TG ? a.kc[(size_t(bh) * TG + JJ) * D + f] : 0.f;
      }
      __syncthreads();
      const float4* qa = reinterpret_cast<const float4*>(sq + warp * D);
      const float4* ka = reinterpret_cast<const float4*>(sk + lane * kStride);
      float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 8
      for (int a4 = 0; a4 < D / 4; a4 += 2) {
        const float4 x0 = qa[a4], y0 = ka[a4], x1 = qa[a4 + 1], y1 = ka[a4 + 1];
        acc0 = fmaf(x0.x, y0.x, acc0); acc0 = fmaf(x0.y, y0.y, acc0);
        acc0 = fmaf(x0.z, y0.z, acc0); acc0 = fmaf(x0.w, y0.w, acc0);
        acc1 = fmaf(x1.x, y1.x, acc1); acc1 = fmaf(x1.y, y1.y, acc1);
        acc1 = fmaf(x1.z, y1.z, acc1); acc1 = fmaf(x1.w, y1.w, acc1);
      }
      if (row_ok && J0 + lane < TG) crow[J0 + lane] = (acc0 + acc1) * a.scale;
    }
    __syncwarp();
    if (row_ok && a.coarse_out)
      for (int J = lane; J < TG; J += 32) a.coarse_out[(size_t(bh) * T + i) * TG + J] = crow[J];
  } else if (row_ok) {
    for (int J = lane; J < TG; J += 32) crow[J] = a.coarse_in[(size_t(bh) * T + i) * TG + J];
  }
  __syncwarp();
  if (!row_ok) return;

  // ---- candidate super-blocks, ascending
  const Threshold thc =
      a.c_hi > 0 ? select_side<KPL>(crow, TG, a.c_hi, false, scratch) : Threshold{0, -1};
  const Threshold tlc =
      a.c_lo > 0 ? select_side<KPL>(crow, TG, a.c_lo, true, scratch) : Threshold{0, -1};
  int nh = 0, nl = 0;
  for (int J0 = 0; J0 < TG; J0 += 32) {
    const int J = J0 + lane;
    bool hi = false, lo = false;
    if (J < TG) {
      const uint32_t o = ordered_bits(crow[J]);
      hi = a.c_hi > 0 && before_or_at(o, J, thc, false);
      lo = a.c_lo > 0 && before_or_at(o, J, tlc, true);
    }
    const uint32_t mh = __ballot_sync(0xFFFFFFFFu, hi), ml = __ballot_sync(0xFFFFFFFFu, lo);
    const uint32_t below = (1u << lane) - 1u;
    if (hi) {
      const int pos = nh + __popc(mh & below);
      if (pos < a.c_hi) list_hi[pos] = J;
    }
    if (lo) {
      const int pos = nl + __popc(ml & below);
      if (pos < a.c_lo) list_lo[pos] = J;
    }
    nh += __popc(mh);
    nl += __popc(ml);
  }
  for (int w = lane; w < 2 * W; w += 32) bits_c[w] = 0u;
  __syncwarp();
  if (nh != a.c_hi || nl != a.c_lo) {  // the selection is exact: cannot happen
    if (lane == 0) set_error(a.err, SLA_ERR_DEVICE);
    return;
  }
  const int tail = TG * G - T;  // missing blocks of the last super-block
  const int nb_hi = a.c_hi == 0 ? 0 : a.c_hi * G - (list_hi[a.c_hi - 1] == TG - 1 ? tail : 0);
  const int nb_lo = a.c_lo == 0 ? 0 : a.c_lo * G - (list_lo[a.c_lo - 1] == TG - 1 ? tail : 0);
  if (a.n_crit > nb_hi || a.n_negl > nb_lo) {  // the host's counts rule this out
    if (lane == 0) set_error(a.err, SLA_ERR_DEVICE);
    return;
  }

  // ---- fine scores of the candidate blocks only
  float* cand_lo = cand + a.cap_hi;
  if (compute) {
    const float* qrow = sq + warp * D;
    const float* kb = a.kbar + size_t(bh) * T * D;
    float* fo = a.fine_out ? a.fine_out + (size_t(bh) * T + i) * T : nullptr;
    fine_scores<D>(qrow, kb, list_hi, nb_hi, G, a.scale, cand, fo);
    fine_scores<D>(qrow, kb, list_lo, nb_lo, G, a.scale, cand_lo, fo);
  } else {
    const float* fr = a.fine_in + (size_t(bh) * T + i) * T;
    for (int p = lane; p < nb_hi; p += 32) cand[p] = fr[cand_block(list_hi, p, G)];
    for (int p = lane; p < nb_lo; p += 32) cand_lo[p] = fr[cand_block(list_lo, p, G)];
  }
  __syncwarp();

  // ---- exact selection inside the candidates (position order = block order)
  if (a.n_crit > 0) {
    const Threshold th = select_side<KPL>(cand, nb_hi, a.n_crit, false, scratch);
    mark_selected(cand, list_hi, nb_hi, G, th, false, bits_c);
  }
  if (a.n_negl > 0) {
    const Threshold tl = select_side<KPL>(cand_lo, nb_lo, a.n_negl, true, scratch);
    mark_selected(cand_lo, list_lo, nb_lo, G, tl, true, bits_n);
  }
  __syncwarp();

  // ---- outputs, as the flat kernel writes them
  const size_t rbase = size_t(bh) * T + i;
  int8_t* crw = a.cls + rbase * T;
  int32_t* idx = a.crit_idx + rbase * a.n_crit;
  uint32_t* mrow = a.marg_bits + rbase * W;
  int written = 0;
  for (int w = 0; w < W; ++w) {
    const int j = w * 32 + lane;
    const uint32_t bc = bits_c[w], bn = bits_n[w];
    const bool in = j < T;
    const bool c = (bc >> lane) & 1u, n = (bn >> lane) & 1u;
    if (in) crw[j] = int8_t(c ? 1 : (n ? -1 : 0));
    if (c) {
      const int pos = written + __popc(bc & ((1u << lane) - 1u));
      if (pos < a.n_crit) idx[pos] = j;
    }
    written += __popc(bc);
    if (lane == 0) {
      const uint32_t valid = (T - w * 32) >= 32 ? 0xFFFFFFFFu : ((1u << (T - w * 32)) - 1u);
      mrow[w] = ~(bc | bn) & valid;
    }
  }
}

// ------------------------------------------------------------------ column CSR
// For every key block j the ascending list of query blocks i with
// cls[i][j] == +1 (offsets relative to the head), in three launches:
//   csr_count_kernel  count -> col_ptr[j+1]
//   csr_scan_kernel   one CTA per head: inclusive scan of col_ptr[1..T] in place
//   csr_fill_kernel   rows in ascending order
// Count and fill: one CTA per 32 key blocks, lane = key block, so each row
// step is one coalesced 32-byte read of cls; warp w scans the contiguous row
// range [w*T/8, (w+1)*T/8), and the fill offsets each warp by the hits of the
// warps before it, which keeps every column's list ascending.
constexpr int kCsrWarps = 8;

__device__ __forceinline__ int csr_count_rows(const int8_t* c, int T, int i0, int i1) {
  int cnt = 0;
#pragma unroll 8
  for (int i = i0; i < i1; ++i) cnt += c[size_t(i) * T] == 1;
  return cnt;
}

__global__ void __launch_bounds__(256) csr_count_kernel(const int8_t* __restrict__ cls,
                                                        int32_t* __restrict__ col_ptr, int T) {
  __shared__ int part[kCsrWarps][32];
  const int bh = blockIdx.y, w = threadIdx.x / 32, lane = lane_id();
  const int j = blockIdx.x * 32 + lane;
  const int i0 = w * T / kCsrWarps, i1 = (w + 1) * T / kCsrWarps;
  part[w][lane] = j < T ? csr_count_rows(cls + size_t(bh) * T * T + j, T, i0, i1) : 0;
  __syncthreads();
  if (w == 0 && j < T) {
    int cnt = 0;
#pragma unroll
    for (int x = 0; x < kCsrWarps; ++x) cnt += part[x][lane];
    col_ptr[size_t(bh) * (T + 1) + j + 1] = cnt;
  }
}

__global__ void __launch_bounds__(1024) csr_scan_kernel(int32_t* __restrict__ col_ptr, int T) {
  __shared__ int wsum[32];
  __shared__ int carry;
  int32_t* ptr = col_ptr + size_t(blockIdx.x) * (T + 1);
  if (threadIdx.x == 0) {
    carry = 0;
    ptr[0] = 0;
  }
  __syncthreads();
  for (int j0 = 1; j0 <= T; j0 += blockDim.x) {
    const int j = j0 + threadIdx.x;
    const int v = j <= T ? ptr[j] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
      if (lane_id() >= o) x += y;
    }
    if (lane_id() == 31) wsum[threadIdx.x / 32] = x;
    __syncthreads();
    if (threadIdx.x < 32) {
      int s = wsum[threadIdx.x];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, s, o);
        if (lane_id() >= o) s += y;
      }
      wsum[threadIdx.x] = s;  // inclusive over warps
    }
    __syncthreads();
    const int warp_off = threadIdx.x >= 32 ? wsum[threadIdx.x / 32 - 1] : 0;
    if (j <= T) ptr[j] = carry + warp_off + x;
    __syncthreads();
    if (threadIdx.x == 0) carry += wsum[31];
    __syncthreads();
  }
}

__global__ void __launch_bounds__(256) csr_fill_kernel(const int8_t* __restrict__ cls,
                                                       const int32_t* __restrict__ col_ptr,
                                                       int32_t* __restrict__ col_idx, int T,
                                                       int n_crit) {
  __shared__ int part[kCsrWarps][32];
  const int bh = blockIdx.y, w = threadIdx.x / 32, lane = lane_id();
  const int j = blockIdx.x * 32 + lane;
  const int i0 = w * T / kCsrWarps, i1 = (w + 1) * T / kCsrWarps;
  const int8_t* c = cls + size_t(bh) * T * T + j;
  part[w][lane] = j < T ? csr_count_rows(c, T, i0, i1) : 0;
  __syncthreads();
  if (j >= T) return;
  int pos = col_ptr[size_t(bh) * (T + 1) + j];
  for (int x = 0; x < w; ++x) pos += part[x][lane];
  int32_t* out = col_idx + size_t(bh) * T * n_crit;
  const int cap = T * n_crit;
#pragma unroll 8
  for (int i = i0; i < i1; ++i) {
    if (c[size_t(i) * T] == 1) {
      if (pos < cap) out[pos] = i;
      ++pos;
    }
  }
}

// ------------------------------------------------------------------ marginal matrix
// bf16 0/1 matrix of marginal pairs, [BH][Tp][Tp] zero-padded, and its
// transpose; the operands of the aggregation GEMMs.  One thread writes 8
// consecutive columns (16 bytes) of one row.
__global__ void __launch_bounds__(256) expand_marginal_kernel(const uint32_t* __restrict__ marg_bits,
                                                              __nv_bfloat16* __restrict__ mmat,
                                                              __nv_bfloat16* __restrict__ mmat_t,
                                                              int T, int Tp) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;  // 8-column group of the whole head
  const int per_row = Tp / 8;
  if (e >= Tp * per_row) return;
  const int r = e / per_row, c0 = (e % per_row) * 8;
  const int words = (T + 31) / 32;
  const uint32_t* mb = marg_bits + size_t(bh) * T * words;
  constexpr uint32_t kOne = 0x3F80u;  // bf16 1.0
  const size_t o = (size_t(bh) * Tp + r) * Tp + c0;
  if (mmat) {
    uint32_t bits = 0;  // bit u: column c0 + u is marginal in row r
    if (r < T && c0 < T) {
      bits = (mb[size_t(r) * words + c0 / 32] >> (c0 % 32)) & 0xFFu;
      if (T - c0 < 8) bits &= (1u << (T - c0)) - 1u;
    }
    uint32_t w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      w[u] = ((bits >> (2 * u)) & 1u ? kOne : 0u) | ((bits >> (2 * u + 1)) & 1u ? kOne << 16 : 0u);
    *reinterpret_cast<uint4*>(mmat + o) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (mmat_t) {  // row r of the transpose = column r of the matrix
    uint32_t bits = 0;
    if (r < T) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = c0 + u;
        if (c < T) bits |= ((mb[size_t(c) * words + r / 32] >> (r % 32)) & 1u) << u;
      }
    }
    uint32_t w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      w[u] = ((bits >> (2 * u)) & 1u ? kOne : 0u) | ((bits >> (2 * u + 1)) & 1u ? kOne << 16 : 0u);
    *reinterpret_cast<uint4*>(mmat_t + o) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace

cudaError_t launch_pool(const Problem& p, const void* q, const void* k, float* qbar,
                        float* kbar, cudaStream_t s) {
  dim3 grid(p.T, p.BH);
  if (p.d == 128)
    pool_kernel<128><<<grid, 128, 0, s>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                          qbar, kbar, p.N, p.T, p.nv);
  else
    pool_kernel<64><<<grid, 128, 0, s>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                         qbar, kbar, p.N, p.T, p.nv);
  return cudaGetLastError();
}

// Scores per lane of a warp's selection (a row of up to 32 * KPL entries):
// the smallest instantiated KPL that holds n entries.
int kpl_for(int n) {
  for (int k : {4, 8, 16, 24, 40, 64, 128})
    if (32 * k >= n) return k;
  return 0;
}

#define SLA_KPL_SWITCH(kpl, CALL)                 \
  switch (kpl) {                                  \
    case 4: return CALL(4);                       \
    case 8: return CALL(8);                       \
    case 16: return CALL(16);                     \
    case 24: return CALL(24);                     \
    case 40: return CALL(40);                     \
    case 64: return CALL(64);                     \
    case 128: return CALL(128);                   \
    default: return cudaErrorInvalidValue;        \
  }

template <int D, int KPL>
cudaError_t launch_classify_t(const Problem& p, size_t smem, const float* qbar, const float* kbar,
                              const float* logits_in, float* logits_out, int8_t* cls,
                              int32_t* crit_idx, uint32_t* marg_bits, cudaStream_t s) {
  const cudaError_t e = cudaFuncSetAttribute(
      classify_kernel<D, KPL>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((p.T + kRowsPerCta - 1) / kRowsPerCta, p.BH);
  classify_kernel<D, KPL><<<grid, 256, smem, s>>>(qbar, kbar, logits_in, logits_out, cls,
                                                  crit_idx, marg_bits, p.T, p.n_crit, p.n_negl,
                                                  p.scale);
  return cudaGetLastError();
}

cudaError_t launch_classify(const Problem& p, const float* qbar, const float* kbar,
                            const float* logits_in, float* logits_out, int8_t* cls,
                            int32_t* crit_idx, uint32_t* marg_bits, cudaStream_t s) {
  const size_t smem = sizeof(float) * (size_t(kRowsPerCta) * p.T + kRowsPerCta * (p.d + 4) +
                                       2 * size_t(kSBuf) + kRowsPerCta * 64);
#define SLA_FLAT(K)                                                                         \
  (p.d == 128 ? launch_classify_t<128, K>(p, smem, qbar, kbar, logits_in, logits_out, cls, \
                                          crit_idx, marg_bits, s)                          \
              : launch_classify_t<64, K>(p, smem, qbar, kbar, logits_in, logits_out, cls,  \
                                         crit_idx, marg_bits, s))
  SLA_KPL_SWITCH(kpl_for(p.T), SLA_FLAT)
#undef SLA_FLAT
}

cudaError_t launch_coarse_keys(const Problem& p, const float* kbar, float* kc, int G,
                               cudaStream_t s) {
  const int TG = (p.T + G - 1) / G;
  coarse_keys_kernel<<<dim3(TG, p.BH), p.d, 0, s>>>(kbar, kc, p.T, TG, G, p.d);
  return cudaGetLastError();
}

size_t hier_smem_bytes(const Problem& p, const HierCounts& h, bool compute, int rows) {
  const int cap_hi = std::min(h.c_hi * h.G, p.T), cap_lo = std::min(h.c_lo * h.G, p.T);
  size_t words = size_t(rows) * hier_warp_words(p.T, h.TG, cap_hi, cap_lo, h.c_hi, h.c_lo);
  if (compute) words += size_t(rows) * p.d + size_t(kKTile) * (p.d + 4);
  return words * 4;
}

template <int D, int KPL>
cudaError_t launch_hier_t(const HierArgs& a, cudaStream_t s) {
  const cudaError_t e = cudaFuncSetAttribute(
      hier_classify_kernel<D, KPL>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(a.smem));
  if (e != cudaSuccess) return e;
  dim3 grid((a.T + a.rows - 1) / a.rows, a.BH);
  hier_classify_kernel<D, KPL><<<grid, 32 * a.rows, a.smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_hier_classify(const Problem& p, const HierCounts& h, const float* qbar,
                                 const float* kbar, const float* kc, const float* fine_in,
                                 const float* coarse_in, float* fine_out, float* coarse_out,
                                 int8_t* cls, int32_t* crit_idx, uint32_t* marg_bits, int* err,
                                 cudaStream_t s) {
  const bool compute = fine_in == nullptr;
  int rows = 8;
  while (rows > 1 && hier_smem_bytes(p, h, compute, rows) > kMaxSmemPerCta) rows /= 2;
  const size_t smem = hier_smem_bytes(p, h, compute, rows);
  if (smem > kMaxSmemPerCta) return cudaErrorInvalidConfiguration;
  HierArgs a;
  a.qbar = qbar; a.kbar = kbar; a.kc = kc; a.fine_in = fine_in; a.coarse_in = coarse_in;
  a.fine_out = fine_out; a.coarse_out = coarse_out;
  a.cls = cls; a.crit_idx = crit_idx; a.marg_bits = marg_bits; a.err = err;
  a.T = p.T; a.TG = h.TG; a.G = h.G; a.c_hi = h.c_hi; a.c_lo = h.c_lo;
  a.cap_hi = std::min(h.c_hi * h.G, p.T); a.cap_lo = std::min(h.c_lo * h.G, p.T);
  a.n_crit = p.n_crit; a.n_negl = p.n_negl; a.rows = rows; a.scale = p.scale; a.BH = p.BH;
  a.smem = smem;
#define SLA_HIER(K) (p.d == 128 ? launch_hier_t<128, K>(a, s) : launch_hier_t<64, K>(a, s))
  SLA_KPL_SWITCH(kpl_for(std::max(h.TG, std::max(a.cap_hi, a.cap_lo))), SLA_HIER)
#undef SLA_HIER
}

cudaError_t launch_crit_csr(const Problem& p, const int8_t* cls, int32_t* col_ptr,
                            int32_t* col_idx, cudaStream_t s) {
  dim3 grid((p.T + 31) / 32, p.BH);
  csr_count_kernel<<<grid, 32 * kCsrWarps, 0, s>>>(cls, col_ptr, p.T);
  csr_scan_kernel<<<p.BH, 1024, 0, s>>>(col_ptr, p.T);
  if (p.n_crit > 0) csr_fill_kernel<<<grid, 32 * kCsrWarps, 0, s>>>(cls, col_ptr, col_idx, p.T, p.n_crit);
  return cudaGetLastError();
}

cudaError_t launch_expand_marginal(const Problem& p, const uint32_t* marg_bits,
                                   __nv_bfloat16* mmat, __nv_bfloat16* mmat_t, cudaStream_t s) {
  dim3 grid((p.Tp * (p.Tp / 8) + 255) / 256, p.BH);
  expand_marginal_kernel<<<grid, 256, 0, s>>>(marg_bits, mmat, mmat_t, p.T, p.Tp);
  return cudaGetLastError();
}

}  // namespace sla
