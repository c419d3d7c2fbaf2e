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

// The n-th element (n >= 1) of one row in the order (score desc, index asc),
// or with `flip` in the reverse order (score asc, index desc), found by one
// warp: an exact radix select on the order-preserving 32-bit score (four
// 8-bit digits, most significant first, histogram in shared memory) followed
// by one pass that breaks ties by index.  Returns the element's (possibly
// complemented) ordered score v and its index jt; an element is at or before
// it in the order iff its value is > v, or == v with index <= jt (>= jt when
// flipped).
struct Threshold {
  uint32_t v;
  int jt;
};

__device__ Threshold warp_select(const float* row, int T, int n, bool flip, uint32_t* hist) {
  constexpr uint32_t kAll = 0xFFFFFFFFu;
  const int lane = lane_id();
  uint32_t prefix = 0, mask = 0;
  int need = n;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int j = lane; j < T; j += 32) {
      uint32_t o = ordered_bits(row[j]);
      if (flip) o = ~o;
      if ((o & mask) == prefix) atomicAdd(&hist[(o >> shift) & 255u], 1u);
    }
    __syncwarp();
    // lane l owns digits 255-8l down to 248-8l; scan from the top digit
    uint32_t c[8];
    int s = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      c[e] = hist[255 - 8 * lane - e];
      s += int(c[e]);
    }
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kAll, incl, o);
      if (lane >= o) incl += y;
    }
    const int excl = incl - s;
    const bool mine = excl < need && need <= incl;
    const int src = __ffs(__ballot_sync(kAll, mine)) - 1;
    int digit = 0, above = 0;
    if (mine) {
      int acc = excl;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (acc + int(c[e]) >= need) {
          digit = 255 - 8 * lane - e;
          above = acc;
          break;
        }
        acc += int(c[e]);
      }
    }
    digit = __shfl_sync(kAll, digit, src);
    above = __shfl_sync(kAll, above, src);
    prefix |= uint32_t(digit) << shift;
    mask |= 255u << shift;
    need -= above;
    __syncwarp();
  }
  // ties on the score: the need-th equal element in index order
  int jt = -1, seen = 0;
  const int last = ((T - 1) / 32) * 32;
  for (int step = 0; step <= last / 32 && jt < 0; ++step) {
    const int j0 = flip ? last - 32 * step : 32 * step;
    const int j = j0 + lane;
    bool eq = false;
    if (j < T) {
      uint32_t o = ordered_bits(row[j]);
      if (flip) o = ~o;
      eq = o == prefix;
    }
    uint32_t m = __ballot_sync(kAll, eq);
    const int cnt = __popc(m);
    if (seen + cnt >= need) {
      for (int k = need - seen; k > 1; --k) m &= flip ? ~(1u << (31 - __clz(m))) : (m - 1);
      jt = j0 + (flip ? 31 - __clz(m) : __ffs(m) - 1);
    }
    seen += cnt;
  }
  return {prefix, jt};
}

__device__ __forceinline__ bool before_or_at(uint32_t o, int j, Threshold t, bool flip) {
  if (flip) o = ~o;
  return o > t.v || (o == t.v && (flip ? j >= t.jt : j <= t.jt));
}

constexpr int kRowsPerCta = 8;  // one warp per query-block row
constexpr int kKTile = 32;      // pooled keys staged per step

// One CTA per 8 rows of one head.  When `logits_in` is null the pooled logits
// are computed from qbar/kbar (fp32), otherwise read from it.
template <int D>
__global__ void __launch_bounds__(256) classify_kernel(
    const float* __restrict__ qbar, const float* __restrict__ kbar,
    const float* __restrict__ logits_in, float* __restrict__ logits_out,
    int8_t* __restrict__ cls, int32_t* __restrict__ crit_idx, uint32_t* __restrict__ marg_bits,
    int T, int n_crit, int n_negl, float scale) {
  extern __shared__ __align__(16) float smem[];
  constexpr int kStride = D + 4;  // padded row of the staged pooled keys
  float* srow = smem;                                // [8][T]
  float* sq = srow + kRowsPerCta * T;                // [8][D]
  float* sk = sq + kRowsPerCta * D;                  // [32][D+4]
  const int bh = blockIdx.y, warp = threadIdx.x / 32, lane = lane_id();
  const int i = blockIdx.x * kRowsPerCta + warp;
  const bool row_ok = i < T;
  float* row = srow + warp * T;

  if (logits_in == nullptr) {
    for (int e = threadIdx.x; e < kRowsPerCta * D; e += blockDim.x) {
      const int r = e / D, a = e % D, ii = blockIdx.x * kRowsPerCta + r;
      sq[e] = ii < T ? qbar[(size_t(bh) * T + ii) * D + a] : 0.f;
    }
    for (int j0 = 0; j0 < T; j0 += kKTile) {
      __syncthreads();
      for (int e = threadIdx.x; e < kKTile * D; e += blockDim.x) {
        const int r = e / D, a = e % D, jj = j0 + r;
        sk[r * kStride + a] = jj < T ? kbar[(size_t(bh) * T + jj) * D + a] : 0.f;
      }
      __syncthreads();
      const int j = j0 + lane;
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
      if (j < T) row[j] = (acc0 + acc1) * scale;
    }
    __syncwarp();
    if (row_ok && logits_out) {
      for (int j = lane; j < T; j += 32) logits_out[(size_t(bh) * T + i) * T + j] = row[j];
    }
  } else {
    if (row_ok)
      for (int j = lane; j < T; j += 32) row[j] = logits_in[(size_t(bh) * T + i) * T + j];
    __syncwarp();
  }
  if (!row_ok) return;

  uint32_t* hist = reinterpret_cast<uint32_t*>(sk + kKTile * kStride) + warp * 256;
  const Threshold th = n_crit > 0 ? warp_select(row, T, n_crit, false, hist) : Threshold{0, -1};
  const Threshold tl = n_negl > 0 ? warp_select(row, T, n_negl, true, hist) : Threshold{0, -1};
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

// ------------------------------------------------------------------ column CSR
// For every key block j the ascending list of query blocks i with
// cls[i][j] == +1 (offsets relative to the head), in three launches:
//   csr_count_kernel  one warp per column: count -> col_ptr[j+1]
//   csr_scan_kernel   one CTA per head: inclusive scan of col_ptr[1..T] in place
//   csr_fill_kernel   one warp per column: rows in ascending order by ballots
constexpr int kCsrWarps = 8;

__global__ void __launch_bounds__(256) csr_count_kernel(const int8_t* __restrict__ cls,
                                                        int32_t* __restrict__ col_ptr, int T) {
  const int bh = blockIdx.y, j = blockIdx.x * kCsrWarps + threadIdx.x / 32, lane = lane_id();
  if (j >= T) return;
  const int8_t* c = cls + size_t(bh) * T * T + j;
  int cnt = 0;
#pragma unroll 4
  for (int i = lane; i < T; i += 32) cnt += c[size_t(i) * T] == 1;
  cnt = __reduce_add_sync(0xFFFFFFFFu, cnt);
  if (lane == 0) col_ptr[size_t(bh) * (T + 1) + j + 1] = cnt;
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
  const int bh = blockIdx.y, j = blockIdx.x * kCsrWarps + threadIdx.x / 32, lane = lane_id();
  if (j >= T) return;
  const int8_t* c = cls + size_t(bh) * T * T + j;
  int32_t* out = col_idx + size_t(bh) * T * n_crit;
  const int cap = T * n_crit;
  int pos = col_ptr[size_t(bh) * (T + 1) + j];
  for (int i0 = 0; i0 < T; i0 += 32) {
    const int i = i0 + lane;
    const bool hit = i < T && c[size_t(i) * T] == 1;
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, hit);
    const int at = pos + __popc(m & ((1u << lane) - 1u));
    if (hit && at < cap) out[at] = i;
    pos += __popc(m);
  }
}

// ------------------------------------------------------------------ marginal matrix
// bf16 0/1 matrix of marginal pairs, [BH][Tp][Tp] zero-padded, and its
// transpose; the operands of the aggregation GEMMs.
__global__ void expand_marginal_kernel(const uint32_t* __restrict__ marg_bits,
                                       __nv_bfloat16* __restrict__ mmat,
                                       __nv_bfloat16* __restrict__ mmat_t, int T, int Tp) {
  const int bh = blockIdx.z;
  const int r = blockIdx.y;                          // row of the output
  const int c = blockIdx.x * blockDim.x + threadIdx.x;  // column
  if (c >= Tp) return;
  const int words = (T + 31) / 32;
  const uint32_t* mb = marg_bits + size_t(bh) * T * words;
  const __nv_bfloat16 one = __float2bfloat16(1.0f), zero = __float2bfloat16(0.0f);
  const size_t o = (size_t(bh) * Tp + r) * Tp + c;
  if (mmat) {
    bool m = r < T && c < T && ((mb[size_t(r) * words + c / 32] >> (c % 32)) & 1u);
    mmat[o] = m ? one : zero;
  }
  if (mmat_t) {
    bool m = r < T && c < T && ((mb[size_t(c) * words + r / 32] >> (r % 32)) & 1u);
    mmat_t[o] = m ? one : zero;
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

cudaError_t launch_classify(const Problem& p, const float* qbar, const float* kbar,
                            const float* logits_in, float* logits_out, int8_t* cls,
                            int32_t* crit_idx, uint32_t* marg_bits, cudaStream_t s) {
  dim3 grid((p.T + kRowsPerCta - 1) / kRowsPerCta, p.BH);
  const size_t smem =
      sizeof(float) * (size_t(kRowsPerCta) * p.T + kRowsPerCta * p.d + kKTile * (p.d + 4)) +
      sizeof(uint32_t) * kRowsPerCta * 256;  // per-warp radix histograms
  cudaError_t e;
  if (p.d == 128) {
    e = cudaFuncSetAttribute(classify_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem));
    if (e != cudaSuccess) return e;
    classify_kernel<128><<<grid, 256, smem, s>>>(qbar, kbar, logits_in, logits_out, cls,
                                                 crit_idx, marg_bits, p.T, p.n_crit, p.n_negl,
                                                 p.scale);
  } else {
    e = cudaFuncSetAttribute(classify_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem));
    if (e != cudaSuccess) return e;
    classify_kernel<64><<<grid, 256, smem, s>>>(qbar, kbar, logits_in, logits_out, cls,
                                                crit_idx, marg_bits, p.T, p.n_crit, p.n_negl,
                                                p.scale);
  }
  return cudaGetLastError();
}

cudaError_t launch_crit_csr(const Problem& p, const int8_t* cls, int32_t* col_ptr,
                            int32_t* col_idx, cudaStream_t s) {
  dim3 grid((p.T + kCsrWarps - 1) / kCsrWarps, p.BH);
  csr_count_kernel<<<grid, 32 * kCsrWarps, 0, s>>>(cls, col_ptr, p.T);
  csr_scan_kernel<<<p.BH, 1024, 0, s>>>(col_ptr, p.T);
  if (p.n_crit > 0) csr_fill_kernel<<<grid, 32 * kCsrWarps, 0, s>>>(cls, col_ptr, col_idx, p.T, p.n_crit);
  return cudaGetLastError();
}

cudaError_t launch_expand_marginal(const Problem& p, const uint32_t* marg_bits,
                                   __nv_bfloat16* mmat, __nv_bfloat16* mmat_t, cudaStream_t s) {
  dim3 grid((p.Tp + 127) / 128, p.Tp, p.BH);
  expand_marginal_kernel<<<grid, 128, 0, s>>>(marg_bits, mmat, mmat_t, p.T, p.Tp);
  return cudaGetLastError();
}

}  // namespace sla
