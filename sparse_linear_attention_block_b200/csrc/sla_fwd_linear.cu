// Combination step of SLA's forward: O = O_s + O_l W_proj with the linear
// branch O_l = phi(Q) H_i / (phi(Q) . Z_i) of each query block i.
//
// SLA (arXiv 2509.24006), abstract / framework step 3 (marginal pairs use
// linear attention; its output is projected and added to the sparse output).
// H_i, Z_i are the aggregated per-block summaries, read as bf16 hi/lo planes
// (value = hi + lo) straight into tensor-core operand tiles by TMA.
//
// One CTA per query block (64 tokens), 128 threads, features on TMEM lanes
// and tokens on TMEM columns so that every product has M = 128 and each
// block meets only its own H_i:
//   NUM^T = H_i^T phi(Q)^T     (M = c, N = 64 tokens, K = a; H_hi + H_lo vs phi_hi)
//   den_t = phi(Q_t) . Z_i      (fp32, from the exact phi values at load time)
//   O_l^T = NUM^T / den         (bf16 hi + lo, an MN-major operand tile)
//   O^T   = W^T O_l^T           (A = W^T held in TMEM; W_proj is exact in bf16)
//   O     = O_s + g O           (bf16 out; den saved for the backward; g = 1
//                                  unless the branch is gated)
// Persistent: two CTAs per SM (96 KB shared memory, 256 TMEM columns each)
// walk the blocks; W^T goes to TMEM once per CTA, and the next block's H tile
// is requested as soon as NUM^T has consumed the current one, so the copy
// overlaps the rest of the block.  d = 64 pads the feature dimension of the
// tiles to 128 with zeros.
#include <cuda_bf16.h>

#include "sla_internal.h"
#include "sla_ptx.cuh"
#include "sla_tile.cuh"

namespace sla {
namespace {

constexpr int kFlH = 32768;  // one H plane tile: 2 chunks x 128 rows x 128 B
constexpr int kFlP = 16384;  // phi(Q) [64 t][a] tile, later O_l^T [c][64 t]
constexpr int kFlSmem = 1024 + 2 * kFlH + 2 * kFlP;

template <int D>
__global__ void __launch_bounds__(128) fwd_linear_kernel(
    const __grid_constant__ CUtensorMap tm_hh, const __grid_constant__ CUtensorMap tm_hl,
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ hz_hi,
    const __nv_bfloat16* __restrict__ hz_lo, const __nv_bfloat16* __restrict__ w_proj,
    const float* __restrict__ o_s, __nv_bfloat16* __restrict__ o, float* __restrict__ den_out,
    float gate, int N, int T, int nv, int nblk, int* err) {
  constexpr int W = D * D + D;
  constexpr int kU = D / 8;               // 16-byte units per token row
  constexpr int kRowsPerPass = 128 / kU;  // token rows covered by one pass of 128 threads
  constexpr int kPass = 64 / kRowsPerPass;
  constexpr uint32_t kNum = 0, kOut = 64, kWt = 128;  // TMEM columns
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = align_smem_1024(smem_raw);
  uint8_t* sHh = base;
  uint8_t* sHl = sHh + kFlH;
  uint8_t* sPh = sHl + kFlH;  // phi(Q) hi, then O_l^T hi (and W staging before either)
  uint8_t* sPl = sPh + kFlP;  // phi(Q) lo, then O_l^T lo
  __shared__ float sZ[D];
  __shared__ float sInv[64];
  __shared__ uint64_t bar_h, bar_n, bar_o;
  __shared__ uint32_t tmem_base;
  const int t = threadIdx.x, warp = t / 32;
  const bool lane_ok = warp * 32 < D;  // this warp's TMEM lanes hold a feature
  const uint32_t lane_base = uint32_t(warp * 32) << 16;
  auto tok_of = [&](int blk) { return size_t(blk / T) * N + size_t(blk % T) * 64; };

  if (warp == 0) tmem_alloc(&tmem_base, 256);
  if (t == 0) {
    mbar_init(&bar_h, 1);
    mbar_init(&bar_n, 1);
    mbar_init(&bar_o, 1);
    fence_barrier_init();
  }
  if (D == 64) {  // zero the padding of the H tiles (features 64..127)
    for (int e = t; e < (kFlH - 8192) / 16; e += 128) {
      reinterpret_cast<uint4*>(sHh + 8192)[e] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(sHl + 8192)[e] = make_uint4(0, 0, 0, 0);
    }
  }
  for (int e = t; e < D * D / 8; e += 128)  // W_proj staging copy, row-major
    reinterpret_cast<uint4*>(sPh)[e] = __ldg(reinterpret_cast<const uint4*>(w_proj) + e);
  fence_proxy_async_smem();  // the padding zeros vs the H tiles' TMA writes
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  auto request_h = [&](int blk) {  // one thread: both planes of block blk's H tile
    mbar_arrive_expect_tx(&bar_h, 2 * D * D * 2);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d(sHh + c * 16384, &bar_h, &tm_hh, c * 64, 0, blk);
      tma_load_3d(sHl + c * 16384, &bar_h, &tm_hl, c * 64, 0, blk);
    }
  };
  if (t == 0) {
    tma_prefetch_desc(&tm_hh);
    tma_prefetch_desc(&tm_hl);
    request_h(blockIdx.x);
  }
  // W^T into TMEM: lane c' holds W[c][c'] for all c, packed in pairs along c
  if (lane_ok) {
    const __nv_bfloat16* sw = reinterpret_cast<const __nv_bfloat16*>(sPh);
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const uint32_t lo = __bfloat16_as_ushort(sw[(c0 + 2 * e) * D + t]);
        const uint32_t hi = __bfloat16_as_ushort(sw[(c0 + 2 * e + 1) * D + t]);
        pk[e] = lo | (hi << 16);
      }
      tmem_st16(tmem + lane_base + kWt + c0 / 2, pk);
    }
  }
  tmem_st_wait();
  // the first block's Q (registers) and Z_i (hi + lo)
  const int u = t % kU, r0 = t / kU;
  uint4 qv[kPass];
  auto load_q = [&](int blk) {
    const size_t tk = tok_of(blk);
#pragma unroll
    for (int b = 0; b < kPass; ++b)
      qv[b] = __ldg(reinterpret_cast<const uint4*>(q + (tk + r0 + b * kRowsPerPass) * D) + u);
  };
  auto load_z = [&](int blk) {
    if (t < D)
      sZ[t] = __bfloat162float(hz_hi[size_t(blk) * W + D * D + t]) +
              __bfloat162float(hz_lo[size_t(blk) * W + D * D + t]);
  };
  load_q(blockIdx.x);
  load_z(blockIdx.x);
  __syncthreads();  // W staging read; sZ written
  bool ok = true;
  int k = 0;
  for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x, ++k) {
    const size_t tok0 = tok_of(blk);
    const int nxt = blk + int(gridDim.x);
    const int vrows = nv - (blk % T) * 64;  // rows of this block that exist (key padding)
    if (t == 0 && nxt < nblk) {  // the next block's Q and O_s rows into L2 meanwhile
      bulk_prefetch_l2(q + tok_of(nxt) * D, 64 * D * 2);
      bulk_prefetch_l2(o_s + tok_of(nxt) * D, 64 * D * 4);
    }
    // phi(Q) as hi/lo K-major tiles [64 t][a]; den_t = phi(Q_t) . Z_i in fp32,
    // each thread's 8 features summed, then over the kU threads of a row
#pragma unroll
    for (int b = 0; b < kPass; ++b) {
      const int rr = r0 + b * kRowsPerPass;
      const uint32_t w4[4] = {qv[b].x, qv[b].y, qv[b].z, qv[b].w};
      uint32_t h[4], l[4];
      float part = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = phi_f(bf16_lo(w4[e])), x1 = phi_f(bf16_hi(w4[e]));
        part = fmaf(x0, sZ[8 * u + 2 * e], fmaf(x1, sZ[8 * u + 2 * e + 1], part));
        split2(x0, x1, h[e], l[e]);
      }
      st_sw128_unit(sPh, 64, rr, 8 * u, make_uint4(h[0], h[1], h[2], h[3]));
      st_sw128_unit(sPl, 64, rr, 8 * u, make_uint4(l[0], l[1], l[2], l[3]));
#pragma unroll
      for (int m = kU / 2; m >= 1; m >>= 1) part += __shfl_xor_sync(0xffffffffu, part, m);
      if (u == 0) {
        // a padded query row (key padding) has no linear output: den = 0
        const float dn = rr < vrows ? part : 0.f;
        sInv[rr] = dn > 0.f ? 1.0f / dn : 0.f;
        den_out[tok0 + rr] = dn;
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // NUM^T = (H_hi + H_lo)^T phi_hi^T
    if (t == 0) {
      ok = mbar_wait(&bar_h, k & 1, err, nullptr);
      if (ok) {
        tc_fence_after();
        constexpr uint32_t id = idesc_bf16(128, 64, 1, 0);
        const uint64_t ah = desc_mnmajor_base(smem_u32(sHh), 128);
        const uint64_t al = desc_mnmajor_base(smem_u32(sHl), 128);
        const uint64_t bp = desc_kmajor_base(smem_u32(sPh));
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t bk = desc_advance(bp, kmajor_step_bytes(64, ks));
          mma_ss(tmem + kNum, desc_advance(ah, mnmajor_step_bytes(ks)), bk, id, ks > 0);
          mma_ss(tmem + kNum, desc_advance(al, mnmajor_step_bytes(ks)), bk, id, 1);
        }
      } else {
        mbar_wait(&bar_h, k & 1, nullptr, nullptr);  // let an in-flight copy land
      }
      mma_commit(&bar_n);  // arrives even when nothing was issued
    }
    ok = mbar_wait(&bar_n, k & 1, err, nullptr) && ok;
    tc_fence_after();
    if (__syncthreads_or(!ok)) break;  // CTA-uniform exit; no copy is in flight
    if (t == 0 && nxt < nblk) request_h(nxt);  // the H tiles are free again
    // O_l^T = NUM^T / den, as hi/lo MN-major tiles [c][64 t] (one 128-byte row per lane)
    if (lane_ok) {
      float v[64];
      tmem_ld32(tmem + lane_base + kNum, reinterpret_cast<float(&)[32]>(v[0]));
      tmem_ld32(tmem + lane_base + kNum + 32, reinterpret_cast<float(&)[32]>(v[32]));
      tmem_ld_wait();
#pragma unroll
      for (int k8 = 0; k8 < 8; ++k8) {
        uint32_t h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tt = 8 * k8 + 2 * e;
          split2(v[tt] * sInv[tt], v[tt + 1] * sInv[tt + 1], h[e], l[e]);
        }
        st_sw128_unit(sPh, 128, t, 8 * k8, make_uint4(h[0], h[1], h[2], h[3]));
        st_sw128_unit(sPl, 128, t, 8 * k8, make_uint4(l[0], l[1], l[2], l[3]));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (t == 0) {  // O^T = W^T (O_l,hi + O_l,lo)^T
      constexpr uint32_t id = idesc_bf16(128, 64, 0, 1);
      const uint64_t bh_ = desc_mnmajor_base(smem_u32(sPh), 128);
      const uint64_t bl_ = desc_mnmajor_base(smem_u32(sPl), 128);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        mma_ts(tmem + kOut, tmem + kWt + ks * 8, desc_advance(bh_, mnmajor_step_bytes(ks)), id,
               ks > 0);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        mma_ts(tmem + kOut, tmem + kWt + ks * 8, desc_advance(bl_, mnmajor_step_bytes(ks)), id, 1);
      mma_commit(&bar_o);
    }
    // while it runs: the next block's Q and Z_i, this block's O_s
    if (nxt < nblk) {
      load_q(nxt);
      load_z(nxt);  // sZ was last read by this block's den
    }
    float os[64];  // all 64 tokens' loads in flight at once
    if (lane_ok) {
#pragma unroll
      for (int j = 0; j < 64; ++j) os[j] = __ldg(o_s + (tok0 + j) * D + t);
    }
    ok = mbar_wait(&bar_o, k & 1, err, nullptr);
    tc_fence_after();
    // O = O_s + O^T (lane = output feature c', 64 tokens), bf16
    if (lane_ok) {
#pragma unroll
      for (int t0 = 0; t0 < 64; t0 += 32) {
        float v[32];
        tmem_ld32(tmem + lane_base + kOut + t0, v);
        tmem_ld_wait();
        if (ok) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            o[(tok0 + t0 + j) * D + t] = __float2bfloat16_rn(fmaf(gate, v[j], os[t0 + j]));
        }
      }
    }
    tc_fence_before();
    if (__syncthreads_or(!ok)) {  // an unfinished product: drain the pending H copy
      if (t == 0 && nxt < nblk) mbar_wait(&bar_h, (k + 1) & 1, nullptr, nullptr);
      break;
    }
    tc_fence_after();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free(tmem, 256);
}
// O = bf16(O_s): the forward's output when the linear branch is dropped.
__global__ void __launch_bounds__(256) os_to_o_kernel(const float4* __restrict__ o_s,
                                                      uint2* __restrict__ o, size_t n4) {
  for (size_t e = blockIdx.x * size_t(256) + threadIdx.x; e < n4; e += size_t(gridDim.x) * 256) {
    const float4 x = __ldg(o_s + e);
    o[e] = make_uint2(pack_bf16(x.x, x.y), pack_bf16(x.z, x.w));
  }
}

}  // namespace

cudaError_t launch_os_to_o(const Problem& p, const float* o_s, void* o, cudaStream_t s) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cudaErrorInvalidValue;
  const size_t n4 = size_t(p.BH) * p.N * p.d / 4;
  os_to_o_kernel<<<4 * sms, 256, 0, s>>>(reinterpret_cast<const float4*>(o_s),
                                         reinterpret_cast<uint2*>(o), n4);
  return cudaGetLastError();
}

cudaError_t launch_fwd_linear(const Problem& p, const void* q, const __nv_bfloat16* hz_hi,
                              const __nv_bfloat16* hz_lo, const void* w_proj, const float* o_s,
                              void* o, float* den, float gate, int* err, cudaStream_t s) {
  CUtensorMap th, tl;
  if (!make_tmap_summary(&th, hz_hi, p.BH * p.T, p.d)) return cudaErrorInvalidValue;
  if (!make_tmap_summary(&tl, hz_lo, p.BH * p.T, p.d)) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cudaErrorInvalidValue;
  const int nblk = p.BH * p.T;
  const int grid = nblk < 2 * sms ? nblk : 2 * sms;
  cudaError_t e;
  if (p.d == 128) {
    e = cudaFuncSetAttribute(fwd_linear_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kFlSmem);
    if (e != cudaSuccess) return e;
    fwd_linear_kernel<128><<<grid, 128, kFlSmem, s>>>(
        th, tl, (const __nv_bfloat16*)q, hz_hi, hz_lo, (const __nv_bfloat16*)w_proj, o_s,
        (__nv_bfloat16*)o, den, gate, p.N, p.T, p.nv, nblk, err);
  } else {
    e = cudaFuncSetAttribute(fwd_linear_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kFlSmem);
    if (e != cudaSuccess) return e;
    fwd_linear_kernel<64><<<grid, 128, kFlSmem, s>>>(
        th, tl, (const __nv_bfloat16*)q, hz_hi, hz_lo, (const __nv_bfloat16*)w_proj, o_s,
        (__nv_bfloat16*)o, den, gate, p.N, p.T, p.nv, nblk, err);
  }
  return cudaGetLastError();
}

}  // namespace sla
