// Warp-parallel sorted union of two block-index lists, used by the sparse
// kernels to walk the critical blocks of a pair of rows (forward) or columns
// (backward) in one pass.
#pragma once

#include <cstdint>

#include "sla_ptx.cuh"

namespace sla {

// One warp.  a[0..na) and b[0..nb) hold block indices (global memory, any
// order, no repeats within a list); values outside [0, T) set SLA_ERR_DEVICE
// in *err and are dropped.  Writes the union in ascending order to idx[] with
// flag[] bit 0 = member of a, bit 1 = member of b, and returns its length
// (the same value in every lane).  bits: 2 * ceil(T/32) words of shared
// scratch.  The caller orders the results for other warps (__syncthreads).
__device__ __forceinline__ int warp_union(const int32_t* a, int na, const int32_t* b, int nb,
                                          int T, uint32_t* bits, uint16_t* idx, uint8_t* flag,
                                          int* err) {
  const int lane = int(lane_id());
  const int nw = (T + 31) / 32;
  uint32_t* ba = bits;
  uint32_t* bb = bits + nw;
  for (int w = lane; w < 2 * nw; w += 32) bits[w] = 0u;
  __syncwarp();
  bool bad = false;
  for (int x = lane; x < na; x += 32) {
    const int v = a[x];
    if (v < 0 || v >= T) bad = true;
    else atomicOr(&ba[v >> 5], 1u << (v & 31));
  }
  for (int x = lane; x < nb; x += 32) {
    const int v = b[x];
    if (v < 0 || v >= T) bad = true;
    else atomicOr(&bb[v >> 5], 1u << (v & 31));
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_error(err, SLA_ERR_DEVICE);
  __syncwarp();
  int base = 0;
  for (int w0 = 0; w0 < nw; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t ua = w < nw ? ba[w] : 0u, ub = w < nw ? bb[w] : 0u;
    uint32_t uu = ua | ub;
    const int cnt = __popc(uu);
    int incl = cnt;  // inclusive prefix sum of the counts over the lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = base + incl - cnt;
    while (uu) {
      const int bit = __ffs(int(uu)) - 1;
      idx[pos] = uint16_t(w * 32 + bit);
      flag[pos] = uint8_t(((ua >> bit) & 1u) | (((ub >> bit) & 1u) << 1));
      ++pos;
      uu &= uu - 1u;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  return base;
}

}  // namespace sla
