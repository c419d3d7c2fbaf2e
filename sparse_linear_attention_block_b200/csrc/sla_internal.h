// Internal declarations shared by the C-ABI layer and the kernels: the
// workspace layout and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "sla.h"

namespace sla {

constexpr int kBlock = 64;       // tokens per block (the only supported block size)
constexpr int kMaxT = 4096;      // blocks per sequence
constexpr size_t kAlign = 1024;  // alignment of every workspace region
// Workspace header (256 bytes): the device error word at 0, the fault
// injection word of sla_debug_inject at 64, the sparse backward's tile counter
// at 128.
constexpr size_t kInjectWordOffset = 64;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Blocks padded to the aggregation GEMM's 128-row tile.
inline int pad128(int T) { return (T + 127) / 128 * 128; }

// Width of one per-block summary row: the d x d matrix followed by the d-vector
// (h_j | z_j, H_i | Z_i, and their backward counterparts).
inline int summary_width(int d) { return d * d + d; }

// Byte offsets of the regions inside the caller's workspace.
struct WorkspaceLayout {
  size_t err;        // the 256-byte header: error word, injection word, tile counter
  size_t qbar;       // fp32 [BH,T,d]   pooled Q
  size_t kbar;       // fp32 [BH,T,d]   pooled K
  size_t summ_hi;    // bf16 [BH,T,d*d+d] (h_j|z_j) forward, (A_i|a_i) backward: high part
  size_t summ_lo;    // bf16 [BH,T,d*d+d] the low part (value = hi + lo)
  size_t dh;         // bf16 [2][BH,T,d*d+d] (dh_j|dz_j) backward: hi plane, lo plane
  size_t mmat;       // bf16 [BH,Tp,Tp] marginal 0/1 matrix, rows = query blocks
  size_t mmat_t;     // bf16 [BH,Tp,Tp] its transpose
  size_t dvec;       // fp32 [BH,N]     D_t = dO_t . O_s,t
  size_t order;      // int32 [BH*ceil(T/2)] key-block pairs of the sparse backward, in order
  size_t ulen;       // int32 [BH*ceil(T/2)] union length of each key-block pair
  size_t ulist;      // uint16 [BH*T*n_crit] each pair's union, in the pair's column-CSR slot
  size_t uflag;      // uint8 [BH*T*n_crit] membership bits of the union entries
  size_t total;
};

WorkspaceLayout workspace_layout(int BH, int N, int d, int n_crit);

// Validated problem description handed to the launchers.
struct Problem {
  int B, H, BH, N, d, T, Tp, n_crit, n_negl;
  int nv;             // valid tokens per sequence (N unless key padding is on)
  float scale;        // softmax scale
  float scale_log2;   // scale * log2(e)
};

// ---- launchers (return cudaGetLastError() of their launches)
cudaError_t launch_pool(const Problem& p, const void* q, const void* k, float* qbar,
                        float* kbar, cudaStream_t s);
cudaError_t launch_classify(const Problem& p, const float* qbar, const float* kbar,
                            const float* logits_in, float* logits_out, int8_t* cls,
                            int32_t* crit_idx, uint32_t* marg_bits, cudaStream_t s);
// Hierarchical selection: super-block size and candidate counts (validated).
struct HierCounts {
  int G, TG, c_hi, c_lo;
};
constexpr size_t kMaxSmemPerCta = 227 * 1024;
cudaError_t launch_coarse_keys(const Problem& p, const float* kbar, float* kc, int G,
                               cudaStream_t s);
cudaError_t launch_hier_classify(const Problem& p, const HierCounts& h, const float* qbar,
                                 const float* kbar, const float* kc, const float* fine_in,
                                 const float* coarse_in, float* fine_out, float* coarse_out,
                                 int8_t* cls, int32_t* crit_idx, uint32_t* marg_bits, int* err,
                                 cudaStream_t s);
cudaError_t launch_crit_csr(const Problem& p, const int8_t* cls, int32_t* col_ptr,
                            int32_t* col_idx, cudaStream_t s);
cudaError_t launch_expand_marginal(const Problem& p, const uint32_t* marg_bits,
                                   __nv_bfloat16* mmat, __nv_bfloat16* mmat_t, cudaStream_t s);
cudaError_t launch_summaries(const Problem& p, const void* k, const void* v,
                             __nv_bfloat16* summ_hi, __nv_bfloat16* summ_lo, int* err,
                             cudaStream_t s);
cudaError_t launch_aggregate(const Problem& p, const __nv_bfloat16* mmat,
                             const __nv_bfloat16* summ_hi, const __nv_bfloat16* summ_lo,
                             __nv_bfloat16* out_hi, __nv_bfloat16* out_lo, int* err,
                             cudaStream_t s);
cudaError_t launch_fwd_sparse(const Problem& p, const void* q, const void* k, const void* v,
                              const int32_t* crit_idx, float* o_s, float* lse, int* err,
                              cudaStream_t s);
cudaError_t launch_fwd_linear(const Problem& p, const void* q, const __nv_bfloat16* hz_hi,
                              const __nv_bfloat16* hz_lo, const void* w_proj, const float* o_s,
                              void* o, float* den, float gate, int* err, cudaStream_t s);
cudaError_t launch_os_to_o(const Problem& p, const float* o_s, void* o, cudaStream_t s);
cudaError_t launch_dvec(const Problem& p, const void* d_o, const float* o_s, float* dvec,
                        cudaStream_t s);
cudaError_t launch_bwd_q(const Problem& p, const void* q, const void* d_o, const void* w_proj,
                         const float* o_s, const float* den, const __nv_bfloat16* hz_hi,
                         const __nv_bfloat16* hz_lo, float* dvec, float* dq,
                         __nv_bfloat16* summ_hi, __nv_bfloat16* summ_lo, float* dw, float gate,
                         float* d_gate, int num_sms, int* err, cudaStream_t s);
// The sparse backward's tiles (key-block pairs): the sorted union of each
// pair's two column lists with membership bits (written into the pair's slot
// of the column CSR), its length, and the tile order: heads in sequence, the
// longest unions of a window of a few heads first.
// `sched` (one int) is reset here for the sparse backward's tile counter.
cudaError_t launch_pair_order(const Problem& p, const int32_t* col_ptr, const int32_t* col_idx,
                              uint16_t* ulist, uint8_t* uflag, int32_t* ulen, int32_t* order,
                              int* sched, int* err, cudaStream_t s);
// Persistent: min(tiles, num_sms) CTAs take the tiles in order from the
// counter `sched` (zero at launch).
cudaError_t launch_bwd_sparse(const Problem& p, const void* q, const void* k, const void* v,
                              const void* d_o, const float* lse, const float* dvec,
                              const int32_t* col_ptr, const uint16_t* ulist, const uint8_t* uflag,
                              const int32_t* ulen, const int32_t* order, int* sched, float* dq,
                              float* dk, float* dv, int num_sms, int* err, cudaStream_t s);
cudaError_t launch_bwd_k(const Problem& p, const void* k, const void* v,
                         const __nv_bfloat16* dh_hi, const __nv_bfloat16* dh_lo, float* dk,
                         float* dv, int num_sms, int* err, cudaStream_t s);

// Opt-in per-kernel profiler (sla_profile_begin / sla_profile_end): while it
// is on, every launch made through launch_named() is bracketed by two CUDA
// events on its stream and recorded under `name`.
bool profiler_on();
cudaError_t profiler_mark(cudaStream_t s, cudaEvent_t* ev);
void profiler_record(const char* name, cudaEvent_t a, cudaEvent_t b);

template <typename F>
cudaError_t launch_named(const char* name, cudaStream_t s, F&& launch) {
  if (!profiler_on()) return launch();
  cudaEvent_t a = nullptr, b = nullptr;
  if (profiler_mark(s, &a) != cudaSuccess) return cudaErrorUnknown;
  const cudaError_t e = launch();
  if (profiler_mark(s, &b) != cudaSuccess) return cudaErrorUnknown;
  profiler_record(name, a, b);
  return e;
}

// TMA descriptor for a bf16 [BH, N, d] tensor viewed as 3D {d, N, BH} with a
// box of {64, rows, 1} and 128-byte swizzle.  Returns false on failure.
bool make_tmap_bhnd(CUtensorMap* map, const void* base, int BH, int N, int d, int box_rows);
// TMA descriptor for a bf16 3D tensor {inner, rows, batch} (row pitch = inner).
bool make_tmap_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                  uint64_t batch, uint32_t box_inner, uint32_t box_rows);
// TMA descriptor for a bf16 3D tensor {d0, d1, d2} with explicit element
// strides of dimensions 1 and 2 (multiples of 8), box {box0, box1, 1}.
bool make_tmap_strided(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint64_t stride1, uint64_t stride2, uint32_t box0, uint32_t box1);
// The d x d block of every per-block summary row of a bf16 plane [rows, d*d+d],
// viewed as {c, a, row} so that a box {64, d, 1} lands as a 128-byte-swizzled
// tile of d rows (a) per 64-column chunk (c).
bool make_tmap_summary(CUtensorMap* map, const void* plane, int rows, int d);
// fp32 [BH][N][d] as {d, N, BH}, 32-column (128-byte) boxes of box_rows rows,
// 128-byte swizzle (a store source: row r's 16-byte unit u at unit u ^ (r % 8)).
bool make_tmap_f32_bhnd(CUtensorMap* map, const float* base, int BH, int N, int d, int box_rows);


}  // namespace sla
