// Shared pieces of the decode kernels: launch parameters, the per-CTA token
// range (sequence, kv head, partition), the cross-warp softmax merge and the
// output / partial-state stores.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>
#include <stdint.h>

#include "../../include/pagedattn.h"

namespace pa {

// Device error word (OR of PA_DEVERR_* bits), one per device.
__device__ unsigned int g_device_errors;

__device__ __forceinline__ void raise_error(unsigned int bit) { atomicOr(&g_device_errors, bit); }

constexpr int kMaxGroup = 8;                     // query heads per kv head handled by one CTA
constexpr int kSliceTokens = 16;                 // tokens one warp processes per step
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s bound on any single tile wait
constexpr uint64_t kDrainLimitNs = 100000000ull;  // 0.1 s bound when draining after a timeout
constexpr float kLog2e = 1.4426950408889634f;

struct DecodeParams {
  const void* q;        // [B][Hq][D]
  void* out;            // [B][Hq][D]
  const void* k_cache;  // [num_blocks][Hkv][bs][D]
  const void* v_cache;
  const int32_t* block_tables;  // [B][max_blocks]
  const int32_t* context_lens;  // [B]
  const void* k_new;            // fused append: the step's new rows [B][Hkv][D] (else null)
  const void* v_new;
  float* ws_o;                  // split-K partial outputs [B][Hq][max_parts][D]
  float* ws_ml;                 // split-K partial (m, l)  [B][Hq][max_parts][2]
  int* queue;                   // dynamic schedule: [0] work-item counter, [1] CTAs finished (zero between calls)
  int* unit_count;              // dynamic schedule: partials stored per (sequence, kv head) (zero between calls)
  int merge_in_kernel;          // dynamic schedule: the last partial of a unit merges it (else the combine kernel)
  int static_items;             // dynamic schedule: items per warp fixed by its index (1 or 2) before claims
  int batch, hq, hkv, group, head_dim;
  int q_len;        // query tokens per sequence (1 for decode; T for the multi-query rows [B][T][Hq][D])
  const int32_t* cu_q;  // prefill: sequence b's query rows are [cu_q[b], cu_q[b+1]) of [total][Hq][D] (else null)
  int q_tile;           // prefill: query tokens per CTA
  int max_q_len;        // prefill: bound on cu_q[b+1] - cu_q[b] (the grid covers it)
  int total_q;          // prefill: rows of q and out (bound on cu_q[B])
  // Cascade: sequences 0 .. n_sharers-1 share positions [0, prefix_len) (a
  // multiple of the partition).  The prefix pass (cascade_prefix = 1) attends
  // them once for all sharers; the other passes start those sequences at
  // prefix_len.
  int cascade_prefix;
  int n_sharers;
  int prefix_len;
  int block_size, log2_bs, max_blocks, num_blocks;
  int window;
  int partition;    // tokens per partition (a multiple of 64); 1 << 30 without split
  int log2_partition;  // dynamic schedule: log2(partition) (its partitions are powers of two)
  int max_parts;    // partitions per sequence in the workspace
  int max_context;  // bound on context_lens[b]
  float scale;      // multiplies q.k
  float softcap;    // > 0 and finite: cap enabled
  float inv_softcap;
  int use_softcap;
};

// Token range one CTA attends.
struct CtaRange {
  int L, s0;         // context length and window start of the sequence
  int lo, hi;        // attended tokens of this CTA: [lo, hi)
  int n_parts;       // partitions the sequence's range spans
  bool final_write;  // this CTA writes the normalised output itself
};

__device__ __forceinline__ int clamp_context(const DecodeParams& p, int b, bool report) {
  int L = p.context_lens[b];
  const int cap = min(p.max_context, p.max_blocks << p.log2_bs);
  if (L < 0 || L > cap) {
    if (report) raise_error(PA_DEVERR_CONTEXT);
    L = L < 0 ? 0 : cap;
  }
  return L;
}

__device__ __forceinline__ int window_start(int L, int window) { return (window > 0 && L > window) ? L - window : 0; }

__device__ __forceinline__ CtaRange cta_range(const DecodeParams& p, int b, int part, bool report) {
  CtaRange r;
  r.L = clamp_context(p, b, report);
  r.s0 = window_start(r.L, p.window);
  const int P = p.partition;
  r.lo = max(r.s0, part * P);
  if (b < p.n_sharers) r.lo = max(r.lo, p.prefix_len);  // the cascade's prefix pass attended the shared prefix
  r.hi = min(r.L, part * P + P);
  r.n_parts = (r.L > r.s0) ? (r.L + P - 1) / P - r.s0 / P : 0;
  r.final_write = (r.n_parts == 1);
  return r;
}

// Row (within the 2-D view [num_blocks*Hkv*bs][D] of the cache) holding token t
// of kv head g, given the token's physical block.
__device__ __forceinline__ int cache_row(const DecodeParams& p, int phys, int g, int t) {
  return (phys * p.hkv + g) * p.block_size + (t & (p.block_size - 1));
}

template <typename T>
__device__ __forceinline__ void store_out(T* dst, float v);
template <>
__device__ __forceinline__ void store_out<float>(float* dst, float v) { *dst = v; }
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* dst, float v) { *dst = __float2bfloat16_rn(v); }

// Zero output rows of the G query heads of (b, g): used when L == 0.
template <typename T>
__device__ void write_zero_rows(const DecodeParams& p, int b, int g) {
  T* out = static_cast<T*>(p.out) + ((size_t)b * p.hq + (size_t)g * p.group) * p.head_dim;
  for (int i = threadIdx.x; i < p.group * p.head_dim; i += blockDim.x) store_out<T>(out + i, 0.f);
}

// Cross-warp merge buffer: per warp w and head h (slot w*gs + h) the running
// max, the sum (log2 domain) and the unnormalised output row.
struct MergeSmem {
  float* m;  // [NW][gs]
  float* l;  // [NW][gs]
  float* o;  // [NW][gs][D]
  int gs;    // head stride
};

template <int NW>
__device__ __forceinline__ MergeSmem merge_smem(void* base, int D, int gs = kMaxGroup) {
  MergeSmem s;
  s.m = static_cast<float*>(base);
  s.l = s.m + NW * gs;
  s.o = s.l + NW * gs;
  s.gs = gs;
  (void)D;
  return s;
}

template <int NW>
__host__ __device__ constexpr int merge_smem_bytes(int D, int gs = kMaxGroup) {
  return (2 * NW * gs + NW * gs * D) * 4;
}

// Where a merged (sequence, kv head) group of G query heads goes: the
// normalised rows (final) or the partial state (m, l in log2 domain, o
// unnormalised), each with its own per-head stride in elements.
template <typename OutT>
struct MergeDest {
  bool final_write;
  OutT* out;  // head h at out + h * D
  float* po;  // head h at po + h * po_stride
  float* pml; // head h at pml + h * pml_stride
  size_t po_stride, pml_stride;
};

// Combine the NW warps' states in `s` for the G heads, using threads
// [tid0, tid0 + nthreads) of the CTA.
template <int NW, typename OutT>
__device__ void merge_warps(const MergeSmem& s, int G, int D, const MergeDest<OutT>& dst, int tid, int nthreads) {
  for (int idx = tid; idx < G * D; idx += nthreads) {
    const int h = idx / D, d = idx - h * D;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, s.m[w * s.gs + h]);
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float mw = s.m[w * s.gs + h];
      if (mw == -CUDART_INF_F) continue;  // this warp saw no token
      const float c = exp2f(mw - M);
      num += c * s.o[(w * s.gs + h) * D + d];
      den += c * s.l[w * s.gs + h];
    }
    if (dst.final_write) {
      store_out<OutT>(dst.out + (size_t)h * D + d, num / den);
    } else {
      dst.po[h * dst.po_stride + d] = num;
      if (d == 0) {
        dst.pml[h * dst.pml_stride + 0] = M;
        dst.pml[h * dst.pml_stride + 1] = den;
      }
    }
  }
}

// The grid-scheduled kernels' destination: output rows of (b, g) or the
// partition's slot in the [B][Hq][max_parts] workspace.
template <typename OutT>
__device__ __forceinline__ MergeDest<OutT> grid_dest(const DecodeParams& p, int b, int g, int part, bool final_write) {
  MergeDest<OutT> d;
  const size_t row = (size_t)b * p.hq + (size_t)g * p.group;
  d.final_write = final_write;
  d.out = static_cast<OutT*>(p.out) + row * p.head_dim;
  d.po = p.ws_o + (row * p.max_parts + part) * p.head_dim;
  d.pml = p.ws_ml + (row * p.max_parts + part) * 2;
  d.po_stride = (size_t)p.max_parts * p.head_dim;
  d.pml_stride = (size_t)p.max_parts * 2;
  return d;
}

}  // namespace pa
