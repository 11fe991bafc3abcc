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
  float* ws_o;                  // split-K partial outputs [B][Hq][max_parts][D]
  float* ws_ml;                 // split-K partial (m, l)  [B][Hq][max_parts][2]
  int batch, hq, hkv, group, head_dim;
  int block_size, log2_bs, max_blocks, num_blocks;
  int window;
  int partition;    // tokens per partition (a multiple of 64); 1 << 30 without split
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
  r.hi = min(r.L, part * P + P);
  r.n_parts = (r.L > r.s0) ? (r.L + P - 1) / P - r.s0 / P : 0;
  r.final_write = (r.n_parts == 1);
  return r;
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

// Cross-warp merge buffer: per warp, per head (max, sum) and the unnormalised
// output row, all in the log2 domain.  Laid over the CTA's ring buffer once
// every warp has finished with it.
struct MergeSmem {
  float* m;  // [NW][kMaxGroup]
  float* l;  // [NW][kMaxGroup]
  float* o;  // [NW][kMaxGroup][D]
};

template <int NW>
__device__ __forceinline__ MergeSmem merge_smem(void* base, int D) {
  MergeSmem s;
  s.m = static_cast<float*>(base);
  s.l = s.m + NW * kMaxGroup;
  s.o = s.l + NW * kMaxGroup;
  (void)D;
  return s;
}

template <int NW>
__host__ __device__ constexpr int merge_smem_bytes(int D) {
  return (2 * NW * kMaxGroup + NW * kMaxGroup * D) * 4;
}

// Combine the NW warps' states and write either the final output (normalised,
// input dtype) or the partition's partial state to the workspace.
template <int NW, typename OutT>
__device__ void merge_and_store(const DecodeParams& p, const MergeSmem& s, int b, int g, int part,
                                bool final_write) {
  const int D = p.head_dim, G = p.group;
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int h = idx / D, d = idx - h * D;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, s.m[w * kMaxGroup + h]);
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float mw = s.m[w * kMaxGroup + h];
      if (mw == -CUDART_INF_F) continue;  // this warp saw no token
      const float c = exp2f(mw - M);
      num += c * s.o[(w * kMaxGroup + h) * D + d];
      den += c * s.l[w * kMaxGroup + h];
    }
    const size_t row = (size_t)b * p.hq + (size_t)g * G + h;
    if (final_write) {
      store_out<OutT>(static_cast<OutT*>(p.out) + row * D + d, num / den);
    } else {
      const size_t slot = row * p.max_parts + part;
      p.ws_o[slot * D + d] = num;
      if (d == 0) {
        p.ws_ml[slot * 2 + 0] = M;
        p.ws_ml[slot * 2 + 1] = den;
      }
    }
  }
}

}  // namespace pa
