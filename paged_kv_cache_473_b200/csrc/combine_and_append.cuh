// The split-K log-sum-exp combine kernel and the KV append (slot scatter) kernel.
#pragma once

#include "decode_common.cuh"

namespace pa {

// ---- split-K combine ----------------------------------------------------------
//
// One CTA per (query head, sequence).  The partitions of the sequence's
// attended range each left (m_p, l_p, o_p) in the workspace (log2 domain, o_p
// unnormalised relative to m_p).  With M = max_p m_p:
//   out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p.
// Sequences whose range fits one partition were written by the decode kernel.
constexpr int kCombineWarps = 8;

template <typename OutT, int D>
__global__ void __launch_bounds__(kCombineWarps * 32) combine_kernel(const DecodeParams p) {
  constexpr int VEC = D / 32;
  extern __shared__ __align__(16) float csm[];  // [max_parts] weights, then [kCombineWarps][D]
  __shared__ float red[kCombineWarps];
  __shared__ float s_M, s_den;

  const int h = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = clamp_context(p, b, false);
  const int s0 = window_start(L, p.window);
  if (L <= s0) return;
  const int P = p.partition;
  const int pb = s0 / P, n = (L + P - 1) / P - pb;
  if (n <= 1) return;

  const size_t row = (size_t)b * p.hq + h;
  const float* ml = p.ws_ml + (row * p.max_parts + pb) * 2;
  const float* po = p.ws_o + (row * p.max_parts + pb) * D;
  float* wts = csm;
  float* acc_s = csm + ((p.max_parts + 3) & ~3);

  float M = -CUDART_INF_F;
  for (int i = threadIdx.x; i < n; i += blockDim.x) M = fmaxf(M, ml[2 * i]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  if (lane == 0) red[warp] = M;
  __syncthreads();
  if (threadIdx.x == 0) {
    float v = red[0];
    for (int w = 1; w < kCombineWarps; ++w) v = fmaxf(v, red[w]);
    s_M = v;
  }
  __syncthreads();
  M = s_M;

  float den = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const float w = exp2f(ml[2 * i] - M);
    wts[i] = w;
    den += w * ml[2 * i + 1];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
  __syncthreads();  // red[] reuse
  if (lane == 0) red[warp] = den;
  __syncthreads();
  if (threadIdx.x == 0) {
    float v = 0.f;
    for (int w = 0; w < kCombineWarps; ++w) v += red[w];
    s_den = v;
  }

  float acc[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
  for (int i = warp; i < n; i += kCombineWarps) {
    const float w = wts[i];
    const float* src = po + (size_t)i * D + lane * VEC;
#pragma unroll
    for (int v = 0; v < VEC; v += 2) {
      const float2 x = *reinterpret_cast<const float2*>(src + v);
      acc[v] = fmaf(w, x.x, acc[v]);
      acc[v + 1] = fmaf(w, x.y, acc[v + 1]);
    }
  }
#pragma unroll
  for (int v = 0; v < VEC; ++v) acc_s[warp * D + lane * VEC + v] = acc[v];
  __syncthreads();
  OutT* out = static_cast<OutT*>(p.out) + row * D;
  const float inv = 1.f / s_den;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kCombineWarps; ++w) s += acc_s[w * D + d];
    store_out<OutT>(out + d, s * inv);
  }
}

// ---- KV append ------------------------------------------------------------------
//
// One thread per 16-byte chunk of one (token, kv head) row of K and of V:
//   cache[slot / bs][h][slot % bs][:] = new[token][h][:].
// Negative slots are padding and skipped; slots past the pool raise
// PA_DEVERR_SLOT and are skipped.
__global__ void __launch_bounds__(256)
    write_kv_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, const int64_t* __restrict__ slots,
                    int num_tokens, uint4* __restrict__ k_cache, uint4* __restrict__ v_cache, int64_t num_slots,
                    int block_size, int num_kv_heads, int chunks_per_row) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)num_tokens * num_kv_heads * chunks_per_row;
  if (idx >= total) return;
  const int c = (int)(idx % chunks_per_row);
  const int64_t rrow = idx / chunks_per_row;  // token * Hkv + head
  const int h = (int)(rrow % num_kv_heads);
  const int64_t i = rrow / num_kv_heads;
  const int64_t s = slots[i];
  if (s < 0) return;
  if (s >= num_slots) {
    if (h == 0 && c == 0) raise_error(PA_DEVERR_SLOT);
    return;
  }
  const int64_t blk = s / block_size, off = s % block_size;
  const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * chunks_per_row + c;
  const int64_t src = rrow * chunks_per_row + c;
  k_cache[dst] = k[src];
  v_cache[dst] = v[src];
}

}  // namespace pa
