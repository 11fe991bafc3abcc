// The split-K log-sum-exp combine kernel and the KV append (slot scatter) kernel.
#pragma once

#include "decode_common.cuh"
#include "ptx.cuh"

namespace pa {

// ---- split-K combine ----------------------------------------------------------
//
// NWR warps per output row (sequence b, query token j, query head h; j = 0
// for decode).  The partitions of the sequence's attended range each left
// (m_p, l_p, o_p) in the workspace (log2 domain, o_p unnormalised relative to
// m_p).  With M = max_p m_p:
//   out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p.
// A partition that held none of a multi-query row's positions left m = -inf,
// l = 0, o = 0 and weighs nothing; a row with no position at all is zero.
// Warp r of a row takes partitions r, r + NWR, ...; lane k computes the
// weights of every 32nd of those and broadcasts them, and each lane
// accumulates D/32 consecutive dims.  With NWR > 1 the row's warps add their
// sums through shared memory.  Sequences whose range fits one partition were
// written by the decode kernel and are skipped here.
constexpr int kCombineWarps = 8;

template <typename OutT, int D, int NWR>
__global__ void __launch_bounds__(kCombineWarps * 32) combine_kernel(const DecodeParams p) {
  constexpr int VEC = D / 32;
  constexpr int ROWS = kCombineWarps / NWR;  // rows per CTA
  constexpr uint32_t FULL = 0xffffffffu;
  __shared__ float red_o[NWR > 1 ? kCombineWarps : 1][NWR > 1 ? D : 1];
  __shared__ float red_l[kCombineWarps];
  pdl_wait();  // the partials come from the preceding decode kernel
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = warp % NWR;
  const int row = blockIdx.x * ROWS + warp / NWR;
  bool active = row < p.batch * p.q_len * p.hq;
  int pb = 0, n = 0;
  if (active) {
    const int b = row / (p.q_len * p.hq);
    const int L = clamp_context(p, b, false);
    const int s0 = window_start(max(L - p.q_len + 1, 0), p.window);  // the first query token's window
    const int P = p.partition;
    pb = s0 / P;
    n = L > s0 ? (L + P - 1) / P - pb : 0;
    active = n > 1;
  }
  float acc[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
  float den = 0.f;
  if (active) {
    const float* ml = p.ws_ml + ((size_t)row * p.max_parts + pb) * 2;
    const float* po = p.ws_o + ((size_t)row * p.max_parts + pb) * D + lane * VEC;
    float M = -CUDART_INF_F;
    for (int i = lane; i < n; i += 32) M = fmaxf(M, ml[2 * i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, off));
    // This warp's partitions: i = r + NWR * j.
    const int nj = (n - r + NWR - 1) / NWR;
    for (int c = 0; c < nj; c += 32) {
      const int j = c + lane;
      float w = 0.f;
      if (j < nj && M != -CUDART_INF_F) {
        const int i = r + NWR * j;
        w = exp2f(ml[2 * i] - M);
        den = fmaf(w, ml[2 * i + 1], den);
      }
      const int cnt = min(32, nj - c);
#pragma unroll 8
      for (int e = 0; e < cnt; ++e) {
        const float wj = __shfl_sync(FULL, w, e);
        const float* src = po + (size_t)(r + NWR * (c + e)) * D;
#pragma unroll
        for (int v = 0; v < VEC; v += 2) {
          const float2 x = *reinterpret_cast<const float2*>(src + v);
          acc[v] = fmaf(wj, x.x, acc[v]);
          acc[v + 1] = fmaf(wj, x.y, acc[v + 1]);
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(FULL, den, off);
  }
  if (NWR > 1) {
#pragma unroll
    for (int v = 0; v < VEC; ++v) red_o[warp][lane * VEC + v] = acc[v];
    if (lane == 0) red_l[warp] = den;
    __syncthreads();
    if (!active || r != 0) return;
    for (int w2 = 1; w2 < NWR; ++w2) {
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[v] += red_o[warp + w2][lane * VEC + v];
      den += red_l[warp + w2];
    }
  } else if (!active) {
    return;
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  OutT* out = static_cast<OutT*>(p.out) + (size_t)row * D + lane * VEC;
#pragma unroll
  for (int v = 0; v < VEC; ++v) store_out<OutT>(out + v, acc[v] * inv);
}

// ---- bounded-wait check ---------------------------------------------------------
//
// One warp waits on an mbarrier that nothing arrives on, with the bounded wait
// of every TMA / MMA completion in this library; when it gives up it raises
// PA_DEVERR_TIMEOUT, as the kernels do, and returns.
__global__ void bounded_wait_check_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_addr(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    mbar_init_fence();
  }
  __syncwarp();
  const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(b, 0, limit_ns));
  if (!ok && threadIdx.x == 0) raise_error(PA_DEVERR_TIMEOUT);
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

// ---- block copies (copy-on-write) ----------------------------------------------------
//
// blockIdx.x: pair i = (src, dst) of pairs[]; threads stride over the block's
// 16-byte chunks (chunks_per_block of them in each cache).  Ids outside the
// pool raise PA_DEVERR_BLOCK and the pair is skipped.
__global__ void __launch_bounds__(256)
    copy_blocks_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache, const int32_t* __restrict__ pairs,
                       int num_blocks, int64_t chunks_per_block) {
  const int src = pairs[2 * blockIdx.x], dst = pairs[2 * blockIdx.x + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0) raise_error(PA_DEVERR_BLOCK);
    return;
  }
  const int64_t s0 = (int64_t)src * chunks_per_block, d0 = (int64_t)dst * chunks_per_block;
  for (int64_t c = (int64_t)blockIdx.y * blockDim.x + threadIdx.x; c < chunks_per_block;
       c += (int64_t)gridDim.y * blockDim.x) {
    k_cache[d0 + c] = k_cache[s0 + c];
    v_cache[d0 + c] = v_cache[s0 + c];
  }
}

}  // namespace pa
