// Paged decode attention on CUDA cores (fp32 or bf16 inputs).
//
// Same CTA decomposition as the tensor-core kernel -- one CTA per
// (partition, kv head, sequence), warp w takes every NW-th 16-token slice --
// but each lane owns D/32 consecutive dims: it keeps those dims of the group's
// query rows in registers, reads the matching dims of each K and V row with one
// vector load from global memory, and the warp sums the per-lane partial dot
// products with shuffles.  Used for fp32 caches and as the CUDA-core baseline
// the tensor-core kernel is measured against.
//
// APPEND (the fused decode step): the CTA whose range ends at the sequence's
// last token takes position L-1's key/value from the step's new rows, and the
// warp that meets it also writes them to the cache slot of that position.
#pragma once

#include "decode_common.cuh"
#include "ptx.cuh"

namespace pa {

template <typename T, int VEC>
struct VecLoad;

// VEC consecutive elements of a row, widened to fp32.
template <int VEC>
struct VecLoad<float, VEC> {
  static __device__ __forceinline__ void load(const float* src, float (&dst)[VEC]) {
    if constexpr (VEC % 4 == 0) {
#pragma unroll
      for (int i = 0; i < VEC; i += 4) {
        const float4 v = *reinterpret_cast<const float4*>(src + i);
        dst[i] = v.x;
        dst[i + 1] = v.y;
        dst[i + 2] = v.z;
        dst[i + 3] = v.w;
      }
    } else {
      static_assert(VEC == 2, "unsupported vector width");
      const float2 v = *reinterpret_cast<const float2*>(src);
      dst[0] = v.x;
      dst[1] = v.y;
    }
  }
};

template <int VEC>
struct VecLoad<__nv_bfloat16, VEC> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* src, float (&dst)[VEC]) {
    if constexpr (VEC == 8) {
      const uint4 v = *reinterpret_cast<const uint4*>(src);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        dst[2 * i] = __uint_as_float(w[i] << 16);
        dst[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
      }
    } else if constexpr (VEC == 4) {
      const uint2 v = *reinterpret_cast<const uint2*>(src);
      dst[0] = __uint_as_float(v.x << 16);
      dst[1] = __uint_as_float(v.x & 0xffff0000u);
      dst[2] = __uint_as_float(v.y << 16);
      dst[3] = __uint_as_float(v.y & 0xffff0000u);
    } else {
      static_assert(VEC == 2, "unsupported vector width");
      const uint32_t v = *reinterpret_cast<const uint32_t*>(src);
      dst[0] = __uint_as_float(v << 16);
      dst[1] = __uint_as_float(v & 0xffff0000u);
    }
  }
};

// GP: group size rounded up to a power of two (heads >= G are padding).
template <typename T, int D, int GP, int NW, bool SPLIT, bool APPEND>
__global__ void __launch_bounds__(NW * 32) decode_simt_kernel(const DecodeParams p) {
  constexpr int VEC = D / 32;
  constexpr int U = 4;  // tokens per inner step
  extern __shared__ __align__(16) uint8_t smem_raw[];
  if (SPLIT) pdl_launch_dependents();  // the combine kernel may launch now and wait for this grid

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = SPLIT ? (int)blockIdx.x : 0;
  const int g = blockIdx.y, b = blockIdx.z;
  const CtaRange r = cta_range(p, b, part, threadIdx.x == 0 && part == 0);
  if (r.lo >= r.hi) {
    if (r.L == r.s0 && part == 0) write_zero_rows<T>(p, b, g);
    return;
  }
  const int G = p.group;

  float q[GP][VEC];
#pragma unroll
  for (int h = 0; h < GP; ++h) {
    if (h < G) {
      const T* qrow = static_cast<const T*>(p.q) + ((size_t)b * p.hq + (size_t)g * G + h) * D + lane * VEC;
      VecLoad<T, VEC>::load(qrow, q[h]);
    } else {
#pragma unroll
      for (int v = 0; v < VEC; ++v) q[h][v] = 0.f;
    }
  }

  float m[GP], l[GP], o[GP][VEC];
#pragma unroll
  for (int h = 0; h < GP; ++h) {
    m[h] = -CUDART_INF_F;
    l[h] = 0.f;
#pragma unroll
    for (int v = 0; v < VEC; ++v) o[h][v] = 0.f;
  }

  const float qk_scale = p.use_softcap ? p.scale : p.scale * kLog2e;
  const int j0 = r.lo / kSliceTokens;
  const int j1 = (r.hi + kSliceTokens - 1) / kSliceTokens;
  const int32_t* table = p.block_tables + (size_t)b * p.max_blocks;
  const T* kc = static_cast<const T*>(p.k_cache);
  const T* vc = static_cast<const T*>(p.v_cache);
  const bool append_cta = APPEND && r.hi == r.L;
  const size_t new_off = ((size_t)b * p.hkv + g) * D + lane * VEC;

  for (int j = j0 + warp; j < j1; j += NW) {
    const int t0 = j * kSliceTokens;
    const int phys = table[t0 >> p.log2_bs];
    if (phys < 0 || phys >= p.num_blocks) {
      if (lane == 0) raise_error(PA_DEVERR_BLOCK);
      continue;
    }
    const size_t row0 = ((size_t)phys * p.hkv + g) * p.block_size + (t0 & (p.block_size - 1));
    for (int u0 = 0; u0 < kSliceTokens; u0 += U) {
      float kr[U][VEC], vr[U][VEC];
      bool valid[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int t = t0 + u0 + u;
        valid[u] = t >= r.lo && t < r.hi;
        if (APPEND && append_cta && t == r.L - 1) {
          // The appended token: read the new rows and store them in the cache.
          const T* kn = static_cast<const T*>(p.k_new) + new_off;
          const T* vn = static_cast<const T*>(p.v_new) + new_off;
          VecLoad<T, VEC>::load(kn, kr[u]);
          VecLoad<T, VEC>::load(vn, vr[u]);
          T* kd = const_cast<T*>(kc) + (row0 + u0 + u) * D + lane * VEC;
          T* vd = const_cast<T*>(vc) + (row0 + u0 + u) * D + lane * VEC;
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            kd[e] = kn[e];
            vd[e] = vn[e];
          }
        } else if (valid[u]) {
          VecLoad<T, VEC>::load(kc + (row0 + u0 + u) * D + lane * VEC, kr[u]);
          VecLoad<T, VEC>::load(vc + (row0 + u0 + u) * D + lane * VEC, vr[u]);
        } else {
#pragma unroll
          for (int v = 0; v < VEC; ++v) kr[u][v] = vr[u][v] = 0.f;
        }
      }
      float x[U][GP];
#pragma unroll
      for (int u = 0; u < U; ++u) {
#pragma unroll
        for (int h = 0; h < GP; ++h) {
          float acc = 0.f;
#pragma unroll
          for (int v = 0; v < VEC; ++v) acc = fmaf(q[h][v], kr[u][v], acc);
          x[u][h] = acc;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int h = 0; h < GP; ++h) x[u][h] += __shfl_xor_sync(0xffffffffu, x[u][h], off);
      }
#pragma unroll
      for (int h = 0; h < GP; ++h) {
        float mx = -CUDART_INF_F;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          float s = x[u][h] * qk_scale;
          if (p.use_softcap) s = p.softcap * tanhf(s * p.inv_softcap) * kLog2e;
          s = valid[u] ? s : -CUDART_INF_F;
          x[u][h] = s;
          mx = fmaxf(mx, s);
        }
        const float mn = fmaxf(m[h], mx);
        if (mn == -CUDART_INF_F) continue;  // nothing valid in this step
        const float al = exp2f(m[h] - mn);
        m[h] = mn;
        l[h] *= al;
#pragma unroll
        for (int v = 0; v < VEC; ++v) o[h][v] *= al;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const float pw = exp2f(x[u][h] - mn);
          l[h] += pw;
#pragma unroll
          for (int v = 0; v < VEC; ++v) o[h][v] = fmaf(pw, vr[u][v], o[h][v]);
        }
      }
    }
  }

  const MergeSmem ms = merge_smem<NW>(smem_raw, D);
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < GP; ++h) {
      ms.m[warp * kMaxGroup + h] = m[h];
      ms.l[warp * kMaxGroup + h] = l[h];
    }
  }
#pragma unroll
  for (int h = 0; h < GP; ++h) {
    if (h < G) {
#pragma unroll
      for (int v = 0; v < VEC; ++v) ms.o[(warp * kMaxGroup + h) * D + lane * VEC + v] = o[h][v];
    }
  }
  __syncthreads();
  merge_warps<NW, T>(ms, G, D, grid_dest<T>(p, b, g, part, !SPLIT || r.final_write), threadIdx.x, blockDim.x);
}

}  // namespace pa
