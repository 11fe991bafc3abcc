// Paged decode attention, bf16, tensor-core (warp MMA) kernel.
//
// One CTA serves one (partition, kv head, sequence).  Each of its NW warps
// owns every NW-th 16-token slice of the CTA's token range and runs its own
// ST-deep ring of shared-memory stages: lane 0 issues 2-D TMA tile loads of the
// slice's K and V rows (the slice lies inside one physical block, found through
// the block table), completion is counted on a per-stage mbarrier, and the
// warp computes on a stage while later ones are in flight.  Warps never wait on
// one another until the final merge.
//
// Per slice, with G <= 8 query heads of the group padded to 8 MMA columns:
//   S^T[16 tok x 8 heads] = K[16 x D] . Q^T[D x 8]          (D/16 MMAs)
//   online softmax over the slice (fp32, log2 domain, warp shuffles)
//   O^T[D x 8 heads]     += V^T[D x 16] . P^T[16 x 8]        (D/16 MMAs)
// K feeds the MMA's A operand straight from shared memory (ldmatrix), V^T via
// ldmatrix.trans, and the probabilities move from the S accumulator layout to
// the B-operand layout with movmatrix.trans, so P never touches shared memory.
//
// Shared-memory tiles come from TMA with 128-byte swizzle: a slice of K (or V)
// is D/64 panels of [16 rows x 128 B]; 16-byte chunk c of row r sits at chunk
// c ^ (r & 7), which keeps every ldmatrix phase free of bank conflicts.
#pragma once

#include "decode_common.cuh"
#include "ptx.cuh"

namespace pa {

template <int D, int NW, int ST>
struct MmaCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kPanelBytes = kSliceTokens * 128;  // 16 rows x 128 B
  static constexpr int kSliceBytes = kPanels * kPanelBytes;
  static constexpr int kStageBytes = 2 * kSliceBytes;  // K then V
  static constexpr int kRingBytes = NW * ST * kStageBytes;
  static constexpr int kBarOffset = kRingBytes;
  static constexpr int kSmemBytes = kRingBytes + NW * ST * 8 + 1024;  // + barriers + alignment slack
  static_assert(merge_smem_bytes<NW>(D) <= kRingBytes, "merge buffer must fit in the ring");
  static_assert(D % 64 == 0, "head_dim must be a multiple of 64");
};

template <int D, int NW, int ST, bool SPLIT>
__global__ void __launch_bounds__(NW * 32)
    decode_mma_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                      const DecodeParams p) {
  using Cfg = MmaCfg<D, NW, ST>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = SPLIT ? (int)blockIdx.x : 0;
  const int g = blockIdx.y, b = blockIdx.z;

  const CtaRange r = cta_range(p, b, part, threadIdx.x == 0 && part == 0);
  if (r.lo >= r.hi) {
    if (r.L == r.s0 && part == 0) write_zero_rows<__nv_bfloat16>(p, b, g);
    return;
  }
  const int G = p.group;

  // Per-warp ring and barriers.
  const uint32_t ring = smem_addr(smem) + warp * ST * Cfg::kStageBytes;
  const uint32_t bars = smem_addr(smem + Cfg::kBarOffset) + warp * ST * 8;
  if (lane == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
#pragma unroll
    for (int s = 0; s < ST; ++s) mbar_init(bars + 8 * s, 1);
    mbar_init_fence();
  }
  __syncwarp();

  const int j0 = r.lo / kSliceTokens;
  const int j1 = (r.hi + kSliceTokens - 1) / kSliceTokens;
  const int n_w = (j1 - j0 > warp) ? (j1 - j0 - warp + NW - 1) / NW : 0;

  const int32_t* table = p.block_tables + (size_t)b * p.max_blocks;
  const int bs_mask = p.block_size - 1;
  // Issue the TMA loads of this warp's i-th slice into stage i % ST (lane 0 only).
  auto issue = [&](int i) {
    const int s = i % ST;
    const uint32_t bar = bars + 8 * s;
    const int t = (j0 + warp + NW * i) * kSliceTokens;
    const int phys = table[t >> p.log2_bs];
    if (phys < 0 || phys >= p.num_blocks) {
      raise_error(PA_DEVERR_BLOCK);
      mbar_arrive(bar);  // complete the phase with no data; the slice computes on stale tiles
      return;
    }
    const int y = (phys * p.hkv + g) * p.block_size + (t & bs_mask);
    const uint32_t kdst = ring + s * Cfg::kStageBytes;
    const uint32_t vdst = kdst + Cfg::kSliceBytes;
    mbar_arrive_expect_tx(bar, Cfg::kStageBytes);
#pragma unroll
    for (int pn = 0; pn < Cfg::kPanels; ++pn) {
      tma_load_2d(kdst + pn * Cfg::kPanelBytes, &kmap, bar, pn * 64, y);
      tma_load_2d(vdst + pn * Cfg::kPanelBytes, &vmap, bar, pn * 64, y);
    }
  };
  if (lane == 0) {
    for (int i = 0; i < ST && i < n_w; ++i) issue(i);
  }

  // Q^T as the B operand of S^T = K Q^T: column n = lane / 4 is query head n of the group.
  uint32_t qf[D / 16][2];
  {
    const int n = lane >> 2;
    const __nv_bfloat16* qrow =
        static_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.hq + (size_t)g * G + (n < G ? n : 0)) * D;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int c = kk * 16 + 2 * (lane & 3);
      qf[kk][0] = n < G ? *reinterpret_cast<const uint32_t*>(qrow + c) : 0u;
      qf[kk][1] = n < G ? *reinterpret_cast<const uint32_t*>(qrow + c + 8) : 0u;
    }
  }

  // Softmax state for heads n0 = 2*(lane%4) and n0+1 (log2 domain); l is this lane's partial sum.
  float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, l0 = 0.f, l1 = 0.f;
  float o[D / 16][4];
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

  const float qk_scale = p.use_softcap ? p.scale : p.scale * kLog2e;
  // Lane-constant parts of the ldmatrix addresses.
  const uint32_t k_lane = ((lane & 7) | (lane & 8)) * 128;      // row = lane%8 + 8*((lane/8)%2)
  const uint32_t v_lane = ((lane & 7) | ((lane >> 4) << 3)) * 128;  // row = lane%8 + 8*(lane/16)
  const uint32_t k_sub = lane >> 4, v_sub = (lane >> 3) & 1, swz = lane & 7;

  bool failed = false;
  int i_done = 0;
  for (int i = 0; i < n_w; ++i) {
    const int s = i % ST;
    bool ok = mbar_wait_bounded(bars + 8 * s, (i / ST) & 1, kWaitLimitNs);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) {
      failed = true;
      break;
    }
    i_done = i + 1;
    const uint32_t kbase = ring + s * Cfg::kStageBytes;
    const uint32_t vbase = kbase + Cfg::kSliceBytes;
    const int t0 = (j0 + warp + NW * i) * kSliceTokens;

    // ---- S^T = K Q^T -------------------------------------------------------
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t chunk = ((kk & 3) << 1) | k_sub;
      const uint32_t addr = kbase + (kk >> 2) * Cfg::kPanelBytes + k_lane + ((chunk ^ swz) << 4);
      uint32_t a0, a1, a2, a3;
      ldsm_x4(addr, a0, a1, a2, a3);
      mma_bf16_16816(sc, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
    }
    // sc[0], sc[1]: token t0 + lane/4, heads n0, n0+1; sc[2], sc[3]: token + 8.
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float v = sc[e] * qk_scale;
      if (p.use_softcap) v = p.softcap * tanhf(v * p.inv_softcap) * kLog2e;
      x[e] = v;
    }
    const bool partial = (t0 < r.lo) || (t0 + kSliceTokens > r.hi);
    uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;
    if (partial) {
      const int ta = t0 + (lane >> 2), tb = ta + 8;
      const bool va = ta >= r.lo && ta < r.hi, vb = tb >= r.lo && tb < r.hi;
      if (!va) x[0] = x[1] = -CUDART_INF_F;
      if (!vb) x[2] = x[3] = -CUDART_INF_F;
      // Tokens held by this lane in the V^T fragments: 2*(lane%4) (+1) and +8.
      const int tc = t0 + 2 * (lane & 3);
      auto ok_tok = [&](int t) { return t >= r.lo && t < r.hi; };
      keep_lo = (ok_tok(tc) ? 0x0000ffffu : 0u) | (ok_tok(tc + 1) ? 0xffff0000u : 0u);
      keep_hi = (ok_tok(tc + 8) ? 0x0000ffffu : 0u) | (ok_tok(tc + 9) ? 0xffff0000u : 0u);
    }

    // ---- online softmax ----------------------------------------------------
    float mx0 = fmaxf(x[0], x[2]), mx1 = fmaxf(x[1], x[3]);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    const uint32_t plo = pack_bf16x2(exp2f(x[0] - mn0), exp2f(x[1] - mn1));
    const uint32_t phi = pack_bf16x2(exp2f(x[2] - mn0), exp2f(x[3] - mn1));
    l0 = l0 * al0 + bf16_lo(plo) + bf16_lo(phi);
    l1 = l1 * al1 + bf16_hi(plo) + bf16_hi(phi);
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      o[mt][0] *= al0;
      o[mt][1] *= al1;
      o[mt][2] *= al0;
      o[mt][3] *= al1;
    }
    const uint32_t pb0 = movmatrix_trans(plo);
    const uint32_t pb1 = movmatrix_trans(phi);

    // ---- O^T += V^T P^T ----------------------------------------------------
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      const uint32_t chunk = ((mt & 3) << 1) | v_sub;
      const uint32_t addr = vbase + (mt >> 2) * Cfg::kPanelBytes + v_lane + ((chunk ^ swz) << 4);
      uint32_t a0, a1, a2, a3;
      ldsm_x4_trans(addr, a0, a1, a2, a3);
      if (partial) {
        a0 &= keep_lo;
        a1 &= keep_lo;
        a2 &= keep_hi;
        a3 &= keep_hi;
      }
      mma_bf16_16816(o[mt], a0, a1, a2, a3, pb0, pb1);
    }

    __syncwarp();
    if (lane == 0 && i + ST < n_w) issue(i + ST);
  }

  if (failed) {
    raise_error(PA_DEVERR_TIMEOUT);
    // Let this warp's loads still in flight land before the CTA exits.
    for (int i = i_done; i < n_w && i < i_done + ST; ++i)
      (void)mbar_wait_bounded(bars + 8 * (i % ST), (i / ST) & 1, kDrainLimitNs);
  }

  // Lane partial sums -> per-head sums (lanes with the same lane%4 share heads).
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }

  __shared__ int cta_failed;
  if (threadIdx.x == 0) cta_failed = 0;
  __syncthreads();  // every warp is done with its ring: reuse it for the merge
  if (failed && lane == 0) cta_failed = 1;

  const MergeSmem ms = merge_smem<NW>(smem, D);
  const int n0 = 2 * (lane & 3);
  if (lane < 4) {
    ms.m[warp * kMaxGroup + n0] = m0;
    ms.m[warp * kMaxGroup + n0 + 1] = m1;
    ms.l[warp * kMaxGroup + n0] = l0;
    ms.l[warp * kMaxGroup + n0 + 1] = l1;
  }
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    const int d = mt * 16 + (lane >> 2);
    if (n0 < G) {
      ms.o[(warp * kMaxGroup + n0) * D + d] = o[mt][0];
      ms.o[(warp * kMaxGroup + n0) * D + d + 8] = o[mt][2];
    }
    if (n0 + 1 < G) {
      ms.o[(warp * kMaxGroup + n0 + 1) * D + d] = o[mt][1];
      ms.o[(warp * kMaxGroup + n0 + 1) * D + d + 8] = o[mt][3];
    }
  }
  __syncthreads();
  if (cta_failed) return;
  merge_and_store<NW, __nv_bfloat16>(p, ms, b, g, part, !SPLIT || r.final_write);
}

}  // namespace pa
