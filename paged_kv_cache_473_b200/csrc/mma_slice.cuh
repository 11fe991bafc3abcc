// One warp's attention over one 16-token slice held in shared memory, on the
// tensor cores (bf16 warp MMA, fp32 accumulation), and the per-warp online
// softmax state it updates.  Shared by the decode kernels.
//
// Shared-memory slice layout (as landed by TMA with 128-byte swizzle): K then V,
// each D/64 panels of [16 rows x 128 B]; 16-byte chunk c of row r sits at
// chunk c ^ (r & 7).
//
// With G <= 8 query heads of the group padded to 8 MMA columns:
//   S^T[16 tok x 8 heads] = K[16 x D] . Q^T[D x 8]          (D/16 MMAs)
//   online softmax over the slice (fp32, log2 domain, warp shuffles)
//   O^T[D x 8 heads]     += V^T[D x 16] . P^T[16 x 8]        (D/16 MMAs)
// K feeds the A operand straight from shared memory (ldmatrix), V^T through
// ldmatrix.trans, and P moves from the S accumulator layout to the B operand
// layout with movmatrix.trans, so it never touches shared memory.
#pragma once

#include "decode_common.cuh"
#include "ptx.cuh"

namespace pa {

constexpr int kPanelBytes = kSliceTokens * 128;  // 16 rows x 128 B

template <int D>
struct SliceBytes {
  static constexpr int kSlice = (D / 64) * kPanelBytes;  // K (or V) of one slice
  static constexpr int kStage = 2 * kSlice;             // K then V
};

// Lane n0 = 2*(lane%4) holds heads n0 and n0+1: running max (log2 domain), its
// partial sum over the tokens it saw, and O^T rows d = mt*16 + lane/4 (+8).
template <int D>
struct WarpAttn {
  float m0, m1, l0, l1;
  float o[D / 16][4];

  __device__ __forceinline__ void reset() {
    m0 = m1 = -CUDART_INF_F;
    l0 = l1 = 0.f;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  }

  // Lane partial sums -> per-head sums (lanes with the same lane%4 share heads).
  __device__ __forceinline__ void reduce_sums() {
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
  }

  // Write this warp's state into the merge buffer: m[warp*gs + h], l[...],
  // o[(warp*gs + h)*D + d] for the G real heads.  Call after reduce_sums().
  __device__ __forceinline__ void dump(float* m, float* l, float* ob, int warp, int gs, int G, int lane) const {
    const int n0 = 2 * (lane & 3);
    if (lane < 4) {
      if (n0 < G) {
        m[warp * gs + n0] = m0;
        l[warp * gs + n0] = l0;
      }
      if (n0 + 1 < G) {
        m[warp * gs + n0 + 1] = m1;
        l[warp * gs + n0 + 1] = l1;
      }
    }
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      const int d = mt * 16 + (lane >> 2);
      if (n0 < G) {
        ob[(warp * gs + n0) * D + d] = o[mt][0];
        ob[(warp * gs + n0) * D + d + 8] = o[mt][2];
      }
      if (n0 + 1 < G) {
        ob[(warp * gs + n0 + 1) * D + d] = o[mt][1];
        ob[(warp * gs + n0 + 1) * D + d + 8] = o[mt][3];
      }
    }
  }
};

// Q^T as the B operand of S^T = K Q^T: column n = lane / 4 is query head n of
// the group; heads >= G are zero.
template <int D>
__device__ __forceinline__ void load_q_frags(uint32_t (&qf)[D / 16][2], const __nv_bfloat16* q_group, int G,
                                             int lane) {
  const int n = lane >> 2;
  const __nv_bfloat16* qrow = q_group + (size_t)(n < G ? n : 0) * D;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const int c = kk * 16 + 2 * (lane & 3);
    qf[kk][0] = n < G ? *reinterpret_cast<const uint32_t*>(qrow + c) : 0u;
    qf[kk][1] = n < G ? *reinterpret_cast<const uint32_t*>(qrow + c + 8) : 0u;
  }
}

// Load one slice (cache rows [y, y+16) of K and of V) into the stage at `dst`
// with 2-D TMA tile loads, one 64-column panel per instruction.  The warp
// calls this together: lane 0 arms the stage's barrier with the byte count and
// lanes 0 .. 2*D/64-1 each issue one panel (issuing from several lanes at once
// costs about as much as one TMA instruction from one lane).  The loads carry
// an evict-first L2 hint: a decode reads each slice once (measured on B200:
// Llama-3-8B step 0.974 -> 1.00 and Gemma-2-2B 0.82 -> 0.87 of the HBM copy
// rate, the partials and tables staying in L2).  y < 0 (a bad block id) arms
// the barrier with no bytes and raises PA_DEVERR_BLOCK.
template <int D>
__device__ __forceinline__ void issue_slice(uint32_t dst, uint32_t bar, const CUtensorMap* kmap,
                                            const CUtensorMap* vmap, int y, int lane) {
  constexpr int kPanels = D / 64;
  if (y < 0) {
    if (lane == 0) {
      raise_error(PA_DEVERR_BLOCK);
      mbar_arrive(bar);  // complete the phase with no data; the slice computes on stale tiles
    }
    return;
  }
  if (lane == 0) mbar_arrive_expect_tx(bar, SliceBytes<D>::kStage);
  __syncwarp();
  if (lane < 2 * kPanels) {
    const int pn = lane % kPanels;
    const bool is_v = lane >= kPanels;
    tma_load_2d_hint(dst + (is_v ? SliceBytes<D>::kSlice : 0) + pn * kPanelBytes, is_v ? vmap : kmap, bar, pn * 64,
                     y, l2_policy_evict_first());
  }
}

// Overwrite row `row` (0..15) of the slice at kbase/vbase with the new key and
// value rows; lane l < D/8 holds 16-byte chunk l of each.
template <int D>
__device__ __forceinline__ void overwrite_slice_row(uint32_t kbase, uint32_t vbase, int row, const uint4& knew,
                                                    const uint4& vnew, int lane) {
  if (lane < D / 8) {
    const uint32_t off = (lane >> 3) * kPanelBytes + row * 128 + (((lane & 7) ^ (row & 7)) << 4);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(kbase + off), "r"(knew.x), "r"(knew.y),
                 "r"(knew.z), "r"(knew.w)
                 : "memory");
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(vbase + off), "r"(vnew.x), "r"(vnew.y),
                 "r"(vnew.z), "r"(vnew.w)
                 : "memory");
    fence_proxy_async_smem();  // before TMA writes this stage again
  }
  __syncwarp();
}

// Per-column token ranges of the lane's two columns n0, n0 + 1 (multi-query
// rows: each query token has its own causal end and window start).
struct ColRange {
  int lo0, hi0, lo1, hi1;
};

// Attend the slice of tokens [t0, t0+16) whose K/V rows sit at kbase/vbase;
// only tokens in [lo, hi) count.  COLS: column n0 (n0 + 1) of this lane only
// counts tokens in [cr.lo0, cr.hi0) ([cr.lo1, cr.hi1)), inside [lo, hi); a
// column may then see no token of the slice at all, which the safe maximum
// below turns into a zero weight.
template <int D, bool COLS = false>
__device__ __forceinline__ void attend_slice(WarpAttn<D>& st, const uint32_t (&qf)[D / 16][2], uint32_t kbase,
                                             uint32_t vbase, int t0, int lo, int hi, float qk_scale,
                                             const DecodeParams& p, int lane, const ColRange& cr = ColRange{}) {
  constexpr uint32_t FULL = 0xffffffffu;
  const uint32_t k_lane = ((lane & 7) | (lane & 8)) * 128;          // row = lane%8 + 8*((lane/8)%2)
  const uint32_t v_lane = ((lane & 7) | ((lane >> 4) << 3)) * 128;  // row = lane%8 + 8*(lane/16)
  const uint32_t k_sub = lane >> 4, v_sub = (lane >> 3) & 1, swz = lane & 7;

  // ---- S^T = K Q^T ---------------------------------------------------------
  float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t chunk = ((kk & 3) << 1) | k_sub;
    const uint32_t addr = kbase + (kk >> 2) * kPanelBytes + k_lane + ((chunk ^ swz) << 4);
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
  const bool partial = (t0 < lo) || (t0 + kSliceTokens > hi);
  uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;
  if (COLS) {
    const int ta = t0 + (lane >> 2), tb = ta + 8;
    if (!(ta >= cr.lo0 && ta < cr.hi0)) x[0] = -CUDART_INF_F;
    if (!(ta >= cr.lo1 && ta < cr.hi1)) x[1] = -CUDART_INF_F;
    if (!(tb >= cr.lo0 && tb < cr.hi0)) x[2] = -CUDART_INF_F;
    if (!(tb >= cr.lo1 && tb < cr.hi1)) x[3] = -CUDART_INF_F;
  }
  if (partial) {
    const int ta = t0 + (lane >> 2), tb = ta + 8;
    if (!COLS) {
      if (!(ta >= lo && ta < hi)) x[0] = x[1] = -CUDART_INF_F;
      if (!(tb >= lo && tb < hi)) x[2] = x[3] = -CUDART_INF_F;
    }
    // Tokens held by this lane in the V^T fragments: 2*(lane%4) (+1) and +8.
    const int tc = t0 + 2 * (lane & 3);
    auto ok = [&](int t) { return t >= lo && t < hi; };
    keep_lo = (ok(tc) ? 0x0000ffffu : 0u) | (ok(tc + 1) ? 0xffff0000u : 0u);
    keep_hi = (ok(tc + 8) ? 0x0000ffffu : 0u) | (ok(tc + 9) ? 0xffff0000u : 0u);
  }

  // ---- online softmax --------------------------------------------------------
  float mx0 = fmaxf(x[0], x[2]), mx1 = fmaxf(x[1], x[3]);
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, off));
    mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, off));
  }
  const float mn0 = fmaxf(st.m0, mx0), mn1 = fmaxf(st.m1, mx1);
  // Reference for the exponentials: the new maximum, or 0 for a column that
  // has seen no token yet (then every weight and the rescale factor are 0).
  const float r0 = (COLS && mn0 == -CUDART_INF_F) ? 0.f : mn0;
  const float r1 = (COLS && mn1 == -CUDART_INF_F) ? 0.f : mn1;
  const float al0 = exp2f(st.m0 - r0), al1 = exp2f(st.m1 - r1);
  st.m0 = mn0;
  st.m1 = mn1;
  const uint32_t plo = pack_bf16x2(exp2f(x[0] - r0), exp2f(x[1] - r1));
  const uint32_t phi = pack_bf16x2(exp2f(x[2] - r0), exp2f(x[3] - r1));
  st.l0 = st.l0 * al0 + bf16_lo(plo) + bf16_lo(phi);
  st.l1 = st.l1 * al1 + bf16_hi(plo) + bf16_hi(phi);
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    st.o[mt][0] *= al0;
    st.o[mt][1] *= al1;
    st.o[mt][2] *= al0;
    st.o[mt][3] *= al1;
  }
  const uint32_t pb0 = movmatrix_trans(plo);
  const uint32_t pb1 = movmatrix_trans(phi);

  // ---- O^T += V^T P^T ---------------------------------------------------------
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    const uint32_t chunk = ((mt & 3) << 1) | v_sub;
    const uint32_t addr = vbase + (mt >> 2) * kPanelBytes + v_lane + ((chunk ^ swz) << 4);
    uint32_t a0, a1, a2, a3;
    ldsm_x4_trans(addr, a0, a1, a2, a3);
    if (partial) {
      a0 &= keep_lo;
      a1 &= keep_lo;
      a2 &= keep_hi;
      a3 &= keep_hi;
    }
    mma_bf16_16816(st.o[mt], a0, a1, a2, a3, pb0, pb1);
  }
}

// Attend two consecutive slices, tokens [t0, t0+16) at kbase0/vbase0 and
// [t0+16, t0+32) at kbase1/vbase1, in one online-softmax step: the same
// arithmetic as attend_slice over a 32-token block (one running-maximum
// update, one rescale of o, one shuffle reduction for both slices), with the
// two S^T products independent of each other.  Only tokens in [lo, hi) count;
// each slice must hold at least one of them.
template <int D>
__device__ __forceinline__ void attend_pair(WarpAttn<D>& st, const uint32_t (&qf)[D / 16][2], uint32_t kbase0,
                                            uint32_t vbase0, uint32_t kbase1, uint32_t vbase1, int t0, int lo,
                                            int hi, float qk_scale, const DecodeParams& p, int lane) {
  constexpr uint32_t FULL = 0xffffffffu;
  const uint32_t k_lane = ((lane & 7) | (lane & 8)) * 128;
  const uint32_t v_lane = ((lane & 7) | ((lane >> 4) << 3)) * 128;
  const uint32_t k_sub = lane >> 4, v_sub = (lane >> 3) & 1, swz = lane & 7;

  // ---- S^T = K Q^T for both slices ---------------------------------------------
  float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * kPanelBytes + k_lane + (((((kk & 3) << 1) | k_sub) ^ swz) << 4);
    uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
    ldsm_x4(kbase0 + off, a0, a1, a2, a3);
    ldsm_x4(kbase1 + off, b0, b1, b2, b3);
    mma_bf16_16816(sc[0], a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
    mma_bf16_16816(sc[1], b0, b1, b2, b3, qf[kk][0], qf[kk][1]);
  }
  // sc[s][0], sc[s][1]: token t0 + 16 s + lane/4, heads n0, n0+1; [2], [3]: token + 8.
  float x[2][4];
#pragma unroll
  for (int s2 = 0; s2 < 2; ++s2) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float v = sc[s2][e] * qk_scale;
      if (p.use_softcap) v = p.softcap * tanhf(v * p.inv_softcap) * kLog2e;
      x[s2][e] = v;
    }
  }
  uint32_t keep_lo[2] = {0xffffffffu, 0xffffffffu}, keep_hi[2] = {0xffffffffu, 0xffffffffu};
  bool partial[2];
#pragma unroll
  for (int s2 = 0; s2 < 2; ++s2) {
    const int ts = t0 + s2 * kSliceTokens;
    partial[s2] = (ts < lo) || (ts + kSliceTokens > hi);
    if (partial[s2]) {
      const int ta = ts + (lane >> 2), tb = ta + 8;
      if (!(ta >= lo && ta < hi)) x[s2][0] = x[s2][1] = -CUDART_INF_F;
      if (!(tb >= lo && tb < hi)) x[s2][2] = x[s2][3] = -CUDART_INF_F;
      const int tc = ts + 2 * (lane & 3);
      auto ok = [&](int t) { return t >= lo && t < hi; };
      keep_lo[s2] = (ok(tc) ? 0x0000ffffu : 0u) | (ok(tc + 1) ? 0xffff0000u : 0u);
      keep_hi[s2] = (ok(tc + 8) ? 0x0000ffffu : 0u) | (ok(tc + 9) ? 0xffff0000u : 0u);
    }
  }

  // ---- online softmax over the 32 tokens ---------------------------------------
  float mx0 = fmaxf(fmaxf(x[0][0], x[0][2]), fmaxf(x[1][0], x[1][2]));
  float mx1 = fmaxf(fmaxf(x[0][1], x[0][3]), fmaxf(x[1][1], x[1][3]));
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, off));
    mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, off));
  }
  const float mn0 = fmaxf(st.m0, mx0), mn1 = fmaxf(st.m1, mx1);
  const float al0 = exp2f(st.m0 - mn0), al1 = exp2f(st.m1 - mn1);
  st.m0 = mn0;
  st.m1 = mn1;
  uint32_t plo[2], phi[2];
#pragma unroll
  for (int s2 = 0; s2 < 2; ++s2) {
    plo[s2] = pack_bf16x2(exp2f(x[s2][0] - mn0), exp2f(x[s2][1] - mn1));
    phi[s2] = pack_bf16x2(exp2f(x[s2][2] - mn0), exp2f(x[s2][3] - mn1));
  }
  st.l0 = st.l0 * al0 + ((bf16_lo(plo[0]) + bf16_lo(phi[0])) + (bf16_lo(plo[1]) + bf16_lo(phi[1])));
  st.l1 = st.l1 * al1 + ((bf16_hi(plo[0]) + bf16_hi(phi[0])) + (bf16_hi(plo[1]) + bf16_hi(phi[1])));
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    st.o[mt][0] *= al0;
    st.o[mt][1] *= al1;
    st.o[mt][2] *= al0;
    st.o[mt][3] *= al1;
  }
  uint32_t pb[2][2];
#pragma unroll
  for (int s2 = 0; s2 < 2; ++s2) {
    pb[s2][0] = movmatrix_trans(plo[s2]);
    pb[s2][1] = movmatrix_trans(phi[s2]);
  }

  // ---- O^T += V^T P^T, one k-step per slice -----------------------------------------
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    const uint32_t off = (mt >> 2) * kPanelBytes + v_lane + (((((mt & 3) << 1) | v_sub) ^ swz) << 4);
#pragma unroll
    for (int s2 = 0; s2 < 2; ++s2) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4_trans((s2 ? vbase1 : vbase0) + off, a0, a1, a2, a3);
      if (partial[s2]) {
        a0 &= keep_lo[s2];
        a1 &= keep_lo[s2];
        a2 &= keep_hi[s2];
        a3 &= keep_hi[s2];
      }
      mma_bf16_16816(st.o[mt], a0, a1, a2, a3, pb[s2][0], pb[s2][1]);
    }
  }
}

// ---- query rows as the MMA M dimension -------------------------------------------
//
// For several query tokens per sequence (multi-query rows) with R = T*G <= 16
// query rows per kv head, the rows fill the 16-row M dimension of the MMA:
//   S[16 rows x 16 tok] = Q[16 x D] . K^T          (2 n-tiles x D/16 MMAs)
//   online softmax per row (fp32, log2 domain, quad shuffles)
//   O[16 x D]          += P[16 x 16] . V[16 x D]     (D/8 n-tiles, one k-step)
// P goes from the S accumulators straight into the A operand of the second
// product (the accumulator and A-operand layouts of m16n8k16 line up), K^T
// is read with ldmatrix and V with ldmatrix.trans from the same swizzled
// stage as the head-column form.  Lane holds rows r0 = lane/4 and r1 = r0 + 8,
// and for each 8-column n-tile the columns 2*(lane%4) and +1.
template <int D>
struct WarpRows {
  float m0, m1, l0, l1;
  float o[D / 8][4];

  __device__ __forceinline__ void reset() {
    m0 = m1 = -CUDART_INF_F;
    l0 = l1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
  }

  // Lane partial sums -> row sums (the four lanes of a row share lane / 4).
  __device__ __forceinline__ void reduce_sums() {
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
  }
};

// Q as the A operand: rows r0, r1 of the 16 (rows >= R are zero); qrow0/qrow1
// point at the rows' query vectors.
template <int D>
__device__ __forceinline__ void load_q_rows(uint32_t (&qa)[D / 16][4], const __nv_bfloat16* qrow0, bool ok0,
                                            const __nv_bfloat16* qrow1, bool ok1, int lane) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const int c = kk * 16 + 2 * (lane & 3);
    qa[kk][0] = ok0 ? *reinterpret_cast<const uint32_t*>(qrow0 + c) : 0u;
    qa[kk][1] = ok1 ? *reinterpret_cast<const uint32_t*>(qrow1 + c) : 0u;
    qa[kk][2] = ok0 ? *reinterpret_cast<const uint32_t*>(qrow0 + c + 8) : 0u;
    qa[kk][3] = ok1 ? *reinterpret_cast<const uint32_t*>(qrow1 + c + 8) : 0u;
  }
}

// Attend the slice of tokens [t0, t0+16) at kbase/vbase for the lane's rows:
// row r0 counts tokens in [cr.lo0, cr.hi0), row r1 in [cr.lo1, cr.hi1); V rows
// outside [lo, hi) (the union) are zeroed.  A row may see no token of the
// slice; the safe reference maximum keeps its weights at zero.
template <int D>
__device__ __forceinline__ void attend_slice_rows(WarpRows<D>& st, const uint32_t (&qa)[D / 16][4], uint32_t kbase,
                                                  uint32_t vbase, int t0, int lo, int hi, const ColRange& cr,
                                                  float qk_scale, const DecodeParams& p, int lane) {
  constexpr uint32_t FULL = 0xffffffffu;
  const int mi = lane >> 3, mj = lane & 7;  // the ldmatrix row this lane addresses: matrix mi, row mj
  const int tq = lane & 3;

  // ---- S = Q K^T: n-tiles 0 (tokens 0-7) and 1 (tokens 8-15) -------------------------
  float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  {
    // matrix mi: tokens (mi >> 1) * 8 + mj, 16-byte chunk 2*kk + (mi & 1)
    const int tok = ((mi >> 1) << 3) | mj;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int chunk = 2 * kk + (mi & 1);
      const uint32_t addr =
          kbase + (chunk >> 3) * kPanelBytes + tok * 128 + ((((chunk & 7) ^ (tok & 7))) << 4);
      uint32_t b00, b01, b10, b11;
      ldsm_x4(addr, b00, b01, b10, b11);
      mma_bf16_16816(s[0], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b00, b01);
      mma_bf16_16816(s[1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b10, b11);
    }
  }
  // s[nt][0..1]: row r0, tokens t0 + 8 nt + 2 tq (+1); s[nt][2..3]: row r1.
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float v = s[nt][e] * qk_scale;
      if (p.use_softcap) v = p.softcap * tanhf(v * p.inv_softcap) * kLog2e;
      const int t = t0 + 8 * nt + 2 * tq + (e & 1);
      const bool ok = e < 2 ? (t >= cr.lo0 && t < cr.hi0) : (t >= cr.lo1 && t < cr.hi1);
      s[nt][e] = ok ? v : -CUDART_INF_F;
    }

  // ---- online softmax per row -----------------------------------------------------
  float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
  float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
#pragma unroll
  for (int off = 1; off < 4; off <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, off));
    mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, off));
  }
  const float mn0 = fmaxf(st.m0, mx0), mn1 = fmaxf(st.m1, mx1);
  const float r0 = mn0 == -CUDART_INF_F ? 0.f : mn0;
  const float r1 = mn1 == -CUDART_INF_F ? 0.f : mn1;
  const float al0 = exp2f(st.m0 - r0), al1 = exp2f(st.m1 - r1);
  st.m0 = mn0;
  st.m1 = mn1;
  // P as the A operand of P V (16 rows x 16 tokens).
  const uint32_t a0 = pack_bf16x2(exp2f(s[0][0] - r0), exp2f(s[0][1] - r0));
  const uint32_t a1 = pack_bf16x2(exp2f(s[0][2] - r1), exp2f(s[0][3] - r1));
  const uint32_t a2 = pack_bf16x2(exp2f(s[1][0] - r0), exp2f(s[1][1] - r0));
  const uint32_t a3 = pack_bf16x2(exp2f(s[1][2] - r1), exp2f(s[1][3] - r1));
  st.l0 = st.l0 * al0 + bf16_lo(a0) + bf16_hi(a0) + bf16_lo(a2) + bf16_hi(a2);
  st.l1 = st.l1 * al1 + bf16_lo(a1) + bf16_hi(a1) + bf16_lo(a3) + bf16_hi(a3);
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) {
    st.o[nt][0] *= al0;
    st.o[nt][1] *= al0;
    st.o[nt][2] *= al1;
    st.o[nt][3] *= al1;
  }

  // V rows outside [lo, hi) may hold anything (NaN canaries): zero them.  This
  // lane's B fragments hold tokens 2 tq, 2 tq + 1 (b0) and 8 + 2 tq, + 1 (b1).
  uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;
  if (t0 < lo || t0 + kSliceTokens > hi) {
    const int tc = t0 + 2 * tq;
    auto ok = [&](int t) { return t >= lo && t < hi; };
    keep_lo = (ok(tc) ? 0x0000ffffu : 0u) | (ok(tc + 1) ? 0xffff0000u : 0u);
    keep_hi = (ok(tc + 8) ? 0x0000ffffu : 0u) | (ok(tc + 9) ? 0xffff0000u : 0u);
  }

  // ---- O += P V: d n-tiles in pairs (2c, 2c+1) ------------------------------------------
  {
    // matrix mi: tokens (mi & 1) * 8 + mj, 16-byte chunk 2c + (mi >> 1)
    const int tok = ((mi & 1) << 3) | mj;
#pragma unroll
    for (int c = 0; c < D / 16; ++c) {
      const int chunk = 2 * c + (mi >> 1);
      const uint32_t addr =
          vbase + (chunk >> 3) * kPanelBytes + tok * 128 + ((((chunk & 7) ^ (tok & 7))) << 4);
      uint32_t v0, v1, v2, v3;
      ldsm_x4_trans(addr, v0, v1, v2, v3);
      mma_bf16_16816(st.o[2 * c], a0, a1, a2, a3, v0 & keep_lo, v1 & keep_hi);
      mma_bf16_16816(st.o[2 * c + 1], a0, a1, a2, a3, v2 & keep_lo, v3 & keep_hi);
    }
  }
}

// attend_slice_rows over two consecutive slices, tokens [t0, t0+16) at
// kbase0/vbase0 and [t0+16, t0+32) at kbase1/vbase1, in one online-softmax
// step: one row maximum, one rescale of o and one running-sum update per 32
// tokens, the two S products independent of each other, and O += P V as two
// k-steps.  Same per-row bounds as attend_slice_rows.
template <int D>
__device__ __forceinline__ void attend_pair_rows(WarpRows<D>& st, const uint32_t (&qa)[D / 16][4], uint32_t kbase0,
                                                 uint32_t vbase0, uint32_t kbase1, uint32_t vbase1, int t0, int lo,
                                                 int hi, const ColRange& cr, float qk_scale, const DecodeParams& p,
                                                 int lane) {
  constexpr uint32_t FULL = 0xffffffffu;
  const int mi = lane >> 3, mj = lane & 7;
  const int tq = lane & 3;

  // ---- S = Q K^T for both slices: s[slice][n-tile][4] ----------------------------------
  float s[2][2][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 2; ++b) s[a][b][0] = s[a][b][1] = s[a][b][2] = s[a][b][3] = 0.f;
  {
    const int tok = ((mi >> 1) << 3) | mj;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int chunk = 2 * kk + (mi & 1);
      const uint32_t off = (chunk >> 3) * kPanelBytes + tok * 128 + ((((chunk & 7) ^ (tok & 7))) << 4);
      uint32_t b00, b01, b10, b11, c00, c01, c10, c11;
      ldsm_x4(kbase0 + off, b00, b01, b10, b11);
      ldsm_x4(kbase1 + off, c00, c01, c10, c11);
      mma_bf16_16816(s[0][0], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b00, b01);
      mma_bf16_16816(s[0][1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b10, b11);
      mma_bf16_16816(s[1][0], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], c00, c01);
      mma_bf16_16816(s[1][1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], c10, c11);
    }
  }
#pragma unroll
  for (int sl = 0; sl < 2; ++sl)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = s[sl][nt][e] * qk_scale;
        if (p.use_softcap) v = p.softcap * tanhf(v * p.inv_softcap) * kLog2e;
        const int t = t0 + 16 * sl + 8 * nt + 2 * tq + (e & 1);
        const bool ok = e < 2 ? (t >= cr.lo0 && t < cr.hi0) : (t >= cr.lo1 && t < cr.hi1);
        s[sl][nt][e] = ok ? v : -CUDART_INF_F;
      }

  // ---- online softmax per row over the 32 tokens -------------------------------------
  float mx0 = -CUDART_INF_F, mx1 = -CUDART_INF_F;
#pragma unroll
  for (int sl = 0; sl < 2; ++sl)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      mx0 = fmaxf(mx0, fmaxf(s[sl][nt][0], s[sl][nt][1]));
      mx1 = fmaxf(mx1, fmaxf(s[sl][nt][2], s[sl][nt][3]));
    }
#pragma unroll
  for (int off = 1; off < 4; off <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, off));
    mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, off));
  }
  const float mn0 = fmaxf(st.m0, mx0), mn1 = fmaxf(st.m1, mx1);
  const float r0 = mn0 == -CUDART_INF_F ? 0.f : mn0;
  const float r1 = mn1 == -CUDART_INF_F ? 0.f : mn1;
  const float al0 = exp2f(st.m0 - r0), al1 = exp2f(st.m1 - r1);
  st.m0 = mn0;
  st.m1 = mn1;
  uint32_t a[2][4];  // P of each slice as the A operand of P V
#pragma unroll
  for (int sl = 0; sl < 2; ++sl) {
    a[sl][0] = pack_bf16x2(exp2f(s[sl][0][0] - r0), exp2f(s[sl][0][1] - r0));
    a[sl][1] = pack_bf16x2(exp2f(s[sl][0][2] - r1), exp2f(s[sl][0][3] - r1));
    a[sl][2] = pack_bf16x2(exp2f(s[sl][1][0] - r0), exp2f(s[sl][1][1] - r0));
    a[sl][3] = pack_bf16x2(exp2f(s[sl][1][2] - r1), exp2f(s[sl][1][3] - r1));
  }
  st.l0 = st.l0 * al0 + ((bf16_lo(a[0][0]) + bf16_hi(a[0][0]) + bf16_lo(a[0][2]) + bf16_hi(a[0][2])) +
                         (bf16_lo(a[1][0]) + bf16_hi(a[1][0]) + bf16_lo(a[1][2]) + bf16_hi(a[1][2])));
  st.l1 = st.l1 * al1 + ((bf16_lo(a[0][1]) + bf16_hi(a[0][1]) + bf16_lo(a[0][3]) + bf16_hi(a[0][3])) +
                         (bf16_lo(a[1][1]) + bf16_hi(a[1][1]) + bf16_lo(a[1][3]) + bf16_hi(a[1][3])));
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) {
    st.o[nt][0] *= al0;
    st.o[nt][1] *= al0;
    st.o[nt][2] *= al1;
    st.o[nt][3] *= al1;
  }

  // V rows outside [lo, hi) may hold anything (NaN canaries): zero them.
  uint32_t keep_lo[2] = {0xffffffffu, 0xffffffffu}, keep_hi[2] = {0xffffffffu, 0xffffffffu};
#pragma unroll
  for (int sl = 0; sl < 2; ++sl) {
    const int ts = t0 + 16 * sl;
    if (ts < lo || ts + kSliceTokens > hi) {
      const int tc = ts + 2 * tq;
      auto ok = [&](int t) { return t >= lo && t < hi; };
      keep_lo[sl] = (ok(tc) ? 0x0000ffffu : 0u) | (ok(tc + 1) ? 0xffff0000u : 0u);
      keep_hi[sl] = (ok(tc + 8) ? 0x0000ffffu : 0u) | (ok(tc + 9) ? 0xffff0000u : 0u);
    }
  }

  // ---- O += P V, one k-step per slice ----------------------------------------------------
  {
    const int tok = ((mi & 1) << 3) | mj;
#pragma unroll
    for (int c = 0; c < D / 16; ++c) {
      const int chunk = 2 * c + (mi >> 1);
      const uint32_t off = (chunk >> 3) * kPanelBytes + tok * 128 + ((((chunk & 7) ^ (tok & 7))) << 4);
#pragma unroll
      for (int sl = 0; sl < 2; ++sl) {
        uint32_t v0, v1, v2, v3;
        ldsm_x4_trans((sl ? vbase1 : vbase0) + off, v0, v1, v2, v3);
        mma_bf16_16816(st.o[2 * c], a[sl][0], a[sl][1], a[sl][2], a[sl][3], v0 & keep_lo[sl], v1 & keep_hi[sl]);
        mma_bf16_16816(st.o[2 * c + 1], a[sl][0], a[sl][1], a[sl][2], a[sl][3], v2 & keep_lo[sl],
                       v3 & keep_hi[sl]);
      }
    }
  }
}

}  // namespace pa
