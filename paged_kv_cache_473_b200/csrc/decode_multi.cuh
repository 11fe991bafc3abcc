// Multi-query paged attention, bf16, tensor cores: T query tokens per sequence
// (speculative-decoding verify, a chunk of a chunked prefill) whose keys and
// values are already in the cache at positions L-T .. L-1.  Query token j sits
// at position p_j = L - T + j and attends the positions [s0_j, p_j + 1) of its
// sequence (causal; s0_j is the sliding-window start).
//
// One CTA per (partition, kv head, sequence).  The T*G query rows of the kv
// head are the N columns of the attention tile, token-major (column
// c = j*G + h); warp w owns columns [8w, 8w + 8) and runs the decode slice
// attention (attend_slice) on them with per-column causal / window bounds.
// Every warp needs every key and value of the range, so the K/V slices are
// loaded once per CTA into a shared ring of ST stages: warp 0 issues the 2-D
// TMA tile loads (full barrier per stage, with the byte count), every warp
// consumes a stage and arrives on the stage's empty barrier, and warp 0 waits
// for that before it refills the stage.  Each warp writes its own columns:
// the normalised rows when the sequence's range is one partition, else the
// partial state for the combine kernel.
//
// Cascade prefix pass (p.cascade_prefix): the same kernel with sharer columns
// (sequence x head) over the shared prefix, addressed through sequence 0's
// table.
#pragma once

#include "decode_common.cuh"
#include "mma_slice.cuh"
#include "ptx.cuh"

namespace pa {

constexpr int kMaxMultiColumns = 64;  // T * G query rows per kv head: 8 warps of 8 columns

template <int D, int ST>
struct MultiCfg {
  static constexpr int kSliceBytes = SliceBytes<D>::kSlice;
  static constexpr int kStageBytes = SliceBytes<D>::kStage;
  static constexpr int kRingBytes = ST * kStageBytes;
  static constexpr int kFullOffset = kRingBytes;           // ST full barriers
  static constexpr int kEmptyOffset = kRingBytes + ST * 8;  // ST empty barriers
  static constexpr int kSmemBytes = kRingBytes + 2 * ST * 8 + 1024;
};

// One query column of the CTA: its output (or workspace) row, its token range
// inside the CTA's partition, and whether it writes the normalised row itself.
struct QueryCol {
  size_t row;
  int lo, hi;
  bool fin;
  bool real;  // false: a padding column (no query, no output)
};

template <int D, int ST, bool SPLIT>
__global__ void __launch_bounds__(kMaxMultiColumns / 8 * 32)
    decode_multi_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                        const DecodeParams p) {
  using Cfg = MultiCfg<D, ST>;
  constexpr uint32_t FULL = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  if (SPLIT) pdl_launch_dependents();  // the combine may launch; it waits for this grid to finish

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NW = blockDim.x >> 5;
  const int g = blockIdx.y;
  const int G = p.group, P = p.partition;
  const bool cascade = p.cascade_prefix != 0;

  // ---- the CTA's K/V range and its query columns ---------------------------------------
  // kv_seq: the sequence whose block table addresses the K/V; [pl, ph): the
  // partition; [ulo, uhi): the positions any column may attend in it (all of
  // them valid cache rows); ncols: real query columns.
  int part = SPLIT ? (int)blockIdx.x : 0;
  int kv_seq, ncols, ulo, uhi;
  int T = 0, j0 = 0, L = 0, n_parts = 0, sbase = 0;
  size_t row0 = 0;
  if (cascade) {
    // Columns: sharer sequences sbase .. x G heads; the K/V are the shared
    // prefix, addressed through the first sharer's table.
    sbase = blockIdx.z * p.q_tile;
    ncols = min(p.q_tile, p.n_sharers - sbase) * G;
    kv_seq = 0;
    if (ncols <= 0) return;
    ulo = part * P;
    uhi = min(ulo + P, p.prefix_len);
  } else {
    kv_seq = blockIdx.z;
    T = p.q_len;
    row0 = (size_t)kv_seq * T;
    const int ntok = T;
    if (ntok <= 0) return;
    ncols = ntok * G;
    L = clamp_context(p, kv_seq, threadIdx.x == 0 && part == 0 && j0 == 0);
    // The union of the tile's ranges is [s0 of its first token, p of its last + 1).
    const int uend = min(L, L - T + j0 + ntok);
    const int ulo_seq = window_start(max(L - T + j0 + 1, 0), p.window);
    n_parts = (uend > ulo_seq) ? (uend + P - 1) / P - ulo_seq / P : 0;
    ulo = max(ulo_seq, part * P);
    uhi = min(uend, part * P + P);
    if (ulo >= uhi) {  // nothing of this sequence falls in this partition
      if (n_parts == 0 && part == 0) {  // no position for any token: zero rows for every query column
        for (int idx = threadIdx.x; idx < ncols * D; idx += blockDim.x) {
          const int c = idx / D;
          static_cast<__nv_bfloat16*>(p.out)[((row0 + c / G) * p.hq + (size_t)g * G + c % G) * D + idx % D] =
              __float2bfloat16_rn(0.f);
        }
      }
      return;
    }
  }
  const int pl = part * P, ph = pl + P;
  const bool cta_final = !SPLIT || n_parts == 1;

  // Column c < ncols.  Token columns (multi-query rows, prefill tiles): token
  // j0 + c / G at position p = L - T + j0 + c / G attends [s0(p + 1), p + 1).
  // Sharer columns (cascade): sequence b = sbase + c / G attends its
  // positions below the prefix length; it writes its row itself only when
  // its whole range is this one partition (or it has no position at all).
  auto column = [&](int c) -> QueryCol {
    QueryCol q;
    const int h = c % G;
    q.real = true;
    if (cascade) {
      const int b = sbase + c / G;
      const int Lb = clamp_context(p, b, false);
      const int s0 = window_start(Lb, p.window);
      const int nb = Lb > s0 ? (Lb + P - 1) / P - s0 / P : 0;
      q.row = (size_t)b * p.hq + (size_t)g * G + h;
      q.lo = max(s0, pl);
      q.hi = min(min(Lb, p.prefix_len), ph);
      q.fin = (nb == 1 && part == s0 / P) || (nb == 0 && part == 0);
    } else {
      const int end = L - T + j0 + c / G + 1;  // p + 1
      q.row = (row0 + c / G) * p.hq + (size_t)g * G + h;
      q.lo = max(window_start(max(end, 0), p.window), pl);
      q.hi = min(end, ph);
      q.fin = cta_final;
    }
    return q;
  };

  // This lane's two accumulator columns and their ranges (padding columns take
  // the union, so that their discarded softmax stays finite).
  const int n0 = 2 * (lane & 3);
  const int c0 = warp * 8 + n0;
  QueryCol qc[2];
  ColRange cr;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    if (c0 + e < ncols) {
      qc[e] = column(c0 + e);
    } else {
      qc[e].row = 0;
      qc[e].lo = ulo;
      qc[e].hi = uhi;
      qc[e].fin = false;
      qc[e].real = false;
    }
  }
  cr.lo0 = qc[0].lo;
  cr.hi0 = qc[0].hi;
  cr.lo1 = qc[1].lo;
  cr.hi1 = qc[1].hi;
  if (cascade && lane < 4) {
    // Every sharer must map the prefix to the same blocks as the first one.
    const int32_t* ref = p.block_tables + (size_t)kv_seq * p.max_blocks;
    for (int e = 0; e < 2; ++e) {
      if (c0 + e >= ncols || (c0 + e) % G) continue;
      const int b = sbase + (c0 + e) / G;
      const int32_t* tb = p.block_tables + (size_t)b * p.max_blocks;
      for (int t = ulo; t < uhi; t += p.block_size)
        if (tb[t >> p.log2_bs] != ref[t >> p.log2_bs]) raise_error(PA_DEVERR_BLOCK);
    }
  }

  const uint32_t ring = smem_addr(smem);
  const uint32_t full = smem_addr(smem + Cfg::kFullOffset);
  const uint32_t empty = smem_addr(smem + Cfg::kEmptyOffset);
  if (threadIdx.x == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
#pragma unroll
    for (int s = 0; s < ST; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, NW);
    }
    mbar_init_fence();
  }
  __syncthreads();

  const int js = ulo / kSliceTokens;  // first 16-token slice
  const int n = (uhi + kSliceTokens - 1) / kSliceTokens - js;

  // Warp 0 issues slice i into stage i % ST.
  const int32_t* table = p.block_tables + (size_t)kv_seq * p.max_blocks;
  auto issue = [&](int i) {
    const int t = (js + i) * kSliceTokens;
    const int phys = table[t >> p.log2_bs];
    const int y = (phys >= 0 && phys < p.num_blocks) ? cache_row(p, phys, g, t) : -1;
    issue_slice<D>(ring + (i % ST) * Cfg::kStageBytes, full + 8 * (i % ST), &kmap, &vmap, y, lane);
  };
  int issued = 0;
  if (warp == 0)
    for (; issued < ST && issued < n; ++issued) issue(issued);

  // Q^T as the B operand: column n = lane / 4 of the warp's 8 is query column
  // 8*warp + n, whose query row is its output row; padding columns are zero.
  uint32_t qf[D / 16][2];
  {
    const int c = warp * 8 + (lane >> 2);
    const QueryCol qcol = c < ncols ? column(c) : QueryCol{0, 0, 0, false, false};
    const bool real = qcol.real;
    const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(p.q) + (real ? qcol.row : 0) * D;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int d = kk * 16 + 2 * (lane & 3);
      qf[kk][0] = real ? *reinterpret_cast<const uint32_t*>(qrow + d) : 0u;
      qf[kk][1] = real ? *reinterpret_cast<const uint32_t*>(qrow + d + 8) : 0u;
    }
  }

  WarpAttn<D> st;
  st.reset();
  const float qk_scale = p.use_softcap ? p.scale : p.scale * kLog2e;
  bool failed = false;
  int i = 0;
  for (; i < n; ++i) {
    const int s = i % ST;
    const uint32_t par = (i / ST) & 1;
    bool ok = mbar_wait_bounded(full + 8 * s, par, kWaitLimitNs);
    ok = __all_sync(FULL, ok);
    if (!ok) {
      failed = true;
      break;
    }
    const uint32_t kbase = ring + s * Cfg::kStageBytes;
    attend_slice<D, true>(st, qf, kbase, kbase + Cfg::kSliceBytes, (js + i) * kSliceTokens, ulo, uhi, qk_scale, p,
                          lane, cr);
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + 8 * s);
    if (warp == 0 && issued < n) {  // refill this stage once every warp has released it
      ok = mbar_wait_bounded(empty + 8 * s, par, kWaitLimitNs);
      ok = __all_sync(FULL, ok);
      if (!ok) {
        failed = true;
        ++i;
        break;
      }
      issue(issued++);
    }
  }

  if (failed) {
    if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
    // Warp 0 owns the loads: let those still in flight land before the CTA exits.
    if (warp == 0)
      for (int k = i; k < issued; ++k) (void)mbar_wait_bounded(full + 8 * (k % ST), (k / ST) & 1, kDrainLimitNs);
    return;
  }
  st.reduce_sums();

  // ---- this warp's columns: final rows or partials, from registers -----------------
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    if (!qc[e].real) continue;
    const float m = e ? st.m1 : st.m0;
    const float l = e ? st.l1 : st.l0;
    const size_t row = qc[e].row;
    if (qc[e].fin) {
      const float inv = l > 0.f ? 1.f / l : 0.f;  // a column with no position gives a zero row
      __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + row * D;
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        const int d = mt * 16 + (lane >> 2);
        o[d] = __float2bfloat16_rn(st.o[mt][e] * inv);
        o[d + 8] = __float2bfloat16_rn(st.o[mt][2 + e] * inv);
      }
    } else {
      float* po = p.ws_o + (row * p.max_parts + part) * D;
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        const int d = mt * 16 + (lane >> 2);
        po[d] = st.o[mt][e];
        po[d + 8] = st.o[mt][2 + e];
      }
      if (lane < 4) {
        float* pml = p.ws_ml + (row * p.max_parts + part) * 2;
        pml[0] = m;
        pml[1] = l;
      }
    }
  }
}

}  // namespace pa
