// Paged decode attention, bf16, tensor cores: the grid-scheduled kernel.
//
// One CTA serves one (partition, kv head, sequence).  Each of its NW warps
// owns every NW-th 16-token slice of the CTA's token range and runs its own
// ST-deep ring of shared-memory stages: lane 0 issues 2-D TMA tile loads of the
// slice's K and V rows (a slice lies inside one physical block, found through
// the block table), completion is counted on a per-stage mbarrier, and the
// warp computes on a stage (attend_slice) while later ones are in flight.
// Warps never wait on one another until the final merge.  The block-table
// entries of a warp's next 32 slices sit one per lane in a register, so
// refilling a stage costs no dependent global load.
//
// APPEND (the fused decode step): the CTA whose range ends at the sequence's
// last token also appends the step's new key/value row: it writes the row to
// the cache slot of position L-1 and, in shared memory, over the stale row the
// TMA load brought for that position, so the attention uses the new row.
#pragma once

#include "decode_common.cuh"
#include "mma_slice.cuh"
#include "ptx.cuh"

namespace pa {

template <int D, int NW, int ST>
struct MmaCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kSliceBytes = SliceBytes<D>::kSlice;
  static constexpr int kStageBytes = SliceBytes<D>::kStage;
  static constexpr int kRingBytes = NW * ST * kStageBytes;
  static constexpr int kBarOffset = kRingBytes;
  static constexpr int kSmemBytes = kRingBytes + NW * ST * 8 + 1024;  // + barriers + alignment slack
  static_assert(merge_smem_bytes<NW>(D) <= kRingBytes, "merge buffer must fit in the ring");
  static_assert(D % 64 == 0, "head_dim must be a multiple of 64");
};

template <int D, int NW, int ST, bool SPLIT, bool APPEND>
__global__ void __launch_bounds__(NW * 32)
    decode_mma_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                      const DecodeParams p) {
  using Cfg = MmaCfg<D, NW, ST>;
  constexpr uint32_t FULL = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  // The combine kernel (a programmatic dependent) may start its launch now; it
  // waits for this grid to finish before it reads anything.
  if (SPLIT) pdl_launch_dependents();

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

  // Block ids of this warp's slices [base, base + 32), one per lane.
  int pg = -1;
  auto load_pages = [&](int base) {
    const int i = base + lane;
    pg = (i < n_w) ? table[((j0 + warp + NW * i) * kSliceTokens) >> p.log2_bs] : -1;
  };
  load_pages(0);

  // Fused append: which warp and local slice index hold position L-1.
  const int j_last = (r.L - 1) / kSliceTokens;
  const bool append_cta = APPEND && r.hi == r.L;
  const bool append_warp = append_cta && ((j_last - j0) % NW) == warp;
  const int i_last = append_warp ? (j_last - j0) / NW : -1;

  // Issue the TMA loads of this warp's i-th slice into stage i % ST.  Called
  // by the whole warp, for i = 0, 1, 2, ... in order.
  auto issue = [&](int i) {
    if (i > 0 && (i & 31) == 0) load_pages(i);
    const int phys = __shfl_sync(FULL, pg, i & 31);
    const int t = (j0 + warp + NW * i) * kSliceTokens;
    const int y = (phys >= 0 && phys < p.num_blocks) ? cache_row(p, phys, g, t) : -1;
    issue_slice<D>(ring + (i % ST) * Cfg::kStageBytes, bars + 8 * (i % ST), &kmap, &vmap, y, lane);
  };
  for (int i = 0; i < ST && i < n_w; ++i) issue(i);

  uint32_t qf[D / 16][2];
  load_q_frags<D>(qf, static_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.hq + (size_t)g * G) * D, G, lane);

  // The appended rows: one 16-byte chunk of K and of V per lane (lanes < D/8).
  uint4 knew = make_uint4(0, 0, 0, 0), vnew = make_uint4(0, 0, 0, 0);
  if (append_warp && lane < D / 8) {
    const size_t off = ((size_t)b * p.hkv + g) * D + lane * 8;
    knew = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.k_new) + off);
    vnew = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.v_new) + off);
    const int phys = table[(r.L - 1) >> p.log2_bs];
    if (phys >= 0 && phys < p.num_blocks) {
      const size_t dst = (size_t)cache_row(p, phys, g, r.L - 1) * D + lane * 8;
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(const_cast<void*>(p.k_cache)) + dst) = knew;
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(const_cast<void*>(p.v_cache)) + dst) = vnew;
    }
  }

  WarpAttn<D> st;
  st.reset();
  const float qk_scale = p.use_softcap ? p.scale : p.scale * kLog2e;

  bool failed = false;
  int i_done = 0;
  for (int i = 0; i < n_w; ++i) {
    const int s = i % ST;
    bool ok = mbar_wait_bounded(bars + 8 * s, (i / ST) & 1, kWaitLimitNs);
    ok = __all_sync(FULL, ok);
    if (!ok) {
      failed = true;
      break;
    }
    i_done = i + 1;
    const uint32_t kbase = ring + s * Cfg::kStageBytes;
    const uint32_t vbase = kbase + Cfg::kSliceBytes;
    const int t0 = (j0 + warp + NW * i) * kSliceTokens;
    if (APPEND && i == i_last) overwrite_slice_row<D>(kbase, vbase, (r.L - 1) & (kSliceTokens - 1), knew, vnew, lane);
    attend_slice<D>(st, qf, kbase, vbase, t0, r.lo, r.hi, qk_scale, p, lane);
    __syncwarp();
    if (i + ST < n_w) issue(i + ST);
  }

  if (failed) {
    raise_error(PA_DEVERR_TIMEOUT);
    // Let this warp's loads still in flight land before the CTA exits.
    for (int i = i_done; i < n_w && i < i_done + ST; ++i)
      (void)mbar_wait_bounded(bars + 8 * (i % ST), (i / ST) & 1, kDrainLimitNs);
  }
  st.reduce_sums();

  __shared__ int cta_failed;
  if (threadIdx.x == 0) cta_failed = 0;
  __syncthreads();  // every warp is done with its ring: reuse it for the merge
  if (failed && lane == 0) cta_failed = 1;

  const MergeSmem ms = merge_smem<NW>(smem, D);
  st.dump(ms.m, ms.l, ms.o, warp, ms.gs, G, lane);
  __syncthreads();
  if (cta_failed) return;
  merge_warps<NW, __nv_bfloat16>(ms, G, D, grid_dest<__nv_bfloat16>(p, b, g, part, !SPLIT || r.final_write),
                                 threadIdx.x, blockDim.x);
}

}  // namespace pa
