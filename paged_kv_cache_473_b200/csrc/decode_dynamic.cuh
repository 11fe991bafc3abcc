// Paged decode attention, bf16, tensor cores: the dynamic (work-queue) split-K
// schedule.
//
// Work items are the non-empty (sequence b, kv head g, partition) triples of
// the split-K decomposition: partition p of sequence b covers tokens
// [p*P, p*P + P) of its attended range [s0, L).  The grid is persistent (as
// many CTAs as fit on the GPU at once); every CTA claims items one at a time
// from a counter in the workspace (atomicAdd), so CTAs on SMs that stream
// faster simply take more items and all finish together.  Items are numbered
// sequence-major: every CTA first builds, with block-wide scans over
// context_lens, the number of items before each sequence, and decodes an item
// number with a binary search in shared memory.
//
// Inside a CTA, warp w takes the item's 16-token slices k with k mod NW == w
// and runs its own ST-deep ring of TMA-filled stages (as the grid-scheduled
// kernel does).  The next item is claimed while the current one is processed,
// so a warp whose share of the current item is issued already loads the next
// item's slices while the CTA merges the current one: the ring stays full
// across item boundaries.  At the end of each item the warps merge their
// softmax states through shared memory; items that cover a whole sequence
// range are normalised and written, the others leave their partial state in
// the [B][Hq][max_parts] workspace for the combine kernel, which also resets
// the counter for the next call.
//
// APPEND (the fused decode step): the item that ends at the sequence's last
// token writes the step's new key/value row to the cache slot of position L-1
// and over the stale row in shared memory.
#pragma once

#include "decode_common.cuh"
#include "mma_slice.cuh"
#include "ptx.cuh"

namespace pa {

constexpr int kMaxDynamicBatch = 2048;  // prefix arrays live in shared memory

// Block-wide exclusive scan over all threads (blockDim.x a multiple of 32).
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  __syncthreads();
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  int before = 0;
  total = 0;
  for (int w = 0; w < nw; ++w) {
    if (w < warp) before += scratch[w];
    total += scratch[w];
  }
  return before + incl - v;
}

__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Partitions of sequence b's attended range [s0, L) (0 when it is empty).
__device__ __forceinline__ int seq_parts(int L, int s0, int P) { return L > s0 ? (L + P - 1) / P - s0 / P : 0; }

struct Item {
  int b, g, part;  // sequence, kv head, absolute partition index
  int L, lo, hi;   // context length; attended tokens [lo, hi) of this item
  int j0, n;       // first 16-token slice and number of slices
  bool whole;      // the item is the sequence's only partition
};

template <int D, int NW, int ST>
struct DynCfg {
  static constexpr int kStageBytes = SliceBytes<D>::kStage;
  static constexpr int kSliceBytes = SliceBytes<D>::kSlice;
  static constexpr int kRingBytes = NW * ST * kStageBytes;
  static constexpr int kThreads = NW * 32;
  // After the 1024-aligned ring: barriers, claim slots, scratch, merge buffer, prefix arrays.
  static constexpr int kBarOffset = kRingBytes;
  static constexpr int kSlotOffset = kBarOffset + NW * ST * 8;  // 2 x {seq, item}
  static constexpr int kScratchOffset = kSlotOffset + 16;
  static constexpr int kMergeOffset = kScratchOffset + 32 * 4;
  static __host__ __device__ constexpr int merge_bytes(int G) { return merge_smem_bytes<NW>(D, G); }
  static __host__ __device__ constexpr int prefix_offset(int G) { return kMergeOffset + merge_bytes(G); }
  static __host__ __device__ constexpr int smem_bytes(int G, int B) {
    return prefix_offset(G) + (2 * B + 1) * 4 + 1024;
  }
};

template <int D, int NW, int ST, bool APPEND>
__global__ void __launch_bounds__(NW * 32)
    decode_dynamic_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                          const DecodeParams p) {
  using Cfg = DynCfg<D, NW, ST>;
  constexpr uint32_t FULL = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int G = p.group, Hkv = p.hkv, P = p.partition, B = p.batch;
  volatile int* slots = reinterpret_cast<volatile int*>(smem + Cfg::kSlotOffset);  // [2][{seq, item}]
  int* scratch = reinterpret_cast<int*>(smem + Cfg::kScratchOffset);  // [0, 31): scans; [31]: abort flag
  volatile int* cta_abort = scratch + 31;
  const MergeSmem ms = merge_smem<NW>(smem + Cfg::kMergeOffset, D, G);
  int* pre = reinterpret_cast<int*>(smem + Cfg::prefix_offset(G));  // [B+1] items before sequence b
  int* lens = pre + B + 1;                                           // [B] clamped context lengths

  pdl_launch_dependents();  // the combine kernel may launch now; it waits for this grid to finish

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const uint32_t ring = smem_addr(smem) + warp * ST * Cfg::kStageBytes;
  const uint32_t bars = smem_addr(smem + Cfg::kBarOffset) + warp * ST * 8;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < ST; ++s) mbar_init(bars + 8 * s, 1);
    mbar_init_fence();
    if (warp == 0) {
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&vmap);
      slots[2] = -1;  // claim slot 1 holds no item yet
      *cta_abort = 0;
    }
  }

  // ---- items before each sequence ---------------------------------------------
  int base = 0;
  for (int b0 = 0; b0 < B; b0 += blockDim.x) {
    const int b = b0 + tid;
    int items = 0;
    if (b < B) {
      const int L = clamp_context(p, b, blockIdx.x == 0);
      lens[b] = L;
      items = Hkv * seq_parts(L, window_start(L, p.window), P);
    }
    int total;
    const int ex = block_exclusive_scan(items, scratch, total);
    if (b < B) pre[b] = base + ex;
    base += total;
  }
  if (tid == 0) {
    pre[B] = base;
    slots[1] = atomicAdd(p.queue, 1);  // the first item
    __threadfence_block();
    slots[0] = 0;
  }
  __syncthreads();
  const int T = pre[B];

  // Item number -> item.
  auto decode = [&](int t) {
    Item it;
    int lo = 0, hi = B - 1;  // largest b with pre[b] <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= t) lo = mid; else hi = mid - 1;
    }
    it.b = lo;
    const int parts = (pre[lo + 1] - pre[lo]) / Hkv;
    const int r = t - pre[lo];
    it.g = r / parts;
    const int L = lens[lo];
    const int s0 = window_start(L, p.window);
    it.part = s0 / P + (r - it.g * parts);
    it.L = L;
    it.lo = max(s0, it.part * P);
    it.hi = min(L, it.part * P + P);
    it.j0 = it.lo / kSliceTokens;
    it.n = (it.hi + kSliceTokens - 1) / kSliceTokens - it.j0;
    it.whole = parts == 1;
    return it;
  };
  // This warp's share of an item's slices: k = warp, warp + NW, ...
  auto share = [&](const Item& it) { return it.n > warp ? (it.n - warp + NW - 1) / NW : 0; };

  int s = 0;  // item sequence number within this CTA
  int t_cur = slots[1];
  if (t_cur >= T) return;  // nothing issued yet: safe to leave

  Item ci = decode(t_cur);
  int cn = share(ci);
  // Issue cursor: item `ii` (sequence number i_seq), slice index ik of in_.
  Item ii = ci;
  int in_ = cn, ik = 0, i_seq = 0;
  int gi = 0, gc = 0;  // slices issued / consumed by this warp (ring position)
  int yrow = -1;       // cache rows of the issue item's warp-slices [kbatch, kbatch + 32), one per lane
  auto load_rows = [&](const Item& it, int base_k) {
    const int i = base_k + lane;
    yrow = -1;
    if (i < share(it)) {
      const int t = (it.j0 + warp + NW * i) * kSliceTokens;
      const int phys = p.block_tables[(size_t)it.b * p.max_blocks + (t >> p.log2_bs)];
      if (phys >= 0 && phys < p.num_blocks) yrow = cache_row(p, phys, it.g, t);
    }
  };
  load_rows(ii, 0);
  uint32_t qf[D / 16][2], qf_next[D / 16][2];
  const __nv_bfloat16* q0 = static_cast<const __nv_bfloat16*>(p.q);
  load_q_frags<D>(qf, q0 + ((size_t)ci.b * p.hq + (size_t)ci.g * G) * D, G, lane);

  bool abort = false;
  // Fill this warp's ring from the issue cursor; moves into the claimed next
  // item once its number is published.  Warp-uniform.
  auto try_issue = [&]() {
    while (!abort && gi - gc < ST) {
      if (ik >= in_) {
        if (i_seq != s) return;  // already in the next item, which is fully issued
        int seq_n = 0, t_n = 0;
        if (lane == 0) {
          seq_n = slots[2 * ((s + 1) & 1)];
          t_n = slots[2 * ((s + 1) & 1) + 1];
        }
        seq_n = __shfl_sync(FULL, seq_n, 0);
        t_n = __shfl_sync(FULL, t_n, 0);
        if (seq_n != s + 1) return;  // the next claim is not published yet
        i_seq = s + 1;
        ik = 0;
        if (t_n >= T) {
          in_ = 0;
          return;
        }
        ii = decode(t_n);
        in_ = share(ii);
        load_rows(ii, 0);
        load_q_frags<D>(qf_next, q0 + ((size_t)ii.b * p.hq + (size_t)ii.g * G) * D, G, lane);
        continue;
      }
      if (ik > 0 && (ik & 31) == 0) load_rows(ii, ik);
      const int y = __shfl_sync(FULL, yrow, ik & 31);
      issue_slice<D>(ring + (gi % ST) * Cfg::kStageBytes, bars + 8 * (gi % ST), &kmap, &vmap, y, lane);
      ++gi;
      ++ik;
    }
  };

  WarpAttn<D> st;
  st.reset();
  const float qk_scale = p.use_softcap ? p.scale : p.scale * kLog2e;
  int t_next = 0;
  if (tid == 0) t_next = atomicAdd(p.queue, 1);  // claim the next item early
  bool published = false;
  auto publish = [&]() {  // thread 0: make the claimed number visible as item s+1
    if (tid == 0 && !published) {
      slots[2 * ((s + 1) & 1) + 1] = t_next;
      __threadfence_block();
      slots[2 * ((s + 1) & 1)] = s + 1;
      published = true;
    }
  };

  while (true) {
    uint4 knew = make_uint4(0, 0, 0, 0), vnew = make_uint4(0, 0, 0, 0);
    const bool append_item = APPEND && ci.hi == ci.L;
    if (append_item && lane < D / 8) {
      const size_t off = ((size_t)ci.b * p.hkv + ci.g) * D + lane * 8;
      knew = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.k_new) + off);
      vnew = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.v_new) + off);
    }
    for (int ck = 0; ck < cn; ++ck) {
      try_issue();
      bool ok = !abort && mbar_wait_bounded(bars + 8 * (gc % ST), (gc / ST) & 1, kWaitLimitNs);
      ok = __all_sync(FULL, ok);
      if (!ok) {
        if (lane == 0) {
          raise_error(PA_DEVERR_TIMEOUT);
          *cta_abort = 1;
        }
        abort = true;
        break;
      }
      const uint32_t kbase = ring + (gc % ST) * Cfg::kStageBytes;
      const uint32_t vbase = kbase + Cfg::kSliceBytes;
      const int js = warp + NW * ck;  // slice within the item
      const int t0 = (ci.j0 + js) * kSliceTokens;
      if (append_item && js == ci.n - 1) {
        // The item's last slice holds position L-1: append the new rows.
        overwrite_slice_row<D>(kbase, vbase, (ci.L - 1) & (kSliceTokens - 1), knew, vnew, lane);
        if (lane < D / 8) {
          const int phys = p.block_tables[(size_t)ci.b * p.max_blocks + ((ci.L - 1) >> p.log2_bs)];
          if (phys >= 0 && phys < p.num_blocks) {
            const size_t dst = (size_t)cache_row(p, phys, ci.g, ci.L - 1) * D + lane * 8;
            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(const_cast<void*>(p.k_cache)) + dst) = knew;
            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(const_cast<void*>(p.v_cache)) + dst) = vnew;
          }
        }
      }
      attend_slice<D>(st, qf, kbase, vbase, t0, ci.lo, ci.hi, qk_scale, p, lane);
      __syncwarp();
      ++gc;
      publish();
    }
    publish();
    try_issue();  // start the next item's loads before merging this one

    // ---- merge this item's warp states -------------------------------------------
    st.reduce_sums();
    st.dump(ms.m, ms.l, ms.o, warp, G, G, lane);
    st.reset();
    named_barrier_sync(1, NW * 32);
    abort = *cta_abort != 0;  // the same decision in every warp from here on
    if (!abort) {
      merge_warps<NW, __nv_bfloat16>(ms, G, D, grid_dest<__nv_bfloat16>(p, ci.b, ci.g, ci.part, ci.whole), tid,
                                     NW * 32);
    }
    named_barrier_sync(1, NW * 32);  // merge buffer free; item s+1 published

    // ---- next item ------------------------------------------------------------------
    ++s;
    t_cur = slots[2 * (s & 1) + 1];
    if (t_cur >= T || abort) break;
    ci = decode(t_cur);
    cn = share(ci);
    if (i_seq == s) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        qf[kk][0] = qf_next[kk][0];
        qf[kk][1] = qf_next[kk][1];
      }
    } else {  // the issue cursor never entered this item
      ii = ci;
      in_ = cn;
      ik = 0;
      i_seq = s;
      load_rows(ii, 0);
      load_q_frags<D>(qf, q0 + ((size_t)ci.b * p.hq + (size_t)ci.g * G) * D, G, lane);
    }
    if (tid == 0) t_next = atomicAdd(p.queue, 1);
    published = false;
  }

  // Every TMA load issued was waited for unless a wait timed out; then give
  // loads still in flight a bounded time to land before the CTA's shared
  // memory is released.
  if (abort && lane == 0) {
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < kDrainLimitNs) {
    }
  }
}

}  // namespace pa
