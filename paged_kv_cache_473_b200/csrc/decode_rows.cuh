// Multi-query rows on the warp-per-item dynamic schedule, for R = T*G query
// rows per kv head (speculative-decoding verify with a few draft tokens):
// MT 16-row tiles per warp, R <= 16 MT, the MT x 16 x D output tiles in
// registers (MT = 2 at head_dim 64, 1 at 128 and 256).
//
// The work items, the persistent grid, the index-fixed first items and the
// claims, each warp's TMA ring, the prologue (inputs prefetched into L2 before
// the grid-dependency wait, a per-warp length scan for small batches) are
// those of the decode kernel (decode_dynamic.cuh); what differs is the attention: the R query rows of
// (sequence b, kv head g) -- token j = r / G, head h = r % G, at position
// p_j = L - T + j -- are the 16-row M dimension of the MMA
// (attend_slice_rows, once per 16-row tile on the same K/V stage), each row
// with its own causal / window range.  The
// sequence's union range is [s0 of token 0, L); an item covers one partition
// of it, and writes either the normalised rows (the sequence's only
// partition) or partials for the combine kernel, which merges [B][T][Hq] rows.
#pragma once

#include "decode_common.cuh"
#include "decode_dynamic.cuh"
#include "mma_slice.cuh"
#include "ptx.cuh"

namespace pa {

// Query rows one warp carries per item: its 16-row MMA tiles times 16.
template <int D>
__host__ __device__ constexpr int rows_tiles() { return D <= 64 ? 2 : 1; }

template <int D, int NW, int ST>
__global__ void __launch_bounds__(NW * 32, dynamic_min_blocks<D>())
    decode_rows_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                       const DecodeParams p) {
  using Cfg = DynCfg<D, NW, ST>;
  constexpr uint32_t FULL = 0xffffffffu;
  constexpr bool kPairs = ST >= 4;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int G = p.group, Hkv = p.hkv, P = p.partition, B = p.batch, T = p.q_len;
  constexpr int MT = rows_tiles<D>();
  const int R = T * G;  // query rows per (sequence, kv head), <= 16 MT
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const bool warp_scan = B <= kWarpScanBatch;
  int* scratch = reinterpret_cast<int*>(smem + Cfg::kScratchOffset);
  // [B+1] items before sequence b, then [B] clamped context lengths: this
  // warp's own arrays (warp_scan), else the CTA's.
  int* pre = reinterpret_cast<int*>(smem + Cfg::kPrefixOffset) + (warp_scan ? warp * (2 * B + 1) : 0);
  int* lens = pre + B + 1;

  pdl_launch_dependents();  // the combine may launch; it waits for this grid to finish

  const uint32_t ring = smem_addr(smem) + warp * ST * Cfg::kStageBytes;
  const uint32_t bars = smem_addr(smem + Cfg::kBarOffset) + warp * ST * 8;
  const int W = gridDim.x * NW, wg = blockIdx.x * NW + warp;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < ST; ++s) mbar_init(bars + 8 * s, 1);
    mbar_init_fence();
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  if (tid == 0) {  // the prologue's small inputs into L2, as in the decode kernel (hints only)
    auto share = [&](const void* base, size_t bytes) {
      const size_t chunk = max((size_t)256, (bytes + gridDim.x - 1) / gridDim.x);
      const size_t off = (size_t)blockIdx.x * chunk;
      if (off < bytes) prefetch_l2(static_cast<const char*>(base) + off, min(chunk, bytes - off));
    };
    share(p.context_lens, (size_t)B * 4);
    share(p.block_tables, (size_t)B * p.max_blocks * 4);
    share(p.q, (size_t)B * T * p.hq * D * 2);
  }
  // Launched as a programmatic dependent: nothing above touched global memory.
  pdl_wait();

  // The union of a sequence's rows' ranges starts at token 0's window start.
  auto union_start = [&](int L) { return window_start(max(L - T + 1, 0), p.window); };

  // ---- items before each sequence ---------------------------------------------
  if (warp_scan) {  // this warp alone (as in the decode kernel)
    warp_items_scan(p, B, Hkv, p.log2_partition, wg == 0, pre, lens, lane,
                    [&](int, int L) { return union_start(L); });
  } else {
#pragma unroll 4
    for (int b = tid; b < B; b += blockDim.x) lens[b] = clamp_context(p, b, blockIdx.x == 0);
    __syncthreads();
    int base = 0;
    for (int b0 = 0; b0 < B; b0 += blockDim.x) {
      const int b = b0 + tid;
      int items = 0;
      if (b < B) {
        const int L = lens[b];
        items = Hkv * seq_parts(L, union_start(L), P);
      }
      int total;
      const int ex = block_exclusive_scan(items, scratch, total);
      if (b < B) pre[b] = base + ex;
      base += total;
    }
    if (tid == 0) pre[B] = base;
    __syncthreads();
  }
  const int T_items = pre[B];
  // Sequences with no position (L == 0) get zero rows; no item covers them.
  // Warp wg takes sequences wg, wg + W, ...
  for (int b = wg; b < B; b += W) {
    if (pre[b + 1] != pre[b]) continue;
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + (size_t)b * T * p.hq * D;
    for (int i = lane; i < T * p.hq * D; i += 32) o[i] = __float2bfloat16_rn(0.f);
  }

  auto decode = [&](int t) {
    Item it;
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= t) lo = mid; else hi = mid - 1;
    }
    it.b = lo;
    const int parts = (pre[lo + 1] - pre[lo]) / Hkv;
    const int r = t - pre[lo];
    it.g = r / parts;
    const int L = lens[lo];
    const int s0 = union_start(L);
    it.pb = s0 / P;
    it.parts = parts;
    it.part = it.pb + (r - it.g * parts);
    it.L = L;
    it.lo = max(s0, it.part * P);
    it.hi = min(L, it.part * P + P);
    it.j0 = it.lo / kSliceTokens;
    it.n = (it.hi + kSliceTokens - 1) / kSliceTokens - it.j0;
    it.whole = parts == 1;
    return it;
  };

  // This lane's rows 16 m + lane / 4 and 16 m + lane / 4 + 8 of tile m of an
  // item: output row index ((b*T + j)*Hq + g*G + h) and token range inside
  // the item.
  const int r0 = lane >> 2;
  auto out_row = [&](const Item& it, int r) {
    return ((size_t)it.b * T + r / G) * p.hq + (size_t)it.g * G + r % G;
  };
  auto row_range = [&](const Item& it, int r, int& lo, int& hi) {
    if (r >= R) {  // padding row: the item's range keeps its softmax finite
      lo = it.lo;
      hi = it.hi;
      return;
    }
    const int end = it.L - T + r / G + 1;  // p_j + 1
    lo = max(window_start(max(end, 0), p.window), it.lo);
    hi = min(end, it.hi);
  };
  const __nv_bfloat16* q0 = static_cast<const __nv_bfloat16*>(p.q);
  auto load_q = [&](uint32_t (&qa)[MT][D / 16][4], const Item& it) {
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const int ra = 16 * m + r0, rb = ra + 8;
      load_q_rows<D>(qa[m], q0 + out_row(it, ra < R ? ra : 0) * D, ra < R, q0 + out_row(it, rb < R ? rb : 0) * D,
                     rb < R, lane);
    }
  };

  const int n_static = p.static_items;
  const int claim_base = n_static * W;
  // Claims are needed only when there are more items than the warps' fixed
  // ones; otherwise no warp touches the counter and no CTA counts out, so a
  // CTA ends with its last warp.
  const bool claims = T_items > claim_base;
  int t_cur = wg;
  int t_next = W + wg;
  bool next_known = n_static >= 2;
  if (t_cur < T_items) {
    int t_claim = 0;
    bool pending = false;
    if (claims && (n_static < 2 || t_next < T_items)) {
      if (lane == 0) t_claim = (n_static < 2 ? W : claim_base) + atomicAdd(p.queue, 1);
      pending = true;
    }
    auto resolve_next = [&]() {
      if (next_known) return;
      t_next = pending ? __shfl_sync(FULL, t_claim, 0) : T_items;
      next_known = true;
      pending = false;
      if (claims && t_next < T_items) {
        if (lane == 0) t_claim = claim_base + atomicAdd(p.queue, 1);
        pending = true;
      }
    };

    Item ci = decode(t_cur);
    Item ii = ci;
    int ik = 0;
    bool i_in_next = false;
    int gi = 0, gc = 0;
    int yrow = -1;
    auto load_rows = [&](const Item& it, int base_k) {
      const int k = base_k + lane;
      yrow = -1;
      if (k < it.n) {
        const int t = (it.j0 + k) * kSliceTokens;
        const int phys = p.block_tables[(size_t)it.b * p.max_blocks + (t >> p.log2_bs)];
        if (phys >= 0 && phys < p.num_blocks) yrow = cache_row(p, phys, it.g, t);
      }
    };
    load_rows(ii, 0);
    uint32_t qa[MT][D / 16][4];  // the next item's rows are loaded when it starts (its K/V are in flight by then)
    load_q(qa, ci);

    auto fill = [&]() {
      while (gi - gc < ST) {
        if (ik >= ii.n) {
          if (i_in_next) return;
          resolve_next();
          if (t_next >= T_items) return;
          ii = decode(t_next);
          ik = 0;
          i_in_next = true;
          load_rows(ii, 0);
          continue;
        }
        if (ik > 0 && (ik & 31) == 0) load_rows(ii, ik);
        const int y = __shfl_sync(FULL, yrow, ik & 31);
        issue_slice<D>(ring + (gi % ST) * Cfg::kStageBytes, bars + 8 * (gi % ST), &kmap, &vmap, y, lane);
        ++gi;
        ++ik;
      }
    };

    WarpRows<D> st[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) st[m].reset();
    const float qk_scale = p.use_softcap ? p.scale : p.scale * kLog2e;
    const int tq = lane & 3;
    bool aborted = false;

    while (true) {
      ColRange cr[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        row_range(ci, 16 * m + r0, cr[m].lo0, cr[m].hi0);
        row_range(ci, 16 * m + r0 + 8, cr[m].lo1, cr[m].hi1);
      }
      for (int ck = 0; ck < ci.n;) {
        fill();
        // Two slices per softmax step where the ring is deep enough to keep
        // loading while both are attended.
        const int step = (kPairs && ck + 1 < ci.n) ? 2 : 1;
        bool ok = mbar_wait_bounded(bars + 8 * (gc % ST), (gc / ST) & 1, kWaitLimitNs);
        if (step == 2) ok = ok && mbar_wait_bounded(bars + 8 * ((gc + 1) % ST), ((gc + 1) / ST) & 1, kWaitLimitNs);
        ok = __all_sync(FULL, ok);
        if (!ok) {
          aborted = true;
          break;
        }
        const uint32_t kbase = ring + (gc % ST) * Cfg::kStageBytes;
        const uint32_t kbase1 = ring + ((gc + 1) % ST) * Cfg::kStageBytes;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (m == 0 || 16 * m < R) {
            if (step == 2)
              attend_pair_rows<D>(st[m], qa[m], kbase, kbase + Cfg::kSliceBytes, kbase1, kbase1 + Cfg::kSliceBytes,
                                  (ci.j0 + ck) * kSliceTokens, ci.lo, ci.hi, cr[m], qk_scale, p, lane);
            else
              attend_slice_rows<D>(st[m], qa[m], kbase, kbase + Cfg::kSliceBytes, (ci.j0 + ck) * kSliceTokens,
                                   ci.lo, ci.hi, cr[m], qk_scale, p, lane);
          }
        }
        __syncwarp();
        gc += step;
        ck += step;
      }
      if (aborted) break;
      fill();  // keep loading the next item while this one is stored

      // ---- store this item's rows from registers ----------------------------------------
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        WarpRows<D>& sm = st[mt];
        sm.reduce_sums();
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int r = 16 * mt + r0 + 8 * e;
          if (r >= R) continue;
          const size_t row = out_row(ci, r);
          const float m = e ? sm.m1 : sm.m0, l = e ? sm.l1 : sm.l0;
          if (ci.whole) {
            const float inv = l > 0.f ? 1.f / l : 0.f;  // a row with no position is zero
            __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + row * D + 2 * tq;
#pragma unroll
            for (int nt = 0; nt < D / 8; ++nt)
              *reinterpret_cast<uint32_t*>(o + nt * 8) = pack_bf16x2(sm.o[nt][2 * e] * inv, sm.o[nt][2 * e + 1] * inv);
          } else {
            float* po = p.ws_o + (row * p.max_parts + ci.part) * D + 2 * tq;
#pragma unroll
            for (int nt = 0; nt < D / 8; ++nt)
              *reinterpret_cast<float2*>(po + nt * 8) = make_float2(sm.o[nt][2 * e], sm.o[nt][2 * e + 1]);
            if (tq == 0) {
              float* pml = p.ws_ml + (row * p.max_parts + ci.part) * 2;
              pml[0] = m;
              pml[1] = l;
            }
          }
        }
        sm.reset();
      }

      // ---- next item ------------------------------------------------------------------
      resolve_next();
      t_cur = t_next;
      if (t_cur >= T_items) break;
      next_known = false;
      if (i_in_next) {
        ci = ii;
        i_in_next = false;
      } else {
        ci = decode(t_cur);
        ii = ci;
        ik = 0;
        load_rows(ii, 0);
      }
      load_q(qa, ci);
    }

    if (pending) t_claim = __shfl_sync(FULL, t_claim, 0);  // every claim lands before the CTA counts out
    if (aborted) {
      if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
      for (int i = gc; i < gi; ++i) (void)mbar_wait_bounded(bars + 8 * (i % ST), (i / ST) & 1, kDrainLimitNs);
    }
  }  // t_cur < T_items

  // The last CTA to finish returns the work counter to zero (when any warp
  // claimed from it).
  if (claims) {
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      if (atomicAdd(p.queue + 1, 1) == (int)gridDim.x - 1) {
        p.queue[0] = 0;
        p.queue[1] = 0;
      }
    }
  }
}

}  // namespace pa
