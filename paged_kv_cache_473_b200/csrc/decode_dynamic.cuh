// Paged decode attention, bf16, tensor cores: the dynamic (work-queue) split-K
// schedule, one work item per warp, with the partition merge done in-kernel.
//
// Work items are the non-empty (sequence b, kv head g, partition) triples of
// the split-K decomposition: partition p of sequence b covers tokens
// [p*P, p*P + P) of its attended range [s0, L).  The grid is persistent (as
// many CTAs as fit on the GPU at once) and every WARP claims items on its own
// from a counter in the workspace (atomicAdd; the first two items of each warp
// are fixed by its index), so warps on SMs that stream faster take more items
// and the whole GPU finishes together.  A warp runs an
// item alone: it streams the item's 16-token slices through its own ST-deep
// ring of TMA-filled shared-memory stages, keeps the online-softmax state in
// registers (attend_slice), and at the end writes either the normalised output
// (the item is the sequence's only partition) or its partial state (m, l, o)
// to the [B][Hq][max_parts] workspace, straight from registers.  No barrier
// joins the warps of a CTA after the prologue, so an SM holds many independent
// streams of loads.  Each warp claims two items ahead and its load cursor runs
// into the next item before the current one is finished, so its ring stays
// full across item boundaries.
//
// Merge: each (sequence, kv head) unit has an arrival counter in the
// workspace.  A warp that stored a partial publishes it (memory fence) and
// counts it; the warp that brings the count to the unit's number of
// partitions reads every partial back from L2, writes the normalised output
// rows (log-sum-exp merge, merge_unit) and returns the counter to zero.  The
// last CTA to finish returns the work counter to zero, so the workspace is
// ready for the next call without a second kernel.
//
// Items are numbered sequence-major; each CTA first builds, with block-wide
// scans over context_lens, the number of items before each sequence and
// decodes an item number with a binary search in shared memory.
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
// The split-K workspace starts with a fixed counter region: [0] work-item
// counter, [1] finished CTAs, then one arrival count per (sequence, kv head).
constexpr int kMaxDynamicUnits = 65534;
constexpr size_t kCounterBytes = (2 + (size_t)kMaxDynamicUnits) * sizeof(int);  // 256 KiB

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

// Partitions of sequence b's attended range [s0, L) (0 when it is empty).
__device__ __forceinline__ int seq_parts(int L, int s0, int P) { return L > s0 ? (L + P - 1) / P - s0 / P : 0; }

// First position this kernel attends for sequence b: the window start, or
// (CASCADE) the end of the shared prefix for a sharer.
template <bool CASCADE>
__device__ __forceinline__ int seq_start(const DecodeParams& p, int b, int L) {
  const int s0 = window_start(L, p.window);
  return (CASCADE && b < p.n_sharers) ? max(s0, p.prefix_len) : s0;
}

struct Item {
  int b, g, part;  // sequence, kv head, absolute partition index
  int L, lo, hi;   // context length; attended tokens [lo, hi) of this item
  int j0, n;       // first 16-token slice and number of slices
  int pb, parts;   // the sequence's first partition index and its number of partitions
  bool whole;      // the item is the sequence's only partition
};

// In-kernel merges take at most this many partials per unit (the host merges
// larger splits with the combine kernel).
constexpr int kMaxMergeParts = 8;

// Log-sum-exp merge of the `n` <= kMaxMergeParts partials [pb, pb + n) of unit
// (b, g) into the normalised output rows of its G query heads:
//   M = max_p m_p,  out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p
// (m in the log2 domain, o unnormalised relative to m).  lph lanes per head (a
// power of two), each covering D / lph dims in chunks of 16; the partials are
// read through L2 (other SMs wrote them).  The merge runs after the unit's
// last partition, on the critical path of the call's tail, so every load of a
// chunk is issued before any is used: one L2 round trip instead of one per
// few partials (kBatch partials at a time where registers are tight).
template <int D>
__device__ __forceinline__ void merge_unit(const DecodeParams& p, int b, int g, int pb, int n, int lane) {
  constexpr int kBatch = D == 128 ? 4 : kMaxMergeParts;  // head_dim 128 runs with a 170-register cap
  const int G = p.group;
  const int lph = min(G == 1 ? 32 : G == 2 ? 16 : G <= 4 ? 8 : 4, D / 16);
  const int h = lane / lph, s = lane & (lph - 1);
  const bool active = h < G;
  const size_t row = (size_t)b * p.hq + (size_t)g * G + (active ? h : 0);
  const float2* ml = reinterpret_cast<const float2*>(p.ws_ml) + row * p.max_parts + pb;
  float2 mlv[kMaxMergeParts];
#pragma unroll
  for (int i = 0; i < kMaxMergeParts; ++i) mlv[i] = i < n ? __ldcg(ml + i) : make_float2(-CUDART_INF_F, 0.f);
  const int E = D / lph;
  const float* po = p.ws_o + (row * p.max_parts + pb) * D + s * E;
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + row * D + s * E;
  for (int c0 = 0; c0 < E; c0 += 16) {
    float acc[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) acc[k] = 0.f;
    float den = 0.f;
#pragma unroll
    for (int i0 = 0; i0 < kMaxMergeParts; i0 += kBatch) {
      if (i0 >= n) break;
      float4 x[kBatch][4];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const float4* src = reinterpret_cast<const float4*>(po + (size_t)(i0 + i) * D + c0);
#pragma unroll
        for (int k = 0; k < 4; ++k) x[i][k] = i0 + i < n ? __ldcg(src + k) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float M = -CUDART_INF_F;
#pragma unroll
      for (int i = 0; i < kMaxMergeParts; ++i) M = fmaxf(M, mlv[i].x);
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const float2 v = mlv[i0 + i];
        const float w = v.x == -CUDART_INF_F ? 0.f : exp2f(v.x - M);  // empty or absent partial: weight 0
        den = fmaf(w, v.y, den);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          acc[4 * k + 0] = fmaf(w, x[i][k].x, acc[4 * k + 0]);
          acc[4 * k + 1] = fmaf(w, x[i][k].y, acc[4 * k + 1]);
          acc[4 * k + 2] = fmaf(w, x[i][k].z, acc[4 * k + 2]);
          acc[4 * k + 3] = fmaf(w, x[i][k].w, acc[4 * k + 3]);
        }
      }
    }
    if (active) {
      const float inv = 1.f / den;
      uint4 lo, hi;
      lo.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
      lo.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
      lo.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
      lo.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
      hi.x = pack_bf16x2(acc[8] * inv, acc[9] * inv);
      hi.y = pack_bf16x2(acc[10] * inv, acc[11] * inv);
      hi.z = pack_bf16x2(acc[12] * inv, acc[13] * inv);
      hi.w = pack_bf16x2(acc[14] * inv, acc[15] * inv);
      reinterpret_cast<uint4*>(out + c0)[0] = lo;
      reinterpret_cast<uint4*>(out + c0)[1] = hi;
    }
  }
}

template <int D, int NW, int ST>
struct DynCfg {
  static constexpr int kStageBytes = SliceBytes<D>::kStage;
  static constexpr int kSliceBytes = SliceBytes<D>::kSlice;
  static constexpr int kRingBytes = NW * ST * kStageBytes;
  static constexpr int kThreads = NW * 32;
  // After the 1024-aligned ring: barriers, scan scratch, prefix arrays.
  static constexpr int kBarOffset = kRingBytes;
  static constexpr int kScratchOffset = kBarOffset + NW * ST * 8;
  static constexpr int kPrefixOffset = kScratchOffset + 32 * 4;
  static __host__ __device__ constexpr int smem_bytes(int B) { return kPrefixOffset + (2 * B + 1) * 4 + 1024; }
};

// Resident CTAs per SM the configurations are sized for (shared memory allows
// that many): the register budget ptxas may use follows from it.
template <int D>
constexpr int dynamic_min_blocks() { return D == 128 ? 3 : 2; }

template <int D, int NW, int ST, bool APPEND, bool CASCADE = false>
__global__ void __launch_bounds__(NW * 32, dynamic_min_blocks<D>())
    decode_dynamic_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                          const DecodeParams p) {
  using Cfg = DynCfg<D, NW, ST>;
  constexpr uint32_t FULL = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int G = p.group, Hkv = p.hkv, P = p.partition, B = p.batch;
  int* scratch = reinterpret_cast<int*>(smem + Cfg::kScratchOffset);
  int* pre = reinterpret_cast<int*>(smem + Cfg::kPrefixOffset);  // [B+1] items before sequence b
  int* lens = pre + B + 1;                                        // [B] clamped context lengths

  // Without the in-kernel merge the combine kernel (a programmatic dependent)
  // may launch now; it waits for this grid to finish before it reads anything.
  if (!p.merge_in_kernel) pdl_launch_dependents();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const uint32_t ring = smem_addr(smem) + warp * ST * Cfg::kStageBytes;
  const uint32_t bars = smem_addr(smem + Cfg::kBarOffset) + warp * ST * 8;
  // A warp's first two items are fixed by its index (W warps in the grid: items
  // w and W + w); later ones are claimed from the counter, offset by 2W, so the
  // launch does not start with every warp contending for one address.
  const int W = gridDim.x * NW, wg = blockIdx.x * NW + warp;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < ST; ++s) mbar_init(bars + 8 * s, 1);
    mbar_init_fence();
    if (warp == 0) {
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&vmap);
    }
  }

  // ---- items before each sequence ---------------------------------------------
  // All lengths are loaded at once (independent loads), then scanned.
#pragma unroll 4
  for (int b = tid; b < B; b += blockDim.x) lens[b] = clamp_context(p, b, blockIdx.x == 0);
  __syncthreads();
  int base = 0;
  for (int b0 = 0; b0 < B; b0 += blockDim.x) {
    const int b = b0 + tid;
    int items = 0;
    if (b < B) {
      const int L = lens[b];
      items = Hkv * seq_parts(L, seq_start<CASCADE>(p, b, L), P);
    }
    int total;
    const int ex = block_exclusive_scan(items, scratch, total);
    if (b < B) pre[b] = base + ex;
    base += total;
  }
  if (tid == 0) pre[B] = base;
  __syncthreads();
  const int T = pre[B];
  // Sequences with nothing to attend (L == 0) get zero rows; no item covers
  // them.  (A cascade sharer whose range lies inside the shared prefix has no
  // item either: the prefix pass writes its rows.)
  for (int b = blockIdx.x; b < B; b += gridDim.x) {
    if (pre[b + 1] != pre[b] || (CASCADE && lens[b] != 0)) continue;
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + (size_t)b * p.hq * D;
    for (int i = tid; i < p.hq * D; i += blockDim.x) o[i] = __float2bfloat16_rn(0.f);
  }

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
    const int st = seq_start<CASCADE>(p, lo, L);
    it.pb = st / P;
    it.parts = parts;
    it.part = it.pb + (r - it.g * parts);
    it.L = L;
    it.lo = max(st, it.part * P);
    it.hi = min(L, it.part * P + P);
    it.j0 = it.lo / kSliceTokens;
    it.n = (it.hi + kSliceTokens - 1) / kSliceTokens - it.j0;
    // (a cascade sharer's prefix partials come from the prefix pass)
    it.whole = parts == 1 && (!CASCADE || st == window_start(L, p.window));
    return it;
  };

  // The first p.static_items (1 or 2) items of a warp are fixed by its index
  // (wg, W + wg); later ones are claimed from the counter, offset by
  // static_items * W.  One claim is always in flight ahead of use and is read
  // only when its item is needed, so no warp waits on the counter at launch.
  const int n_static = p.static_items;
  const int claim_base = n_static * W;
  // Claims are needed only when there are more items than the warps' fixed
  // ones; otherwise no warp touches the counter and no CTA counts out, so a
  // CTA ends with its last warp.
  const bool claims = T > claim_base;
  int t_cur = wg;       // item being computed
  int t_next = W + wg;  // item after it, valid when next_known
  bool next_known = n_static >= 2;
  if (t_cur < T) {  // else this warp has no item; it still joins the final barrier
    int t_claim = 0;       // lane 0: the claim in flight (for t_next when !next_known, else the item after)
    bool pending = false;  // a claim is in flight (warp-uniform)
    if (claims && (n_static < 2 || t_next < T)) {
      if (lane == 0) t_claim = (n_static < 2 ? W : claim_base) + atomicAdd(p.queue, 1);
      pending = true;
    }
    // Make t_next known (read the claim in flight) and put the next claim in flight.
    auto resolve_next = [&]() {
      if (next_known) return;
      t_next = pending ? __shfl_sync(FULL, t_claim, 0) : T;
      next_known = true;
      pending = false;
      if (claims && t_next < T) {
        if (lane == 0) t_claim = claim_base + atomicAdd(p.queue, 1);
        pending = true;
      }
    };

    Item ci = decode(t_cur);
    // Load cursor: slice ik of item ii (ii == ci, or the next item once ci is fully issued).
    Item ii = ci;
    int ik = 0;
    bool i_in_next = false;
    int gi = 0, gc = 0;  // slices issued / consumed (ring position)
    int yrow = -1;       // cache rows of the load item's slices [kbatch, kbatch + 32), one per lane
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
    uint32_t qf[D / 16][2], qf_next[D / 16][2];
    const __nv_bfloat16* q0 = static_cast<const __nv_bfloat16*>(p.q);
    load_q_frags<D>(qf, q0 + ((size_t)ci.b * p.hq + (size_t)ci.g * G) * D, G, lane);

    // Keep ST slices in flight: finish the current item's loads, then run into the next item.
    auto fill = [&]() {
      while (gi - gc < ST) {
        if (ik >= ii.n) {
          if (i_in_next) return;
          resolve_next();
          if (t_next >= T) return;
          ii = decode(t_next);
          ik = 0;
          i_in_next = true;
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
    const int n0 = 2 * (lane & 3);
    bool aborted = false;

    while (true) {
      uint4 knew = make_uint4(0, 0, 0, 0), vnew = make_uint4(0, 0, 0, 0);
      const bool append_item = APPEND && ci.hi == ci.L;
      if (append_item && lane < D / 8) {
        const size_t off = ((size_t)ci.b * p.hkv + ci.g) * D + lane * 8;
        knew = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.k_new) + off);
        vnew = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.v_new) + off);
      }
      for (int ck = 0; ck < ci.n; ++ck) {
        fill();
        bool ok = mbar_wait_bounded(bars + 8 * (gc % ST), (gc / ST) & 1, kWaitLimitNs);
        ok = __all_sync(FULL, ok);
        if (!ok) {
          aborted = true;
          break;
        }
        const uint32_t kbase = ring + (gc % ST) * Cfg::kStageBytes;
        const uint32_t vbase = kbase + Cfg::kSliceBytes;
        if (append_item && ck == ci.n - 1) {
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
        attend_slice<D>(st, qf, kbase, vbase, (ci.j0 + ck) * kSliceTokens, ci.lo, ci.hi, qk_scale, p, lane);
        __syncwarp();
        ++gc;
      }
      if (aborted) break;
      fill();  // keep loading the next item while this one is stored

      // ---- store this item's result from registers ------------------------------------
      st.reduce_sums();
      const size_t row0 = (size_t)ci.b * p.hq + (size_t)ci.g * G;
      if (ci.whole) {
        const float inv0 = 1.f / st.l0, inv1 = 1.f / st.l1;
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + row0 * D;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          const int d = mt * 16 + (lane >> 2);
          if (n0 < G) {
            out[(size_t)n0 * D + d] = __float2bfloat16_rn(st.o[mt][0] * inv0);
            out[(size_t)n0 * D + d + 8] = __float2bfloat16_rn(st.o[mt][2] * inv0);
          }
          if (n0 + 1 < G) {
            out[(size_t)(n0 + 1) * D + d] = __float2bfloat16_rn(st.o[mt][1] * inv1);
            out[(size_t)(n0 + 1) * D + d + 8] = __float2bfloat16_rn(st.o[mt][3] * inv1);
          }
        }
      } else {
        const size_t slot0 = (row0 + n0) * p.max_parts + ci.part;  // head n0; head n0+1 is max_parts further
        float* po = p.ws_o + slot0 * D;
        const size_t hstride = (size_t)p.max_parts * D;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          const int d = mt * 16 + (lane >> 2);
          if (n0 < G) {
            po[d] = st.o[mt][0];
            po[d + 8] = st.o[mt][2];
          }
          if (n0 + 1 < G) {
            po[hstride + d] = st.o[mt][1];
            po[hstride + d + 8] = st.o[mt][3];
          }
        }
        if (lane < 4) {
          float* pml = p.ws_ml + slot0 * 2;
          if (n0 < G) {
            pml[0] = st.m0;
            pml[1] = st.l0;
          }
          if (n0 + 1 < G) {
            pml[(size_t)p.max_parts * 2 + 0] = st.m1;
            pml[(size_t)p.max_parts * 2 + 1] = st.l1;
          }
        }
        if (p.merge_in_kernel) {
          // Publish the partial, then count it (release); the unit's last
          // partial merges them all (acquire).
          fence_acq_rel_gpu();
          __syncwarp();
          int* cnt = p.unit_count + (size_t)ci.b * Hkv + ci.g;
          int last = 0;
          if (lane == 0) last = atomicAdd(cnt, 1) == ci.parts - 1;
          if (__shfl_sync(FULL, last, 0)) {
            fence_acq_rel_gpu();
            merge_unit<D>(p, ci.b, ci.g, ci.pb, ci.parts, lane);
            if (lane == 0) *cnt = 0;  // every partial of the unit has arrived: ready for the next call
          }
        }
      }
      st.reset();

      // ---- next item ------------------------------------------------------------------
      resolve_next();
      t_cur = t_next;
      if (t_cur >= T) break;
      next_known = false;  // the claim in flight is for the item after t_cur
      if (i_in_next) {
        ci = ii;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          qf[kk][0] = qf_next[kk][0];
          qf[kk][1] = qf_next[kk][1];
        }
        i_in_next = false;
      } else {  // the load cursor had not reached this item yet
        ci = decode(t_cur);
        ii = ci;
        ik = 0;
        load_rows(ii, 0);
        load_q_frags<D>(qf, q0 + ((size_t)ci.b * p.hq + (size_t)ci.g * G) * D, G, lane);
      }
    }

    if (pending) t_claim = __shfl_sync(FULL, t_claim, 0);  // every claim lands before the CTA counts out
    if (aborted) {
      if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
      // Give this warp's loads still in flight a bounded time to land before the
      // CTA's shared memory is released.
      for (int i = gc; i < gi; ++i) (void)mbar_wait_bounded(bars + 8 * (i % ST), (i / ST) & 1, kDrainLimitNs);
    }
  }  // t_cur < T

  // Every claim of this CTA's warps has returned: count the CTA out; the last
  // CTA returns the work counter (and this count) to zero for the next call.
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
  // In a cascade this grid is a programmatic dependent of the prefix pass
  // (which it does not read): it finishes only after that pass has, so the
  // combine that waits for this grid also sees the prefix partials.
  if (CASCADE) pdl_wait();
}

}  // namespace pa
