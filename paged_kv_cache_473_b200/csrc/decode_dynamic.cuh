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
// registers (attend_slice; two slices per softmax step, attend_pair, where the
// ring has at least four stages: a warp's time per slice is its own dependent
// latency, not the memory's, so halving the softmax steps shortens it), and at
// the end writes either the normalised output
// (the item is the sequence's only partition) or its partial state (m, l, o)
// to the [B][Hq][max_parts] workspace, straight from registers.  No barrier
// joins the warps of a CTA after the prologue, so an SM holds many independent
// streams of loads.  Each warp claims two items ahead and its load cursor runs
// into the next item before the current one is finished, so its ring stays
// full across item boundaries.
//
// Merge (small steps): each (sequence, kv head) unit has an arrival counter in
// the workspace.  A warp that stored a partial publishes and counts it with
// one acquire-release atomic; the warp that brings the count to the unit's number of
// partitions reads every partial back through L2 in partition order (the same
// bits whichever warp merges), merges them (log-sum-exp) and writes the
// normalised output rows; it returns the counter to zero.  (Measured on
// B200 and not kept: counting arrivals before the stores, so that the last
// warp merges without storing its own partial; the waits it adds cost more
// than the store and fence it saves.)  The last CTA to
// finish returns the work counter to zero, so the workspace is ready for the
// next call without a second kernel.  Larger steps leave the merge to the
// combine kernel.
//
// Items are numbered sequence-major.  The number of items before each sequence
// is a scan over context_lens, and an item number is decoded with a binary
// search over that prefix in shared memory.  For batches of up to
// kWarpScanBatch sequences every warp scans the lengths itself, into its own
// slice of shared memory, so that no barrier across the CTA's warps stands
// between a warp's start and its first TMA issue; larger batches share one
// CTA-wide scan.
//
// The kernel is launched as a programmatic dependent of whatever precedes it
// on the stream: everything before griddepcontrol.wait (barrier set-up, the
// tensor-map prefetch) overlaps that kernel's tail, and no global memory is
// touched before the wait (the cascade's own-range pass waits at its end).
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
// Batches up to this size are scanned by every warp for itself (per-warp prefix
// arrays, up to eight sequences per lane); larger ones by the CTA together.
constexpr int kWarpScanBatch = 256;


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
// The same for a partition of 2^lp tokens.
__device__ __forceinline__ int seq_parts_sh(int L, int s0, int lp) {
  return L > s0 ? ((L + (1 << lp) - 1) >> lp) - (s0 >> lp) : 0;
}

// One warp's scan of the items before each sequence, for B <= kWarpScanBatch:
// lane l takes sequences [c l, c l + c), c = ceil(B / 32), their lengths in
// registers; items(b) = Hkv * (partitions of b's range); a warp shuffle scan
// gives each lane its base.  Writes lens[b], pre[b] for b < B and pre[B].
template <typename RangeStart>
__device__ __forceinline__ void warp_items_scan(const DecodeParams& p, int B, int Hkv, int lp, bool report,
                                                int* pre, int* lens, int lane, RangeStart start) {
  constexpr uint32_t FULL = 0xffffffffu;
  const int c = (B + 31) >> 5, b0 = lane * c;
  int L[8], n[8];
  int sum = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    L[k] = n[k] = 0;
    if (k < c && b0 + k < B) {
      L[k] = clamp_context(p, b0 + k, report);
      n[k] = Hkv * seq_parts_sh(L[k], start(b0 + k, L[k]), lp);
    }
    sum += n[k];
  }
  int incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(FULL, incl, off);
    if (lane >= off) incl += y;
  }
  int base = incl - sum;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    if (k < c && b0 + k < B) {
      lens[b0 + k] = L[k];
      pre[b0 + k] = base;
      base += n[k];
    }
  }
  if (lane == 31) pre[B] = incl;
  __syncwarp();
}

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

// In-kernel merge.  A unit's partials are stored in LANE ORDER: the D floats of
// head h's slot for partition i hold, at [r * D/8 + 2 * mt + e], dimension
// mt * 16 + r + 8 e, where r = lane / 4 is the row group of the lane that holds
// that value in the MMA accumulator layout (WarpAttn: lane holds heads 2 (lane
// % 4) and + 1, dimensions mt * 16 + lane / 4 (+ 8)).  So each lane writes, and
// the merging warp's same lane reads, its own D/8 values per head as whole
// 16-byte vectors, and the merge needs no exchange between lanes.  (m, l) sit
// in the [row][part][2] array as for the combine.

// This warp's partial state of its G heads into partition `part`'s slots.
template <int D>
__device__ __forceinline__ void store_partial_lanes(const WarpAttn<D>& st, const DecodeParams& p, size_t row0,
                                                    int part, int G, int lane) {
  const int n0 = 2 * (lane & 3), r = lane >> 2;
  const size_t slot0 = (row0 + n0) * p.max_parts + part;  // head n0; head n0 + 1 is max_parts slots further
  float4* po0 = reinterpret_cast<float4*>(p.ws_o + slot0 * D + r * (D / 8));
  float4* po1 = reinterpret_cast<float4*>(p.ws_o + (slot0 + p.max_parts) * D + r * (D / 8));
#pragma unroll
  for (int k = 0; k < D / 32; ++k) {  // vector k: mt = 2k and 2k + 1
    if (n0 < G) po0[k] = make_float4(st.o[2 * k][0], st.o[2 * k][2], st.o[2 * k + 1][0], st.o[2 * k + 1][2]);
    if (n0 + 1 < G) po1[k] = make_float4(st.o[2 * k][1], st.o[2 * k][3], st.o[2 * k + 1][1], st.o[2 * k + 1][3]);
  }
  if (lane < 4) {
    float2* pml = reinterpret_cast<float2*>(p.ws_ml) + slot0;
    if (n0 < G) pml[0] = make_float2(st.m0, st.l0);
    if (n0 + 1 < G) pml[p.max_parts] = make_float2(st.m1, st.l1);
  }
}

// Log-sum-exp merge of a unit's n <= kMaxMergeParts partitions into `st`:
//   M = max_i m_i,  o = sum_i 2^(m_i - M) o_i,  l = sum_i 2^(m_i - M) l_i
// (m in the log2 domain, o unnormalised relative to m), the sums taken in
// partition order, so the result is the same bits whichever warp merges.  The
// merging warp's own partition `own` has been stored like the others; its
// (m, l) come from registers.
// The loads of kB partials are issued before any is used (one L2 round trip
// per batch), the first batch together with the (m, l) loads.
// Partials per batch (kB): at head_dim 64 with six-stage rings all of them, so
// that every load of the merge, (m, l) included, is in one L2 round trip (two
// CTAs per SM are set by shared memory, so the registers cost no occupancy);
// the configurations sized for three CTAs per SM run at a 168-register cap.
template <int D, int kB>
__device__ __forceinline__ void merge_lanes(WarpAttn<D>& st, const DecodeParams& p, size_t row0, int pb, int n,
                                            int own, int G, int lane) {
  constexpr int V = D / 32;                // 16-byte vectors per head per lane
  const int n0 = 2 * (lane & 3), r = lane >> 2;
  const bool h0 = n0 < G, h1 = n0 + 1 < G;
  const size_t slot0 = (row0 + n0) * p.max_parts + pb;
  const float2* ml = reinterpret_cast<const float2*>(p.ws_ml) + slot0;
  float2 a[kMaxMergeParts], c[kMaxMergeParts];
#pragma unroll
  for (int i = 0; i < kMaxMergeParts; ++i) {
    const bool other = i < n && i != own;
    a[i] = i == own ? make_float2(st.m0, st.l0)
                    : (other && h0 ? __ldcg(ml + i) : make_float2(-CUDART_INF_F, 0.f));
    c[i] = i == own ? make_float2(st.m1, st.l1)
                    : (other && h1 ? __ldcg(ml + p.max_parts + i) : make_float2(-CUDART_INF_F, 0.f));
  }
  const float* base0 = p.ws_o + slot0 * D + r * (D / 8);
  const float* base1 = p.ws_o + (slot0 + p.max_parts) * D + r * (D / 8);
  float4 x0[kB][V], x1[kB][V];
  auto load_batch = [&](int i0) {
#pragma unroll
    for (int j = 0; j < kB; ++j) {
      const int i = i0 + j;
      const float4* s0 = reinterpret_cast<const float4*>(base0 + (size_t)i * D);
      const float4* s1 = reinterpret_cast<const float4*>(base1 + (size_t)i * D);
#pragma unroll
      for (int k = 0; k < V; ++k) {
        x0[j][k] = i < n && h0 ? __ldcg(s0 + k) : make_float4(0.f, 0.f, 0.f, 0.f);
        x1[j][k] = i < n && h1 ? __ldcg(s1 + k) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  };
  load_batch(0);  // in flight with the (m, l) loads: the maximum below needs only the latter
  float M0 = -CUDART_INF_F, M1 = -CUDART_INF_F;
#pragma unroll
  for (int i = 0; i < kMaxMergeParts; ++i) {
    M0 = fmaxf(M0, a[i].x);
    M1 = fmaxf(M1, c[i].x);
  }
  st.l0 = st.l1 = 0.f;
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) st.o[mt][0] = st.o[mt][1] = st.o[mt][2] = st.o[mt][3] = 0.f;
#pragma unroll
  for (int i0 = 0; i0 < kMaxMergeParts; i0 += kB) {
    if (i0 >= n) break;
    if (i0 > 0) load_batch(i0);
#pragma unroll
    for (int j = 0; j < kB; ++j) {
      const int i = i0 + j;
      if (i >= kMaxMergeParts) break;
      const float wa = a[i].x == -CUDART_INF_F ? 0.f : exp2f(a[i].x - M0);  // absent partition: weight 0
      const float wc = c[i].x == -CUDART_INF_F ? 0.f : exp2f(c[i].x - M1);
      st.l0 = fmaf(wa, a[i].y, st.l0);
      st.l1 = fmaf(wc, c[i].y, st.l1);
#pragma unroll
      for (int k = 0; k < V; ++k) {
        st.o[2 * k][0] = fmaf(wa, x0[j][k].x, st.o[2 * k][0]);
        st.o[2 * k][2] = fmaf(wa, x0[j][k].y, st.o[2 * k][2]);
        st.o[2 * k + 1][0] = fmaf(wa, x0[j][k].z, st.o[2 * k + 1][0]);
        st.o[2 * k + 1][2] = fmaf(wa, x0[j][k].w, st.o[2 * k + 1][2]);
        st.o[2 * k][1] = fmaf(wc, x1[j][k].x, st.o[2 * k][1]);
        st.o[2 * k][3] = fmaf(wc, x1[j][k].y, st.o[2 * k][3]);
        st.o[2 * k + 1][1] = fmaf(wc, x1[j][k].z, st.o[2 * k + 1][1]);
        st.o[2 * k + 1][3] = fmaf(wc, x1[j][k].w, st.o[2 * k + 1][3]);
      }
    }
  }
  st.m0 = M0;
  st.m1 = M1;
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
  // decode_dynamic_kernel: one prefix / length array per warp up to
  // kWarpScanBatch sequences, one per CTA above.
  static __host__ __device__ constexpr int decode_smem_bytes(int B) {
    return kPrefixOffset + (B <= kWarpScanBatch ? NW : 1) * (2 * B + 1) * 4 + 1024;
  }
};

// Resident CTAs per SM the configurations are sized for (shared memory allows
// that many): the register budget ptxas may use follows from it.
template <int D>
__host__ __device__ constexpr int dynamic_min_blocks() { return D == 128 ? 3 : 2; }
// The decode kernel's: head_dim 64 with rings of at most four stages (the
// configuration for steps merged by the combine kernel) runs three CTAs.
template <int D, int ST>
__host__ __device__ constexpr int decode_min_blocks() { return D == 64 && ST <= 4 ? 3 : dynamic_min_blocks<D>(); }
template <int D, int ST>
__host__ __device__ constexpr int merge_batch() { return D == 64 ? (decode_min_blocks<D, ST>() == 2 ? kMaxMergeParts : 2) : 1; }

template <int D, int NW, int ST, bool APPEND, bool CASCADE = false>
__global__ void __launch_bounds__(NW * 32, decode_min_blocks<D, ST>())
    decode_dynamic_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                          const DecodeParams p) {
  using Cfg = DynCfg<D, NW, ST>;
  constexpr uint32_t FULL = 0xffffffffu;
  constexpr bool kPairs = ST >= 4;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int G = p.group, Hkv = p.hkv, P = p.partition, B = p.batch;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const bool warp_scan = B <= kWarpScanBatch;
  int* scratch = reinterpret_cast<int*>(smem + Cfg::kScratchOffset);
  // [B+1] items before sequence b, then [B] clamped context lengths: this
  // warp's own arrays (warp_scan), else the CTA's.
  int* pre = reinterpret_cast<int*>(smem + Cfg::kPrefixOffset) + (warp_scan ? warp * (2 * B + 1) : 0);
  int* lens = pre + B + 1;

  // The next kernel on the stream (the combine, or the next step when it is a
  // programmatic dependent too) may launch now; it waits for this grid to
  // finish before it touches global memory.
  pdl_launch_dependents();

  const uint32_t ring = smem_addr(smem) + warp * ST * Cfg::kStageBytes;
  const uint32_t bars = smem_addr(smem + Cfg::kBarOffset) + warp * ST * 8;
  // A warp's first two items are fixed by its index (W warps in the grid: items
  // w and W + w); later ones are claimed from the counter, offset by 2W, so the
  // launch does not start with every warp contending for one address.
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < ST; ++s) mbar_init(bars + 8 * s, 1);
    mbar_init_fence();
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  if (tid == 0) {
    // The small inputs the prologue reads one after another (lengths, then
    // block tables and queries), brought into L2 while the preceding kernel
    // finishes: each CTA a share.  Prefetches only warm L2; they read no value
    // this grid uses before the wait below.
    auto share = [&](const void* base, size_t bytes) {
      const size_t chunk = max((size_t)256, (bytes + gridDim.x - 1) / gridDim.x);
      const size_t off = (size_t)blockIdx.x * chunk;
      if (off < bytes) prefetch_l2(static_cast<const char*>(base) + off, min(chunk, bytes - off));
    };
    share(p.context_lens, (size_t)B * 4);
    share(p.block_tables, (size_t)B * p.max_blocks * 4);
    share(p.q, (size_t)B * p.hq * D * 2);
    if (APPEND) {
      share(p.k_new, (size_t)B * Hkv * D * 2);
      share(p.v_new, (size_t)B * Hkv * D * 2);
    }
  }
  // Nothing above touched global memory; the preceding kernel's writes (and
  // its reads of what this grid writes) are complete after this.  (The
  // cascade's own-range pass reads nothing its preceding prefix pass writes
  // and waits for it at its end instead, so the two passes overlap.)
  if (!CASCADE) pdl_wait();

  // ---- items before each sequence ---------------------------------------------
  const int W = gridDim.x * NW, wg = blockIdx.x * NW + warp;
  if (warp_scan) {
    // This warp alone.
    warp_items_scan(p, B, Hkv, p.log2_partition, wg == 0, pre, lens, lane,
                    [&](int b, int L) { return seq_start<CASCADE>(p, b, L); });
  } else {
    // The CTA together: all lengths loaded at once (independent loads), then scanned.
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
  }
  const int T = pre[B];
  // Sequences with nothing to attend (L == 0) get zero rows; no item covers
  // them.  (A cascade sharer whose range lies inside the shared prefix has no
  // item either: the prefix pass writes its rows.)  Warp wg takes sequences
  // wg, wg + W, ...
  for (int b = wg; b < B; b += W) {
    if (pre[b + 1] != pre[b] || (CASCADE && lens[b] != 0)) continue;
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + (size_t)b * p.hq * D;
    for (int i = lane; i < p.hq * D; i += 32) o[i] = __float2bfloat16_rn(0.f);
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
      for (int ck = 0; ck < ci.n;) {
        fill();
        // Two slices per step where the ring is deep enough to keep loading
        // while both are attended.
        const int step = (kPairs && ck + 1 < ci.n) ? 2 : 1;
        bool ok = mbar_wait_bounded(bars + 8 * (gc % ST), (gc / ST) & 1, kWaitLimitNs);
        if (step == 2) ok = ok && mbar_wait_bounded(bars + 8 * ((gc + 1) % ST), ((gc + 1) / ST) & 1, kWaitLimitNs);
        ok = __all_sync(FULL, ok);
        if (!ok) {
          aborted = true;
          break;
        }
        const uint32_t kbase = ring + (gc % ST) * Cfg::kStageBytes;
        const uint32_t vbase = kbase + Cfg::kSliceBytes;
        const uint32_t kbase1 = ring + ((gc + 1) % ST) * Cfg::kStageBytes;
        const uint32_t vbase1 = kbase1 + Cfg::kSliceBytes;
        if (append_item && ck + step == ci.n) {
          // The item's last slice holds position L-1: append the new rows.
          overwrite_slice_row<D>(step == 2 ? kbase1 : kbase, step == 2 ? vbase1 : vbase,
                                 (ci.L - 1) & (kSliceTokens - 1), knew, vnew, lane);
          if (lane < D / 8) {
            const int phys = p.block_tables[(size_t)ci.b * p.max_blocks + ((ci.L - 1) >> p.log2_bs)];
            if (phys >= 0 && phys < p.num_blocks) {
              const size_t dst = (size_t)cache_row(p, phys, ci.g, ci.L - 1) * D + lane * 8;
              *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(const_cast<void*>(p.k_cache)) + dst) = knew;
              *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(const_cast<void*>(p.v_cache)) + dst) = vnew;
            }
          }
        }
        if (step == 2) {
          attend_pair<D>(st, qf, kbase, vbase, kbase1, vbase1, (ci.j0 + ck) * kSliceTokens, ci.lo, ci.hi, qk_scale,
                         p, lane);
        } else {
          attend_slice<D>(st, qf, kbase, vbase, (ci.j0 + ck) * kSliceTokens, ci.lo, ci.hi, qk_scale, p, lane);
        }
        __syncwarp();
        gc += step;
        ck += step;
      }
      if (aborted) break;
      fill();  // keep loading the next item while this one is stored

      // ---- store this item's result from registers ------------------------------------
      st.reduce_sums();
      const size_t row0 = (size_t)ci.b * p.hq + (size_t)ci.g * G;
      bool write_rows = ci.whole;
      if (!ci.whole && !p.merge_in_kernel) {  // the combine kernel merges: [row][part][D] partials
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
      } else if (!ci.whole) {  // merged in this kernel
        // Publish the partial and count it with one acquire-release atomic
        // (lane 0, after the warp barrier that orders every lane's stores
        // before it); the unit's last partial merges them all, its lanes'
        // loads ordered after the acquire by a second warp barrier.  (One
        // atomic with both orderings measured 0.6 us shorter on B200 than a
        // release fence followed by a relaxed count and an acquire fence.)
        store_partial_lanes<D>(st, p, row0, ci.part, G, lane);
        __syncwarp();
        int* cnt = p.unit_count + (size_t)ci.b * Hkv + ci.g;
        int last = 0;
        if (lane == 0) last = atom_add_acq_rel_gpu(cnt, 1) == ci.parts - 1;
        if (__shfl_sync(FULL, last, 0)) {
          __syncwarp();
          merge_lanes<D, merge_batch<D, ST>()>(st, p, row0, ci.pb, ci.parts, ci.part - ci.pb, G, lane);
          write_rows = true;
          if (lane == 0) *cnt = 0;  // every partial of the unit has arrived: ready for the next call
        }
      }
      if (write_rows) {  // the normalised rows of the G heads, from registers
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
