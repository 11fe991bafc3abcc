// Paged prefill attention on the 5th-generation tensor cores (tcgen05 / UMMA,
// accumulators in tensor memory).
//
// One CTA takes 128 query rows of one sequence and kv head: TQ = 128 / G query
// tokens x G heads, row r = (token j0 + r / G, head r % G), the token at
// position p = L - T + j attending the positions [s0(p + 1), p] of its
// sequence (causal, sliding window).  The K and V of the union of those ranges
// stream through two rings of 64-token tiles (2-D TMA boxes of 16 rows per
// physical block, SWIZZLE_128B, which is the canonical K-major layout for K
// and the MN-major layout for V).  The rings are separate so that a K stage is
// refilled as soon as its S = Q K^T is done and a V stage as soon as its P V
// is: K runs two tiles ahead of S without waiting for the P V of the tile
// before.  Per tile:
//   S = Q K^T        UMMA M=128, N=64, K=D     into one of two TMEM S buffers
//   softmax          warps 0-3: each thread owns one query row (its TMEM lane):
//                    tcgen05.ld of its 64 scores, scale / softcap / masks,
//                    online max and sum, O rescale in TMEM when the max moved,
//                    P (bf16) back into the TMEM columns its S came from
//   O += P V         UMMA M=128, N=D, K=64, A (P) from TMEM     into TMEM
// P never goes through shared memory, which leaves room for a third K stage.
// Warp 5 issues the TMA loads (one box per lane), refilling each stage as soon
// as the MMA that reads it is done.  Warp 4 issues the MMAs from lane 0: S for
// the next tile before waiting for this tile's P, so the tensor core computes
// S(i+1) while the softmax warps work on S(i).  (A per-tile timeline of the
// version with one K+V ring and one warp for loads and MMAs, on B200: the
// softmax warps waited 1-1.6 us per tile for S, whose K tile was loaded only
// after the previous P V had freed the stage.)  Completion
// travels through mbarriers (TMA bytes, tcgen05.commit); every wait is
// bounded.  V rows of a tile outside the union range are zeroed in shared
// memory before P V (P is 0 there, and a NaN canary would still poison it).
#pragma once

#include "decode_common.cuh"
#include "ptx.cuh"
#include "umma.cuh"

namespace pa {

template <int D>
struct PrefillCfg {
  static constexpr int kPanels = D / 64;         // 64-element (128-byte) column panels
  static constexpr int kTile = 64;               // K/V tokens per stage
  static constexpr int kKStages = D <= 64 ? 4 : 3;  // K ring
  static constexpr int kVStages = D <= 64 ? 4 : 2;  // V ring
  static constexpr int kRows = 128;              // query rows per CTA (UMMA M)
  static constexpr int kQPanelBytes = kRows * 128;
  static constexpr int kKVPanelBytes = kTile * 128;
  static constexpr int kKBytes = kPanels * kKVPanelBytes;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kPanels * kQPanelBytes;
  static constexpr int kVOff = kKOff + kKStages * kKBytes;
  static constexpr int kBarOff = kVOff + kVStages * kKBytes;
  static constexpr int kBarBytes = 256;
  // Exactly the layout plus the barrier area (the dynamic shared-memory base is
  // 1024-byte aligned; the kernel checks it), and at least 80 KB so that no more
  // CTAs share an SM than its 512 tensor-memory columns hold (kTmemCols each):
  // two CTAs per SM for head_dim 64 and 128, one for 256.
  static constexpr int kSmemBytes = (kBarOff + kBarBytes) > 80 * 1024 ? (kBarOff + kBarBytes) : 80 * 1024;
  static_assert(16 * (kKStages + kVStages) + 48 <= kBarBytes, "barrier area");
  static constexpr int kSCol = 0;                // two S buffers: columns [0, 64) and [64, 128)
  static constexpr int kOCol = 2 * kTile;        // O: columns [128, 128 + D)
  static constexpr int kTmemCols = (2 * kTile + D) <= 256 ? 256 : 512;
  static constexpr int kThreads = 192;           // 4 softmax warps, the MMA warp, the TMA warp
  // Register budget: two resident CTAs per SM for head_dim <= 128.
  static constexpr int kBoundThreads = 192;
  static constexpr int kMinBlocks = D <= 128 ? 2 : 1;
};

template <int D>
__global__ void __launch_bounds__(PrefillCfg<D>::kBoundThreads, PrefillCfg<D>::kMinBlocks)
    prefill_umma_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                        const DecodeParams p) {
  using C = PrefillCfg<D>;
  constexpr uint32_t FULL = 0xffffffffu;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  // Grid (kv heads, sequences, query tiles): blockIdx.z counts a sequence's
  // query tiles back from its last one, so every sequence's longest tiles (the
  // most keys under the causal mask) are dispatched first and the short ones
  // fill the end of the launch.
  const int g = blockIdx.x, b = blockIdx.y, back = blockIdx.z, G = p.group;
  const int TQ = C::kRows / G;
  if (smem_addr(smem) & 1023) {  // the swizzled tiles need 1024-byte alignment
    if (tid == 0) raise_error(PA_DEVERR_LAYOUT);
    return;
  }

  // ---- this CTA's query tokens and K/V range ------------------------------------------
  const int a = p.cu_q[b], e = p.cu_q[b + 1];
  if (a < 0 || e < a || e > p.total_q || e - a > p.max_q_len) {  // malformed offsets: report, write nothing
    if (back == 0 && g == 0 && tid == 0) raise_error(PA_DEVERR_CONTEXT);
    return;
  }
  const int T = e - a;
  const int tile = (T + TQ - 1) / TQ - 1 - back;
  if (tile < 0) return;
  const int j0 = tile * TQ;
  const int ntok = min(TQ, T - j0);
  if (ntok <= 0) return;
  const int L = clamp_context(p, b, back == 0 && g == 0 && tid == 0);
  const int ulo = window_start(max(L - T + j0 + 1, 0), p.window);
  const int uhi = min(L, L - T + j0 + ntok);
  const size_t row0 = (size_t)a + j0;  // q / out row of token j0
  if (ulo >= uhi) {  // no token of the tile has a position: zero rows
    for (int idx = tid; idx < ntok * G * D; idx += blockDim.x) {
      const int r = idx / D;
      static_cast<__nv_bfloat16*>(p.out)[((row0 + r / G) * p.hq + (size_t)g * G + r % G) * D + idx % D] =
          __float2bfloat16_rn(0.f);
    }
    return;
  }
  const int kt0 = (ulo / C::kTile) * C::kTile;
  const int n_kv = (uhi - kt0 + C::kTile - 1) / C::kTile;

  const uint32_t s_base = smem_addr(smem);
  const uint32_t q_s = s_base + C::kQOff, k_s = s_base + C::kKOff, v_s = s_base + C::kVOff;
  const uint32_t bar = s_base + C::kBarOff;
  // Barrier area: kfull/kempty[kKStages], vfull/vempty[kVStages], sfull[2],
  // pready, odone, the TMEM address slot and the abort flag.
  constexpr int NK = C::kKStages, NV = C::kVStages;
  const uint32_t kfull_b = bar, kempty_b = bar + 8 * NK;
  const uint32_t vfull_b = bar + 16 * NK, vempty_b = bar + 16 * NK + 8 * NV;
  const uint32_t sfull_b = bar + 16 * (NK + NV);
  const uint32_t pready_b = sfull_b + 16, odone_b = sfull_b + 24, drain_b = sfull_b + 32;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + 16 * (NK + NV) + 40);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kBarOff + 16 * (NK + NV) + 44);

  if (tid == 0) {
    for (int s = 0; s < NK; ++s) {
      mbar_init(kfull_b + 8 * s, 1);
      mbar_init(kempty_b + 8 * s, 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(vfull_b + 8 * s, 1);
      mbar_init(vempty_b + 8 * s, 1);
    }
    mbar_init(sfull_b, 1);
    mbar_init(sfull_b + 8, 1);
    mbar_init(pready_b, 4);
    mbar_init(odone_b, 1);
    mbar_init(drain_b, 1);
    *abort_flag = 0;
    mbar_init_fence();
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  if (warp == 0) umma::alloc(smem_addr(tmem_slot), C::kTmemCols);

  // ---- Q tile into shared memory (canonical K-major SWIZZLE_128B) ------------------------
  if (tid < C::kRows) {
    const int r = tid;
    const bool real = r / G < ntok;
    const __nv_bfloat16* qrow =
        static_cast<const __nv_bfloat16*>(p.q) + ((row0 + r / G) * p.hq + (size_t)g * G + r % G) * D;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      const uint4 v = real ? *reinterpret_cast<const uint4*>(qrow + c * 8) : make_uint4(0, 0, 0, 0);
      const uint32_t dst = q_s + (c >> 3) * C::kQPanelBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                   : "memory");
    }
  }
  fence_proxy_async_smem();
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = *tmem_slot;
  const float qk_scale = p.use_softcap ? p.scale : p.scale * kLog2e;
  const int32_t* table = p.block_tables + (size_t)b * p.max_blocks;

  // Wait for completion number `use` of a barrier (completions alternate parity).
  auto wait_use = [&](uint32_t b, int use) { return __all_sync(FULL, mbar_wait_bounded(b, use & 1, kWaitLimitNs)); };
  if (warp == 5) {
    // ================= TMA producer =================
    // K (kv = 0) or V (kv = 1) of tile i into its ring's stage: one 2-D box per
    // lane (slice s = lane / panels, panel).
    int issued[2] = {0, 0};
    // Physical blocks of the 16-token slices, per ring: lane l holds slice
    // wb + l (cur) and wb + 32 + l (nxt), and the window after is loaded as soon
    // as a ring moves on, so no load waits on a block-table read (with the read
    // in line, the producer took one L2 round trip per tile and set the pace).
    auto page_of = [&](int q) {  // slice q of the K/V range; -1 past the attended range
      const int t = kt0 + q * kSliceTokens;
      return t < uhi ? table[t >> p.log2_bs] : -1;
    };
    int wb[2] = {0, 0}, wcur[2], wnxt[2];
    wcur[0] = wcur[1] = page_of(lane);
    wnxt[0] = wnxt[1] = page_of(32 + lane);
    auto issue_kv = [&](int i, int kv) {
      const int stage = i % (kv ? NV : NK);
      const uint32_t full = (kv ? vfull_b : kfull_b) + 8 * stage;
      const int kt = kt0 + i * C::kTile;
      if (4 * i >= wb[kv] + 32) {  // tiles advance one at a time: the window moves by 32 slices
        wb[kv] += 32;
        wcur[kv] = wnxt[kv];
        wnxt[kv] = page_of(wb[kv] + 32 + lane);
      }
      const int box = lane;
      const int s = box / C::kPanels, pn = box % C::kPanels;
      const int t = kt + s * kSliceTokens;
      const int page = __shfl_sync(FULL, wcur[kv], (4 * i + (s & 3) - wb[kv]) & 31);
      bool valid = false;
      int y = -1;
      if (box < 4 * C::kPanels && t + kSliceTokens > ulo && t < uhi) {
        const int phys = page;
        if (phys >= 0 && phys < p.num_blocks) {
          valid = true;
          y = cache_row(p, phys, g, t);
        } else if (kv == 0 && pn == 0) {
          raise_error(PA_DEVERR_BLOCK);
        }
      }
      const uint32_t nvalid = __popc(__ballot_sync(FULL, valid));
      if (lane == 0) {
        if (nvalid) mbar_arrive_expect_tx(full, nvalid * kSliceTokens * 128);
        else mbar_arrive(full);
      }
      __syncwarp();
      if (valid) {
        const uint32_t dst = (kv ? v_s : k_s) + stage * C::kKBytes + pn * C::kKVPanelBytes + s * kSliceTokens * 128;
        tma_load_2d(dst, kv ? &vmap : &kmap, full, pn * 64, y);
      }
      issued[kv] = i + 1;
    };
    // A K stage frees when the S that read it is done, a V stage when its P V
    // is.  The MMAs complete in issue order, S(m + 1) before P V(m), so the
    // refills go in that order: K(m + 1 + NK) after S(m + 1), V(m + NV) after
    // P V(m).
    auto refill = [&](int j, int kv) {  // tile j into the stage tile j - N (N = the ring's stages) used
      const int n = kv ? NV : NK, u = j - n;
      if (!wait_use((kv ? vempty_b : kempty_b) + 8 * (u % n), u / n)) return false;
      issue_kv(j, kv);
      return true;
    };
    bool ok = true;
    for (int i = 0; i < NK && i < n_kv; ++i) issue_kv(i, 0);
    for (int i = 0; i < NV && i < n_kv; ++i) issue_kv(i, 1);
    if (NK < n_kv) ok = refill(NK, 0);
    for (int m = 0; ok && (m + 1 + NK < n_kv || m + NV < n_kv); ++m) {
      if (*abort_flag) break;
      if (m + 1 + NK < n_kv) ok = refill(m + 1 + NK, 0);
      if (ok && m + NV < n_kv) ok = refill(m + NV, 1);
    }
    if (!ok) {
      if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
    if (!ok || *abort_flag) {
      // Before the CTA releases its shared memory: give the last loads of each
      // ring a bounded time to land (earlier ones have, their stages were reused).
      for (int kv = 0; kv < 2; ++kv) {
        const int n = kv ? NV : NK;
        for (int j = max(issued[kv] - n, 0); j < issued[kv]; ++j)
          (void)mbar_wait_bounded((kv ? vfull_b : kfull_b) + 8 * (j % n), (j / n) & 1, kDrainLimitNs);
      }
    }
  } else if (warp == 4) {
    // ================= MMA issuer (lane 0) =================
    const uint32_t idesc_s = umma::idesc_bf16(128, C::kTile, 0, 0);
    const uint32_t idesc_o = umma::idesc_bf16(128, D, 0, 1);
    auto issue_s = [&](int i) {  // S(i) = Q K(i)^T into buffer i % 2
      const uint32_t kst = k_s + (i % NK) * C::kKBytes;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t ad = umma::desc_sw128(q_s + (kk >> 2) * C::kQPanelBytes + (kk & 3) * 32, 16, 1024);
        const uint64_t bd = umma::desc_sw128(kst + (kk >> 2) * C::kKVPanelBytes + (kk & 3) * 32, 16, 1024);
        umma::mma_f16(tmem + C::kSCol + (i & 1) * C::kTile, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
      }
      umma::commit(sfull_b + 8 * (i & 1));
      umma::commit(kempty_b + 8 * (i % NK));
    };
    auto issue_o = [&](int i) {  // O += P V(i), P (bf16 pairs) in the columns of S buffer i % 2
      const uint32_t vst = v_s + (i % NV) * C::kKBytes;
      const uint32_t pcol = tmem + C::kSCol + (i & 1) * C::kTile;
#pragma unroll
      for (int k = 0; k < C::kTile / 16; ++k) {
        const uint64_t bd = umma::desc_sw128(vst + k * 16 * 128, C::kKVPanelBytes, 1024);
        umma::mma_f16_tmem_a(tmem + C::kOCol, pcol + k * 8, bd, idesc_o, (i > 0 || k > 0) ? 1u : 0u);
      }
      umma::commit(odone_b);
      umma::commit(vempty_b + 8 * (i % NV));
    };
    auto s_when_ready = [&](int j) {
      if (!wait_use(kfull_b + 8 * (j % NK), j / NK)) return false;
      umma::fence_after();
      if (lane == 0) issue_s(j);
      __syncwarp();
      return true;
    };
    bool ok = s_when_ready(0);
    for (int i = 0; ok && i < n_kv; ++i) {
      if (i + 1 < n_kv && !(ok = s_when_ready(i + 1))) break;
      ok = wait_use(pready_b, i);
      if (!ok || *abort_flag) break;
      if (!(ok = wait_use(vfull_b + 8 * (i % NV), i / NV))) break;
      umma::fence_after();
      if (lane == 0) issue_o(i);
      __syncwarp();
    }
    if (!ok) {
      if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
    if (!ok || *abort_flag) {  // the MMAs issued get a bounded time to finish before TMEM is freed
      if (lane == 0) umma::commit(drain_b);
      (void)mbar_wait_bounded(drain_b, 0, kDrainLimitNs);
    }
  } else {
    // ================= softmax warps 0-3: one query row per thread =================
    const int r = tid;  // TMEM lane = row
    const bool real = r / G < ntok;
    const int end_r = L - T + j0 + r / G + 1;  // p + 1
    const int lo_r = real ? max(window_start(max(end_r, 0), p.window), 0) : ulo;
    const int hi_r = real ? min(end_r, L) : uhi;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
    // Tiles that need no mask for any row of this warp: [w_lo, w_hi) is valid
    // for all of them.
    const int w_lo = __reduce_max_sync(FULL, lo_r), w_hi = __reduce_min_sync(FULL, hi_r);
    float m = -CUDART_INF_F, l = 0.f;
    bool ok = true;
    for (int i = 0; i < n_kv; ++i) {
      ok = __all_sync(FULL, mbar_wait_bounded(sfull_b + 8 * (i & 1), (i >> 1) & 1, kWaitLimitNs));
      if (!ok || *abort_flag) break;
      umma::fence_after();
      const int kt = kt0 + i * C::kTile;
      float x[C::kTile];
      {
        uint32_t u[C::kTile / 16][16];
#pragma unroll
        for (int c = 0; c < C::kTile / 16; ++c)
          umma::ld16_nowait(lane_base + C::kSCol + (i & 1) * C::kTile + c * 16, u[c]);
        umma::wait_ld();
#pragma unroll
        for (int c = 0; c < C::kTile / 16; ++c)
#pragma unroll
          for (int k = 0; k < 16; ++k) x[c * 16 + k] = __uint_as_float(u[c][k]);
      }
      // x becomes the log2-domain score (scaled, softcapped) in place; the
      // masks apply only where some row of the warp needs them.
      float mt = -CUDART_INF_F;
      const bool masked = kt < w_lo || kt + C::kTile > w_hi;
      if (p.use_softcap) {
#pragma unroll
        for (int k = 0; k < C::kTile; ++k) x[k] = p.softcap * tanhf(x[k] * qk_scale * p.inv_softcap) * kLog2e;
      }
      const float xs = p.use_softcap ? 1.f : qk_scale;  // scale still to apply to x
      if (masked) {
#pragma unroll
        for (int k = 0; k < C::kTile; ++k) {
          const int t = kt + k;
          x[k] = (t >= lo_r && t < hi_r) ? x[k] : -CUDART_INF_F;
        }
      }
      {  // eight independent chains, then a tree: the 64-long dependent chain took 0.2 us a tile
        float mx[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) mx[c] = x[c];
#pragma unroll
        for (int k = 8; k < C::kTile; ++k) mx[k & 7] = fmaxf(mx[k & 7], x[k]);
        mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      }
      mt *= xs;  // xs > 0: the maximum of the scaled scores
      // Lazy rescaling: keep the reference m while the tile's maximum exceeds
      // it by at most 8 (log2 units): the weights stay <= 256 and the sum and
      // output share the reference, so the result is exact; O is rescaled only
      // when the reference moves.
      const float mn = (m == -CUDART_INF_F || mt > m + 8.f) ? mt : m;
      const float ref = mn == -CUDART_INF_F ? 0.f : mn;
      const float alpha = exp2f(m - ref);
      m = mn;
      // p = 2^(xs x - ref) (one FMA and one ex2 each); the row sum in four
      // independent chains.
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[C::kTile / 2];
#pragma unroll
      for (int k = 0; k < C::kTile / 2; ++k) {
        float e0, e1;
        asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e0) : "f"(fmaf(x[2 * k], xs, -ref)));
        asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e1) : "f"(fmaf(x[2 * k + 1], xs, -ref)));
        ps[k & 3] += e0 + e1;
        pk[k] = pack_bf16x2(e0, e1);
      }
      l = l * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
      // P row r into this lane's first 32 columns of S buffer i % 2 (its S
      // values are in registers; P V(i-1) reads the other buffer).
      {
        const uint32_t pcol = lane_base + C::kSCol + (i & 1) * C::kTile;
        uint32_t (&pk0)[16] = *reinterpret_cast<uint32_t(*)[16]>(&pk[0]);
        uint32_t (&pk1)[16] = *reinterpret_cast<uint32_t(*)[16]>(&pk[16]);
        umma::st16_nowait(pcol, pk0);
        umma::st16_nowait(pcol + 16, pk1);
      }
      if (i > 0) {  // P V(i-1) must be done before O is rescaled
        ok = __all_sync(FULL, mbar_wait_bounded(odone_b, (i - 1) & 1, kWaitLimitNs));
        if (!ok) break;
        umma::fence_after();
        if (__any_sync(FULL, alpha != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < D / 16; ++c) {
            float v[16];
            umma::ld16(lane_base + C::kOCol + c * 16, v);
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] *= alpha;
            umma::st16(lane_base + C::kOCol + c * 16, v);
          }
        }
      }
      umma::wait_st();
      // V rows of this tile outside [ulo, uhi): zero (stale or canary data, P = 0 there),
      // once V(i) has landed.
      if (kt < ulo || kt + C::kTile > uhi) {
        ok = __all_sync(FULL, mbar_wait_bounded(vfull_b + 8 * (i % NV), (i / NV) & 1, kWaitLimitNs));
        if (!ok) break;
        const uint32_t vst = v_s + (i % NV) * C::kKBytes;
        for (int idx = tid; idx < C::kTile * C::kPanels * 8; idx += C::kRows) {
          const int row = idx / (C::kPanels * 8), rem = idx % (C::kPanels * 8);
          const int t = kt + row;
          if (t < ulo || t >= uhi) {
            const uint32_t dst = vst + (rem >> 3) * C::kKVPanelBytes + row * 128 + ((rem & 7) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
          }
        }
        fence_proxy_async_smem();  // the zeros are visible to the tensor core's reads
      }
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pready_b);
    }
    // ---- epilogue: O / l to the output rows ---------------------------------------------
    if (ok && !*abort_flag) ok = __all_sync(FULL, mbar_wait_bounded(odone_b, (n_kv - 1) & 1, kWaitLimitNs));
    if (ok && !*abort_flag) {
      umma::fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow =
          static_cast<__nv_bfloat16*>(p.out) + ((row0 + r / G) * p.hq + (size_t)g * G + r % G) * D;
#pragma unroll 1
      for (int c = 0; c < D / 16; ++c) {
        float v[16];
        umma::ld16(lane_base + C::kOCol + c * 16, v);
        if (real) {
          uint4 lo, hi;
          lo.x = pack_bf16x2(v[0] * inv, v[1] * inv);
          lo.y = pack_bf16x2(v[2] * inv, v[3] * inv);
          lo.z = pack_bf16x2(v[4] * inv, v[5] * inv);
          lo.w = pack_bf16x2(v[6] * inv, v[7] * inv);
          hi.x = pack_bf16x2(v[8] * inv, v[9] * inv);
          hi.y = pack_bf16x2(v[10] * inv, v[11] * inv);
          hi.z = pack_bf16x2(v[12] * inv, v[13] * inv);
          hi.w = pack_bf16x2(v[14] * inv, v[15] * inv);
          reinterpret_cast<uint4*>(orow + c * 16)[0] = lo;
          reinterpret_cast<uint4*>(orow + c * 16)[1] = hi;
        }
      }
    } else if (lane == 0) {
      raise_error(PA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
  }
  // Every tcgen05 access is complete (waited); free the tensor memory.
  umma::fence_before();
  __syncthreads();
  if (warp == 0) {
    umma::fence_after();
    umma::dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace pa
