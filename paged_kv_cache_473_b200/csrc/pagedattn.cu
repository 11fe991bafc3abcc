// C ABI of the paged KV cache library: host-side argument checks, tensor-map
// set-up, kernel selection and launches.  See include/pagedattn.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <algorithm>
#include <utility>
#include <vector>

#include "../../include/pagedattn.h"
#include "../../include/block_manager.h"
#include "combine_and_append.cuh"
#include "decode_common.cuh"
#include "decode_mma.cuh"
#include "decode_simt.cuh"
#include "decode_dynamic.cuh"
#include "decode_multi.cuh"
#include "decode_rows.cuh"
#include "prefill_umma.cuh"

namespace {

using pa::DecodeParams;

thread_local int32_t t_last_launches = 0;
thread_local int32_t t_last_schedule = PA_SCHEDULE_NONE;

constexpr int kNoSplitPartition = 1 << 30;
constexpr int kMaxPartsPerSeq = 8192;
constexpr int kMaxGridYZ = 65535;
// Split-K auto partition: aim for at least this many (partition, kv head,
// sequence) work units, i.e. several resident CTAs for each of B200's 148 SMs.
constexpr long long kTargetWorkUnits = 8LL * 148;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
int ilog2(int x) {
  int r = 0;
  while ((1 << r) < x) ++r;
  return r;
}

// ---- tensor maps ---------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool tensor_map_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// The cache viewed as a 2-D bf16 tensor [rows = num_blocks*Hkv*bs][head_dim];
// a box is 64 columns (128 B) x 16 rows, landed with 128-byte swizzle.
bool encode_cache_map(CUtensorMap* map, const void* base, int head_dim, long long rows) {
  cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)head_dim * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)pa::kSliceTokens};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor maps of the K and V caches, encoded once per (base addresses, rows,
// head_dim) and reused: a map holds only the address, the shape and the fixed
// box / swizzle, so a cached one is exactly what a fresh encode would give.
// A small per-thread table (no lock); the oldest entry is replaced.
bool cache_maps(const void* kbase, const void* vbase, int head_dim, long long rows, CUtensorMap* kmap,
                CUtensorMap* vmap) {
  struct Entry {
    const void* k;
    const void* v;
    long long rows;
    int d;
    CUtensorMap kmap, vmap;
  };
  constexpr int kEntries = 16;
  thread_local Entry table[kEntries] = {};
  thread_local int next = 0;
  for (const Entry& e : table) {
    if (e.k == kbase && e.v == vbase && e.rows == rows && e.d == head_dim && kbase) {
      *kmap = e.kmap;
      *vmap = e.vmap;
      return true;
    }
  }
  if (!tensor_map_encoder()) return false;
  if (!encode_cache_map(kmap, kbase, head_dim, rows) || !encode_cache_map(vmap, vbase, head_dim, rows)) return false;
  Entry& e = table[next];
  next = (next + 1) % kEntries;
  e.k = kbase;
  e.v = vbase;
  e.rows = rows;
  e.d = head_dim;
  e.kmap = *kmap;
  e.vmap = *vmap;
  return true;
}

// ---- argument checks -------------------------------------------------------------

struct Shape {
  int batch, hq, hkv, d, bs, max_blocks, num_blocks;
};

pa_status_t check_decode_args(const void* q, const void* kc, const void* vc, const int32_t* bt, const int32_t* cl,
                              const Shape& s, float softcap, const void* out, pa_dtype_t dt, pa_kernel_t kernel) {
  if (s.batch < 0 || s.hq <= 0 || s.hkv <= 0 || s.d <= 0 || s.bs <= 0 || s.max_blocks <= 0 || s.num_blocks <= 0)
    return PA_ERR_INVALID;
  if (s.hq % s.hkv != 0) return PA_ERR_INVALID;
  if (dt != PA_F32 && dt != PA_BF16) return PA_ERR_INVALID;
  if (kernel != PA_KERNEL_AUTO && kernel != PA_KERNEL_CUDA_CORE && kernel != PA_KERNEL_MMA) return PA_ERR_INVALID;
  if (std::isnan(softcap)) return PA_ERR_INVALID;
  if (s.batch > 0) {
    if (!q || !kc || !vc || !bt || !cl || !out) return PA_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(kc, 16) || !aligned(vc, 16) || !aligned(out, 16) || !aligned(bt, 4) ||
        !aligned(cl, 4))
      return PA_ERR_INVALID;
  }
  if (s.d != 64 && s.d != 128 && s.d != 256) return PA_ERR_UNSUPPORTED;
  if (!pow2(s.bs) || s.bs < 16 || s.bs > 256) return PA_ERR_UNSUPPORTED;
  if (s.hq / s.hkv > pa::kMaxGroup) return PA_ERR_UNSUPPORTED;
  if (s.batch > kMaxGridYZ || s.hkv > kMaxGridYZ) return PA_ERR_UNSUPPORTED;
  if ((long long)s.num_blocks * s.hkv * s.bs >= (1LL << 31)) return PA_ERR_UNSUPPORTED;
  if ((long long)s.max_blocks * s.bs >= (1LL << 30)) return PA_ERR_UNSUPPORTED;
  if (kernel == PA_KERNEL_MMA && dt != PA_BF16) return PA_ERR_UNSUPPORTED;
  return PA_OK;
}

DecodeParams make_params(const void* q, const void* kc, const void* vc, const int32_t* bt, const int32_t* cl,
                         const Shape& s, float scale, float softcap, int32_t window, void* out) {
  DecodeParams p{};
  p.q = q;
  p.out = out;
  p.k_cache = kc;
  p.v_cache = vc;
  p.block_tables = bt;
  p.context_lens = cl;
  p.batch = s.batch;
  p.hq = s.hq;
  p.hkv = s.hkv;
  p.group = s.hq / s.hkv;
  p.head_dim = s.d;
  p.block_size = s.bs;
  p.log2_bs = ilog2(s.bs);
  p.max_blocks = s.max_blocks;
  p.num_blocks = s.num_blocks;
  p.window = window;
  p.partition = kNoSplitPartition;
  p.max_parts = 1;
  p.max_context = s.max_blocks * s.bs;
  p.scale = scale;
  p.use_softcap = (softcap > 0.f && std::isfinite(softcap)) ? 1 : 0;
  p.softcap = p.use_softcap ? softcap : 0.f;
  p.inv_softcap = p.use_softcap ? 1.f / softcap : 0.f;
  p.q_len = 1;
  return p;
}

// ---- launches ---------------------------------------------------------------------

// Opt a kernel in to more than 48 KB of dynamic shared memory, once per device
// (the flag word is per kernel instantiation: one bit per device ordinal < 64).
template <typename Kernel>
cudaError_t set_smem(Kernel k, int bytes, std::atomic<uint64_t>& done) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Launch `kern` with cudaLaunchKernelEx; `pdl` lets it start while the
// preceding kernel on the stream finishes (it must call griddepcontrol.wait
// before reading that kernel's output).
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, int smem, cudaStream_t st, bool pdl,
                      Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  if (pdl) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

template <int D, int NW, int ST, bool SPLIT, bool APPEND>
cudaError_t launch_mma_t(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  using Cfg = pa::MmaCfg<D, NW, ST>;
  CUtensorMap kmap, vmap;
  const long long rows = (long long)p.num_blocks * p.hkv * p.block_size;
  if (!cache_maps(p.k_cache, p.v_cache, D, rows, &kmap, &vmap)) return cudaErrorInvalidValue;
  auto kern = pa::decode_mma_kernel<D, NW, ST, SPLIT, APPEND>;
  static std::atomic<uint64_t> smem_done{0};
  cudaError_t e = set_smem(kern, Cfg::kSmemBytes, smem_done);
  if (e != cudaSuccess) return e;
  return launch_ex(kern, grid, dim3(NW * 32), Cfg::kSmemBytes, st, false, kmap, vmap, p);
}

template <bool SPLIT, bool APPEND>
cudaError_t launch_mma(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  switch (p.head_dim) {
    case 64:
      return launch_mma_t<64, 4, 4, SPLIT, APPEND>(p, grid, st);
    case 128:
      return launch_mma_t<128, 4, 3, SPLIT, APPEND>(p, grid, st);
    default:
      return launch_mma_t<256, 2, 3, SPLIT, APPEND>(p, grid, st);
  }
}

template <int D, int ST, bool SPLIT>
cudaError_t launch_multi_t(const DecodeParams& p, dim3 grid, int warps, cudaStream_t st) {
  using Cfg = pa::MultiCfg<D, ST>;
  CUtensorMap kmap, vmap;
  const long long rows = (long long)p.num_blocks * p.hkv * p.block_size;
  if (!cache_maps(p.k_cache, p.v_cache, D, rows, &kmap, &vmap)) return cudaErrorInvalidValue;
  auto kern = pa::decode_multi_kernel<D, ST, SPLIT>;
  static std::atomic<uint64_t> smem_done{0};
  cudaError_t e = set_smem(kern, Cfg::kSmemBytes, smem_done);
  if (e != cudaSuccess) return e;
  return launch_ex(kern, grid, dim3(warps * 32), Cfg::kSmemBytes, st, false, kmap, vmap, p);
}

// Multi-query rows: one warp per 8 of the T*G query columns of a kv head (or
// of the q_tile*G columns of a cascade sharer group); the CTA's shared ring
// holds 32-64 KB of K/V slices.
template <bool SPLIT>
cudaError_t launch_multi(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  const int warps = ((p.cascade_prefix ? p.q_tile : p.q_len) * p.group + 7) / 8;
  switch (p.head_dim) {
    case 64:
      return launch_multi_t<64, 8, SPLIT>(p, grid, warps, st);
    case 128:
      return launch_multi_t<128, 6, SPLIT>(p, grid, warps, st);
    default:
      return launch_multi_t<256, 4, SPLIT>(p, grid, warps, st);
  }
}

template <typename T, int D, int GP, bool SPLIT, bool APPEND>
cudaError_t launch_simt_t(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  constexpr int NW = 4;
  const int smem = pa::merge_smem_bytes<NW>(D);
  auto kern = pa::decode_simt_kernel<T, D, GP, NW, SPLIT, APPEND>;
  static std::atomic<uint64_t> smem_done{0};
  cudaError_t e = set_smem(kern, smem, smem_done);
  if (e != cudaSuccess) return e;
  return launch_ex(kern, grid, dim3(NW * 32), smem, st, false, p);
}

template <typename T, int D, bool SPLIT, bool APPEND>
cudaError_t launch_simt_d(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  const int G = p.group;
  if (G <= 1) return launch_simt_t<T, D, 1, SPLIT, APPEND>(p, grid, st);
  if (G <= 2) return launch_simt_t<T, D, 2, SPLIT, APPEND>(p, grid, st);
  if (G <= 4) return launch_simt_t<T, D, 4, SPLIT, APPEND>(p, grid, st);
  return launch_simt_t<T, D, 8, SPLIT, APPEND>(p, grid, st);
}

template <typename T, bool SPLIT, bool APPEND>
cudaError_t launch_simt(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  switch (p.head_dim) {
    case 64:
      return launch_simt_d<T, 64, SPLIT, APPEND>(p, grid, st);
    case 128:
      return launch_simt_d<T, 128, SPLIT, APPEND>(p, grid, st);
    default:
      return launch_simt_d<T, 256, SPLIT, APPEND>(p, grid, st);
  }
}

template <bool SPLIT, bool APPEND>
cudaError_t launch_decode(const DecodeParams& p, pa_dtype_t dt, pa_kernel_t kernel, dim3 grid, cudaStream_t st) {
  const bool use_mma = (kernel == PA_KERNEL_MMA) || (kernel == PA_KERNEL_AUTO && dt == PA_BF16);
  if (use_mma) return launch_mma<SPLIT, APPEND>(p, grid, st);
  if (dt == PA_BF16) return launch_simt<__nv_bfloat16, SPLIT, APPEND>(p, grid, st);
  return launch_simt<float, SPLIT, APPEND>(p, grid, st);
}

template <typename OutT, int NWR>
cudaError_t launch_combine_n(const DecodeParams& p, cudaStream_t st) {
  constexpr int rows_per_cta = pa::kCombineWarps / NWR;
  const int rows = p.batch * p.q_len * p.hq;
  dim3 grid((rows + rows_per_cta - 1) / rows_per_cta);
  dim3 block(pa::kCombineWarps * 32);
  switch (p.head_dim) {
    case 64:
      return launch_ex(pa::combine_kernel<OutT, 64, NWR>, grid, block, 0, st, true, p);
    case 128:
      return launch_ex(pa::combine_kernel<OutT, 128, NWR>, grid, block, 0, st, true, p);
    default:
      return launch_ex(pa::combine_kernel<OutT, 256, NWR>, grid, block, 0, st, true, p);
  }
}

// One warp per row when rows have few partitions; eight when they have many.
template <typename OutT>
cudaError_t launch_combine(const DecodeParams& p, cudaStream_t st) {
  return p.max_parts > 16 ? launch_combine_n<OutT, 8>(p, st) : launch_combine_n<OutT, 1>(p, st);
}

int sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 64) {
    const int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// Opt in to `bytes` of dynamic shared memory (growing only), once per device
// and size, for kernels whose size depends on the launch.
template <typename Kernel>
cudaError_t set_smem_at_least(Kernel k, int bytes, std::atomic<int>* done /* [64] */) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && done[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev < 64) {
    int cur = done[dev].load(std::memory_order_acquire);
    while (cur < bytes && !done[dev].compare_exchange_weak(cur, bytes)) {
    }
  }
  return e;
}

// Resident CTAs per SM of `kern` at `threads` x `smem`, on the current device:
// queried once per (kernel, shared-memory size, device) and remembered (one
// entry per device for each kernel instantiation; `cache` is that kernel's).
template <typename Kernel>
cudaError_t occupancy(Kernel kern, int threads, int smem, std::atomic<long long>* cache /* [64] */, int* occ) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64) {
    const long long v = cache[dev].load(std::memory_order_acquire);
    if (v > 0 && (v >> 16) == smem) {
      *occ = (int)(v & 0xffff);
      return cudaSuccess;
    }
  }
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(occ, kern, threads, smem);
  if (e == cudaSuccess && dev < 64 && *occ > 0 && *occ < 0x10000)
    cache[dev].store(((long long)smem << 16) | *occ, std::memory_order_release);
  return e;
}

// Paged prefill attention on tcgen05: one CTA per 128 query rows (128 / G
// tokens) of one sequence and kv head; grid (kv heads, sequences, query tiles
// counted back from each sequence's end), so the longest tiles go first.
template <int D>
cudaError_t launch_prefill_t(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  using Cfg = pa::PrefillCfg<D>;
  CUtensorMap kmap, vmap;
  const long long rows = (long long)p.num_blocks * p.hkv * p.block_size;
  if (!cache_maps(p.k_cache, p.v_cache, D, rows, &kmap, &vmap)) return cudaErrorInvalidValue;
  auto kern = pa::prefill_umma_kernel<D>;
  static std::atomic<uint64_t> smem_done{0};
  cudaError_t e = set_smem(kern, Cfg::kSmemBytes, smem_done);
  if (e != cudaSuccess) return e;
  // The whole shared-memory carveout, so that kMinBlocks CTAs fit per SM.
  static std::once_flag carveout_once;
  std::call_once(carveout_once, [&] {
    (void)cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  });
  return launch_ex(kern, grid, dim3(Cfg::kThreads), Cfg::kSmemBytes, st, false, kmap, vmap, p);
}

cudaError_t launch_prefill(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  switch (p.head_dim) {
    case 64:
      return launch_prefill_t<64>(p, grid, st);
    case 128:
      return launch_prefill_t<128>(p, grid, st);
    default:
      return launch_prefill_t<256>(p, grid, st);
  }
}

// Launch the dynamic schedule with the persistent grid (as many CTAs as are
// resident at once).  Sets p.merge_in_kernel: the partitions of each unit are
// merged in-kernel when the step is small next to the resident warps (at most
// 8 partitions per sequence and at most two work items per resident warp, a
// bound from the host-known sizes), where the combine kernel's fixed cost
// (launch, grid drain, L2 round trips) would be a large share of the step;
// otherwise the combine kernel merges them with full-GPU parallelism after
// the decode grid, and the merging warps do not stall their loads.
template <int D, int NW, int ST, bool APPEND, bool CASCADE>
cudaError_t launch_dynamic_t(DecodeParams& p, cudaStream_t st, bool pdl, bool allow_merge) {
  using Cfg = pa::DynCfg<D, NW, ST>;
  CUtensorMap kmap, vmap;
  const long long rows = (long long)p.num_blocks * p.hkv * p.block_size;
  if (!cache_maps(p.k_cache, p.v_cache, D, rows, &kmap, &vmap)) return cudaErrorInvalidValue;
  auto kern = pa::decode_dynamic_kernel<D, NW, ST, APPEND, CASCADE>;
  const int smem = Cfg::decode_smem_bytes(p.batch);
  static std::atomic<int> smem_done[64];
  cudaError_t e = set_smem_at_least(kern, smem, smem_done);
  if (e != cudaSuccess) return e;
  int occ = 0;
  static std::atomic<long long> occ_cache[64];
  e = occupancy(kern, Cfg::kThreads, smem, occ_cache, &occ);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  const int grid = occ * sm_count();
  const long long unit_bound = (long long)p.batch * p.hkv * p.max_parts;
  p.merge_in_kernel = (allow_merge && p.max_parts <= pa::kMaxMergeParts && unit_bound <= 2LL * grid * NW) ? 1 : 0;
  if (!pow2(p.partition)) return cudaErrorInvalidValue;  // the schedule's partitions are powers of two
  p.log2_partition = ilog2(p.partition);
  p.static_items = 2;
  return launch_ex(kern, dim3(grid), dim3(Cfg::kThreads), smem, st, pdl, kmap, vmap, p);
}

// Launched as a programmatic dependent of the preceding kernel on the stream
// (the kernel waits for it before touching global memory).  CASCADE: the
// cascade's own-range pass (sharers start at the prefix end), which overlaps
// the prefix pass and is merged by the combine.
template <bool APPEND, bool CASCADE = false>
cudaError_t launch_dynamic(DecodeParams& p, cudaStream_t st) {
  const bool pdl = true, allow_merge = !CASCADE;
  switch (p.head_dim) {
    // Warps are independent (one work item each); CTAs of a few warps with a
    // 2-6 stage ring each put ~192 KB of loads in flight per SM.
    case 64: {
      // Steps small enough for the in-kernel merge (bounded on the host as in
      // launch_dynamic_t, for two resident CTAs of four warps): 8 warps per SM
      // with six-stage rings, the merge's loads in one L2 round trip.  Larger
      // steps, merged by the combine kernel: 12 warps per SM (three CTAs,
      // four-stage rings), so more items stream at once (measured on B200:
      // TinyLlama shape with 128 sequences 47.2 -> 42.7 us; at 64 sequences,
      // merged in-kernel, the six-stage configuration is 1.8 us faster).
      const long long unit_bound = (long long)p.batch * p.hkv * p.max_parts;
      const bool merge = allow_merge && p.max_parts <= pa::kMaxMergeParts && unit_bound <= 2LL * (2 * 4) * sm_count();
      if (merge) return launch_dynamic_t<64, 4, 6, APPEND, CASCADE>(p, st, pdl, true);
      return launch_dynamic_t<64, 4, 4, APPEND, CASCADE>(p, st, pdl, false);
    }
    case 128:
      return launch_dynamic_t<128, 4, 2, APPEND, CASCADE>(p, st, pdl, allow_merge);
    default:
      return launch_dynamic_t<256, 2, 2, APPEND, CASCADE>(p, st, pdl, allow_merge);
  }
}

// Multi-query rows with T*G <= 16 on the dynamic warp-per-item schedule (the
// combine merges the partials).
template <int D, int NW, int ST>
cudaError_t launch_rows_t(DecodeParams& p, cudaStream_t st) {
  using Cfg = pa::DynCfg<D, NW, ST>;
  CUtensorMap kmap, vmap;
  const long long rows = (long long)p.num_blocks * p.hkv * p.block_size;
  if (!cache_maps(p.k_cache, p.v_cache, D, rows, &kmap, &vmap)) return cudaErrorInvalidValue;
  auto kern = pa::decode_rows_kernel<D, NW, ST>;
  const int smem = Cfg::decode_smem_bytes(p.batch);
  static std::atomic<int> smem_done[64];
  cudaError_t e = set_smem_at_least(kern, smem, smem_done);
  if (e != cudaSuccess) return e;
  int occ = 0;
  static std::atomic<long long> occ_cache[64];
  e = occupancy(kern, Cfg::kThreads, smem, occ_cache, &occ);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  p.merge_in_kernel = 0;
  p.static_items = 2;
  if (!pow2(p.partition)) return cudaErrorInvalidValue;  // the schedule's partitions are powers of two
  p.log2_partition = ilog2(p.partition);
  // A programmatic dependent of the preceding kernel: it waits for it before
  // touching global memory.
  return launch_ex(kern, dim3(occ * sm_count()), dim3(Cfg::kThreads), smem, st, true, kmap, vmap, p);
}

cudaError_t launch_rows(DecodeParams& p, cudaStream_t st) {
  switch (p.head_dim) {
    case 64:
      return launch_rows_t<64, 4, 6>(p, st);
    case 128:
      return launch_rows_t<128, 4, 2>(p, st);
    default:
      return launch_rows_t<256, 2, 2>(p, st);
  }
}


int32_t auto_partition(int32_t batch, int32_t num_kv_heads, int32_t max_context_len, int32_t partition_tokens) {
  if (partition_tokens > 0) return partition_tokens;
  const long long work = (long long)(batch > 0 ? batch : 1) * (num_kv_heads > 0 ? num_kv_heads : 1) *
                         (max_context_len > 0 ? max_context_len : 1);
  int P = 512;
  while (P > 64 && work / P < kTargetWorkUnits) P >>= 1;
  return P;
}

// Partition size of the dynamic schedule, where one warp runs one item: a
// per-head_dim default (from a sweep on B200: long items cut the partials, the
// combine's work and the per-item overhead; short ones cut the tail when the
// last items finish), halved while there would be fewer items than resident
// warps.
int32_t dynamic_partition(int32_t batch, int32_t num_kv_heads, int32_t max_context_len, int32_t head_dim) {
  const long long work = (long long)(batch > 0 ? batch : 1) * (num_kv_heads > 0 ? num_kv_heads : 1) *
                         (max_context_len > 0 ? max_context_len : 1);
  const int warps_per_sm = head_dim <= 64 ? 8 : head_dim <= 128 ? 12 : 6;
  // head_dim 128: 512-token partitions past 16K tokens keep the combine's
  // per-row chain short; 256 below that balances the tail better.
  int P = head_dim <= 64 ? 256 : head_dim <= 128 ? (max_context_len > 16384 ? 512 : 256) : 128;
  while (P > 64 && work / P < (long long)warps_per_sm * 148) P >>= 1;
  return P;
}

long long splitk_parts(int32_t max_context_len, int32_t P) {
  return ((long long)(max_context_len > 0 ? max_context_len : 1) + P - 1) / P;
}

// Split-K workspace layout, for every schedule: a fixed-size counter region
// first (the dynamic schedule's work-item counter, its count of finished CTAs
// and one arrival count per (sequence, kv head)), then the partial outputs
// [B][Hq][parts][D] and the partial (m, l) [B][Hq][parts][2].  The counters sit
// at the same place whatever the call's shape, and no call writes partials
// there, so counters that one call leaves at zero are zero for the next call
// of any shape or schedule.
size_t workspace_size(int32_t batch, int32_t num_q_heads, int32_t head_dim, int32_t max_context_len, int32_t P,
                      int32_t q_len = 1) {
  const size_t rows = (size_t)batch * q_len * num_q_heads * (size_t)splitk_parts(max_context_len, P);
  return pa::kCounterBytes + align256(rows * head_dim * 4) + align256(rows * 2 * 4);
}

size_t dynamic_counter_bytes(int32_t batch, int32_t num_kv_heads) {
  return (2 + (size_t)batch * num_kv_heads) * sizeof(int);
}

// ---- the allocation-free call's scratch ---------------------------------------------

// Split-K scratch of pa_decode_splitk_noalloc: reserved in device memory by the
// module itself on every device that loads the library, so that call allocates
// nothing.  In host code the name is a host-side stand-in, not a device
// address; noalloc_scratch() asks the runtime for the device address.
static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_get_id = nullptr;
std::once_flag g_ctx_once;

// Unique id of the calling thread's current context, or 0 when no context is
// current (or the driver cannot tell).
unsigned long long current_context_id() {
  std::call_once(g_ctx_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 4000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    fn = nullptr;
    q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &fn, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
  });
  if (!g_ctx_current || !g_ctx_get_id) return 0;
  CUcontext ctx = nullptr;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  unsigned long long id = 0;
  return g_ctx_get_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}

// Device address of g_noalloc_scratch in the current device's context, or null
// when the runtime cannot give it.  The lookup allocates nothing; it runs on
// the first call on a device and again whenever that device's context has
// changed since (a cudaDeviceReset unloads the module, and the array is placed
// anew when the library is next used), so no stale address is ever handed to
// a kernel.  Any device ordinal is served.
void* noalloc_scratch() {
  struct Entry {
    int dev;
    unsigned long long ctx;  // 0: unknown, look the address up again
    void* addr;
  };
  static std::mutex mu;
  static std::vector<Entry> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  Entry* e = nullptr;
  for (auto& x : cache)
    if (x.dev == dev) e = &x;
  const unsigned long long ctx = current_context_id();
  if (e && ctx != 0 && e->ctx == ctx) return e->addr;
  void* a = nullptr;
  if (cudaGetSymbolAddress(&a, g_noalloc_scratch) != cudaSuccess || !a) return nullptr;
  const unsigned long long now = current_context_id();  // the lookup may have made the context current
  if (e) {
    e->ctx = now;
    e->addr = a;
  } else {
    cache.push_back(Entry{dev, now, a});
  }
  return a;
}

// Everything the decode entry points share.  split: partitioned launch plus
// the combine; append: the fused decode step (k_new / v_new appended at L-1).
struct DecodeCall {
  const void* q;
  const void* k_new;
  const void* v_new;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  Shape shape;
  float scale, softcap;
  int32_t window;
  void* out;
  pa_dtype_t dtype;
  bool split, append;
  int32_t partition_tokens, max_context_len;
  void* workspace;
  size_t workspace_bytes;
  bool noalloc;  // split-K scratch is the library's own array (workspace ignored)
  pa_kernel_t kernel;
  cudaStream_t stream;
};

pa_status_t run_decode(const DecodeCall& c) {
  t_last_schedule = PA_SCHEDULE_NONE;
  const Shape& s = c.shape;
  pa_status_t st = check_decode_args(c.q, c.k_cache, c.v_cache, c.block_tables, c.context_lens, s, c.softcap,
                                     c.out, c.dtype, c.kernel);
  if (st != PA_OK) return st;
  if (c.append && s.batch > 0) {
    if (!c.k_new || !c.v_new || !aligned(c.k_new, 16) || !aligned(c.v_new, 16)) return PA_ERR_INVALID;
  }
  int P = kNoSplitPartition;
  long long parts = 1;
  bool dynamic = false;
  if (c.split) {
    if (c.partition_tokens < 0 || (c.partition_tokens > 0 && c.partition_tokens % 64 != 0)) return PA_ERR_INVALID;
    if (c.max_context_len <= 0) return PA_ERR_INVALID;
    const bool mma = (c.kernel == PA_KERNEL_MMA) || (c.kernel == PA_KERNEL_AUTO && c.dtype == PA_BF16);
    dynamic = c.partition_tokens == 0 && mma && s.batch <= pa::kMaxDynamicBatch &&
              (long long)s.batch * s.hkv <= pa::kMaxDynamicUnits;
    P = dynamic ? dynamic_partition(s.batch, s.hkv, c.max_context_len, s.d)
                : auto_partition(s.batch, s.hkv, c.max_context_len, c.partition_tokens);
    parts = splitk_parts(c.max_context_len, P);
    if (parts > kMaxPartsPerSeq) return PA_ERR_UNSUPPORTED;
    const size_t need = workspace_size(s.batch, s.hq, s.d, c.max_context_len, P);
    if (c.noalloc) {
      if (need > PA_NOALLOC_SCRATCH_BYTES) return PA_ERR_WORKSPACE;
    } else if (s.batch > 0 && (!c.workspace || !aligned(c.workspace, 16) || c.workspace_bytes < need)) {
      return PA_ERR_WORKSPACE;
    }
  }
  if (s.batch == 0) return PA_OK;
  void* workspace = c.workspace;
  if (c.split && c.noalloc) {  // every host check has passed: only now touch the device
    workspace = noalloc_scratch();
    if (!workspace) return PA_ERR_CUDA;
  }

  DecodeParams p = make_params(c.q, c.k_cache, c.v_cache, c.block_tables, c.context_lens, s, c.scale, c.softcap,
                               c.window, c.out);
  p.k_new = c.k_new;
  p.v_new = c.v_new;
  cudaError_t e;
  if (c.split) {
    p.partition = P;
    p.max_parts = (int)parts;
    p.max_context = c.max_context_len < p.max_context ? c.max_context_len : p.max_context;
    const size_t rows = (size_t)s.batch * s.hq * parts;
    char* ws = static_cast<char*>(workspace);
    p.ws_o = reinterpret_cast<float*>(ws + pa::kCounterBytes);
    p.ws_ml = reinterpret_cast<float*>(ws + pa::kCounterBytes + align256(rows * s.d * 4));
    if (dynamic) {  // resets its counters itself; merges in-kernel or through the combine
      if (c.noalloc) {
        // The shared array keeps what the last call left in it.  A call that
        // completed left the counters (the start of the array) at zero, one
        // that timed out may not have: clear the ones this call uses.
        const size_t len = std::min(dynamic_counter_bytes(s.batch, s.hkv), pa::kCounterBytes);
        if (cudaMemsetAsync(ws, 0, len, c.stream) != cudaSuccess) return PA_ERR_CUDA;
      }
      p.queue = reinterpret_cast<int*>(ws);
      p.unit_count = p.queue + 2;
      e = c.append ? launch_dynamic<true>(p, c.stream) : launch_dynamic<false>(p, c.stream);
      if (e != cudaSuccess) return PA_ERR_CUDA;
      t_last_launches = 1;
      t_last_schedule = p.merge_in_kernel ? PA_SCHEDULE_DYNAMIC_MERGED : PA_SCHEDULE_DYNAMIC;
      if (!p.merge_in_kernel && parts > 1) {
        e = launch_combine<__nv_bfloat16>(p, c.stream);
        if (e != cudaSuccess) return PA_ERR_CUDA;
        t_last_launches = 2;
      }
      return PA_OK;
    }
    dim3 grid((unsigned)parts, s.hkv, s.batch);
    e = c.append ? launch_decode<true, true>(p, c.dtype, c.kernel, grid, c.stream)
                 : launch_decode<true, false>(p, c.dtype, c.kernel, grid, c.stream);
    if (e != cudaSuccess) return PA_ERR_CUDA;
    t_last_schedule = PA_SCHEDULE_GRID;
    if (parts > 1) {
      e = c.dtype == PA_BF16 ? launch_combine<__nv_bfloat16>(p, c.stream) : launch_combine<float>(p, c.stream);
      if (e != cudaSuccess) return PA_ERR_CUDA;
      t_last_launches = 2;
    } else {
      t_last_launches = 1;
    }
  } else {
    dim3 grid(1, s.hkv, s.batch);
    e = c.append ? launch_decode<false, true>(p, c.dtype, c.kernel, grid, c.stream)
                 : launch_decode<false, false>(p, c.dtype, c.kernel, grid, c.stream);
    if (e != cudaSuccess) return PA_ERR_CUDA;
    t_last_launches = 1;
    t_last_schedule = PA_SCHEDULE_SINGLE;
  }
  return PA_OK;
}

}  // namespace

extern "C" {

pa_status_t pa_write_kv(const void* k, const void* v, const int64_t* slot_mapping, int32_t num_tokens,
                        void* k_cache, void* v_cache, int32_t num_blocks, int32_t block_size,
                        int32_t num_kv_heads, int32_t head_dim, pa_dtype_t dtype, pa_stream_t stream) {
  t_last_launches = 0;
  if (num_tokens < 0 || num_blocks <= 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return PA_ERR_INVALID;
  if (dtype != PA_F32 && dtype != PA_BF16) return PA_ERR_INVALID;
  const int elt = dtype == PA_F32 ? 4 : 2;
  if ((head_dim * elt) % 16 != 0) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !slot_mapping || !k_cache || !v_cache) return PA_ERR_INVALID;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(slot_mapping, 8))
    return PA_ERR_INVALID;
  const int chunks = head_dim * elt / 16;
  const long long total = (long long)num_tokens * num_kv_heads * chunks;
  const long long blocks = (total + 255) / 256;
  if (blocks > INT_MAX) return PA_ERR_UNSUPPORTED;
  pa::write_kv_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping, num_tokens,
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), (int64_t)num_blocks * block_size, block_size,
      num_kv_heads, chunks);
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  t_last_launches = 1;
  return PA_OK;
}

pa_status_t pa_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                      const int32_t* context_lens, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                      int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq, int32_t num_blocks,
                      float scale, float softcap, int32_t window, void* out, pa_dtype_t dtype,
                      pa_kernel_t kernel, pa_stream_t stream) {
  t_last_launches = 0;
  DecodeCall c{};
  c.q = q;
  c.k_cache = k_cache;
  c.v_cache = v_cache;
  c.block_tables = block_tables;
  c.context_lens = context_lens;
  c.shape = Shape{batch, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks};
  c.scale = scale;
  c.softcap = softcap;
  c.window = window;
  c.out = out;
  c.dtype = dtype;
  c.kernel = kernel;
  c.stream = stream;
  return run_decode(c);
}

int32_t pa_decode_splitk_partition(int32_t batch, int32_t num_kv_heads, int32_t max_context_len,
                                   int32_t partition_tokens) {
  return auto_partition(batch, num_kv_heads, max_context_len, partition_tokens);
}

size_t pa_decode_splitk_workspace_size(int32_t batch, int32_t num_q_heads, int32_t head_dim,
                                       int32_t max_context_len, int32_t partition_tokens,
                                       int32_t num_kv_heads) {
  if (batch <= 0 || num_q_heads <= 0 || head_dim <= 0) return 0;
  const int P = auto_partition(batch, num_kv_heads, max_context_len, partition_tokens);
  if (P <= 0) return 0;
  size_t n = workspace_size(batch, num_q_heads, head_dim, max_context_len, P);
  if (partition_tokens == 0) {  // may select the dynamic schedule: its partition and its counters
    const int Pd = dynamic_partition(batch, num_kv_heads, max_context_len, head_dim);
    n = std::max(n, workspace_size(batch, num_q_heads, head_dim, max_context_len, Pd));
  }
  return n;
}

pa_status_t pa_decode_splitk(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                             const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
                             int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                             int32_t max_blocks_per_seq, int32_t num_blocks, float scale, float softcap,
                             int32_t window, void* out, pa_dtype_t dtype, int32_t partition_tokens,
                             int32_t max_context_len, void* workspace, size_t workspace_bytes,
                             pa_kernel_t kernel, pa_stream_t stream) {
  t_last_launches = 0;
  DecodeCall c{};
  c.q = q;
  c.k_cache = k_cache;
  c.v_cache = v_cache;
  c.block_tables = block_tables;
  c.context_lens = context_lens;
  c.shape = Shape{batch, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks};
  c.scale = scale;
  c.softcap = softcap;
  c.window = window;
  c.out = out;
  c.dtype = dtype;
  c.split = true;
  c.partition_tokens = partition_tokens;
  c.max_context_len = max_context_len;
  c.workspace = workspace;
  c.workspace_bytes = workspace_bytes;
  c.kernel = kernel;
  c.stream = stream;
  return run_decode(c);
}

pa_status_t pa_decode_step(const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                           const int32_t* block_tables, const int32_t* context_lens, int32_t batch,
                           int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                           int32_t max_blocks_per_seq, int32_t num_blocks, float scale, float softcap,
                           int32_t window, void* out, pa_dtype_t dtype, int32_t partition_tokens,
                           int32_t max_context_len, void* workspace, size_t workspace_bytes, pa_kernel_t kernel,
                           pa_stream_t stream) {
  t_last_launches = 0;
  DecodeCall c{};
  c.q = q;
  c.k_new = k_new;
  c.v_new = v_new;
  c.k_cache = k_cache;
  c.v_cache = v_cache;
  c.block_tables = block_tables;
  c.context_lens = context_lens;
  c.shape = Shape{batch, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks};
  c.scale = scale;
  c.softcap = softcap;
  c.window = window;
  c.out = out;
  c.dtype = dtype;
  c.append = true;
  c.split = partition_tokens >= 0;
  c.partition_tokens = partition_tokens;
  c.max_context_len = max_context_len;
  c.workspace = workspace;
  c.workspace_bytes = workspace_bytes;
  c.kernel = kernel;
  c.stream = stream;
  return run_decode(c);
}

// Whether multi-query rows run on the dynamic warp-per-item schedule: at most
// 32 query rows (T * G) per kv head at head_dim 64, 16 at 128 and 256, and a batch the schedule
// takes.
bool multi_rows_path(int32_t batch, int32_t q_len, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim) {
  const int rows = head_dim <= 64 ? 16 * pa::rows_tiles<64>() : 16 * pa::rows_tiles<128>();
  return (long long)q_len * (num_q_heads / num_kv_heads) <= rows &&
         batch <= pa::kMaxDynamicBatch && (long long)batch * num_kv_heads <= pa::kMaxDynamicUnits;
}

// Multi-query partition: the requested one; else the dynamic schedule's choice
// on that path, the grid schedule's otherwise.
int32_t multi_partition(int32_t batch, int32_t q_len, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                        int32_t max_context_len, int32_t partition_tokens) {
  if (partition_tokens > 0) return partition_tokens;
  if (!multi_rows_path(batch, q_len, num_q_heads, num_kv_heads, head_dim))
    return auto_partition(batch, num_kv_heads, max_context_len, 0);
  // The rows path writes T*G partial rows per item, twice the decode's at
  // T*G = 16: at head_dim 128 512-token partitions keep the partials and the
  // combine small (a sweep on B200: Llama-3 T=4, 0.76 -> 0.89 of HBM peak; at
  // head_dim 256, Gemma-2 T=8: 128 / 256 / 512 tokens gave 155 / 139 / 161
  // us); halved, as for decode, while there are fewer items than resident warps.
  const long long work = (long long)(batch > 0 ? batch : 1) * (num_kv_heads > 0 ? num_kv_heads : 1) *
                         (max_context_len > 0 ? max_context_len : 1);
  int P = head_dim <= 64 ? 256 : head_dim <= 128 ? 512 : 256;
  const int warps_per_sm = head_dim <= 64 ? 8 : head_dim <= 128 ? 12 : 6;
  while (P > 64 && work / P < (long long)warps_per_sm * 148) P >>= 1;
  return P;
}

pa_status_t pa_decode_multi(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                            const int32_t* context_lens, int32_t batch, int32_t q_len, int32_t num_q_heads,
                            int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq,
                            int32_t num_blocks, float scale, float softcap, int32_t window, void* out,
                            pa_dtype_t dtype, int32_t partition_tokens, int32_t max_context_len, void* workspace,
                            size_t workspace_bytes, pa_stream_t stream) {
  t_last_launches = 0;
  const Shape s{batch, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks};
  pa_status_t st = check_decode_args(q, k_cache, v_cache, block_tables, context_lens, s, softcap, out, dtype,
                                     PA_KERNEL_MMA);
  if (st != PA_OK) return st;
  if (q_len <= 0) return PA_ERR_INVALID;
  if ((long long)q_len * (num_q_heads / num_kv_heads) > pa::kMaxMultiColumns) return PA_ERR_UNSUPPORTED;
  const bool split = partition_tokens >= 0;
  const bool rows_path = split && multi_rows_path(batch, q_len, num_q_heads, num_kv_heads, head_dim);
  int P = kNoSplitPartition;
  long long parts = 1;
  if (split) {
    if (partition_tokens > 0 && partition_tokens % 64 != 0) return PA_ERR_INVALID;
    if (max_context_len <= 0) return PA_ERR_INVALID;
    P = multi_partition(batch, q_len, num_q_heads, num_kv_heads, head_dim, max_context_len, partition_tokens);
    parts = splitk_parts(max_context_len, P);
    if (parts > kMaxPartsPerSeq) return PA_ERR_UNSUPPORTED;
    const size_t need = workspace_size(batch, num_q_heads, head_dim, max_context_len, P, q_len);
    if (batch > 0 && (!workspace || !aligned(workspace, 16) || workspace_bytes < need)) return PA_ERR_WORKSPACE;
  }
  if (batch == 0) return PA_OK;
  DecodeParams p = make_params(q, k_cache, v_cache, block_tables, context_lens, s, scale, softcap, window, out);
  p.q_len = q_len;
  cudaError_t e;
  if (split) {
    p.partition = P;
    p.max_parts = (int)parts;
    p.max_context = max_context_len < p.max_context ? max_context_len : p.max_context;
    const size_t rows = (size_t)batch * q_len * num_q_heads * parts;
    char* ws = static_cast<char*>(workspace);
    p.ws_o = reinterpret_cast<float*>(ws + pa::kCounterBytes);
    p.ws_ml = reinterpret_cast<float*>(ws + pa::kCounterBytes + align256(rows * head_dim * 4));
    if (rows_path) {  // one warp per (sequence, kv head, partition) item, dynamic schedule
      p.queue = reinterpret_cast<int*>(ws);
      p.unit_count = p.queue + 2;
      e = launch_rows(p, stream);
    } else {
      e = launch_multi<true>(p, dim3((unsigned)parts, num_kv_heads, batch), stream);
    }
    if (e != cudaSuccess) return PA_ERR_CUDA;
    t_last_launches = 1;
    if (parts > 1) {
      e = launch_combine<__nv_bfloat16>(p, stream);
      if (e != cudaSuccess) return PA_ERR_CUDA;
      t_last_launches = 2;
    }
  } else {
    e = launch_multi<false>(p, dim3(1, num_kv_heads, batch), stream);
    if (e != cudaSuccess) return PA_ERR_CUDA;
    t_last_launches = 1;
  }
  return PA_OK;
}

pa_status_t pa_prefill(const void* q, const void* k_new, const void* v_new, const int64_t* slot_mapping,
                       const int32_t* cu_q_lens, int32_t total_q, int32_t max_q_len, void* k_cache, void* v_cache,
                       const int32_t* block_tables, const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
                       int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq,
                       int32_t num_blocks, float scale, float softcap, int32_t window, void* out, pa_dtype_t dtype,
                       pa_stream_t stream) {
  t_last_launches = 0;
  const Shape s{batch, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks};
  pa_status_t st = check_decode_args(q, k_cache, v_cache, block_tables, context_lens, s, softcap, out, dtype,
                                     PA_KERNEL_MMA);
  if (st != PA_OK) return st;
  if (total_q < 0 || max_q_len < 0) return PA_ERR_INVALID;
  if (batch == 0 || total_q == 0 || max_q_len == 0) return PA_OK;
  if (!cu_q_lens || !aligned(cu_q_lens, 4)) return PA_ERR_INVALID;
  const bool append = k_new != nullptr || v_new != nullptr;
  if (append) {
    if (!k_new || !v_new || !slot_mapping) return PA_ERR_INVALID;
    st = pa_write_kv(k_new, v_new, slot_mapping, total_q, k_cache, v_cache, num_blocks, block_size, num_kv_heads,
                     head_dim, dtype, stream);
    if (st != PA_OK) return st;
  }
  const int G = num_q_heads / num_kv_heads;
  const int q_tile = 128 / G;  // one CTA: 128 query rows = q_tile tokens x G heads
  const long long tiles = ((long long)max_q_len + q_tile - 1) / q_tile;
  if (tiles > kMaxGridYZ) return PA_ERR_UNSUPPORTED;
  DecodeParams p = make_params(q, k_cache, v_cache, block_tables, context_lens, s, scale, softcap, window, out);
  p.cu_q = cu_q_lens;
  p.q_tile = q_tile;
  p.max_q_len = max_q_len;
  p.total_q = total_q;
  cudaError_t e = launch_prefill(p, dim3(num_kv_heads, batch, (unsigned)tiles), stream);
  if (e != cudaSuccess) return PA_ERR_CUDA;
  t_last_launches = append ? 2 : 1;
  return PA_OK;
}

// Whether the cascade's own-range pass runs the dynamic schedule (the library
// chooses the partition and the shape fits it).
bool cascade_dynamic(int32_t batch, int32_t num_kv_heads, int32_t partition_tokens) {
  return partition_tokens == 0 && batch <= pa::kMaxDynamicBatch &&
         (long long)batch * num_kv_heads <= pa::kMaxDynamicUnits;
}

// Cascade partition: the requested one (it must divide prefix_len), or the
// library's choice (the dynamic schedule's, else the grid's) halved until it
// divides prefix_len (a multiple of 64).
int32_t cascade_partition(int32_t batch, int32_t num_kv_heads, int32_t max_context_len, int32_t prefix_len,
                          int32_t partition_tokens, int32_t head_dim) {
  if (partition_tokens > 0) return prefix_len % partition_tokens == 0 ? partition_tokens : -1;
  int32_t P = cascade_dynamic(batch, num_kv_heads, partition_tokens)
                  ? dynamic_partition(batch, num_kv_heads, max_context_len, head_dim)
                  : auto_partition(batch, num_kv_heads, max_context_len, 0);
  while (P > 64 && prefix_len % P != 0) P >>= 1;
  return P;
}

pa_status_t pa_decode_cascade(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                              const int32_t* context_lens, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                              int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq, int32_t num_blocks,
                              float scale, float softcap, int32_t window, void* out, pa_dtype_t dtype,
                              int32_t n_sharers, int32_t prefix_len, int32_t partition_tokens,
                              int32_t max_context_len, void* workspace, size_t workspace_bytes, pa_stream_t stream) {
  t_last_launches = 0;
  const Shape s{batch, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks};
  pa_status_t st = check_decode_args(q, k_cache, v_cache, block_tables, context_lens, s, softcap, out, dtype,
                                     PA_KERNEL_MMA);
  if (st != PA_OK) return st;
  if (n_sharers < 0 || n_sharers > batch || prefix_len < 0 || max_context_len <= 0) return PA_ERR_INVALID;
  if (partition_tokens < 0 || (partition_tokens > 0 && partition_tokens % 64 != 0)) return PA_ERR_INVALID;
  if (prefix_len % 64 != 0 || prefix_len % block_size != 0 || prefix_len > max_context_len ||
      (long long)prefix_len > (long long)max_blocks_per_seq * block_size)
    return PA_ERR_INVALID;
  if (n_sharers == 0 || prefix_len == 0)  // nothing shared: the plain split-K call
    return pa_decode_splitk(q, k_cache, v_cache, block_tables, context_lens, batch, num_q_heads, num_kv_heads,
                            head_dim, block_size, max_blocks_per_seq, num_blocks, scale, softcap, window, out, dtype,
                            partition_tokens, max_context_len, workspace, workspace_bytes, PA_KERNEL_MMA, stream);
  const int32_t P =
      cascade_partition(batch, num_kv_heads, max_context_len, prefix_len, partition_tokens, head_dim);
  if (P <= 0) return PA_ERR_INVALID;
  const bool dynamic = cascade_dynamic(batch, num_kv_heads, partition_tokens);
  const long long parts = splitk_parts(max_context_len, P);
  if (parts > kMaxPartsPerSeq) return PA_ERR_UNSUPPORTED;
  const size_t need = workspace_size(batch, num_q_heads, head_dim, max_context_len, P);
  if (!workspace || !aligned(workspace, 16) || workspace_bytes < need) return PA_ERR_WORKSPACE;

  DecodeParams p = make_params(q, k_cache, v_cache, block_tables, context_lens, s, scale, softcap, window, out);
  p.partition = P;
  p.max_parts = (int)parts;
  p.max_context = max_context_len < p.max_context ? max_context_len : p.max_context;
  const size_t rows = (size_t)batch * num_q_heads * parts;
  char* ws = static_cast<char*>(workspace);
  p.ws_o = reinterpret_cast<float*>(ws + pa::kCounterBytes);
  p.ws_ml = reinterpret_cast<float*>(ws + pa::kCounterBytes + align256(rows * head_dim * 4));
  p.n_sharers = n_sharers;
  p.prefix_len = prefix_len;
  // 1. The shared prefix, once per (partition, kv head) for up to 64/G sharers per CTA.
  DecodeParams pp = p;
  pp.cascade_prefix = 1;
  pp.q_tile = pa::kMaxMultiColumns / (num_q_heads / num_kv_heads);
  const unsigned groups = (unsigned)((n_sharers + pp.q_tile - 1) / pp.q_tile);
  cudaError_t e = launch_multi<true>(pp, dim3((unsigned)(prefix_len / P), num_kv_heads, groups), stream);
  if (e != cudaSuccess) return PA_ERR_CUDA;
  // 2. Every sequence's own range (sharers from prefix_len on), split-K: the
  // dynamic schedule as a programmatic dependent of the prefix pass (the two
  // overlap; it waits for the prefix pass only before it exits), merged by
  // the combine; or the grid schedule after it.
  if (dynamic) {
    p.queue = reinterpret_cast<int*>(ws);
    p.unit_count = p.queue + 2;
    e = launch_dynamic<false, true>(p, stream);
  } else {
    e = launch_decode<true, false>(p, dtype, PA_KERNEL_MMA, dim3((unsigned)parts, num_kv_heads, batch), stream);
  }
  if (e != cudaSuccess) return PA_ERR_CUDA;
  // 3. Merge the prefix and suffix partials.
  e = launch_combine<__nv_bfloat16>(p, stream);
  if (e != cudaSuccess) return PA_ERR_CUDA;
  t_last_launches = 3;
  return PA_OK;
}

size_t pa_decode_cascade_workspace_size(int32_t batch, int32_t num_q_heads, int32_t head_dim,
                                        int32_t max_context_len, int32_t prefix_len, int32_t partition_tokens,
                                        int32_t num_kv_heads) {
  if (batch <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len <= 0 || prefix_len < 0) return 0;
  if (prefix_len == 0)
    return pa_decode_splitk_workspace_size(batch, num_q_heads, head_dim, max_context_len, partition_tokens,
                                           num_kv_heads);
  const int32_t P =
      cascade_partition(batch, num_kv_heads, max_context_len, prefix_len, partition_tokens, head_dim);
  if (P <= 0) return 0;
  return std::max(workspace_size(batch, num_q_heads, head_dim, max_context_len, P),
                  pa_decode_splitk_workspace_size(batch, num_q_heads, head_dim, max_context_len, partition_tokens,
                                                  num_kv_heads));
}

size_t pa_decode_multi_workspace_size(int32_t batch, int32_t q_len, int32_t num_q_heads, int32_t head_dim,
                                      int32_t max_context_len, int32_t partition_tokens, int32_t num_kv_heads) {
  if (batch <= 0 || q_len <= 0 || num_q_heads <= 0 || head_dim <= 0 || partition_tokens < 0) return 0;
  if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return 0;
  const int P =
      multi_partition(batch, q_len, num_q_heads, num_kv_heads, head_dim, max_context_len, partition_tokens);
  if (P <= 0) return 0;
  return workspace_size(batch, num_q_heads, head_dim, max_context_len, P, q_len);
}

pa_status_t pa_decode_splitk_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* block_tables, const int32_t* context_lens, int32_t batch,
                                     int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                     int32_t block_size, int32_t max_blocks_per_seq, int32_t num_blocks,
                                     float scale, float softcap, int32_t window, void* out, pa_dtype_t dtype,
                                     int32_t partition_tokens, int32_t max_context_len, pa_kernel_t kernel,
                                     pa_stream_t stream) {
  t_last_launches = 0;
  // The documented limit: what pa_decode_splitk would ask of a caller's workspace.
  if (batch > 0 && num_q_heads > 0 && head_dim > 0 && max_context_len > 0 && partition_tokens >= 0) {
    const size_t need = pa_decode_splitk_workspace_size(batch, num_q_heads, head_dim, max_context_len,
                                                        partition_tokens, num_kv_heads);
    if (need > PA_NOALLOC_SCRATCH_BYTES) return PA_ERR_WORKSPACE;
  }
  DecodeCall c{};
  c.q = q;
  c.k_cache = k_cache;
  c.v_cache = v_cache;
  c.block_tables = block_tables;
  c.context_lens = context_lens;
  c.shape = Shape{batch, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks};
  c.scale = scale;
  c.softcap = softcap;
  c.window = window;
  c.out = out;
  c.dtype = dtype;
  c.split = true;
  c.partition_tokens = partition_tokens;
  c.max_context_len = max_context_len;
  c.noalloc = true;  // the scratch is looked up, and its counters cleared, only once every check has passed
  c.kernel = kernel;
  c.stream = stream;
  return run_decode(c);
}

pa_status_t pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* pairs, int32_t n, int32_t num_blocks,
                           int32_t block_size, int32_t num_kv_heads, int32_t head_dim, pa_dtype_t dtype,
                           pa_stream_t stream) {
  t_last_launches = 0;
  if (n < 0 || num_blocks <= 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0) return PA_ERR_INVALID;
  if (dtype != PA_F32 && dtype != PA_BF16) return PA_ERR_INVALID;
  if (n == 0) return PA_OK;
  if (!k_cache || !v_cache || !pairs || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(pairs, 4))
    return PA_ERR_INVALID;
  const int64_t bytes = (int64_t)num_kv_heads * block_size * head_dim * (dtype == PA_F32 ? 4 : 2);
  if (bytes % 16 != 0) return PA_ERR_UNSUPPORTED;
  const int64_t chunks = bytes / 16;
  const unsigned ys = (unsigned)std::min<int64_t>((chunks + 255) / 256, 64);
  pa::copy_blocks_kernel<<<dim3((unsigned)n, ys), 256, 0, stream>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), pairs, num_blocks, chunks);
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  t_last_launches = 1;
  return PA_OK;
}

pa_status_t pa_check_bounded_wait(uint64_t limit_ns, pa_stream_t stream) {
  t_last_launches = 0;
  if (limit_ns == 0 || limit_ns > pa::kWaitLimitNs) return PA_ERR_INVALID;
  pa::bounded_wait_check_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  t_last_launches = 1;
  return PA_OK;
}

pa_status_t pa_device_errors(uint32_t* bits, int32_t clear) {
  if (!bits) return PA_ERR_INVALID;
  unsigned int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return PA_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&v, pa::g_device_errors, sizeof v) != cudaSuccess) return PA_ERR_CUDA;
  *bits = v;
  if (clear) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(pa::g_device_errors, &zero, sizeof zero) != cudaSuccess) return PA_ERR_CUDA;
  }
  return PA_OK;
}

const char* pa_error_string(pa_status_t status) {
  switch (status) {
    case PA_OK:
      return "ok";
    case PA_ERR_INVALID:
      return "invalid argument (null or misaligned pointer, or a bad size)";
    case PA_ERR_UNSUPPORTED:
      return "unsupported shape or dtype (head_dim, block_size, group size, or pool too large)";
    case PA_ERR_WORKSPACE:
      return "split-K workspace missing, misaligned or too small";
    case PA_ERR_CUDA:
      return "CUDA runtime error or failed launch";
  }
  return "unknown status";
}

int32_t pa_last_launch_count(void) { return t_last_launches; }

int32_t pa_last_decode_schedule(void) { return t_last_schedule; }

}  // extern "C"
