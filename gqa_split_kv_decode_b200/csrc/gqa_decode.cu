// libgqadecode.so: the C ABI declared in include/gqa_decode.h.
//
// Host responsibilities only: argument checks, tensor-map encoding, the
// workspace, and kernel launches on the caller's stream.  Every step of the
// computation runs in the kernels of decode_tc.cuh (bf16), decode_simt.cuh
// (fp32) and split_merge.cuh (merge).
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>

#include "gqa_decode.h"
#include "gqa_prefill.h"
#include "decode_persist.cuh"
#include "decode_simt.cuh"
#include "decode_tc.cuh"
#include "prefill_tc.cuh"
#include "split_merge.cuh"

namespace {

using namespace gqa;

constexpr int kMaxSlots = 1024;
constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultTimeoutNs = 1000000000ull;

std::atomic<unsigned long long> g_timeout_ns{kDefaultTimeoutNs};

// ------------------------------------------------------------------ helpers

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

// Heads handled by one CTA for each path, and the number of head blocks.
inline int tc_heads_per_cta(int G) { return G <= 8 ? 8 : 16; }
inline int simt_heads_per_cta(int G) {
  int hb = 1;
  while (hb < G && hb < 16) hb <<= 1;
  return hb;
}
inline int heads_per_cta(int dtype, int G) {
  return dtype == GQA_BF16 ? tc_heads_per_cta(G) : simt_heads_per_cta(G);
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D view (d, kv head, row) of a bf16 cache of `rows` rows; box = 64 d x 1
// head x 16 rows, 128-byte swizzle.  Rows below 0 (a shifted first tile) and
// at or past `rows` read zero fill.  rows < 0 (not given): the extent is
// 2^31, a clip bound only (the kernels address no row past the batch's last).
bool encode_cache_map(CUtensorMap* map, const void* base, int h_kv, int D, long long rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t extent = rows > 0 ? static_cast<cuuint64_t>(rows)
                                     : static_cast<cuuint64_t>(rows == 0 ? 1u : 1u << 31);
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(h_kv), extent};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                                 static_cast<cuuint64_t>(h_kv) * D * 2};
  const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(kTileKeys)};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Decode cache maps of recent calls.  A map is a pure function of (base
// address, h_kv, D, rows), so a cached map is exactly what encoding again
// would give; the cache only saves the driver call on the launch path.  Per
// host thread, a few entries replaced round-robin.
struct CacheMapEntry {
  const void* base;
  int h_kv, D;
  long long rows;
  CUtensorMap map;
};

bool cached_cache_map(CUtensorMap* map, const void* base, int h_kv, int D, long long rows) {
  constexpr int kEntries = 16;
  thread_local CacheMapEntry entries[kEntries] = {};
  thread_local int next = 0;
  for (int i = 0; i < kEntries; ++i) {
    const CacheMapEntry& e = entries[i];
    if (e.base == base && e.h_kv == h_kv && e.D == D && e.rows == rows) {
      *map = e.map;
      return true;
    }
  }
  if (!encode_cache_map(map, base, h_kv, D, rows)) return false;
  CacheMapEntry& e = entries[next];
  next = (next + 1) % kEntries;
  e.base = base;
  e.h_kv = h_kv;
  e.D = D;
  e.rows = rows;
  e.map = *map;
  return true;
}

// One-time (per device) opt-in to large dynamic shared memory for a kernel.
template <typename K>
int ensure_smem_attr(K kernel, int bytes, std::atomic<uint64_t>& done) {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return GQA_ERR_CUDA;
  const uint64_t bit = 1ull << dev;
  if (done.load(std::memory_order_acquire) & bit) return GQA_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return GQA_ERR_CUDA;
  done.fetch_or(bit, std::memory_order_acq_rel);
  return GQA_OK;
}

int after_launch() {
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

// Launches with programmatic stream serialization: the kernel may begin
// launching while the previous kernel of the stream drains; every kernel
// here waits for its prerequisites (griddepcontrol.wait) before it touches
// global memory, so results do not depend on what precedes it.
template <typename... Params, typename... Args>
int launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
               Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_CUDA;
  }
  return after_launch();
}

// ---------------------------------------------------------- kernel dispatch

// Tensor-core kernel shape: NW warps per CTA, NS stages per warp (build-time
// constants; -DGQA_TC_WARPS / -DGQA_TC_STAGES override them).
#ifndef GQA_TC_WARPS
#define GQA_TC_WARPS 4
#endif
#ifndef GQA_TC_STAGES
#define GQA_TC_STAGES 3
#endif
constexpr int kTcWarps = GQA_TC_WARPS;
constexpr int kTcStages = GQA_TC_STAGES;

// Tiles per warp that the bf16 kernels' first-wave CTAs prefetch into L2
// before their dependency wait (-DGQA_HINT_TILES overrides it; 0: none).
// Measured on B200 over 2000 back-to-back calls: none, 6, 8 and 12 tiles ran
// the 70B-shaped call (B 8, 64/8 heads, 8192 keys) in 46.7, 45.6, 46.0 and
// 46.7 us and the 7B-shaped one (B 1, 32/32 heads, 4096 keys) in 16.6, 14.8,
// 15.3 and 15.3 us; on another box 4, 5, 6 and 7 tiles ran them in 45.2,
// 45.1, 45.1, 45.4 and 14.4, 14.25, 14.5, 14.8 us.  Deeper prefetches evict
// each other and delay the running call's own loads.
#ifndef GQA_HINT_TILES
#define GQA_HINT_TILES 5
#endif
constexpr int kHintTiles = GQA_HINT_TILES;

int sm_count() {
  static std::atomic<int> cached[kMaxDevices];
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return -1;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

// CTAs of `kern` resident on the current device at once (per-device cache).
template <typename K>
int resident_ctas(K kern, int threads, int smem, std::atomic<int>* per_sm) {
  const int dev = current_device();
  const int sms = sm_count();
  if (dev < 0 || dev >= kMaxDevices || sms <= 0) return -1;
  int occ = per_sm[dev].load(std::memory_order_relaxed);
  if (occ <= 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, smem) != cudaSuccess ||
        occ <= 0) {
      cudaGetLastError();
      return -1;
    }
    per_sm[dev].store(occ, std::memory_order_relaxed);
  }
  return sms * occ;
}

template <int D, int NT, int MODE, int NS = kTcStages>
int launch_tc(DecodeArgs a, dim3 grid, cudaStream_t st) {
  constexpr int NW = kTcWarps;
  constexpr int smem = tc_dynamic_smem<D, NW, NS>();
  static std::atomic<uint64_t> attr_done{0};
  static std::atomic<int> per_sm[kMaxDevices];
  auto kern = decode_tc_bf16<D, NT, NW, NS, MODE>;
  if (int rc = ensure_smem_attr(kern, smem, attr_done)) return rc;
  if (a.hint_tiles > 0) {  // the grid's first wave prefetches
    a.hint_ctas = resident_ctas(kern, NW * 32, smem, per_sm);
    if (a.hint_ctas < 0) return GQA_ERR_CUDA;
  }
  CUtensorMap kmap, vmap;
  if (!cached_cache_map(&kmap, a.k, a.h_kv, D, a.kv_rows) ||
      !cached_cache_map(&vmap, a.v, a.h_kv, D, a.kv_rows))
    return GQA_ERR_CUDA;
  return launch_pdl(kern, grid, dim3(NW * 32), smem, st, kmap, vmap, a);
}


// Launch plans of the fused bf16 path, chosen from the grid size alone (the
// sequence lengths live on the device).  R = CTAs of the per-split kernel
// (4 warps x 3 stages) that fit on the GPU at once, by shared memory.
//   units <= R      one wave: per-split grid, in-kernel ticket merge (1 launch)
//   units <= 4 R    a few waves: persistent CTAs + row merge (2 launches), so
//                   no later wave starts cold
//   otherwise       many waves: per-split grid with 2 stages (more CTAs per
//                   SM), whose tails overlap other CTAs' streaming (1 launch)
enum FusedPlan { kPlanOneWave = 0, kPlanPersistent = 1, kPlanManyWaves = 2 };

int fused_plan(long long units, int D) {
  const int sms = sm_count();
  if (sms <= 0) return -1;
  const int smem = D == 128 ? tc_dynamic_smem<128, kTcWarps, kTcStages>()
                            : tc_dynamic_smem<64, kTcWarps, kTcStages>();
  const long long per_sm = (228 * 1024) / (smem + 1024);  // 1 KiB reserved per CTA
  const long long R = (long long)sms * (per_sm > 0 ? per_sm : 1);
  if (units <= R) return kPlanOneWave;
  if (units <= 4 * R) return kPlanPersistent;
  return kPlanManyWaves;
}

// The row merge of the fused paths that store split triplets first: one warp
// per row over the row's non-empty splits (programmatic dependent launch).
int launch_merge_rows(const DecodeArgs& a, int D, cudaStream_t st) {
  const long long rows = (long long)a.B * a.h_q;
  const dim3 grid((unsigned)((rows + 3) / 4));
  if (D == 128) return launch_pdl(merge_rows_kernel<4>, grid, dim3(128), 0, st, a, D);
  return launch_pdl(merge_rows_kernel<2>, grid, dim3(128), 0, st, a, D);
}

// One-wave plan: whether the splits' triplets are merged by a second kernel
// rather than by the CTA that finishes a group last.  That CTA merges the
// group's G rows alone, at the very end of the call: with one row (G = 1) it
// is quicker than a second launch, with G >= 8 rows the second kernel, which
// spreads the rows over many CTAs, is (measured on B200: 16.3 against
// 16.8 us at G = 1, 49.6 against 47.4 us at G = 8).
inline bool one_wave_merge_kernel(int G) { return G >= 8; }

// Fused bf16: persistent CTAs over the non-empty splits (as many as fit on
// the GPU at once), then the row merge.  Both launches overlap their
// predecessor's tail (programmatic dependent launch).
template <int D, int NT, bool PARTIAL>
int launch_persist(const DecodeArgs& a, cudaStream_t st) {
  constexpr int NW = 4, NS = kTcStages;
  constexpr int smem = persist_dynamic_smem<D, NT, NW, NS>();
  static std::atomic<uint64_t> attr_done{0};
  static std::atomic<int> per_sm[kMaxDevices];
  auto kern = decode_tc_bf16_persist<D, NT, NW, NS, PARTIAL>;
  if (int rc = ensure_smem_attr(kern, smem, attr_done)) return rc;
  const int resident = resident_ctas(kern, NW * 32, smem, per_sm);
  if (resident <= 0) return GQA_ERR_CUDA;
  const long long units_max = (long long)a.n_slots * a.h_kv * a.n_hb * a.B;
  // As few CTAs as take the units in the same number of rounds, so every CTA
  // gets the same number of units (to one): with all 296 resident CTAs, the
  // 512 units of the Llama-70B-shaped call leave 80 CTAs without a second
  // unit while the others stream it; with 256 every CTA takes two.  Measured
  // on B200 (2000 back-to-back calls): 45.2 -> 44.0 us on that call, 640 ->
  // 633 us on the 1M-key one.
  const long long rounds = (units_max + resident - 1) / resident;
  const int ctas = (int)((units_max + rounds - 1) / rounds);
  DecodeArgs b = a;
  b.hint_ctas = ctas;  // one wave: every CTA prefetches
  CUtensorMap kmap, vmap;
  if (!cached_cache_map(&kmap, a.k, a.h_kv, D, a.kv_rows) ||
      !cached_cache_map(&vmap, a.v, a.h_kv, D, a.kv_rows))
    return GQA_ERR_CUDA;
  if (int rc = launch_pdl(kern, dim3(ctas), dim3(NW * 32), smem, st, kmap, vmap, b)) return rc;
  return PARTIAL ? GQA_OK : launch_merge_rows(a, D, st);
}

template <int D, int HB, int MODE>
int launch_simt(DecodeArgs a, dim3 grid, cudaStream_t st) {
  constexpr int NW = 4;
  static std::atomic<int> per_sm[kMaxDevices];
  auto kern = decode_simt_f32<D, HB, NW, MODE>;
  if (a.hint_tiles > 0) {  // the grid's first wave prefetches
    a.hint_ctas = resident_ctas(kern, NW * 32, 0, per_sm);
    if (a.hint_ctas < 0) return GQA_ERR_CUDA;
  }
  return launch_pdl(kern, grid, dim3(NW * 32), 0, st, a);
}

template <int D, int MODE>
int launch_simt_hb(const DecodeArgs& a, int hb, dim3 grid, cudaStream_t st) {
  switch (hb) {
    case 1: return launch_simt<D, 1, MODE>(a, grid, st);
    case 2: return launch_simt<D, 2, MODE>(a, grid, st);
    case 4: return launch_simt<D, 4, MODE>(a, grid, st);
    case 8: return launch_simt<D, 8, MODE>(a, grid, st);
    default: return launch_simt<D, 16, MODE>(a, grid, st);
  }
}

// One CTA per (split, kv head, head block, b).
template <int MODE>
int launch_decode(DecodeArgs a, int dtype, int D, cudaStream_t st) {
  const int hb = heads_per_cta(dtype, a.G);
  a.n_hb = (a.G + hb - 1) / hb;
  const dim3 grid(a.n_slots, a.h_kv * a.n_hb, a.B);
  if (dtype == GQA_BF16) {
    const bool wide = hb == 16;
    if (MODE == kFused) {
      const long long units = (long long)grid.x * grid.y * grid.z;
      switch (fused_plan(units, D)) {
        case kPlanOneWave:
          if (one_wave_merge_kernel(a.G)) {
            int rc;
            if (D == 128)
              rc = wide ? launch_tc<128, 2, kPartial>(a, grid, st) : launch_tc<128, 1, kPartial>(a, grid, st);
            else
              rc = wide ? launch_tc<64, 2, kPartial>(a, grid, st) : launch_tc<64, 1, kPartial>(a, grid, st);
            if (rc) return rc;
            return launch_merge_rows(a, D, st);
          }
          if (D == 128)
            return wide ? launch_tc<128, 2, kFused>(a, grid, st) : launch_tc<128, 1, kFused>(a, grid, st);
          return wide ? launch_tc<64, 2, kFused>(a, grid, st) : launch_tc<64, 1, kFused>(a, grid, st);
        case kPlanPersistent:
          if (D == 128)
            return wide ? launch_persist<128, 2, false>(a, st) : launch_persist<128, 1, false>(a, st);
          return wide ? launch_persist<64, 2, false>(a, st) : launch_persist<64, 1, false>(a, st);
        case kPlanManyWaves:
          if (D == 128)
            return wide ? launch_tc<128, 2, kFused, 2>(a, grid, st)
                        : launch_tc<128, 1, kFused, 2>(a, grid, st);
          return wide ? launch_tc<64, 2, kFused, 2>(a, grid, st) : launch_tc<64, 1, kFused, 2>(a, grid, st);
        default:
          return GQA_ERR_CUDA;
      }
    }
    // Partial call: a grid of a few waves runs on the persistent CTAs too
    // (every split's triplet stored, empty ones included; no merge).
    if (fused_plan((long long)grid.x * grid.y * grid.z, D) == kPlanPersistent) {
      if (D == 128)
        return wide ? launch_persist<128, 2, true>(a, st) : launch_persist<128, 1, true>(a, st);
      return wide ? launch_persist<64, 2, true>(a, st) : launch_persist<64, 1, true>(a, st);
    }
    if (D == 128)
      return wide ? launch_tc<128, 2, kPartial>(a, grid, st) : launch_tc<128, 1, kPartial>(a, grid, st);
    return wide ? launch_tc<64, 2, kPartial>(a, grid, st) : launch_tc<64, 1, kPartial>(a, grid, st);
  }
  if (D == 128) return launch_simt_hb<128, MODE>(a, hb, grid, st);
  return launch_simt_hb<64, MODE>(a, hb, grid, st);
}

// Split count chosen for the caller (n_splits == 0 on a fused call): the
// largest count whose grid still fits on the GPU in one wave (R CTAs), capped
// so a split keeps >= 256 keys when max_seqlen is known (> 0).  One wave
// avoids the grids just past R, where a few leftover splits run alone.
int auto_splits(int B, int h_q, int h_kv, int D, int max_seqlen) {
  if (B < 1 || h_kv < 1 || h_q < h_kv || h_q % h_kv) return -GQA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return -GQA_ERR_UNSUPPORTED;
  const int sms = sm_count();
  if (sms <= 0) return -GQA_ERR_CUDA;
  const int smem = D == 128 ? tc_dynamic_smem<128, kTcWarps, kTcStages>()
                            : tc_dynamic_smem<64, kTcWarps, kTcStages>();
  const long long R = (long long)sms * ((228 * 1024) / (smem + 1024));
  const int G = h_q / h_kv;
  const long long bh = (long long)B * h_kv * (G <= 16 ? 1 : (G + 15) / 16);
  long long n = bh >= R ? 1 : R / bh;
  if (max_seqlen > 0) {
    const long long cap = (max_seqlen + 255) / 256;
    if (n > cap) n = cap;
  }
  if (n < 1) n = 1;
  if (n > kMaxSlots) n = kMaxSlots;
  return (int)n;
}

// ------------------------------------------------------------ validation

struct Shape {
  int B, h_q, h_kv, D, n_slots, n_splits, chunk_len, dtype;
  float scale;
};

// Size / value checks that need no pointers.
int check_shape(const Shape& s) {
  if (s.B < 0 || s.h_q < 1 || s.h_kv < 1 || s.h_q % s.h_kv != 0) return GQA_ERR_INVALID_ARG;
  if (s.dtype != GQA_F32 && s.dtype != GQA_BF16) return GQA_ERR_INVALID_ARG;
  if (!std::isfinite(s.scale)) return GQA_ERR_INVALID_ARG;
  if (s.D != 64 && s.D != 128) return s.D > 0 ? GQA_ERR_UNSUPPORTED : GQA_ERR_INVALID_ARG;
  if (s.n_slots < 1 || s.n_slots > kMaxSlots) return GQA_ERR_INVALID_ARG;
  if (s.B > 65535) return GQA_ERR_UNSUPPORTED;
  const int G = s.h_q / s.h_kv;
  const int hb = heads_per_cta(s.dtype, G);
  if ((long long)s.h_kv * ((G + hb - 1) / hb) > 65535) return GQA_ERR_UNSUPPORTED;
  return GQA_OK;
}

int check_common(const void* q, const void* k, const void* v, const int32_t* seqlens,
                 long long kv_rows, const Shape& s) {
  if (int rc = check_shape(s)) return rc;
  if (kv_rows < -1) return GQA_ERR_INVALID_ARG;
  if (kv_rows > 0x7fffffffLL) return GQA_ERR_UNSUPPORTED;  // int32 row coordinates
  if (s.B == 0) return GQA_OK;
  if (!q || !k || !v || !seqlens) return GQA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(seqlens, 4))
    return GQA_ERR_INVALID_ARG;
  return GQA_OK;
}

Shape split_shape(int B, int h_q, int h_kv, int D, int n_splits, float scale, int dtype) {
  return Shape{B, h_q, h_kv, D, n_splits, n_splits, 0, dtype, scale};
}

Shape chunk_shape(int B, int h_q, int h_kv, int D, int chunk_len, int max_seqlen, float scale,
                  int dtype) {
  int slots = -1;
  if (chunk_len >= 1 && max_seqlen >= 0) {
    const long long n = ((long long)max_seqlen + chunk_len - 1) / chunk_len;
    slots = n < 1 ? 1 : (n > kMaxSlots ? kMaxSlots + 1 : (int)n);
  }
  return Shape{B, h_q, h_kv, D, slots, 0, chunk_len, dtype, scale};
}

DecodeArgs make_args(const void* q, const void* k, const void* v, const int32_t* seqlens,
                     long long kv_rows, const Shape& s) {
  DecodeArgs a{};
  a.kv_rows = kv_rows;
  // the prefetch addresses are only provably inside the cache when its rows
  // are known; the fp32 kernel prefetches its warps' first batch of keys
  a.hint_tiles = kv_rows < 0 ? 0 : (s.dtype == GQA_BF16 ? kHintTiles : 1);
  a.q = q;
  a.k = k;
  a.v = v;
  a.seqlens = seqlens;
  a.B = s.B;
  a.h_q = s.h_q;
  a.h_kv = s.h_kv;
  a.G = s.h_q / s.h_kv;
  a.n_splits = s.n_splits;
  a.chunk_len = s.chunk_len;
  a.n_slots = s.n_slots;
  a.scale_log2 = s.scale * kLog2e;
  a.timeout_ns = g_timeout_ns.load(std::memory_order_relaxed);
  return a;
}

// ------------------------------------------------------------- workspace

struct WsLayout {
  size_t tickets, m, l, o, total;
};

// Workspace = a fixed 256 KiB ticket area, then the fp32 triplets.  The ticket
// area has the same size and place for every shape, and each call returns the
// tickets it used to zero, so the area is all zeros at rest whatever shapes
// used the workspace before (triplets of one shape never land on tickets of
// another).  Both paths split a group into ceil(G / 16) head blocks when
// G > 16 and use one block otherwise, so the layout does not depend on dtype.
constexpr size_t kTicketBytes = 256 * 1024;

size_t n_tickets(const Shape& s) {
  const int G = s.h_q / s.h_kv;
  return (size_t)s.B * s.h_kv * (G <= 16 ? 1 : (G + 15) / 16);
}

WsLayout ws_layout(const Shape& s) {
  const size_t rows = (size_t)s.B * s.h_q;
  WsLayout w;
  w.tickets = 0;
  w.m = kTicketBytes;
  w.l = w.m + round_up(rows * s.n_slots * sizeof(float), 256);
  w.o = w.l + round_up(rows * s.n_slots * sizeof(float), 256);
  w.total = w.o + round_up(rows * s.n_slots * s.D * sizeof(float), 256);
  return w;
}

struct LibWorkspace {
  void* ptr = nullptr;
  size_t bytes = 0;
};
std::mutex g_ws_mu;
LibWorkspace g_ws[kMaxDevices];

// Library-owned, zero-filled, grow-only workspace of the current device.
int lib_workspace(size_t need, void** out) {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return GQA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_ws_mu);
  LibWorkspace& w = g_ws[dev];
  if (w.bytes < need) {
    if (w.ptr) {
      if (cudaDeviceSynchronize() != cudaSuccess) return GQA_ERR_CUDA;
      cudaFree(w.ptr);
      w.ptr = nullptr;
      w.bytes = 0;
    }
    const size_t bytes = round_up(need, 1 << 20);
    void* p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) return GQA_ERR_WORKSPACE;
    if (cudaMemset(p, 0, bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
      cudaFree(p);
      return GQA_ERR_CUDA;
    }
    w.ptr = p;
    w.bytes = bytes;
  }
  *out = w.ptr;
  return GQA_OK;
}

// The token to append and the per-sequence capacity of a padded cache
// ([B][cap][h_kv][d]); all zero for the plain packed-cache calls.
struct Append {
  const void* k_new = nullptr;
  const void* v_new = nullptr;
  long long cap = 0;
};

int fused(const void* q, const void* k, const void* v, const int32_t* seqlens, long long kv_rows,
          float* out, const Shape& s, void* workspace, size_t workspace_bytes, void* stream,
          const Append& app = Append()) {
  if (int rc = check_common(q, k, v, seqlens, kv_rows, s)) return rc;
  if (n_tickets(s) * sizeof(int) > kTicketBytes) return GQA_ERR_UNSUPPORTED;
  if (s.B == 0) return GQA_OK;
  if (!out || !aligned(out, 16)) return GQA_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(s);
  void* ws = workspace;
  if (ws) {
    if (workspace_bytes < w.total || !aligned(ws, 256)) return GQA_ERR_WORKSPACE;
  } else if (int rc = lib_workspace(w.total, &ws)) {
    return rc;
  }
  DecodeArgs a = make_args(q, k, v, seqlens, kv_rows, s);
  a.k_new = app.k_new;
  a.v_new = app.v_new;
  a.cap = app.cap;
  uint8_t* base = static_cast<uint8_t*>(ws);
  a.tickets = reinterpret_cast<int*>(base + w.tickets);
  a.m = reinterpret_cast<float*>(base + w.m);
  a.l = reinterpret_cast<float*>(base + w.l);
  a.o = reinterpret_cast<float*>(base + w.o);
  a.out = out;
  return launch_decode<kFused>(a, s.dtype, s.D, as_stream(stream));
}

int partial(const void* q, const void* k, const void* v, const int32_t* seqlens, long long kv_rows,
            float* m, float* l, float* o, const Shape& s, void* stream) {
  if (int rc = check_common(q, k, v, seqlens, kv_rows, s)) return rc;
  if (s.B == 0) return GQA_OK;
  if (!m || !l || !o || !aligned(m, 16) || !aligned(l, 16) || !aligned(o, 16))
    return GQA_ERR_INVALID_ARG;
  DecodeArgs a = make_args(q, k, v, seqlens, kv_rows, s);
  a.m = m;
  a.l = l;
  a.o = o;
  return launch_decode<kPartial>(a, s.dtype, s.D, as_stream(stream));
}

// ------------------------------------------------ allocation-free variant

// Scratch for gqa_decode_attn_noalloc: a fixed array in this module's global
// memory, so that entry point never allocates.  Every device that loads the
// library holds these bytes until the process exits.  The first 256 KiB are
// the ticket area, the rest holds the triplets, exactly as in a caller's
// workspace.
constexpr size_t kNoAllocScratchBytes = 40ull << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array, looked up once per device.  In host
// code `g_noalloc_scratch` only names a host-side stand-in; handing that name
// to a kernel would read the wrong memory, so the address always comes from
// cudaGetSymbolAddress with the device current.
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices];

int noalloc_scratch(void** out) {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return GQA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return GQA_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return GQA_OK;
}

__global__ void selftest_wait_kernel(unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  // No thread ever arrives on `bar`: the wait must run out and report it.
  if (threadIdx.x == 0 && !mbar_wait_bounded(smem_u32(&bar), 0, timeout_ns))
    raise_status(kStatusTimeout);
}

#ifdef GQA_CHECKED
// Self-test of the index checks: one check whose index equals its extent.
// It fails, and the store it guards is skipped.
__global__ void selftest_bounds_kernel(int* sink) {
  if (threadIdx.x == 0 && in_bounds(1, 1, kSiteSelftest)) *sink = 1;
}
#endif

// ------------------------------------------------------------ prefill

// 3-D view (d = 128, head, row) of a packed bf16 [rows][heads][128] tensor;
// box = 64 d x 1 head x box_rows rows, 128-byte swizzle.  The row extent is
// the tensor's own, so a tile that runs past the last row reads zeros.
bool encode_rows_map(CUtensorMap* map, const void* base, int heads, int rows, int box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kPfD), static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kPfD) * 2,
                                 static_cast<cuuint64_t>(heads) * kPfD * 2};
  const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int prefill(const void* q, const void* k, const void* v, const int32_t* seqlens, float* out,
            int B, int total_rows, int max_seqlen, int h_q, int h_kv, int d_head, float scale,
            int dtype, void* stream) {
  if (B < 0 || total_rows < 0 || max_seqlen < 0 || h_q < 1 || h_kv < 1 || h_q % h_kv != 0)
    return GQA_ERR_INVALID_ARG;
  if (dtype != GQA_F32 && dtype != GQA_BF16) return GQA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return GQA_ERR_INVALID_ARG;
  if (d_head < 1) return GQA_ERR_INVALID_ARG;
  if (d_head != kPfD || dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED;
  if (B == 0 || total_rows == 0) return GQA_OK;
  if (max_seqlen == 0) return GQA_ERR_INVALID_ARG;   // rows exist, so some S_b > 0
  if (!q || !k || !v || !seqlens || !out) return GQA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(seqlens, 4))
    return GQA_ERR_INVALID_ARG;
  const int n_qtiles = (max_seqlen + kPfRows - 1) / kPfRows;
  if (B > 65535 || h_q > 65535 || n_qtiles > 65535) return GQA_ERR_UNSUPPORTED;
  static std::atomic<uint64_t> attr_done{0};
  if (int rc = ensure_smem_attr(prefill_tc_bf16, kPfDynSmem, attr_done)) return rc;
  CUtensorMap qmap, kmap, vmap;
  if (!encode_rows_map(&qmap, q, h_q, total_rows, kPfRows) ||
      !encode_rows_map(&kmap, k, h_kv, total_rows, kPfKeys) ||
      !encode_rows_map(&vmap, v, h_kv, total_rows, kPfKeys))
    return GQA_ERR_CUDA;
  PrefillArgs a{};
  a.seqlens = seqlens;
  a.out = out;
  a.total_rows = total_rows;
  a.B = B;
  a.h_q = h_q;
  a.h_kv = h_kv;
  a.G = h_q / h_kv;
  a.n_qtiles = n_qtiles;
  a.scale_log2 = scale * kLog2e;
  a.timeout_ns = g_timeout_ns.load(std::memory_order_relaxed);
  return launch_pdl(prefill_tc_bf16, dim3(h_q, B, n_qtiles), dim3(kPfThreads), kPfDynSmem,
                    as_stream(stream), qmap, kmap, vmap, a);
}

}  // namespace

// ====================================================================== ABI

extern "C" {

int gqa_decode_version(void) { return 300; }

const char* gqa_decode_error_string(int status) {
  switch (status) {
    case GQA_OK: return "GQA_OK";
    case GQA_ERR_INVALID_ARG: return "GQA_ERR_INVALID_ARG: invalid argument";
    case GQA_ERR_UNSUPPORTED: return "GQA_ERR_UNSUPPORTED: valid but unsupported shape";
    case GQA_ERR_CUDA: return "GQA_ERR_CUDA: a CUDA call failed";
    case GQA_ERR_WORKSPACE: return "GQA_ERR_WORKSPACE: workspace too small, misaligned or not allocatable";
    case GQA_ERR_DEVICE_TIMEOUT: return "GQA_ERR_DEVICE_TIMEOUT: a bounded wait in a kernel ran out";
    case GQA_ERR_DEVICE_SEQLEN: return "GQA_ERR_DEVICE_SEQLEN: a kernel saw S_b < 0 or S_b > max_seqlen";
    case GQA_ERR_DEVICE_BOUNDS: return "GQA_ERR_DEVICE_BOUNDS: an index check of the checked build failed";
    default: return "unknown gqa_status";
  }
}

size_t gqa_decode_workspace_size(int B, int h_q, int h_kv, int d_head, int n_splits) {
  if (n_splits == 0 && B > 0) {
    n_splits = auto_splits(B, h_q, h_kv, d_head, 0);
    if (n_splits < 0) return 0;
  }
  const Shape s = split_shape(B, h_q, h_kv, d_head, n_splits, 1.f, GQA_BF16);
  if (check_shape(s) || n_tickets(s) * sizeof(int) > kTicketBytes) return 0;
  return ws_layout(s).total;
}

size_t gqa_decode_chunked_workspace_size(int B, int h_q, int h_kv, int d_head, int chunk_len,
                                         int max_seqlen) {
  const Shape s = chunk_shape(B, h_q, h_kv, d_head, chunk_len, max_seqlen, 1.f, GQA_BF16);
  if (check_shape(s) || n_tickets(s) * sizeof(int) > kTicketBytes) return 0;
  return ws_layout(s).total;
}

int gqa_decode_attn(const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* seqlens, long long kv_rows, float* out, int B, int h_q,
                    int h_kv, int d_head, int n_splits, float scale, int dtype, void* workspace,
                    size_t workspace_bytes, void* stream) {
  if (n_splits == 0 && B > 0) {
    n_splits = auto_splits(B, h_q, h_kv, d_head, 0);
    if (n_splits < 0) return -n_splits;
  }
  return fused(q, k_cache, v_cache, seqlens, kv_rows, out,
               split_shape(B, h_q, h_kv, d_head, n_splits, scale, dtype), workspace,
               workspace_bytes, stream);
}

int gqa_decode_attn_noalloc(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* seqlens, long long kv_rows, float* out, int B, int h_q,
                            int h_kv, int d_head, int n_splits, float scale, int dtype,
                            void* stream) {
  if (n_splits == 0 && B > 0) {
    n_splits = auto_splits(B, h_q, h_kv, d_head, 0);
    if (n_splits < 0) return -n_splits;
  }
  const Shape s = split_shape(B, h_q, h_kv, d_head, n_splits, scale, dtype);
  if (int rc = check_common(q, k_cache, v_cache, seqlens, kv_rows, s)) return rc;
  if (n_tickets(s) * sizeof(int) > kTicketBytes) return GQA_ERR_UNSUPPORTED;
  if (s.B == 0) return GQA_OK;
  const size_t need = ws_layout(s).total;
  if (need > kNoAllocScratchBytes) return GQA_ERR_WORKSPACE;  // beyond the fixed scratch
  void* scratch = nullptr;
  if (int rc = noalloc_scratch(&scratch)) return rc;
  // The array keeps whatever the previous call left; the tickets must start
  // at zero, so clear this call's part of the ticket area first.  A call
  // that merges in a second kernel (two launches) reads no ticket and needs
  // no clearing.
  const bool uses_tickets =
      gqa_decode_launches_per_call(B, h_q, h_kv, d_head, s.n_slots, dtype) != 2;
  if (uses_tickets &&
      cudaMemsetAsync(scratch, 0, n_tickets(s) * sizeof(int), as_stream(stream)) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_CUDA;
  }
  return fused(q, k_cache, v_cache, seqlens, kv_rows, out, s, scratch, kNoAllocScratchBytes,
               stream);
}

int gqa_decode_attn_append(const void* q, const void* k_new, const void* v_new, void* k_cache,
                           void* v_cache, const int32_t* seqlens, float* out, int B, int h_q,
                           int h_kv, int d_head, int cache_capacity, int n_splits, float scale,
                           int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  if (n_splits == 0 && B > 0) {
    n_splits = auto_splits(B, h_q, h_kv, d_head, cache_capacity);
    if (n_splits < 0) return -n_splits;
  }
  const Shape s = split_shape(B, h_q, h_kv, d_head, n_splits, scale, dtype);
  if (cache_capacity < 1) return GQA_ERR_INVALID_ARG;
  if ((long long)B * cache_capacity > 0x7fffffffLL) return GQA_ERR_UNSUPPORTED;  // int32 rows
  if (B > 0 && (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16)))
    return GQA_ERR_INVALID_ARG;
  Append app;
  app.k_new = k_new;
  app.v_new = v_new;
  app.cap = cache_capacity;
  // the padded cache's B * cache_capacity rows bound every read
  return fused(q, k_cache, v_cache, seqlens, (long long)B * cache_capacity, out, s, workspace,
               workspace_bytes, stream, app);
}

int gqa_decode_attn_chunked(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* seqlens, long long kv_rows, float* out, int B, int h_q,
                            int h_kv, int d_head, int chunk_len, int max_seqlen, float scale,
                            int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  return fused(q, k_cache, v_cache, seqlens, kv_rows, out,
               chunk_shape(B, h_q, h_kv, d_head, chunk_len, max_seqlen, scale, dtype), workspace,
               workspace_bytes, stream);
}

int gqa_decode_partial(const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* seqlens, long long kv_rows, float* m, float* l, float* o,
                       int B, int h_q, int h_kv, int d_head, int n_splits, float scale, int dtype,
                       void* stream) {
  return partial(q, k_cache, v_cache, seqlens, kv_rows, m, l, o,
                 split_shape(B, h_q, h_kv, d_head, n_splits, scale, dtype), stream);
}

int gqa_decode_partial_chunked(const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* seqlens, long long kv_rows, float* m, float* l,
                               float* o, int B, int h_q, int h_kv, int d_head, int chunk_len,
                               int max_seqlen, float scale, int dtype, void* stream) {
  return partial(q, k_cache, v_cache, seqlens, kv_rows, m, l, o,
                 chunk_shape(B, h_q, h_kv, d_head, chunk_len, max_seqlen, scale, dtype), stream);
}

int mlo_merge(const float* m, const float* l, const float* o, float* out, int rows, int n_splits,
              int d_head, void* stream) {
  if (rows < 0 || n_splits < 1 || d_head < 1 || d_head > 256) return GQA_ERR_INVALID_ARG;
  if (rows == 0) return GQA_OK;
  if (!m || !l || !o || !out) return GQA_ERR_INVALID_ARG;
  if (!aligned(m, 4) || !aligned(l, 4) || !aligned(o, 4) || !aligned(out, 4))
    return GQA_ERR_INVALID_ARG;
  const dim3 grid((rows + 3) / 4);
  cudaStream_t st = as_stream(stream);
  if (d_head <= 64)
    return launch_pdl(mlo_merge_kernel<2>, grid, dim3(128), 0, st, m, l, o, out, rows, n_splits, d_head);
  if (d_head <= 128)
    return launch_pdl(mlo_merge_kernel<4>, grid, dim3(128), 0, st, m, l, o, out, rows, n_splits, d_head);
  return launch_pdl(mlo_merge_kernel<8>, grid, dim3(128), 0, st, m, l, o, out, rows, n_splits, d_head);
}

int mlo_merge_ranked(const float* m, const float* l, const float* o, float* out, int rows,
                     int n_ranks, int n_splits, int d_head, long long rank_stride_ml,
                     long long rank_stride_o, void* stream) {
  if (rows < 0 || n_ranks < 1 || n_splits < 1 || d_head < 1 || d_head > 256)
    return GQA_ERR_INVALID_ARG;
  if ((long long)n_ranks * n_splits > (1 << 20)) return GQA_ERR_INVALID_ARG;
  if (rows == 0) return GQA_OK;
  // each rank's block must not overlap the next one's
  if (n_ranks > 1 && (rank_stride_ml < (long long)rows * n_splits ||
                      rank_stride_o < (long long)rows * n_splits * d_head))
    return GQA_ERR_INVALID_ARG;
  if (!m || !l || !o || !out) return GQA_ERR_INVALID_ARG;
  if (!aligned(m, 4) || !aligned(l, 4) || !aligned(o, 4) || !aligned(out, 4))
    return GQA_ERR_INVALID_ARG;
  const dim3 grid((rows + 3) / 4);
  cudaStream_t st = as_stream(stream);
  const size_t sml = (size_t)rank_stride_ml, so = (size_t)rank_stride_o;
  if (d_head <= 64)
    return launch_pdl(mlo_merge_ranked_kernel<2>, grid, dim3(128), 0, st, m, l, o, out, rows,
                      n_ranks, n_splits, d_head, sml, so);
  if (d_head <= 128)
    return launch_pdl(mlo_merge_ranked_kernel<4>, grid, dim3(128), 0, st, m, l, o, out, rows,
                      n_ranks, n_splits, d_head, sml, so);
  return launch_pdl(mlo_merge_ranked_kernel<8>, grid, dim3(128), 0, st, m, l, o, out, rows,
                    n_ranks, n_splits, d_head, sml, so);
}

int gqa_decode_auto_splits(int B, int h_q, int h_kv, int d_head, int max_seqlen) {
  return auto_splits(B, h_q, h_kv, d_head, max_seqlen);
}

int gqa_decode_launches_per_call(int B, int h_q, int h_kv, int d_head, int n_slots, int dtype) {
  const Shape s = split_shape(B, h_q, h_kv, d_head, n_slots, 1.f, dtype);
  if (check_shape(s)) return -GQA_ERR_INVALID_ARG;
  if (B == 0) return 0;
  if (dtype != GQA_BF16) return 1;
  const int G = h_q / h_kv;
  const int hb = tc_heads_per_cta(G);
  const long long units = (long long)n_slots * h_kv * ((G + hb - 1) / hb) * B;
  const int plan = fused_plan(units, d_head);
  if (plan < 0) return -GQA_ERR_CUDA;
  return (plan == kPlanPersistent || (plan == kPlanOneWave && one_wave_merge_kernel(G))) ? 2 : 1;
}

int gqa_decode_fused_plan(int B, int h_q, int h_kv, int d_head, int n_slots, int dtype) {
  const Shape s = split_shape(B, h_q, h_kv, d_head, n_slots, 1.f, dtype);
  if (check_shape(s) || B == 0) return -GQA_ERR_INVALID_ARG;
  if (dtype != GQA_BF16) return GQA_PLAN_SIMT;
  const int G = h_q / h_kv;
  const int hb = tc_heads_per_cta(G);
  const long long units = (long long)n_slots * h_kv * ((G + hb - 1) / hb) * B;
  switch (fused_plan(units, d_head)) {
    case kPlanOneWave: return GQA_PLAN_ONE_WAVE;
    case kPlanPersistent: return GQA_PLAN_PERSISTENT;
    case kPlanManyWaves: return GQA_PLAN_MANY_WAVES;
    default: return -GQA_ERR_CUDA;
  }
}

int gqa_prefill_attn(const void* q, const void* k, const void* v, const int32_t* seqlens,
                     float* out, int B, int total_rows, int max_seqlen, int h_q, int h_kv,
                     int d_head, float scale, int dtype, void* stream) {
  return prefill(q, k, v, seqlens, out, B, total_rows, max_seqlen, h_q, h_kv, d_head, scale,
                 dtype, stream);
}

int gqa_decode_get_status(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return GQA_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_status, sizeof(word)) != cudaSuccess) return GQA_ERR_CUDA;
  if (word) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return GQA_ERR_CUDA;
  }
  if (word & kStatusTimeout) return GQA_ERR_DEVICE_TIMEOUT;
  if (word & kStatusBounds) return GQA_ERR_DEVICE_BOUNDS;
  if (word & (kStatusNegSeqlen | kStatusSeqlenOverMax)) return GQA_ERR_DEVICE_SEQLEN;
  return GQA_OK;
}

int gqa_decode_checked_build(void) {
#ifdef GQA_CHECKED
  return 1;
#else
  return 0;
#endif
}

unsigned long long gqa_decode_bounds_report(void* stream) {
#ifdef GQA_CHECKED
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return ~0ull;
  unsigned long long rec = 0;
  if (cudaMemcpyFromSymbol(&rec, g_bounds_first, sizeof(rec)) != cudaSuccess) return ~0ull;
  if (rec) {
    const unsigned long long zero = 0;
    if (cudaMemcpyToSymbol(g_bounds_first, &zero, sizeof(zero)) != cudaSuccess) return ~0ull;
  }
  return rec;
#else
  (void)stream;
  return 0;
#endif
}

int gqa_decode_selftest_bounds(void* stream) {
#ifdef GQA_CHECKED
  // The guarded store's target: one int per device, never freed (the
  // failing check skips the store, but the pointer is a real one regardless).
  static std::mutex mu;
  static int* sink[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return GQA_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (!sink[dev] && cudaMalloc(&sink[dev], sizeof(int)) != cudaSuccess) return GQA_ERR_CUDA;
  }
  selftest_bounds_kernel<<<1, 32, 0, as_stream(stream)>>>(sink[dev]);
  return after_launch();
#else
  (void)stream;
  return GQA_ERR_UNSUPPORTED;
#endif
}

int gqa_decode_set_wait_timeout_ns(unsigned long long timeout_ns) {
  g_timeout_ns.store(timeout_ns ? timeout_ns : kDefaultTimeoutNs, std::memory_order_relaxed);
  return GQA_OK;
}

int gqa_decode_selftest_wait_timeout(unsigned long long timeout_ns, void* stream) {
  if (timeout_ns == 0 || timeout_ns > 10ull * kDefaultTimeoutNs) return GQA_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 32, 0, as_stream(stream)>>>(timeout_ns);
  return after_launch();
}

int gqa_decode_release(void) {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return GQA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_ws_mu);
  LibWorkspace& w = g_ws[dev];
  if (w.ptr) {
    if (cudaDeviceSynchronize() != cudaSuccess) return GQA_ERR_CUDA;
    cudaFree(w.ptr);
    w.ptr = nullptr;
    w.bytes = 0;
  }
  return GQA_OK;
}

}  // extern "C"
