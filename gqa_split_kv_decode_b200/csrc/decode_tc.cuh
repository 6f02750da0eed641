// bf16 decode attention: TMA-fed K/V tiles, tensor-core logits and PV.
//
// One CTA owns one (split, kv head g, head block, b).  Each of its NW warps
// runs its own NS-stage TMA ring: a stage holds KT = 16 consecutive keys of K
// and V for kv head g (one 64-element, 128-byte-swizzled box per half of
// d_head), loaded once from HBM and shared by every query head of the group
// (exllama "Llama 2 is out": broadcast the kv head to its group instead of
// copying the cache).  Warp w takes the split's tiles w, w + NW, ..., so the
// warps of a CTA are sub-splits whose triplets are merged in shared memory at
// the end -- the page's merge rule once more.
//
// The products are oriented so the group, not the keys, is the narrow side:
//   S^T[key][head] = K[key][:] . Q^T[:][head]     mma m16n8k16, M = 16 keys,
//                                                 N = 8 heads, K = d
//   o^T[d][head]  += V^T[d][key] . P^T[key][head] M = 16 dims, N = 8 heads,
//                                                 K = 16 keys
// so a group of 8 (Llama-70B) fills N exactly.  Q^T stays in registers for
// the whole split; the S^T accumulator becomes P^T's B fragment through one
// movmatrix transpose per 8x8 block.  Softmax statistics are fp32 in base 2
// (scale * log2 e is folded into one multiply), reduced with shuffles across
// the 8 lanes that share a head.  P enters the PV product as two bf16 parts
// (hi + lo) so its rounding stays near fp32 level.
//
// The last tile of a split that is not a whole tile is loaded as the KT rows
// that END at the split's end (shifted back) and the rows before the tile's
// first new key are masked by index, so no load ever reaches past the
// batch's last cache row.  A shift below row 0 reads TMA zero fill.
#pragma once

#include "split_merge.cuh"

namespace gqa {

constexpr int kTileKeys = 16;
constexpr int kBoxBytes = kTileKeys * 128;  // 16 rows x 64 bf16 (one d half)

template <int D>
struct TcShape {
  static constexpr int kHalves = D / 64;
  static constexpr int kStageBytes = 2 * kHalves * kBoxBytes;  // K halves, then V halves
  static constexpr int kSteps = D / 16;                        // k-steps of S^T, d-tiles of o^T
};

template <int D, int NW, int NS>
constexpr int tc_dynamic_smem() {
  return NW * NS * TcShape<D>::kStageBytes + 1024;  // + slack for 1024-byte alignment
}

// Q^T as the B operand of S^T = K Q^T: thread holds head (lane / 4) of the
// n-tile and d = 16 * ks + 2 * (lane % 4) + {0, 1} (b0) and + {8, 9} (b1).
// Heads at or past G (padding of a partial block) read as zero.
template <int D, int NT>
__device__ __forceinline__ void load_q_frags(uint32_t (&qf)[NT][D / 16][2], const DecodeArgs& a,
                                             int b, int g, int hb, int lane) {
  constexpr int HB = NT * 8;
  const uint32_t* qw = static_cast<const uint32_t*>(a.q);  // bf16 pairs
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int gi = hb * HB + nt * 8 + (lane >> 2);
    const bool ok = gi < a.G && in_bounds((long long)query_row(a, b, g, gi), (long long)a.B * a.h_q,
                                          kSiteQ);
    const size_t base = (query_row(a, b, g, ok ? gi : 0) * D) / 2 + (lane & 3);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      qf[nt][ks][0] = ok ? __ldg(qw + base + ks * 8) : 0u;
      qf[nt][ks][1] = ok ? __ldg(qw + base + ks * 8 + 4) : 0u;
    }
  }
}

// Online-softmax state of one warp over the keys it has seen: per head
// column (2 per lane and n-tile) the running max m (base 2) and this lane's
// share of the denominator l; o^T accumulators in mma C-fragment layout
// (d = 16 dt + lane/4 (+8), head = 8 nt + 2 (lane%4) (+1)).
template <int D, int NT>
struct WarpAcc {
  float m[NT][2], l[NT][2];
  float o[D / 16][NT][4];

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m[nt][0] = m[nt][1] = -INFINITY;
      l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
      for (int dt = 0; dt < D / 16; ++dt)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[dt][nt][e] = 0.f;
    }
  }

  // Sums each head's denominator over the 8 lanes that share its column.
  __device__ __forceinline__ void reduce_l() {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int o2 = 4; o2 < 32; o2 <<= 1) l[nt][j] += __shfl_xor_sync(kFull, l[nt][j], o2);
  }
};

// One 16-key tile held in shared memory at kbase (K) / vbase (V), 128-byte
// swizzled boxes of 16 rows x 64 d: S^T = K Q^T, masking, online softmax and
// o^T += V^T P^T.  valid0 / valid1: whether key rows lane/4 and lane/4 + 8 of
// the tile belong to the range (at least one row of a tile always does).
template <int D, int NT>
__device__ __forceinline__ void tc_tile(WarpAcc<D, NT>& acc, const uint32_t (&qf)[NT][D / 16][2],
                                        uint32_t kbase, uint32_t vbase, bool valid0, bool valid1,
                                        float scale_log2, int lane) {
  constexpr int STEPS = D / 16;
  // ---- S^T = K Q^T (16 keys x 8 heads per n-tile)
  float sacc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
  {
    const int r = lane & 15;  // key row of this lane's ldmatrix address
#pragma unroll
    for (int ks = 0; ks < STEPS; ++ks) {
      const int half = ks >> 2;
      const int chunk = ((ks & 3) << 1) + (lane >> 4);  // 16-byte chunk within the half
      uint32_t af[4];
      ldsm_x4(kbase + half * kBoxBytes + r * 128 + ((chunk ^ (r & 7)) << 4), af);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(sacc[nt], af, qf[nt][ks][0], qf[nt][ks][1]);
    }
  }

  // ---- mask, online softmax (base 2)
  float p[NT][4];
  bool rescale = false;
  float alpha[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const float s0 = valid0 ? sacc[nt][0] * scale_log2 : -INFINITY;
    const float s1 = valid0 ? sacc[nt][1] * scale_log2 : -INFINITY;
    const float s2 = valid1 ? sacc[nt][2] * scale_log2 : -INFINITY;
    const float s3 = valid1 ? sacc[nt][3] * scale_log2 : -INFINITY;
    float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, o));
    }
    // every tile holds at least one valid key, so the new maxima are finite
    const float mn0 = fmaxf(acc.m[nt][0], mx0), mn1 = fmaxf(acc.m[nt][1], mx1);
    alpha[nt][0] = exp2f(acc.m[nt][0] - mn0);
    alpha[nt][1] = exp2f(acc.m[nt][1] - mn1);
    rescale |= (alpha[nt][0] != 1.f) | (alpha[nt][1] != 1.f);
    acc.m[nt][0] = mn0;
    acc.m[nt][1] = mn1;
    p[nt][0] = exp2f(s0 - mn0);
    p[nt][1] = exp2f(s1 - mn1);
    p[nt][2] = exp2f(s2 - mn0);
    p[nt][3] = exp2f(s3 - mn1);
    acc.l[nt][0] = fmaf(acc.l[nt][0], alpha[nt][0], p[nt][0] + p[nt][2]);
    acc.l[nt][1] = fmaf(acc.l[nt][1], alpha[nt][1], p[nt][1] + p[nt][3]);
  }
  if (__any_sync(kFull, rescale)) {
#pragma unroll
    for (int dt = 0; dt < STEPS; ++dt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        acc.o[dt][nt][0] *= alpha[nt][0];
        acc.o[dt][nt][1] *= alpha[nt][1];
        acc.o[dt][nt][2] *= alpha[nt][0];
        acc.o[dt][nt][3] *= alpha[nt][1];
      }
  }

  // ---- o^T += V^T P^T.  P enters the bf16 product as hi + lo, two bf16
  // parts whose sum carries ~16 significant bits, so a split of a few keys
  // with large, opposite V rows keeps fp32-level accuracy.
  uint32_t pb[NT][2][2];  // [n-tile][hi, lo][keys 0-7, keys 8-15]
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const uint32_t h01 = pack_bf16x2(p[nt][0], p[nt][1]);
    const uint32_t h23 = pack_bf16x2(p[nt][2], p[nt][3]);
    const uint32_t l01 = pack_bf16x2(p[nt][0] - bf16lo_to_f32(h01), p[nt][1] - bf16hi_to_f32(h01));
    const uint32_t l23 = pack_bf16x2(p[nt][2] - bf16lo_to_f32(h23), p[nt][3] - bf16hi_to_f32(h23));
    pb[nt][0][0] = movmatrix_trans(h01);  // keys 0-7  -> B rows k 0-7
    pb[nt][0][1] = movmatrix_trans(h23);  // keys 8-15 -> B rows k 8-15
    pb[nt][1][0] = movmatrix_trans(l01);
    pb[nt][1][1] = movmatrix_trans(l23);
  }
  {
    const int key = (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
    for (int dt = 0; dt < STEPS; ++dt) {
      const int chunk = dt * 2 + ((lane >> 3) & 1);  // 16-byte chunk along d
      const int half = chunk >> 3, cc = chunk & 7;
      uint32_t af[4];
      ldsm_x4_trans(vbase + half * kBoxBytes + key * 128 + ((cc ^ (key & 7)) << 4), af);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        mma_bf16_16816(acc.o[dt][nt], af, pb[nt][0][0], pb[nt][0][1]);
        mma_bf16_16816(acc.o[dt][nt], af, pb[nt][1][0], pb[nt][1][1]);
      }
    }
  }
}

// Folds one more key into a warp's online-softmax state: the token being
// appended, read from global memory (d bf16 values of k and of v for this kv
// head) rather than from a stage.  Register-only.
template <int D, int NT>
__device__ __forceinline__ void tc_extra_key(WarpAcc<D, NT>& acc, const uint32_t (&qf)[NT][D / 16][2],
                                             const __nv_bfloat16* kn, const __nv_bfloat16* vn,
                                             float scale_log2, int lane) {
  constexpr int STEPS = D / 16;
  const uint32_t* kw = reinterpret_cast<const uint32_t*>(kn);
  float s_own[NT];  // logit of head 8 nt + lane/4 (the B-fragment head of this lane)
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float part = 0.f;
#pragma unroll
    for (int ks = 0; ks < STEPS; ++ks) {
      const uint32_t k0 = __ldg(kw + ks * 8 + (lane & 3));
      const uint32_t k1 = __ldg(kw + ks * 8 + 4 + (lane & 3));
      part = fmaf(bf16lo_to_f32(qf[nt][ks][0]), bf16lo_to_f32(k0), part);
      part = fmaf(bf16hi_to_f32(qf[nt][ks][0]), bf16hi_to_f32(k0), part);
      part = fmaf(bf16lo_to_f32(qf[nt][ks][1]), bf16lo_to_f32(k1), part);
      part = fmaf(bf16hi_to_f32(qf[nt][ks][1]), bf16hi_to_f32(k1), part);
    }
    part += __shfl_xor_sync(kFull, part, 1);
    part += __shfl_xor_sync(kFull, part, 2);
    s_own[nt] = part * scale_log2;
  }
  float alpha[NT][2], p[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      // this lane's accumulator column is head 8 nt + 2 (lane%4) + j
      const float s = __shfl_sync(kFull, s_own[nt], 4 * (2 * (lane & 3) + j));
      const float mn = fmaxf(acc.m[nt][j], s);
      alpha[nt][j] = exp2f(acc.m[nt][j] - mn);
      p[nt][j] = exp2f(s - mn);
      acc.m[nt][j] = mn;
      // the 8 lanes of a column each hold part of l: count the new weight once
      acc.l[nt][j] = acc.l[nt][j] * alpha[nt][j] + ((lane >> 2) == 0 ? p[nt][j] : 0.f);
    }
#pragma unroll
  for (int dt = 0; dt < STEPS; ++dt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int d = dt * 16 + (lane >> 2) + ((e >> 1) << 3);
      const float v = __bfloat162float(vn[d]);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        acc.o[dt][nt][e] = fmaf(acc.o[dt][nt][e], alpha[nt][e & 1], p[nt][e & 1] * v);
    }
}

// Stores the appended token's k and v rows (d bf16 each) into the cache row
// `dst_row` of kv head g.  Whole warp.
template <int D>
__device__ __forceinline__ void store_new_row(const DecodeArgs& a, const __nv_bfloat16* kn,
                                              const __nv_bfloat16* vn, long long dst_row, int g,
                                              int lane) {
  constexpr int CH = D / 8;  // 16-byte chunks per row
  const size_t base = ((size_t)dst_row * a.h_kv + g) * D;
  if (lane < 2 * CH && in_bounds(dst_row, (long long)a.B * a.cap, kSiteAppend)) {
    const bool isv = lane >= CH;
    const int c = isv ? lane - CH : lane;
    const uint4 val = __ldg(reinterpret_cast<const uint4*>(isv ? vn : kn) + c);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(const_cast<void*>(isv ? a.v : a.k)) + base) + c;
    *dst = val;
  }
}

// Zeroes V rows [0, n) of a stage.  In a padded cache the rows before a
// sequence's first key are the previous sequence's unused tail and may hold
// anything; masking their weights to 0 would still leave 0 * NaN in P V.
template <int D>
__device__ __forceinline__ void zero_v_rows(uint32_t vbase, int n, int lane) {
  constexpr int CH = (D / 64) * 8;  // 16-byte chunks per row, both d halves
  for (int c = lane; c < n * CH; c += 32) {
    const int r = c / CH, rem = c % CH;
    const uint32_t addr = vbase + (rem >> 3) * kBoxBytes + r * 128 + (rem & 7) * 16;
    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0) : "memory");
  }
  __syncwarp();
}

// Issues the TMA loads of one stage: both d halves of K then of V for the
// 16 rows starting at packed row `row` of kv head g.
template <int D>
__device__ __forceinline__ void tc_issue_stage(uint32_t dst, uint32_t bar, const CUtensorMap* kmap,
                                               const CUtensorMap* vmap, int g, int row,
                                               uint64_t policy) {
  constexpr int HALVES = TcShape<D>::kHalves;
  mbar_arrive_expect_tx(bar, TcShape<D>::kStageBytes);
#pragma unroll
  for (int h = 0; h < HALVES; ++h) tma_load_3d(dst + h * kBoxBytes, kmap, h * 64, g, row, bar, policy);
#pragma unroll
  for (int h = 0; h < HALVES; ++h)
    tma_load_3d(dst + (HALVES + h) * kBoxBytes, vmap, h * 64, g, row, bar, policy);
}

template <int D>
__device__ __forceinline__ void tc_prefetch_stage(const CUtensorMap* kmap, const CUtensorMap* vmap,
                                                  int g, int row) {
#pragma unroll
  for (int h = 0; h < TcShape<D>::kHalves; ++h) tma_prefetch_3d(kmap, h * 64, g, row);
#pragma unroll
  for (int h = 0; h < TcShape<D>::kHalves; ++h) tma_prefetch_3d(vmap, h * 64, g, row);
}

// 1024-byte-aligned start of the dynamic shared memory (128-byte swizzle
// atoms repeat every 1024 bytes).
__device__ __forceinline__ uint8_t* aligned_dyn_smem(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) &
                                    ~static_cast<uintptr_t>(1023));
}

// One CTA per (split, kv head g, head block, b) writes that split's triplet;
// fused, the CTA that finishes a (b, g, head block) last merges its splits.
template <int D, int NT, int NW, int NS, int MODE>
__global__ void __launch_bounds__(NW * 32)
    decode_tc_bf16(const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const DecodeArgs a) {
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(NT == 1 || NT == 2, "heads per CTA: 8 or 16");
  constexpr int HB = NT * 8;
  constexpr int KT = kTileKeys;
  constexpr int HALVES = TcShape<D>::kHalves;
  constexpr int STAGE = TcShape<D>::kStageBytes;
  constexpr int STEPS = TcShape<D>::kSteps;
  static_assert(HB * D * 4 <= NS * STAGE, "per-warp o staging must fit in the warp's stages");

  extern __shared__ uint8_t dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[NW * NS];
  __shared__ float sm_m[NW * HB], sm_l[NW * HB];
  __shared__ int sm_flag;

  uint8_t* stages = aligned_dyn_smem(dyn_smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = blockIdx.x, b = blockIdx.z;
  const int g = blockIdx.y / a.n_hb, hb = blockIdx.y % a.n_hb;

  if (threadIdx.x == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
#pragma unroll
    for (int i = 0; i < NW * NS; ++i) mbar_init(smem_u32(&full_bar[i]), 1);
    fence_barrier_init();
  }
  if (a.hint_tiles > 0 &&
      blockIdx.x + gridDim.x * (blockIdx.y + (long long)gridDim.y * blockIdx.z) < a.hint_ctas) {
    // While the previous grid drains: L2 prefetch of this warp's first tiles,
    // at rows from lengths read before the wait (possibly stale, so every
    // box is checked against the cache's rows; the split is located again
    // after the wait).
    const Split h = locate_split<true>(a, b, slot, lane, false);
    if (lane == 0 && slot < h.n_active)
      for (int s = 0; s < a.hint_tiles; ++s) {
        const int ts = h.lo + (warp + s * NW) * KT;
        if (ts >= h.cached_hi) break;
        const long long row = h.off + ((ts + KT <= h.cached_hi) ? ts : h.cached_hi - KT);
        if (row >= 0 && row + KT <= a.kv_rows) tc_prefetch_stage<D>(&kmap, &vmap, g, (int)row);
      }
  }
  grid_dependency_wait();
  allow_dependent_launch();
  __syncthreads();

  const Split sp = locate_split(a, b, slot, lane,
                                warp == 0 && lane == 0 && slot == 0 && blockIdx.y == 0);
  if (slot >= sp.n_active) {
    if (MODE == kPartial) emit_empty_triplet<HB, D>(a, b, g, hb, slot);
    return;
  }

  const int len = sp.cached_hi > sp.lo ? sp.cached_hi - sp.lo : 0;  // keys read from the cache
  const int ntiles = (len + KT - 1) / KT;
  const uint64_t policy = l2_policy_evict_first();
  const uint32_t stage0 = smem_u32(stages) + warp * NS * STAGE;
  const uint32_t bar0 = smem_u32(&full_bar[warp * NS]);

  // First row (relative to the sequence) that tile t loads.
  auto tile_row0 = [&](int t) {
    const int ts = sp.lo + t * KT;
    return (ts + KT <= sp.cached_hi) ? ts : sp.cached_hi - KT;
  };
  auto issue = [&](int t, int s) {
    tc_issue_stage<D>(stage0 + s * STAGE, bar0 + s * 8, &kmap, &vmap, g,
                      static_cast<int>(sp.off + tile_row0(t)), policy);
  };

  // q is requested before any K/V tile, so it is not queued behind the
  // grid's first burst of TMA traffic.
  uint32_t qf[NT][STEPS][2];
  load_q_frags<D, NT>(qf, a, b, g, hb, lane);
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      const int t = warp + s * NW;
      if (t < ntiles) issue(t, s);
    }
  }
  __syncwarp();
  WarpAcc<D, NT> acc;
  acc.reset();

  int it = 0;
  bool failed = false;
  for (int t = warp; t < ntiles; t += NW, ++it) {
    const int s = it % NS;
    const uint32_t parity = (it / NS) & 1;
    const bool ok = mbar_wait_bounded(bar0 + s * 8, parity, a.timeout_ns);
    if (!__all_sync(kFull, ok)) {
      failed = true;
      break;
    }
    const uint32_t kbase = stage0 + s * STAGE;
    const int ts = sp.lo + t * KT;
    const int row0 = tile_row0(t);
    if (a.cap > 0 && row0 < 0) zero_v_rows<D>(kbase + HALVES * kBoxBytes, -row0, lane);
    tc_tile<D, NT>(acc, qf, kbase, kbase + HALVES * kBoxBytes, row0 + (lane >> 2) >= ts,
                   row0 + (lane >> 2) + 8 >= ts, a.scale_log2, lane);
    __syncwarp();
    // refill this stage with the warp's tile NS steps ahead
    const int tn = t + NS * NW;
    if (lane == 0 && tn < ntiles) {
      fence_proxy_async_smem();
      issue(tn, s);
    }
  }

  if (failed) {
    // Record the error, then let every load this warp issued land (bounded)
    // before the CTA reuses or releases its shared memory.
    if (lane == 0) raise_status(kStatusTimeout);
    const int my_tiles = (ntiles > warp) ? (ntiles - warp + NW - 1) / NW : 0;
    const int last = min(it + NS, my_tiles);
    for (int i = it; i < last; ++i) mbar_wait_bounded(bar0 + (i % NS) * 8, (i / NS) & 1, a.timeout_ns);
    acc.reset();
  }
  if (sp.has_new && warp == ntiles % NW &&  // the appended token, after the cached keys
      in_bounds((long long)b * a.h_kv + g, (long long)a.B * a.h_kv, kSiteAppend)) {
    const size_t nr = ((size_t)b * a.h_kv + g) * D;
    const __nv_bfloat16* kn = static_cast<const __nv_bfloat16*>(a.k_new) + nr;
    const __nv_bfloat16* vn = static_cast<const __nv_bfloat16*>(a.v_new) + nr;
    tc_extra_key<D, NT>(acc, qf, kn, vn, a.scale_log2, lane);
    if (hb == 0) store_new_row<D>(a, kn, vn, sp.off + sp.cached_hi, g, lane);
  }
  acc.reduce_l();

  __syncthreads();  // every warp is done with its stages: reuse them for o
  float* sm_o = reinterpret_cast<float*>(stages);
  if (lane < 4) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        sm_m[warp * HB + nt * 8 + 2 * lane + j] = acc.m[nt][j];
        sm_l[warp * HB + nt * 8 + 2 * lane + j] = acc.l[nt][j];
      }
  }
#pragma unroll
  for (int dt = 0; dt < STEPS; ++dt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int d = dt * 16 + (lane >> 2) + ((e >> 1) << 3);
        const int head = nt * 8 + 2 * (lane & 3) + (e & 1);
        sm_o[(warp * HB + head) * D + d] = acc.o[dt][nt][e];
      }
  __syncthreads();
  emit_split_triplet<NW, HB, D>(sm_m, sm_l, sm_o, a, b, g, hb, slot);
  if (MODE == kFused) fused_finish<NW, HB, D>(a, b, g, hb, sp.n_active, &sm_flag);
}

}  // namespace gqa
