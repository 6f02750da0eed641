// bf16 decode over persistent CTAs: the fused call (then a merge kernel over
// all rows) and, for grids of a few waves, the partial call.
//
// The per-split grid runs one CTA per (split, kv head, head block, b); when
// there are more splits than resident CTAs the second wave starts cold and
// every wave pays its start-up and drain with the memory system idle.  Here
// the grid is C CTAs that all fit at once -- as few as take the units in the
// same number of rounds, so every CTA gets the same number of units (to
// one) -- and CTA c takes the
// non-empty splits ("units") c, c + C, c + 2C, ... in the per-split grid's
// order (split fastest, then kv head / head block, then b), so CTAs that run
// together still read neighbouring cache rows.  Each warp keeps one TMA ring
// across its CTA's units: while the warps of a CTA reduce one split, the
// first tiles of their next split are already in flight.
//
// Per unit, the warps' partial triplets are combined pairwise through an
// 8 KiB exchange buffer (named barriers), and warp 0 stores the split's
// triplet (kernbench "_attention_mesh_mlo.py": "One-shot local partial
// attention").  merge_rows_kernel then merges each row's non-empty splits
// with the page's log-sum-exp rule and normalises ("Final normalize").
#pragma once

#include "decode_tc.cuh"

namespace gqa {

// Geometry of one unit (non-empty split of one (b, kv head / head block)).
struct Unit {
  int b, gy, slot;
  int lo, hi;      // keys [lo, hi) of the split, relative to the sequence
  int cached_hi;   // min(hi, cached keys): the split's keys read from the cache
  bool has_new;    // the split holds the appended token (key number cached_hi)
  int ntiles;      // 16-key tiles of [lo, cached_hi)
  long long off;   // cache row of the sequence's first key
};

// Non-empty splits of a sequence attending S keys: ceil(S / L), clipped to
// n_slots (0 when S == 0).  L as in locate_split.  32-bit: S < 2^31 and the
// host keeps every unit and cache-row count below 2^31.
__device__ __forceinline__ int active_splits(const DecodeArgs& a, int S, int& L) {
  if (S <= 0) {
    L = 1;
    return 0;
  }
  L = a.n_splits > 0 ? (int)(((unsigned)S + a.n_splits - 1) / (unsigned)a.n_splits) : a.chunk_len;
  const int n = (int)(((unsigned)S + L - 1) / (unsigned)L);
  return n < a.n_slots ? n : a.n_slots;
}

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += x;
  }
  return v;
}

// One pass over the sequences (whole warp): the number of units, and -- when
// u < that number -- unit u itself.  A unit is a non-empty split of one
// (b, kv head / head block); units are numbered b-major, then kv head / head
// block, then split.
template <bool HINT = false>
__device__ Unit scan_units(const DecodeArgs& a, int H, int u, int lane, int* total) {
  int units = 0, rows = 0;
  Unit x{};
  bool found = false;
  for (int base = 0; base < a.B; base += 32) {
    const int b = base + lane;
    const SeqKeys kk = seq_keys(a, b < a.B ? load_seqlen<HINT>(a.seqlens + b) : 0);
    int L;
    const int n = b < a.B ? active_splits(a, kk.total, L) : 0;
    const int cu = H * n, cr = kk.cached;
    const int iu = warp_incl_scan(cu, lane), ir = warp_incl_scan(cr, lane);
    const unsigned hit = found ? 0u : __ballot_sync(kFull, units + iu > u);
    if (hit) {
      const int j = __ffs(hit) - 1;
      found = true;
      x.b = base + j;
      const int r = u - (units + __shfl_sync(kFull, iu - cu, j));
      x.off = a.cap > 0 ? (long long)x.b * a.cap : (long long)rows + __shfl_sync(kFull, ir - cr, j);
      const int St = __shfl_sync(kFull, kk.total, j), Sc = __shfl_sync(kFull, kk.cached, j);
      const bool app = __shfl_sync(kFull, (int)kk.append, j) != 0;
      const int nj = __shfl_sync(kFull, n, j), Lj = __shfl_sync(kFull, L, j);
      x.gy = r / nj;
      x.slot = r - x.gy * nj;
      const int lo = x.slot * Lj;
      const int hi = (St - lo < Lj) ? St : lo + Lj;
      x.lo = lo;
      x.hi = hi;
      x.cached_hi = hi < Sc ? hi : Sc;
      x.has_new = app && lo <= Sc && Sc < hi;
      const int len = x.cached_hi > x.lo ? x.cached_hi - x.lo : 0;
      x.ntiles = (len + kTileKeys - 1) / kTileKeys;
      if (!total) return x;
    }
    units += __shfl_sync(kFull, iu, 31);
    rows += __shfl_sync(kFull, ir, 31);
  }
  if (total) *total = units;
  return x;
}

// Unit u, 0 <= u < the number of units (whole warp).
__device__ __forceinline__ Unit unit_at(const DecodeArgs& a, int H, long long u, int lane) {
  return scan_units(a, H, (int)u, lane, nullptr);
}

__device__ __forceinline__ void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// A warp's partial triplet in the exchange buffer: m and l per head column,
// then the o fragments stored element-major ([i][lane]) so every store and
// load of a warp touches 32 consecutive words.
template <int D, int NT>
struct XSlot {
  static constexpr int kFrag = (D / 16) * NT * 4;  // o floats per lane
  static constexpr int kFloats = 2 * NT * 8 + kFrag * 32;
};

template <int D, int NT>
__device__ __forceinline__ void xslot_store(float* x, const WarpAcc<D, NT>& acc, int lane) {
  if (lane < 4) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        x[nt * 8 + 2 * lane + j] = acc.m[nt][j];
        x[NT * 8 + nt * 8 + 2 * lane + j] = acc.l[nt][j];
      }
  }
  float* xo = x + 2 * NT * 8;
  int i = 0;
#pragma unroll
  for (int dt = 0; dt < D / 16; ++dt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e, ++i) xo[i * 32 + lane] = acc.o[dt][nt][e];
}

// acc <- merge(acc, partial in x) with the log-sum-exp rule (base-2 m).
template <int D, int NT>
__device__ __forceinline__ void xslot_merge(WarpAcc<D, NT>& acc, const float* x, int lane) {
  float sa[NT][2], sb[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int h = nt * 8 + 2 * (lane & 3) + j;
      const float mb = x[h], lb = x[NT * 8 + h];
      const float M = fmaxf(acc.m[nt][j], mb);
      sa[nt][j] = M == -INFINITY ? 0.f : exp2f(acc.m[nt][j] - M);
      sb[nt][j] = M == -INFINITY ? 0.f : exp2f(mb - M);
      acc.l[nt][j] = acc.l[nt][j] * sa[nt][j] + lb * sb[nt][j];
      acc.m[nt][j] = M;
    }
  const float* xo = x + 2 * NT * 8;
  int i = 0;
#pragma unroll
  for (int dt = 0; dt < D / 16; ++dt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e, ++i)
        acc.o[dt][nt][e] = acc.o[dt][nt][e] * sa[nt][e & 1] + xo[i * 32 + lane] * sb[nt][e & 1];
}

template <int D, int NT, int NW, int NS>
constexpr int persist_dynamic_smem() {
  return NW * NS * TcShape<D>::kStageBytes + 2 * XSlot<D, NT>::kFloats * 4 + 1024;
}

// PARTIAL: the call returns every split slot (gqa_decode_partial), so after
// its units each CTA also writes the empty triplets (-inf, 0, 0) of the
// slots past a sequence's non-empty splits, for a share of the (b, kv head /
// head block) pairs.
template <int D, int NT, int NW, int NS, bool PARTIAL>
__global__ void __launch_bounds__(NW * 32)
    decode_tc_bf16_persist(const __grid_constant__ CUtensorMap kmap,
                           const __grid_constant__ CUtensorMap vmap, const DecodeArgs a) {
  static_assert(NW == 4, "the pairwise exchange assumes four warps");
  constexpr int HB = NT * 8;
  constexpr int STAGE = TcShape<D>::kStageBytes;
  constexpr int STEPS = TcShape<D>::kSteps;
  constexpr int HALVES = TcShape<D>::kHalves;
  constexpr int XF = XSlot<D, NT>::kFloats;

  extern __shared__ uint8_t dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[NW * NS];
  uint8_t* stages = aligned_dyn_smem(dyn_smem);
  float* xbuf = reinterpret_cast<float*>(stages + NW * NS * STAGE);  // 2 slots of XF floats

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = a.h_kv * a.n_hb;

  if (threadIdx.x == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
#pragma unroll
    for (int i = 0; i < NW * NS; ++i) mbar_init(smem_u32(&full_bar[i]), 1);
    fence_barrier_init();
  }
  if (a.hint_tiles > 0 && blockIdx.x < a.hint_ctas) {
    // While the previous grid drains: L2 prefetch of this warp's first tiles
    // of the CTA's first unit, at rows from lengths read before the wait
    // (possibly stale, so every box is checked against the cache's rows; the
    // units are scanned again after the wait).
    const Unit h = scan_units<true>(a, H, blockIdx.x, lane, nullptr);
    if (lane == 0)
      for (int s = 0; s < a.hint_tiles; ++s) {
        const int t = warp + s * NW;
        if (t >= h.ntiles) break;
        const int ts = h.lo + t * kTileKeys;
        const long long row =
            h.off + ((ts + kTileKeys <= h.cached_hi) ? ts : h.cached_hi - kTileKeys);
        if (row >= 0 && row + kTileKeys <= a.kv_rows)
          tc_prefetch_stage<D>(&kmap, &vmap, h.gy / a.n_hb, (int)row);
      }
  }
  grid_dependency_wait();
  allow_dependent_launch();
  __syncthreads();

  if (blockIdx.x == 0 && threadIdx.x < 32) {  // report bad lengths once
    long long rows = 0;
    for (int b = lane; b < a.B; b += 32) {
      const int S = __ldg(a.seqlens + b);
      report_length(a, S, true);
      if (a.chunk_len > 0 && (long long)seq_keys(a, S).total > (long long)a.n_slots * a.chunk_len)
        raise_status(kStatusSeqlenOverMax);
      rows += S > 0 ? S : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rows += __shfl_xor_sync(kFull, rows, o);
    if (lane == 0 && a.cap == 0 && a.kv_rows >= 0 && rows > a.kv_rows)  // cache rows past the cache
      raise_status(kStatusSeqlenOverMax);
  }

  int A32 = 0;
  const Unit first = scan_units(a, H, blockIdx.x, lane, &A32);  // count + first unit, one pass
  const long long A = A32;
  const uint64_t policy = l2_policy_evict_first();
  const uint32_t stage0 = smem_u32(stages) + warp * NS * STAGE;
  const uint32_t bar0 = smem_u32(&full_bar[warp * NS]);


  // ---- issue cursor: the next tile of this warp's sequence (warp-uniform)
  long long ia = blockIdx.x;
  Unit iu{};
  int it = warp;
  bool more = false;
  if (ia < A) {
    iu = first;
    more = true;
    while (more && it >= iu.ntiles) {  // no tile of this unit for this warp
      ia += gridDim.x;
      if (ia >= A) {
        more = false;
      } else {
        iu = unit_at(a, H, ia, lane);
        it = warp;
      }
    }
  }
  uint32_t issued = 0, used = 0;
  auto issue_next = [&]() {
    if (lane == 0) {
      const int ts = iu.lo + it * kTileKeys;
      const int row0 = (ts + kTileKeys <= iu.cached_hi) ? ts : iu.cached_hi - kTileKeys;
      tc_issue_stage<D>(stage0 + (issued % NS) * STAGE, bar0 + (issued % NS) * 8, &kmap, &vmap,
                        iu.gy / a.n_hb, static_cast<int>(iu.off + row0), policy);
    }
    ++issued;
    it += NW;
    while (it >= iu.ntiles) {
      ia += gridDim.x;
      if (ia >= A) {
        more = false;
        break;
      }
      iu = unit_at(a, H, ia, lane);
      it = warp;
    }
  };
  for (int s = 0; s < NS && more; ++s) issue_next();
  __syncwarp();

  // q of the first unit (an L2 hit) is requested after the first K/V tiles,
  // whose DRAM latency it then overlaps.
  uint32_t qf[NT][STEPS][2];
  int q_b = -1, q_gy = -1;
  if (blockIdx.x < A) {
    load_q_frags<D, NT>(qf, a, first.b, first.gy / a.n_hb, first.gy % a.n_hb, lane);
    q_b = first.b;
    q_gy = first.gy;
  }

  WarpAcc<D, NT> acc;
  bool failed = false;

  for (long long u = blockIdx.x; u < A; u += gridDim.x) {
    const Unit cu = u == blockIdx.x ? first : unit_at(a, H, u, lane);
    const int g = cu.gy / a.n_hb, hb = cu.gy % a.n_hb;
    if (cu.b != q_b || cu.gy != q_gy) {
      load_q_frags<D, NT>(qf, a, cu.b, g, hb, lane);
      q_b = cu.b;
      q_gy = cu.gy;
    }
    acc.reset();
    for (int t = warp; t < cu.ntiles && !failed; t += NW) {
      const int s = used % NS;
      const bool ok = mbar_wait_bounded(bar0 + s * 8, (used / NS) & 1, a.timeout_ns);
      if (!__all_sync(kFull, ok)) {
        failed = true;
        break;
      }
      const int ts = cu.lo + t * kTileKeys;
      const int row0 = (ts + kTileKeys <= cu.cached_hi) ? ts : cu.cached_hi - kTileKeys;
      const uint32_t kbase = stage0 + s * STAGE;
      if (a.cap > 0 && row0 < 0) zero_v_rows<D>(kbase + HALVES * kBoxBytes, -row0, lane);
      tc_tile<D, NT>(acc, qf, kbase, kbase + HALVES * kBoxBytes, row0 + (lane >> 2) >= ts,
                     row0 + (lane >> 2) + 8 >= ts, a.scale_log2, lane);
      ++used;
      __syncwarp();
      if (more) {
        if (lane == 0) fence_proxy_async_smem();
        issue_next();
      }
    }
    if (failed) {
      // Record the error, let this warp's issued loads land (bounded); the
      // warp's partials read as empty from here on.
      if (lane == 0) raise_status(kStatusTimeout);
      for (uint32_t i = used; i < issued; ++i)
        mbar_wait_bounded(bar0 + (i % NS) * 8, (i / NS) & 1, a.timeout_ns);
      used = issued;
      more = false;
      acc.reset();
    }
    if (cu.has_new && warp == cu.ntiles % NW &&  // the appended token, after the cached keys
        in_bounds((long long)cu.b * a.h_kv + g, (long long)a.B * a.h_kv, kSiteAppend)) {
      const size_t nr = ((size_t)cu.b * a.h_kv + g) * D;
      const __nv_bfloat16* kn = static_cast<const __nv_bfloat16*>(a.k_new) + nr;
      const __nv_bfloat16* vn = static_cast<const __nv_bfloat16*>(a.v_new) + nr;
      tc_extra_key<D, NT>(acc, qf, kn, vn, a.scale_log2, lane);
      if (hb == 0) store_new_row<D>(a, kn, vn, cu.off + cu.cached_hi, g, lane);
    }
    acc.reduce_l();

    // ---- combine the four warps' partials: (2,3) -> (0,1), then 1 -> 0
    named_barrier(1, NW * 32);  // every warp done with this unit and with xbuf
    if (warp >= 2) xslot_store<D, NT>(xbuf + (warp - 2) * XF, acc, lane);
    named_barrier(1, NW * 32);
    if (warp < 2) {
      xslot_merge<D, NT>(acc, xbuf + warp * XF, lane);
      named_barrier(2, 64);
      if (warp == 1) xslot_store<D, NT>(xbuf, acc, lane);
      named_barrier(3, 64);
      if (warp == 0) {
        xslot_merge<D, NT>(acc, xbuf, lane);
        // ---- store the split's triplet (m in natural-log units)
        const bool row_ok = in_bounds(   // the block's last head row: its highest slot index
            (long long)(query_row(a, cu.b, g, min(hb * HB + HB - 1, a.G - 1)) * a.n_slots + cu.slot),
            (long long)a.B * a.h_q * a.n_slots, kSiteTriplet);
        if (row_ok && lane < 4) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int gi = hb * HB + nt * 8 + 2 * lane + j;
              if (gi < a.G) {
                const size_t r = query_row(a, cu.b, g, gi) * a.n_slots + cu.slot;
                a.m[r] = acc.m[nt][j] == -INFINITY ? -INFINITY : acc.m[nt][j] * kLn2;
                a.l[r] = acc.l[nt][j];
              }
            }
        }
#pragma unroll
        for (int dt = 0; dt < STEPS; ++dt)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int gi = hb * HB + nt * 8 + 2 * (lane & 3) + (e & 1);
              if (row_ok && gi < a.G) {
                const int d = dt * 16 + (lane >> 2) + ((e >> 1) << 3);
                a.o[(query_row(a, cu.b, g, gi) * a.n_slots + cu.slot) * D + d] = acc.o[dt][nt][e];
              }
            }
      }
    }
  }

  if (PARTIAL) {
    const long long pairs = (long long)a.B * H;
    for (long long p = blockIdx.x; p < pairs; p += gridDim.x) {
      const int b = (int)(p / H), gy = (int)(p % H);
      int L;
      const int n = active_splits(a, seq_keys(a, __ldg(a.seqlens + b)).total, L);
      for (int slot = n; slot < a.n_slots; ++slot)
        emit_empty_triplet<HB, D>(a, b, gy / a.n_hb, gy % a.n_hb, slot);
    }
  }
}

// Merge of every row's non-empty splits (fused path): one warp per row;
// a row of an empty sequence is 0.  The row's first triplets are requested
// together with its sequence length (every slot of the workspace row may be
// read; only the n active ones are used).
template <int MAXK>
__global__ void __launch_bounds__(128) merge_rows_kernel(const DecodeArgs a, int D) {
  grid_dependency_wait();
  allow_dependent_launch();
  const long long row = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
  if (row >= (long long)a.B * a.h_q) return;
  const int b = (int)(row / a.h_q);
  const int S = __ldg(a.seqlens + b);
  const int lane = threadIdx.x & 31;
  const float *m = a.m + row * a.n_slots, *l = a.l + row * a.n_slots, *o = a.o + row * a.n_slots * D;
  RowMerge<MAXK> r;
  r.prefetch(m, l, o, a.n_slots, D, lane, ContiguousSplits());
  int L;
  const int n = active_splits(a, seq_keys(a, S).total, L);
  float* out = a.out + row * D;
  if (n == 0) {
    for (int d = lane; d < D; d += 32) out[d] = 0.f;
    return;
  }
  r.finish(m, l, o, n, D, out, lane, ContiguousSplits());
}

}  // namespace gqa
