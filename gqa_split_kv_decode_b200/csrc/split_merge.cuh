// Split assignment, triplet emission and the log-sum-exp merge shared by the
// decode kernels and mlo_merge.
//
// Method (kernbench "_attention_mesh_mlo.py", attention_mesh_mlo_kernel): each
// shard of the sequence yields a triplet (m, l, o) -- the maximum logit, the
// softmax denominator relative to it and the unnormalised weighted sum of V
// ("One-shot local partial attention"); triplets combine with
// m_c = max(m, m'), l = l e^{m-m_c} + l' e^{m'-m_c}, o = o e^{m-m_c} +
// o' e^{m'-m_c}, and the answer is o / l ("Final normalize").  Merging all n
// triplets against their common maximum M is the same rule applied n - 1
// times, written in one pass.
#pragma once

#include "device_common.cuh"

namespace gqa {

// Everything a decode kernel needs besides the tensor maps.
struct DecodeArgs {
  const void* q;            // [B][h_q][D]
  const void* k;            // cache: packed [rows][h_kv][D], or [B][cap][h_kv][D]
  const void* v;
  const int32_t* seqlens;   // [B]
  float* m;                 // triplets: m, l [B*h_q][n_slots], o [B*h_q][n_slots][D]
  float* l;
  float* o;
  float* out;               // fused: [B*h_q][D]
  int* tickets;             // fused: one counter per (b, blockIdx.y)
  const void* k_new;        // append: the new token's k and v, [B][h_kv][D]; null otherwise
  const void* v_new;
  long long cap;            // > 0: cache rows per sequence ([B][cap][h_kv][D]); 0: packed
  long long kv_rows;        // rows of the cache; no cache row at or past it is read.  < 0:
                            //   not given (packed calls that do not pass it)
  int hint_tiles;           // > 0: a CTA prefetches its warps' first hint_tiles tiles into L2
                            //   before the dependency wait (needs kv_rows >= 0)
  int hint_ctas;            // only CTAs whose linear index is below it prefetch (first wave)
  int B, h_q, h_kv, G, n_hb;
  int n_splits;             // > 0: split by count
  int chunk_len;            // > 0: split by fixed chunks
  int n_slots;              // triplet slots per row == gridDim.x
  float scale_log2;         // scale * log2(e): logits are kept in base 2
  unsigned long long timeout_ns;
};

enum { kPartial = 0, kFused = 1 };

// Tickets in the workspace's fixed ticket area (256 KiB of int32).
constexpr long long kTicketCount = 65536;

// Keys of one sequence: `cached` rows are read from the cache; `total` keys
// are attended, the new token being key number `cached` when appending and
// the sequence's cache rows have room for it.
struct SeqKeys {
  int cached, total;
  bool append;
};

__device__ __forceinline__ SeqKeys seq_keys(const DecodeArgs& a, int S) {
  SeqKeys k;
  k.cached = S > 0 ? S : 0;
  if (a.cap > 0 && k.cached > a.cap) k.cached = (int)a.cap;
  k.append = a.k_new != nullptr && k.cached < a.cap;
  k.total = k.cached + (k.append ? 1 : 0);
  return k;
}

// Reports (once, by the caller's choice of `report`) lengths the call cannot
// honour: negative, above max_seqlen in chunked mode, above the capacity of a
// padded cache, or with no room left to append.
__device__ __forceinline__ void report_length(const DecodeArgs& a, int S, bool report) {
  if (!report) return;
  if (S < 0) raise_status(kStatusNegSeqlen);
  if (a.cap > 0 && (long long)S + (a.k_new ? 1 : 0) > a.cap) raise_status(kStatusSeqlenOverMax);
}

struct Split {
  long long off;  // cache row of the sequence's first key
  int S;          // keys attended (cached, plus the new token when appending)
  int lo, hi;     // this split's keys [lo, hi), relative to the sequence
  int cached_hi;  // min(hi, cached keys): the split's keys that come from the cache
  bool has_new;   // the split holds the appended token (key number `cached`)
  int n_active;   // splits of this sequence that hold keys (>= 1)
};

// Sequence b's first cache row and the key range of split `slot` (whole
// warp).  Split i covers [i*L, min((i+1)*L, S)) with L = ceil(S / n_splits)
// or L = chunk_len.  n_active = max(1, ceil(S / L)): the number of splits
// the fused merge waits for (split 0 stands in for an empty sequence).
// HINT: lengths read with relaxed loads before the dependency wait, for L2
// prefetch addresses only (the split is located again after the wait).
template <bool HINT = false>
__device__ __forceinline__ int load_seqlen(const int32_t* p) {
  return HINT ? ld_relaxed_s32(p) : __ldg(p);
}

template <bool HINT = false>
__device__ __forceinline__ Split locate_split(const DecodeArgs& a, int b, int slot, int lane,
                                              bool report) {
  long long acc = 0;
  if (a.cap > 0) {
    acc = (long long)b * a.cap;
  } else {
    for (int j = lane; j < b; j += 32) {
      const int s = load_seqlen<HINT>(a.seqlens + j);
      acc += s > 0 ? s : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
  }
  const int Sraw = load_seqlen<HINT>(a.seqlens + b);
  report_length(a, Sraw, report);
  // the sequence's cache rows end past the cache
  if (report && a.cap == 0 && a.kv_rows >= 0 && acc + (Sraw > 0 ? Sraw : 0) > a.kv_rows)
    raise_status(kStatusSeqlenOverMax);
  const SeqKeys kk = seq_keys(a, Sraw);
  const int S = kk.total;
  const long long L =
      a.n_splits > 0 ? ((long long)S + a.n_splits - 1) / a.n_splits : (long long)a.chunk_len;
  int n_active = S > 0 ? (int)(((long long)S + L - 1) / L) : 1;
  if (n_active > a.n_slots) {
    if (report) raise_status(kStatusSeqlenOverMax);
    n_active = a.n_slots;
  }
  long long lo = (long long)slot * L;
  if (lo > S) lo = S;
  long long hi = lo + L;
  if (hi > S) hi = S;
  Split sp;
  sp.off = acc;
  sp.S = S;
  sp.lo = (int)lo;
  sp.hi = (int)hi;
  sp.cached_hi = (int)(hi < kk.cached ? hi : kk.cached);
  sp.has_new = kk.append && lo <= kk.cached && kk.cached < hi;
  sp.n_active = n_active;
  return sp;
}

__device__ __forceinline__ size_t query_row(const DecodeArgs& a, int b, int g, int gi) {
  return (size_t)b * a.h_q + (size_t)g * a.G + gi;
}

// Writes the empty triplet (-inf, 0, 0) of split `slot` for the CTA's heads.
template <int HB, int D>
__device__ void emit_empty_triplet(const DecodeArgs& a, int b, int g, int hb, int slot) {
  for (int idx = threadIdx.x; idx < HB * D; idx += blockDim.x) {
    const int hh = idx / D, dd = idx % D;
    const int gi = hb * HB + hh;
    if (gi >= a.G) continue;
    const size_t row = query_row(a, b, g, gi);
    if (!in_bounds((long long)(row * a.n_slots + slot), (long long)a.B * a.h_q * a.n_slots,
                   kSiteTriplet))
      continue;
    a.o[(row * a.n_slots + slot) * D + dd] = 0.f;
    if (dd == 0) {
      a.m[row * a.n_slots + slot] = -INFINITY;
      a.l[row * a.n_slots + slot] = 0.f;
    }
  }
}

// Combines the NW per-warp triplets held in shared memory (m in base 2:
// sm_m[w*HB+h]; sm_l likewise; sm_o[(w*HB+h)*D + d]) into this CTA's split
// triplet and stores it at slot `slot` (m converted to natural-log units).
template <int NW, int HB, int D>
__device__ void emit_split_triplet(const float* sm_m, const float* sm_l, const float* sm_o,
                                   const DecodeArgs& a, int b, int g, int hb, int slot) {
  for (int idx = threadIdx.x; idx < HB * D; idx += blockDim.x) {
    const int hh = idx / D, dd = idx % D;
    const int gi = hb * HB + hh;
    if (gi >= a.G) continue;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, sm_m[w * HB + hh]);
    float ov = 0.f, lv = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float sc = exp2f(sm_m[w * HB + hh] - M);
        ov = fmaf(sm_o[(w * HB + hh) * D + dd], sc, ov);
        lv = fmaf(sm_l[w * HB + hh], sc, lv);
      }
    }
    const size_t row = query_row(a, b, g, gi);
    if (!in_bounds((long long)(row * a.n_slots + slot), (long long)a.B * a.h_q * a.n_slots,
                   kSiteTriplet))
      continue;
    a.o[(row * a.n_slots + slot) * D + dd] = ov;
    if (dd == 0) {
      a.m[row * a.n_slots + slot] = (M == -INFINITY) ? -INFINITY : M * kLn2;
      a.l[row * a.n_slots + slot] = lv;
    }
  }
}

// Split j of a row is at element j of its m / l rows and at o + j * d ...
struct ContiguousSplits {
  __device__ __forceinline__ size_t ml(int j) const { return (size_t)j; }
  __device__ __forceinline__ size_t o(int j, int d) const { return (size_t)j * d; }
};
// ... or, for triplets gathered from several shards (shard r's block of
// rows x n_inner splits `stride_ml` elements after shard r-1's for m and l,
// `stride_o` for o), split j is split j % n_inner of shard j / n_inner.
struct ShardedSplits {
  int n_inner;
  size_t stride_ml, stride_o;
  __device__ __forceinline__ size_t ml(int j) const {
    return (size_t)(j / n_inner) * stride_ml + (size_t)(j % n_inner);
  }
  __device__ __forceinline__ size_t o(int j, int d) const {
    return (size_t)(j / n_inner) * stride_o + (size_t)(j % n_inner) * d;
  }
};

// Merges the n triplets of one row and normalises: the whole warp
// cooperates, lane j owning elements j, j+32, ... (d <= 32*MAXK).  Splits are
// combined strictly in index order, so every element's result is
// deterministic and identical wherever this runs.  m in natural-log units.
//
// Two halves, so the first loads can leave before n is known: prefetch()
// requests the o rows of the first 8 of `n_pre` slots together with their m
// and l (n_pre >= n: slots in [n, n_pre) are read but never used), finish()
// merges n splits, requesting each later batch of 8 o rows before any of its
// rows is used.  A merge of up to 8 splits costs about one memory round trip.
template <int MAXK, typename SplitIndex = ContiguousSplits>
struct RowMerge {
  static constexpr int BATCH = 8;
  float ov[BATCH][MAXK];
  float mi, li;

  __device__ __forceinline__ void load_batch(const float* o, int j0, int n, int d, int lane,
                                             SplitIndex at) {
#pragma unroll
    for (int u = 0; u < BATCH; ++u) {
      const float* oj = o + at.o(j0 + u < n ? j0 + u : 0, d);
#pragma unroll
      for (int k = 0; k < MAXK; ++k) {
        const int dd = lane + 32 * k;
        ov[u][k] = (j0 + u < n && dd < d) ? __ldcg(oj + dd) : 0.f;
      }
    }
  }

  __device__ __forceinline__ void prefetch(const float* m, const float* l, const float* o,
                                           int n_pre, int d, int lane, SplitIndex at) {
    load_batch(o, 0, n_pre, d, lane, at);
    mi = lane < n_pre ? __ldcg(m + at.ml(lane)) : -INFINITY;
    li = lane < n_pre ? __ldcg(l + at.ml(lane)) : 0.f;
  }

  __device__ __forceinline__ void finish(const float* m, const float* l, const float* o, int n,
                                         int d, float* out, int lane, SplitIndex at) {
    if (lane >= n) {
      mi = -INFINITY;
      li = 0.f;
    }
    float M = mi;
    for (int j = 32 + lane; j < n; j += 32) M = fmaxf(M, __ldcg(m + at.ml(j)));
    M = warp_max(M);

    float acc[MAXK];
#pragma unroll
    for (int k = 0; k < MAXK; ++k) acc[k] = 0.f;
    float L = 0.f;
    if (M != -INFINITY) {
      for (int base = 0; base < n; base += 32) {
        if (base > 0) {
          mi = base + lane < n ? __ldcg(m + at.ml(base + lane)) : -INFINITY;
          li = base + lane < n ? __ldcg(l + at.ml(base + lane)) : 0.f;
        }
        const float wi = exp2f((mi - M) * kLog2e);  // 0 for an empty split
        const int cnt = min(32, n - base);
        for (int j0 = 0; j0 < cnt; j0 += BATCH) {
          if (base + j0 > 0) load_batch(o, base + j0, n, d, lane, at);
#pragma unroll
          for (int u = 0; u < BATCH; ++u) {
            const int j = j0 + u;
            const float wj = __shfl_sync(kFull, wi, j & 31);
            const float lj = __shfl_sync(kFull, li, j & 31);
            if (j < cnt) {
              L = fmaf(lj, wj, L);
#pragma unroll
              for (int k = 0; k < MAXK; ++k) acc[k] = fmaf(ov[u][k], wj, acc[k]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int k = 0; k < MAXK; ++k) {
      const int dd = lane + 32 * k;
      if (dd < d) out[dd] = L > 0.f ? acc[k] / L : 0.f;
    }
  }
};

template <int MAXK, typename SplitIndex = ContiguousSplits>
__device__ __forceinline__ void merge_row_warp(const float* m, const float* l, const float* o,
                                               int n, int d, float* out, int lane,
                                               SplitIndex at = SplitIndex()) {
  RowMerge<MAXK, SplitIndex> r;
  r.prefetch(m, l, o, n, d, lane, at);
  r.finish(m, l, o, n, d, out, lane, at);
}

// Fused finish: after this CTA's triplet is stored, take a ticket for the
// (b, kv head, head block); the CTA that takes the last one merges the
// group's rows over the n_active splits and writes `out`.  Nothing waits on
// another CTA, so there is no inter-CTA spin.  The last CTA also resets the
// ticket to 0 for the next call.
//
// Ordering: the barrier puts every thread's triplet stores before thread 0's
// ticket; the ticket is a gpu-scope acq_rel atomic, so it releases them
// (cumulatively) to the CTA that takes the last ticket, and that CTA's
// acquire, passed on to its other threads by the second barrier, makes every
// released triplet visible to the merge's L2 loads.  The reset needs no
// ordering within the call: no CTA of this call takes the ticket after the
// last one, and the next call reads it only after this grid has ended.
template <int NW, int HB, int D>
__device__ void fused_finish(const DecodeArgs& a, int b, int g, int hb, int n_active,
                             int* sm_flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    const long long ti = (long long)b * gridDim.y + blockIdx.y;
    int last = 0;
    if (in_bounds(ti, kTicketCount, kSiteTicket)) {
      int* t = a.tickets + ti;
      const int prev = atom_add_acq_rel_gpu(t, 1);
      last = (prev == n_active - 1);
      if (last) *t = 0;
    }
    *sm_flag = last;
  }
  __syncthreads();
  if (!*sm_flag) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int hh = warp; hh < HB; hh += NW) {
    const int gi = hb * HB + hh;
    if (gi >= a.G) break;
    const size_t row = query_row(a, b, g, gi);
    if (!in_bounds((long long)row, (long long)a.B * a.h_q, kSiteMergeRow)) break;
    merge_row_warp<D / 32>(a.m + row * a.n_slots, a.l + row * a.n_slots,
                           a.o + row * a.n_slots * D, n_active, D, a.out + row * D, lane);
  }
}

// Stand-alone merge: one warp per row.
template <int MAXK>
__global__ void __launch_bounds__(128) mlo_merge_kernel(const float* __restrict__ m,
                                                        const float* __restrict__ l,
                                                        const float* __restrict__ o,
                                                        float* __restrict__ out, int rows, int n,
                                                        int d) {
  grid_dependency_wait();
  allow_dependent_launch();
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (row >= rows) return;
  merge_row_warp<MAXK>(m + (size_t)row * n, l + (size_t)row * n, o + (size_t)row * n * d, n, d,
                       out + (size_t)row * d, threadIdx.x & 31);
}

// Merge of triplets gathered from n_ranks shards: rank r's m / l block
// [rows][n_splits] starts r * stride_ml elements in, its o block
// [rows][n_splits][d] r * stride_o elements in; a row's splits are taken in
// rank-major order.  One warp per row.
template <int MAXK>
__global__ void __launch_bounds__(128) mlo_merge_ranked_kernel(
    const float* __restrict__ m, const float* __restrict__ l, const float* __restrict__ o,
    float* __restrict__ out, int rows, int n_ranks, int n_splits, int d, size_t stride_ml,
    size_t stride_o) {
  grid_dependency_wait();
  allow_dependent_launch();
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const ShardedSplits at{n_splits, stride_ml, stride_o};
  merge_row_warp<MAXK>(m + (size_t)row * n_splits, l + (size_t)row * n_splits,
                       o + (size_t)row * n_splits * d, n_ranks * n_splits, d, out + (size_t)row * d,
                       threadIdx.x & 31, at);
}

}  // namespace gqa
