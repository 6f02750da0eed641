// Fused bf16 decode attention with an even, persistent split of the work.
//
// Every kv head (head block) gy sees the same sequence of 16-key tiles: the
// tiles of every unit (b, split), in that order, T1 tiles in all.  The grid
// holds exactly the CTAs that fit on the GPU at once.  Its warps are laid out
// head-minor: warp w serves head gy = w % H and takes run k = w / H of that
// head's tiles, [k*T1/Wk, (k+1)*T1/Wk), so every warp streams the same number
// of bytes, no second wave starts cold, and the warps that share k (the four
// warps of a CTA, and their neighbours) read the same cache rows of
// different kv heads together -- a cache row holds every kv head's keys side
// by side, so that keeps DRAM pages open.  A warp keeps its TMA ring running
// across unit boundaries and emits one partial triplet (a "piece",
// kernbench "_attention_mesh_mlo.py": "One-shot local partial attention" over
// the keys it saw) for each unit it touches; a piece never spans two splits,
// so the user's split structure is preserved.  The pieces of a group (b, gy)
// are merged with the page's log-sum-exp rule by the warp that completes the
// group's last tile (a per-group counter of finished tiles, incremented once
// per piece; nothing waits on another warp), which also normalises and
// writes out.
//
// Piece storage: within head gy, piece (u, k) exists iff run k meets unit u;
// ordered by tile position each next piece increments u, k or both, so
// u + k is unique in [0, U1 + Wk) (U1 = non-empty units per head) and piece
// (gy, u, k) lives at slot gy * (U1 + Wk) + u + k.
#pragma once

#include "decode_tc.cuh"

namespace gqa {

// Split geometry of one sequence (16-key tiles).
struct SeqGeom {
  int S;      // length (negative lengths read as 0)
  int L;      // split length
  int n_act;  // non-empty splits (0 when S == 0)
  int tps;    // tiles of a full split
  int tlast;  // tiles of the last non-empty split
  int Tg;     // tiles per (b, gy): (n_act - 1) * tps + tlast
};

__device__ __forceinline__ SeqGeom seq_geom(const DecodeArgs& a, int S) {
  SeqGeom q;
  q.S = S > 0 ? S : 0;
  if (q.S == 0) {
    q.L = 1;
    q.n_act = q.tps = q.tlast = q.Tg = 0;
    return q;
  }
  const long long L =
      a.n_splits > 0 ? ((long long)q.S + a.n_splits - 1) / a.n_splits : (long long)a.chunk_len;
  long long n = ((long long)q.S + L - 1) / L;
  if (n > a.n_slots) n = a.n_slots;  // chunked mode, S above max_seqlen: tail ignored
  long long last = (long long)q.S - (n - 1) * L;
  if (last > L) last = L;
  q.L = (int)L;
  q.n_act = (int)n;
  q.tps = (int)((L + kTileKeys - 1) / kTileKeys);
  q.tlast = (int)((last + kTileKeys - 1) / kTileKeys);
  q.Tg = (q.n_act - 1) * q.tps + q.tlast;
  return q;
}

__device__ __forceinline__ int tiles_in(const SeqGeom& q, int slot) {
  return slot == q.n_act - 1 ? q.tlast : q.tps;
}

// Position of a warp in its head's tile sequence (identical in every lane).
struct Cursor {
  int b, slot, tile;
  long long off;  // packed row of sequence b's first key
  long long F;    // per-head tile index of (b, split 0, tile 0)
  long long U;    // per-head unit index of (b, split 0)
  SeqGeom q;
};

__device__ __forceinline__ long long scan_incl(long long v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long x = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += x;
  }
  return v;
}

// Cursor at per-head tile t0 (0 <= t0 < T1).  Whole warp.
__device__ Cursor locate_tile(const DecodeArgs& a, long long t0, int lane) {
  long long F = 0, U = 0, off = 0;
  for (int base = 0; base < a.B; base += 32) {
    const int b = base + lane;
    const int S = b < a.B ? __ldg(a.seqlens + b) : 0;
    const SeqGeom q = seq_geom(a, S);
    const long long tiles = q.Tg, units = q.n_act, rows = q.S;
    const long long ti = scan_incl(tiles, lane), ui = scan_incl(units, lane), ri = scan_incl(rows, lane);
    const unsigned hit = __ballot_sync(kFull, F + ti > t0);
    if (hit) {
      const int j = __ffs(hit) - 1;
      Cursor c;
      c.b = base + j;
      c.F = F + __shfl_sync(kFull, ti - tiles, j);
      c.U = U + __shfl_sync(kFull, ui - units, j);
      c.off = off + __shfl_sync(kFull, ri - rows, j);
      c.q = seq_geom(a, __shfl_sync(kFull, S, j));
      const int r = (int)(t0 - c.F);
      int slot = r / c.q.tps;
      if (slot > c.q.n_act - 1) slot = c.q.n_act - 1;
      c.slot = slot;
      c.tile = r - slot * c.q.tps;
      return c;
    }
    F += __shfl_sync(kFull, ti, 31);
    U += __shfl_sync(kFull, ui, 31);
    off += __shfl_sync(kFull, ri, 31);
  }
  Cursor none{};  // not reached for t0 < T1
  return none;
}

// Moves the cursor to the next tile; the caller guarantees one exists.
__device__ __forceinline__ void advance(Cursor& c, const DecodeArgs& a) {
  if (++c.tile < tiles_in(c.q, c.slot)) return;
  c.tile = 0;
  if (++c.slot < c.q.n_act) return;
  c.slot = 0;
  c.F += c.q.Tg;
  c.U += c.q.n_act;
  c.off += c.q.S;
  for (;;) {  // skip empty sequences (they add no rows, tiles or units)
    ++c.b;
    c.q = seq_geom(a, __ldg(a.seqlens + c.b));
    if (c.q.Tg > 0) break;
  }
}

// Rows of the tile under the cursor, relative to its sequence: the first
// new key ts, and the first loaded row row0 (= ts, or shifted back so the
// 16 loaded rows end at the split's end).
__device__ __forceinline__ void tile_rows(const Cursor& c, int& ts, int& row0) {
  const long long lo = (long long)c.slot * c.q.L;
  long long hi = lo + c.q.L;
  if (hi > c.q.S) hi = c.q.S;
  const long long t = lo + (long long)c.tile * kTileKeys;
  ts = (int)t;
  row0 = (int)((t + kTileKeys <= hi) ? t : hi - kTileKeys);
}

// Warp that owns tile t: the largest w with floor(w*T/Wv) <= t.
__device__ __forceinline__ long long owner_of(long long t, long long T, long long Wv) {
  return ((t + 1) * Wv - 1) / T;
}

struct PieceStore {
  float* m;   // [slots][HBs], base 2
  float* l;   // [slots][HBs]
  float* o;   // [slots][HBs][D]
  int HBs;    // heads stored per piece = min(HB, G)
};

// Merges every piece of group (b, gy) in split and run order, normalises,
// and writes the group's rows of out.  Whole warp.
template <int D, int NT>
__device__ __noinline__ void merge_group(const DecodeArgs& a, const PieceStore ps, int b, int gy,
                                         SeqGeom q, long long Fb, long long Ub, long long T1,
                                         long long Wk, long long U1, int lane) {
  constexpr int HB = NT * 8;
  constexpr int PER = D / 32;  // contiguous elements of d per lane
  const int g = gy / a.n_hb, hb = gy % a.n_hb;
  const long long Fg = Fb;
  const long long Ug = (long long)gy * (U1 + Wk) + Ub;
  const long long T = T1, Wv = Wk;
  const int HBs = ps.HBs;

  float M[HB];
#pragma unroll
  for (int h = 0; h < HB; ++h) M[h] = -INFINITY;
  for (int s0 = 0; s0 < q.n_act; s0 += 32) {
    const int slot = s0 + lane;
    if (slot < q.n_act) {
      const long long Fu = Fg + (long long)slot * q.tps;
      const long long w0 = owner_of(Fu, T, Wv), w1 = owner_of(Fu + tiles_in(q, slot) - 1, T, Wv);
      for (long long w = w0; w <= w1; ++w) {
        const long long P = Ug + slot + w;
#pragma unroll
        for (int h = 0; h < HB; ++h)
          if (h < HBs) M[h] = fmaxf(M[h], __ldcg(ps.m + P * HBs + h));
      }
    }
  }
#pragma unroll
  for (int h = 0; h < HB; ++h) M[h] = warp_max(M[h]);

  float acc[HB][PER], Lh[HB];
#pragma unroll
  for (int h = 0; h < HB; ++h) {
    Lh[h] = 0.f;
#pragma unroll
    for (int k = 0; k < PER; ++k) acc[h][k] = 0.f;
  }
  for (int s0 = 0; s0 < q.n_act; s0 += 32) {
    const int slot = s0 + lane;
    long long w0 = 0, cnt = 0;
    if (slot < q.n_act) {
      const long long Fu = Fg + (long long)slot * q.tps;
      w0 = owner_of(Fu, T, Wv);
      cnt = owner_of(Fu + tiles_in(q, slot) - 1, T, Wv) - w0 + 1;
    }
    const int nj = min(32, q.n_act - s0);
    for (int j = 0; j < nj; ++j) {
      const long long P0 = Ug + s0 + j + __shfl_sync(kFull, w0, j);
      const int n = (int)__shfl_sync(kFull, cnt, j);
      for (int p = 0; p < n; ++p) {
        const long long P = P0 + p;
#pragma unroll
        for (int h = 0; h < HB; ++h) {
          if (h < HBs) {
            const float wgt = exp2f(__ldcg(ps.m + P * HBs + h) - M[h]);
            Lh[h] = fmaf(__ldcg(ps.l + P * HBs + h), wgt, Lh[h]);
            const float* src = ps.o + (P * HBs + h) * D + lane * PER;
            if constexpr (PER == 4) {
              const float4 v = __ldcg(reinterpret_cast<const float4*>(src));
              acc[h][0] = fmaf(v.x, wgt, acc[h][0]);
              acc[h][1] = fmaf(v.y, wgt, acc[h][1]);
              acc[h][2] = fmaf(v.z, wgt, acc[h][2]);
              acc[h][3] = fmaf(v.w, wgt, acc[h][3]);
            } else {
              const float2 v = __ldcg(reinterpret_cast<const float2*>(src));
              acc[h][0] = fmaf(v.x, wgt, acc[h][0]);
              acc[h][1] = fmaf(v.y, wgt, acc[h][1]);
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int h = 0; h < HB; ++h) {
    const int gi = hb * HB + h;
    if (h < HBs && gi < a.G) {
      float* dst = a.out + query_row(a, b, g, gi) * D + lane * PER;
#pragma unroll
      for (int k = 0; k < PER; ++k) dst[k] = Lh[h] > 0.f ? acc[h][k] / Lh[h] : 0.f;
    }
  }
}

template <int D, int NT, int NW, int NS>
__global__ void __launch_bounds__(NW * 32)
    decode_tc_bf16_streamk(const __grid_constant__ CUtensorMap kmap,
                           const __grid_constant__ CUtensorMap vmap, const DecodeArgs a,
                           const PieceStore ps) {
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(NT == 1 || NT == 2, "heads per CTA: 8 or 16");
  constexpr int STAGE = TcShape<D>::kStageBytes;
  constexpr int STEPS = TcShape<D>::kSteps;
  constexpr int HALVES = TcShape<D>::kHalves;

  extern __shared__ uint8_t dyn_smem[];
  __shared__ __align__(8) uint64_t full_bar[NW * NS];
  uint8_t* stages = aligned_dyn_smem(dyn_smem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long W = (long long)gridDim.x * NW;
  const long long wid = (long long)blockIdx.x * NW + warp;
  const int H = a.h_kv * a.n_hb;

  if (threadIdx.x == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
#pragma unroll
    for (int i = 0; i < NW * NS; ++i) mbar_init(smem_u32(&full_bar[i]), 1);
    fence_barrier_init();
  }
  __syncthreads();  // the only CTA-wide barrier: warps run independently from here

  // Per-head tiles T1 and units U1; rows of empty sequences are written
  // (zeros) by warp b % W.
  long long T1 = 0, U1 = 0;
  for (int base = 0; base < a.B; base += 32) {
    const int b = base + lane;
    const int S = b < a.B ? __ldg(a.seqlens + b) : 0;
    if (wid == 0 && S < 0) raise_status(kStatusNegSeqlen);
    const SeqGeom q = seq_geom(a, S);
    if (wid == 0 && b < a.B && a.chunk_len > 0 &&
        (long long)q.S > (long long)a.n_slots * a.chunk_len)
      raise_status(kStatusSeqlenOverMax);
    T1 += __shfl_sync(kFull, scan_incl(q.Tg, lane), 31);
    U1 += __shfl_sync(kFull, scan_incl(q.n_act, lane), 31);
    unsigned empty = __ballot_sync(kFull, b < a.B && q.S == 0 && (b % W) == wid);
    while (empty) {
      const int j = __ffs(empty) - 1;
      empty &= empty - 1;
      float* dst = a.out + (size_t)(base + j) * a.h_q * D;
      for (int i = lane; i < a.h_q * D; i += 32) dst[i] = 0.f;
    }
  }
  if (T1 == 0) return;
  long long Wg = W / H;
  if (Wg < 1) Wg = 1;
  const long long Wk = T1 < Wg ? T1 : Wg;  // runs per head

  const uint64_t policy = l2_policy_evict_first();
  const uint32_t stage0 = smem_u32(stages) + warp * NS * STAGE;
  const uint32_t bar0 = smem_u32(&full_bar[warp * NS]);
  uint32_t phase_base = 0;  // uses of this warp's stages so far (for mbarrier parity)

  // Virtual warps vw = wid, wid + W, ... (more than one only when H > W).
  for (long long vw = wid; vw < Wg * H; vw += W) {
    const int gy = (int)(vw % H);
    const long long k = vw / H;
    if (k >= Wk) continue;
    const long long t0 = k * T1 / Wk, t1 = (k + 1) * T1 / Wk;
    const int g = gy / a.n_hb, hb = gy % a.n_hb;

    Cursor cc = locate_tile(a, t0, lane);  // tile being computed
    Cursor ic = cc;                        // next tile to load
    auto issue = [&](const Cursor& c, int s) {
      int ts, row0;
      tile_rows(c, ts, row0);
      tc_issue_stage<D>(stage0 + s * STAGE, bar0 + s * 8, &kmap, &vmap, g,
                        static_cast<int>(c.off + row0), policy);
    };
    const long long n_pro = (t1 - t0) < NS ? (t1 - t0) : NS;
    for (int i = 0; i < n_pro; ++i) {
      if (lane == 0) issue(ic, (int)((phase_base + i) % NS));
      if (t0 + i + 1 < t1) advance(ic, a);
    }
    __syncwarp();

    uint32_t qf[NT][STEPS][2];
    load_q_frags<D, NT>(qf, a, cc.b, g, hb, lane);
    WarpAcc<D, NT> acc;
    acc.reset();
    int piece_tiles = 0;

    for (long long t = t0; t < t1; ++t) {
      const uint32_t use = phase_base + (uint32_t)(t - t0);
      const int s = (int)(use % NS);
      const uint32_t parity = (use / NS) & 1;
      const bool ok = mbar_wait_bounded(bar0 + s * 8, parity, a.timeout_ns);
      if (!__all_sync(kFull, ok)) {
        // Record the error, let this warp's issued loads land (bounded), stop.
        if (lane == 0) raise_status(kStatusTimeout);
        const uint32_t end = phase_base + (uint32_t)(t1 - t0);
        const uint32_t last = (use + NS < end) ? use + NS : end;
        for (uint32_t i = use; i < last; ++i)
          mbar_wait_bounded(bar0 + (i % NS) * 8, (i / NS) & 1, a.timeout_ns);
        return;
      }
      int ts, row0;
      tile_rows(cc, ts, row0);
      const uint32_t kbase = stage0 + s * STAGE;
      tc_tile<D, NT>(acc, qf, kbase, kbase + HALVES * kBoxBytes, row0 + (lane >> 2) >= ts,
                     row0 + (lane >> 2) + 8 >= ts, a.scale_log2, lane);
      ++piece_tiles;
      __syncwarp();
      // refill this stage with the tile NS ahead
      if (t + NS < t1) {
        if (lane == 0) {
          fence_proxy_async_smem();
          issue(ic, s);
        }
        if (t + NS + 1 < t1) advance(ic, a);
      }

      const bool range_end = (t + 1 == t1);
      if (range_end || cc.tile + 1 == tiles_in(cc.q, cc.slot)) {
        // ---- this warp's piece of unit (b, gy, slot) is complete
        acc.reduce_l();
        const long long P = (long long)gy * (U1 + Wk) + cc.U + cc.slot + k;
        const int HBs = ps.HBs;
        if (lane < 4) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int h = nt * 8 + 2 * lane + j;
              if (h < HBs) {
                ps.m[P * HBs + h] = acc.m[nt][j];
                ps.l[P * HBs + h] = acc.l[nt][j];
              }
            }
        }
#pragma unroll
        for (int dt = 0; dt < STEPS; ++dt)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int h = nt * 8 + 2 * (lane & 3) + (e & 1);
              const int d = dt * 16 + (lane >> 2) + ((e >> 1) << 3);
              if (h < HBs) ps.o[(P * HBs + h) * D + d] = acc.o[dt][nt][e];
            }
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) {
          int* ticket = a.tickets + (size_t)cc.b * H + gy;
          const int prev = atomicAdd(ticket, piece_tiles);
          last = (prev + piece_tiles == cc.q.Tg);
          if (last) atomicExch(ticket, 0);
        }
        last = __shfl_sync(kFull, last, 0);
        if (last) {
          __threadfence();
          merge_group<D, NT>(a, ps, cc.b, gy, cc.q, cc.F, cc.U, T1, Wk, U1, lane);
        }
        acc.reset();
        piece_tiles = 0;
      }
      if (!range_end) {
        const int b_prev = cc.b;
        advance(cc, a);
        if (cc.b != b_prev) load_q_frags<D, NT>(qf, a, cc.b, g, hb, lane);
      }
    }
    phase_base += (uint32_t)(t1 - t0);
  }
}

}  // namespace gqa
