// Causal prefill attention (S_q = T > 1) on the fifth-generation tensor
// cores: the compute-bound counterpart of decode, the "flash-attention style"
// SDPA of the tt-metal "[Llama2] Perf burndown" page (Prefill 2k list), whose
// arithmetic intensity grows with T (scaling-book "All About Transformer
// Inference", the prefill discussion).
//
// Query i of sequence b attends keys 0..i of the same sequence:
//   O_i = sum_{j<=i} e^{s_ij - m_i} v_j / sum_{j<=i} e^{s_ij - m_i},
//   s_ij = scale <q_i, k_j>,  query head h reading kv head h / (h_q / h_kv).
//
// One CTA = 128 query rows of one head of one sequence; two CTAs share an
// SM, so one's tensor-core work fills the other's softmax time.  Six warps:
//   warps 0-3  softmax: thread r owns row r (TMEM lane r) -- reads S from
//              TMEM, keeps the row's reference max and denominator, writes P
//              back into TMEM over the S it came from, rescales O when the
//              max moves, and finally normalises O and stores it;
//   warp 4     TMA producer: Q once, then 64-key K and V tiles through
//              two-stage rings;
//   warp 5     MMA issuer (one thread): S_j = Q K_j^T from shared memory
//              into one of two TMEM S buffers, then O += P_j V_j with P read
//              from TMEM.
// TMEM (256 columns, fp32, lane = query row): S0 [0,64), S1 [64,128),
// O [128,256).  P_j replaces S_j in place: keys 32c..32c+31 of the tile
// (S columns [32c, 32c+32)) become their bf16 hi parts in columns
// [32c, 32c+16) and lo parts (p - hi, rounded) in [32c+16, 32c+32); S_{j+2}
// is issued right after PV_j, which reads them (one CTA's MMAs run in order).
//
// Precision: the P V product normally takes the hi parts only (one bf16 P).
// A (128-row, 64-key) block also adds the lo parts -- so its P is exact to
// ~2^-17 -- whenever some row's tile mass exceeds a third of that row's
// running denominator; that covers every short row and every tile that
// carries a row's dominant keys, where a single bf16 rounding of the
// weights would show in the output.
#pragma once

#include "device_common.cuh"
#include "tcgen05.cuh"

namespace gqa {

constexpr int kPfRows = 128;                   // query rows per CTA (MMA M)
constexpr int kPfKeys = 64;                    // keys per K/V tile
constexpr int kPfD = 128;                      // head dim
constexpr int kPfThreads = 192;
constexpr int kPfQHalf = kPfRows * 128;        // 64 dims x 128 rows: 16 KiB
constexpr int kPfKvHalf = kPfKeys * 128;       // 64 dims x 64 keys: 8 KiB
constexpr int kPfQBytes = 2 * kPfQHalf;        // 32 KiB
constexpr int kPfKvBytes = 2 * kPfKvHalf;      // 16 KiB
// Shared memory: Q, K[2], V[2], 1024-byte aligned.
constexpr int kPfSmemQ = 0;
constexpr int kPfSmemK = kPfSmemQ + kPfQBytes;
constexpr int kPfSmemV = kPfSmemK + 2 * kPfKvBytes;
constexpr int kPfSmemBytes = kPfSmemV + 2 * kPfKvBytes;   // 96 KiB
constexpr int kPfDynSmem = kPfSmemBytes + 1024;          // + alignment slack
constexpr uint32_t kPfTmemCols = 256;
constexpr uint32_t kPfColO = 128;
constexpr int kPfStageStride = kPfD * 4 + 16;          // output staging row, padded
static_assert(kPfRows * kPfStageStride <= kPfSmemBytes, "output staging must fit");
constexpr float kPfRescaleLog2 = 8.f;   // lazy rescale: keep the max unless it grew by > 2^8
constexpr float kPfLoShare = 1.f / 3;  // a tile above this share of a row's mass takes lo parts

struct PrefillArgs {
  const int32_t* seqlens;   // [B] device
  float* out;               // [total_rows][h_q][128] fp32
  long long total_rows;     // rows of the packed q / k / v (sum of S_b)
  int B, h_q, h_kv, G;      // G = h_q / h_kv
  int n_qtiles;             // ceil(max_seqlen / 128): the grid's tile extent
  float scale_log2;         // scale * log2(e)
  unsigned long long timeout_ns;
};

// Barriers and flags of one CTA (shared memory).
struct PfBars {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2];
  uint64_t v_full[2], v_empty[2];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t drain;
  int lo_tile[2];           // j + 1 when tile j's block needs the lo parts
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ uint32_t bar_addr(uint64_t& b) { return smem_u32(&b); }

// Bounded wait shared by every role: false (and the CTA's abort flag set,
// the timeout recorded) when the wait ran out or another role gave up.
__device__ __forceinline__ bool pf_wait(PfBars& sb, uint64_t& bar, uint32_t parity,
                                        unsigned long long timeout_ns) {
  if (*reinterpret_cast<volatile int*>(&sb.abort)) return false;
  if (mbar_wait_bounded(bar_addr(bar), parity, timeout_ns)) return true;
  *reinterpret_cast<volatile int*>(&sb.abort) = 1;
  raise_status(kStatusTimeout);
  return false;
}

// Warp-uniform version for the softmax warps (their TMEM accesses are
// warp-collective, so every lane must take the same branch).
__device__ __forceinline__ bool pf_wait_warp(PfBars& sb, uint64_t& bar, uint32_t parity,
                                             unsigned long long timeout_ns) {
  const bool ok = pf_wait(sb, bar, parity, timeout_ns);
  return __all_sync(kFull, ok);
}

// Loads a rows x 128-dim bf16 tile as two 64-dim boxes (128-byte swizzle):
// dims [0,64) at dst, [64,128) at dst + half_bytes.
__device__ __forceinline__ void pf_load_tile(uint32_t dst, uint32_t half_bytes,
                                             const CUtensorMap* map, int head, long long row,
                                             uint32_t bar, uint64_t policy) {
  mbar_arrive_expect_tx(bar, 2 * half_bytes);
  tma_load_3d(dst, map, 0, head, (int)row, bar, policy);
  tma_load_3d(dst + half_bytes, map, 64, head, (int)row, bar, policy);
}

// Warp 4, one thread: Q, then K_j / V_j for j = 0 .. nt-1 through the rings.
// Stage s = j & 1 is refilled once the MMA that read its previous tile
// (S_{j-2} for K, PV_{j-2} for V) has completed.  At the end it waits for
// every copy it issued, so none lands after the CTA has gone.
__device__ __forceinline__ void pf_producer(PfBars& sb, uint32_t smem, const CUtensorMap* qmap,
                                            const CUtensorMap* kmap, const CUtensorMap* vmap,
                                            int h, int g, long long qrow, long long krow0, int nt,
                                            unsigned long long tmo) {
  const uint64_t pol_q = l2_policy_evict_first();
  const uint64_t pol_kv = l2_policy_evict_last();
  pf_load_tile(smem + kPfSmemQ, kPfQHalf, qmap, h, qrow, bar_addr(sb.q_full), pol_q);
  int issued = 0;
  for (int j = 0; j < nt; ++j) {
    const int s = j & 1;
    const uint32_t par = ((j >> 1) - 1) & 1;
    const long long row = krow0 + (long long)j * kPfKeys;
    if (j >= 2 && !pf_wait(sb, sb.k_empty[s], par, tmo)) break;
    pf_load_tile(smem + kPfSmemK + s * kPfKvBytes, kPfKvHalf, kmap, g, row,
                 bar_addr(sb.k_full[s]), pol_kv);
    if (j >= 2 && !pf_wait(sb, sb.v_empty[s], par, tmo)) {
      issued = 2 * j + 1;
      break;
    }
    pf_load_tile(smem + kPfSmemV + s * kPfKvBytes, kPfKvHalf, vmap, g, row,
                 bar_addr(sb.v_full[s]), pol_kv);
    issued = 2 * j + 2;
  }
  // Drain: the last K and V load of each stage (earlier ones are implied,
  // since a stage is refilled only after its previous load was consumed).
  if (!mbar_wait_bounded(bar_addr(sb.q_full), 0, tmo)) raise_status(kStatusTimeout);
  for (int n = issued - 1; n >= 0 && n >= issued - 4; --n) {
    const int j = n >> 1;
    uint64_t& bar = (n & 1) ? sb.v_full[j & 1] : sb.k_full[j & 1];
    if (!mbar_wait_bounded(bar_addr(bar), (j >> 1) & 1, tmo)) raise_status(kStatusTimeout);
  }
}

// S_j = Q K_j^T (M = 128 rows, N = 64 keys, K = 128 dims): eight K = 16
// steps, both operands K-major, each step 32 bytes further along the
// swizzled 128-byte rows, dims 64..127 in each tile's second half.
__device__ __forceinline__ void pf_issue_qk(uint32_t smem, uint32_t tmem, int j) {
  constexpr uint32_t idesc = umma_idesc_bf16_f32(kPfRows, kPfKeys, false);
  const SDesc qa = umma_sdesc_sw128_split(smem + kPfSmemQ, 16, 1024);
  const SDesc kb = umma_sdesc_sw128_split(smem + kPfSmemK + (j & 1) * kPfKvBytes, 16, 1024);
  const uint32_t d = tmem + (j & 1) * kPfKeys;
#pragma unroll
  for (int k = 0; k < kPfD / 16; ++k)
    umma_bf16_ss_step(d, qa, ((k >> 2) * kPfQHalf + (k & 3) * 32) >> 4, kb,
                      ((k >> 2) * kPfKvHalf + (k & 3) * 32) >> 4, idesc, k > 0);
}

// O (+)= P V_j (M = 128 rows, N = 128 dims, K = 64 keys): P from TMEM (the
// hi or lo columns of each 32-key chunk), V MN-major (its dims contiguous):
// 16 keys = two 8-row swizzle groups = 2 KiB per step, the two 64-dim halves
// 8 KiB apart.
__device__ __forceinline__ void pf_issue_pv(uint32_t tmem, int j, uint32_t vb, bool lo,
                                            bool overwrite) {
  constexpr uint32_t idesc = umma_idesc_bf16_f32(kPfRows, kPfD, true);
  const uint32_t p = tmem + (j & 1) * kPfKeys + (lo ? 16 : 0);
  const SDesc v = umma_sdesc_sw128_split(vb, kPfKvHalf, 1024);
#pragma unroll
  for (int k = 0; k < kPfKeys / 16; ++k)
    umma_bf16_ts_step(tmem + kPfColO, p + (k >> 1) * 32 + (k & 1) * 8, v, (k * 2048) >> 4, idesc,
                      (overwrite && k == 0) ? 0u : 1u);
}

// Warp 5, one thread.  S_0 and S_1 first; then, polling without blocking,
// S_k as soon as PV_{k-2}, which reads P_{k-2} from the same TMEM buffer, is
// issued (and K_k is in), and PV_j as soon as P_j and V_j are ready (with
// the lo parts when the softmax asked for them).  S goes first when both
// are ready: the softmax waits for it.  No progress for the wait limit
// aborts the CTA.
__device__ __forceinline__ void pf_mma(PfBars& sb, uint32_t smem, uint32_t tmem, int nt,
                                       unsigned long long tmo) {
  if (pf_wait(sb, sb.q_full, 0, tmo)) {
    tc_fence_after_sync();
    bool ok = true;
    for (int j = 0; j < 2 && j < nt && ok; ++j) {
      ok = pf_wait(sb, sb.k_full[j], 0, tmo);
      if (!ok) break;
      tc_fence_after_sync();
      pf_issue_qk(smem, tmem, j);
      umma_commit(bar_addr(sb.s_full[j]));
      umma_commit(bar_addr(sb.k_empty[j]));
    }
    int next_s = 2, next_pv = 0;
    uint64_t t_progress = globaltimer_ns();
    uint32_t idle = 0;
    while (ok && next_pv < nt) {
      bool progress = false;
      // S_k overwrites the TMEM columns of P_{k-2}: it goes in once PV_{k-2}
      // is issued, since the tensor core executes one CTA's MMAs in issue
      // order (PV_{k-2} has read P before S_k writes).
      if (next_s < nt && next_s - 2 < next_pv) {
        const int k = next_s, s = k & 1;
        if (mbar_test_wait(bar_addr(sb.k_full[s]), (k >> 1) & 1)) {
          tc_fence_after_sync();
          pf_issue_qk(smem, tmem, k);
          umma_commit(bar_addr(sb.s_full[s]));
          umma_commit(bar_addr(sb.k_empty[s]));
          ++next_s;
          progress = true;
        }
      }
      {
        const int j = next_pv, s = j & 1;
        const uint32_t par = (j >> 1) & 1;
        if (mbar_test_wait(bar_addr(sb.p_full[s]), par) &&
            mbar_test_wait(bar_addr(sb.v_full[s]), par)) {
          tc_fence_after_sync();
          const uint32_t vb = smem + kPfSmemV + s * kPfKvBytes;
          pf_issue_pv(tmem, j, vb, false, j == 0);
          if (*reinterpret_cast<volatile int*>(&sb.lo_tile[s]) == j + 1)
            pf_issue_pv(tmem, j, vb, true, false);
          umma_commit(bar_addr(sb.pv_done[s]));
          umma_commit(bar_addr(sb.v_empty[s]));
          ++next_pv;
          progress = true;
        }
      }
      if (progress) {
        idle = 0;
      } else if ((++idle & 255u) == 0 &&   // the clock is read now and then only
                 (*reinterpret_cast<volatile int*>(&sb.abort) ||
                  (idle == 256 ? (t_progress = globaltimer_ns(), false)
                               : globaltimer_ns() - t_progress > tmo))) {
        if (!*reinterpret_cast<volatile int*>(&sb.abort)) {
          *reinterpret_cast<volatile int*>(&sb.abort) = 1;
          raise_status(kStatusTimeout);
        }
        ok = false;
      }
    }
  }
  // Nothing issued may still run when TMEM is freed.
  umma_commit(bar_addr(sb.drain));
  if (!mbar_wait_bounded(bar_addr(sb.drain), 0, tmo)) raise_status(kStatusTimeout);
}

// Multiplies this thread's O row (TMEM) by f, 32 columns at a time.
__device__ __forceinline__ void pf_rescale_o(uint32_t trow, float f) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t o[32];
    tmem_ld32(trow + kPfColO + c * 32, o);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
    tmem_st32(trow + kPfColO + c * 32, o);
  }
  tmem_wait_st();
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Max (MIN: min) of the 64 logits, keys c > lim excluded when MASKED: eight
// independent 3-input chains, then a small tree, so the latency is short.
template <bool MASKED, bool MIN>
__device__ __forceinline__ float pf_tile_reduce(const float (&x)[kPfKeys], int lim) {
  constexpr float kFill = MIN ? INFINITY : -INFINITY;
  float m[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) m[u] = kFill;
#pragma unroll
  for (int c = 0; c < kPfKeys; c += 16) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c0 = c + 2 * u, c1 = c0 + 1;
      const float a0 = (!MASKED || c0 <= lim) ? x[c0] : kFill;
      const float a1 = (!MASKED || c1 <= lim) ? x[c1] : kFill;
      m[u] = MIN ? fmin3(m[u], a0, a1) : fmax3(m[u], a0, a1);
    }
  }
  if (MIN)
    return fminf(fmin3(fmin3(m[0], m[1], m[2]), fmin3(m[3], m[4], m[5]), m[6]), m[7]);
  return fmaxf(fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]), m[6]), m[7]);
}

// Row max (or min, for a negative scale) of the 64 logits.
template <bool MASKED>
__device__ __forceinline__ float pf_tile_extreme(const float (&x)[kPfKeys], int lim, float sl2) {
  return sl2 >= 0.f ? pf_tile_reduce<MASKED, false>(x, lim) : pf_tile_reduce<MASKED, true>(x, lim);
}

// Packed two-lane fp32 arithmetic of sm_100 (one instruction for a pair).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// x <- P = 2^(x * sl2 - m) in place (0 for keys c > lim when MASKED);
// returns the row's tile mass T.  Exponent arguments and sums go two keys
// per instruction.
template <bool MASKED>
__device__ __forceinline__ float pf_tile_exp(float (&x)[kPfKeys], int lim, float sl2, float neg) {
  const float2 s2 = make_float2(sl2, sl2), n2 = make_float2(neg, neg);
  float2 ts[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int c = 0; c < kPfKeys; c += 2) {
    const float2 arg = ffma2(make_float2(x[c], x[c + 1]), s2, n2);
    x[c] = (!MASKED || c <= lim) ? ex2_approx(arg.x) : 0.f;
    x[c + 1] = (!MASKED || c + 1 <= lim) ? ex2_approx(arg.y) : 0.f;
    ts[(c >> 1) & 1] = fadd2(ts[(c >> 1) & 1], make_float2(x[c], x[c + 1]));
  }
  return (ts[0].x + ts[0].y) + (ts[1].x + ts[1].y);
}

// Warps 0-3: thread r owns query row r of the tile (TMEM lane r).  Per K/V
// tile j: read S_j, mask (key c of the tile is causal while
// c <= r + 128 t - 64 j; only the two tiles that straddle the diagonal
// need it), update the row's reference max m (base 2, kept unless the
// tile's max exceeds it by more than 2^8: then O and the denominator are
// rescaled), write P = 2^(s * scale * log2e - m) into TMEM as bf16 hi
// parts, and -- in warps where some row's tile mass exceeds a third of its
// running mass, which then also flag the block for the lo MMA -- the lo
// parts p - hi (zeros elsewhere), and accumulate the fp32 denominator.
// Finally O / l is stored for the rows that exist.
__device__ __forceinline__ void pf_softmax(PfBars& sb, uint32_t smem, uint32_t tmem, int warp,
                                           int lane, int t,
                                           int nt, const PrefillArgs& a, long long out_row0,
                                           int rows_valid, int h, unsigned long long tmo) {
  const int r = warp * 32 + lane;
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
  const float sl2 = a.scale_log2;
  float m_used = -INFINITY, l = 0.f;
  bool ok = true;
  for (int j = 0; j < nt; ++j) {
    const int s = j & 1;
    if (!(ok = pf_wait_warp(sb, sb.s_full[s], (j >> 1) & 1, tmo))) break;
    tc_fence_after_sync();
    const uint32_t sbuf = trow + s * kPfKeys;
    float x[kPfKeys];
    {
      uint32_t v[2][32];
      tmem_ld32(sbuf, v[0]);
      tmem_ld32(sbuf + 32, v[1]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < kPfKeys; ++c) x[c] = __uint_as_float(v[c >> 5][c & 31]);
    }
    const bool masked = j >= 2 * t;                  // warp-uniform
    const int lim = r + kPfRows * t - kPfKeys * j;   // keys c <= lim are causal
    const float ext = masked ? pf_tile_extreme<true>(x, lim, sl2)
                             : pf_tile_extreme<false>(x, lim, sl2);
    const float mt = sl2 != 0.f ? ext * sl2 : 0.f;
    const float m_new = fmaxf(m_used, mt);
    const bool resc = m_new > m_used + kPfRescaleLog2;   // always true on the first tile
    float factor = 1.f;
    if (resc) {
      factor = ex2_approx(m_used - m_new);                 // 0 on the first tile
      l *= factor;
      m_used = m_new;
    }
    // O may be rescaled once PV_{j-1} has completed.
    if (j >= 1 && __any_sync(kFull, resc)) {
      if (!(ok = pf_wait_warp(sb, sb.pv_done[s ^ 1], ((j - 1) >> 1) & 1, tmo))) break;
      tc_fence_after_sync();
      pf_rescale_o(trow, factor);
    }

    const float T = masked ? pf_tile_exp<true>(x, lim, sl2, -m_used)
                           : pf_tile_exp<false>(x, lim, sl2, -m_used);
    const bool need_lo = T > kPfLoShare * (l + T);
    l += T;
    const bool warp_lo = __any_sync(kFull, need_lo);
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint32_t hi[16], lo[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) hi[e] = pack_bf16x2(x[c * 32 + 2 * e], x[c * 32 + 2 * e + 1]);
      tmem_st16(sbuf + c * 32, hi);
      if (warp_lo) {
#pragma unroll
        for (int e = 0; e < 16; ++e)
          lo[e] = pack_bf16x2(x[c * 32 + 2 * e] - bf16lo_to_f32(hi[e]),
                              x[c * 32 + 2 * e + 1] - bf16hi_to_f32(hi[e]));
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) lo[e] = 0u;
      }
      tmem_st16(sbuf + c * 32 + 16, lo);
    }
    if (need_lo) sb.lo_tile[s] = j + 1;
    tmem_wait_st();
    tc_fence_before_sync();
    __syncwarp();   // one arrival per warp: 128 arrivals on one barrier serialise
    if (lane == 0) mbar_arrive(bar_addr(sb.p_full[s]));
  }
  if (!ok) return;

  // Epilogue: O / l for the rows of this tile that exist.  Once the last PV
  // is done no MMA or copy touches shared memory any more, so each thread
  // stages its normalised row there (rows 528 bytes apart: conflict-free)
  // and sends it to global memory with one 512-byte bulk copy.
  if (!pf_wait_warp(sb, sb.pv_done[(nt - 1) & 1], ((nt - 1) >> 1) & 1, tmo)) return;
  tc_fence_after_sync();
  const float inv = l > 0.f ? 1.f / l : 0.f;
  const uint32_t srow = smem + r * kPfStageStride;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t o[32];
    tmem_ld32(trow + kPfColO + c * 32, o);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; e += 4)
      asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(srow + (c * 32 + e) * 4),
                   "f"(__uint_as_float(o[e]) * inv), "f"(__uint_as_float(o[e + 1]) * inv),
                   "f"(__uint_as_float(o[e + 2]) * inv), "f"(__uint_as_float(o[e + 3]) * inv)
                   : "memory");
  }
  fence_proxy_async_smem();   // generic-proxy writes -> bulk-copy reads
  if (r < rows_valid && in_bounds(out_row0 + r, a.total_rows, kSitePrefillOut)) {
    float* dst = a.out + ((out_row0 + r) * a.h_q + h) * (long long)kPfD;
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(srow), "r"(kPfD * 4)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    // Only the shared-memory reads need to be over before the CTA goes (the
    // global writes complete with the grid); the slot frees up sooner.
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
  }
}

// Grid (h_q, B, n_qtiles): block (h, b, z) takes q-tile t = n_qtiles-1-z of
// head h of sequence b, so the longest rows (most K/V tiles) start first and
// the heads of one kv group run side by side (their K/V tiles shared in L2).
__global__ void __launch_bounds__(kPfThreads, 2)
    prefill_tc_bf16(const __grid_constant__ CUtensorMap qmap,
                    const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap, const PrefillArgs a) {
  __shared__ PfBars sb;
  extern __shared__ uint8_t pf_dyn[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x, b = blockIdx.y;
  const int t = a.n_qtiles - 1 - (int)blockIdx.z;

  grid_dependency_wait();
  // Sequence b: first row (prefix sum of the non-negative lengths) and length.
  long long off = 0;
  for (int i = lane; i < b; i += 32) {
    const int v = a.seqlens[i];
    off += v > 0 ? v : 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) off += __shfl_xor_sync(kFull, off, o);
  const int Sraw = a.seqlens[b];
  long long S = Sraw > 0 ? Sraw : 0;
  if (threadIdx.x == 0 && h == 0 && t == 0) {
    if (Sraw < 0) raise_status(kStatusNegSeqlen);
    if (S > (long long)a.n_qtiles * kPfRows || off + S > a.total_rows)
      raise_status(kStatusSeqlenOverMax);
  }
  if (off + S > a.total_rows) S = a.total_rows > off ? a.total_rows - off : 0;
  const long long row0 = (long long)t * kPfRows;   // first query position of the tile
  if (row0 >= S) return;                             // the whole CTA: no rows here
  allow_dependent_launch();

  const long long rows_left = S - row0;
  const int rows_valid = rows_left < kPfRows ? (int)rows_left : kPfRows;
  // K/V tiles covering keys [0, row0 + rows_valid): the causal reach of the tile.
  const int nt = (int)((row0 + rows_valid + kPfKeys - 1) / kPfKeys);
  const long long qrow = off + row0;
  const uint32_t smem = (smem_u32(pf_dyn) + 1023u) & ~1023u;

  if (threadIdx.x == 0) {
    mbar_init(bar_addr(sb.q_full), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_addr(sb.k_full[s]), 1);
      mbar_init(bar_addr(sb.k_empty[s]), 1);
      mbar_init(bar_addr(sb.v_full[s]), 1);
      mbar_init(bar_addr(sb.v_empty[s]), 1);
      mbar_init(bar_addr(sb.s_full[s]), 1);
      mbar_init(bar_addr(sb.p_full[s]), 4);
      mbar_init(bar_addr(sb.pv_done[s]), 1);
      sb.lo_tile[s] = 0;
    }
    mbar_init(bar_addr(sb.drain), 1);
    sb.abort = 0;
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tensormap(&qmap);
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  if (warp == 5) tmem_alloc(smem_u32(&sb.tmem_base), kPfTmemCols);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = sb.tmem_base;

  if (warp < 4) {
    pf_softmax(sb, smem, tmem, warp, lane, t, nt, a, qrow, rows_valid, h, a.timeout_ns);
  } else if (warp == 4) {
    if (lane == 0)
      pf_producer(sb, smem, &qmap, &kmap, &vmap, h, h / a.G, qrow, off, nt, a.timeout_ns);
  } else {
    if (lane == 0) pf_mma(sb, smem, tmem, nt, a.timeout_ns);
  }
  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kPfTmemCols);
  }
}

}  // namespace gqa
