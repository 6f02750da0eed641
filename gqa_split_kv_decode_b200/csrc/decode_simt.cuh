// fp32 decode attention on the CUDA cores.
//
// fp32 inputs must not go through TF32 or bf16 tensor-core products (the fp32
// tolerance is 1e-5), so this path uses plain FMA.  It serves the small fp32
// workloads, which are latency-bound: a warp streams its keys in batches,
// each key row read with 16-byte (D = 128) or 8-byte (D = 64) loads per lane,
// all HB query heads of the block reuse each row, and the online softmax is
// kept per warp in base 2.
#pragma once

#include "split_merge.cuh"

namespace gqa {

// L2 prefetch of `bytes` bytes at `p` (16-byte aligned, a multiple of 16).
__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)),
               "r"(bytes)
               : "memory");
}

template <int D, int HB, int NW, int MODE>
__global__ void __launch_bounds__(NW * 32) decode_simt_f32(const DecodeArgs a) {
  static_assert(D == 64 || D == 128, "head dim");
  constexpr int PER = D / 32;  // contiguous elements per lane
  __shared__ float sm_m[NW * HB], sm_l[NW * HB];
  __shared__ __align__(16) float sm_o[NW * HB * D];
  __shared__ int sm_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = blockIdx.x, b = blockIdx.z;
  const int g = blockIdx.y / a.n_hb, hb = blockIdx.y % a.n_hb;
  // Keys in batches of U per warp (see the key loop below).
  constexpr int U = (HB * PER <= 8) ? 16 : (HB * PER <= 16) ? 8 : 4;
  if (a.hint_tiles > 0 &&
      blockIdx.x + gridDim.x * (blockIdx.y + (long long)gridDim.y * blockIdx.z) < a.hint_ctas) {
    // While the previous grid drains: L2 prefetch of the K and V rows of this
    // warp's first batch, at rows from lengths read before the wait
    // (possibly stale, so every row is checked against the cache's rows; the
    // split is located again after the wait).
    const Split h = locate_split<true>(a, b, slot, lane, false);
    const long long row = h.off + h.lo + warp + (long long)lane * NW;
    if (slot < h.n_active && lane < U && h.lo + warp + lane * NW < h.cached_hi && row >= 0 &&
        row < a.kv_rows) {
      const size_t at = ((size_t)row * a.h_kv + g) * D;
      bulk_prefetch_l2(static_cast<const float*>(a.k) + at, D * 4);
      bulk_prefetch_l2(static_cast<const float*>(a.v) + at, D * 4);
    }
  }
  grid_dependency_wait();
  allow_dependent_launch();
  const Split sp = locate_split(a, b, slot, lane,
                                warp == 0 && lane == 0 && slot == 0 && blockIdx.y == 0);
  if (slot >= sp.n_active) {
    if (MODE == kPartial) emit_empty_triplet<HB, D>(a, b, g, hb, slot);
    return;
  }

  const float* __restrict__ qp = static_cast<const float*>(a.q);
  const float* __restrict__ kp = static_cast<const float*>(a.k);
  const float* __restrict__ vp = static_cast<const float*>(a.v);

  float qr[HB][PER];
#pragma unroll
  for (int hh = 0; hh < HB; ++hh) {
    const int gi = hb * HB + hh;
    const bool ok = gi < a.G && in_bounds((long long)query_row(a, b, g, gi), (long long)a.B * a.h_q,
                                          kSiteQ);
    const float* src = qp + query_row(a, b, g, ok ? gi : 0) * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; ++e) qr[hh][e] = ok ? src[e] : 0.f;
  }

  float m_run[HB], l_run[HB], o_acc[HB][PER];
#pragma unroll
  for (int hh = 0; hh < HB; ++hh) {
    m_run[hh] = -INFINITY;
    l_run[hh] = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) o_acc[hh][e] = 0.f;
  }

  const size_t new_base = ((size_t)b * a.h_kv + g) * D + lane * PER;
  // Keys in batches of U per warp (keys j0, j0 + NW, ..., j0 + (U-1) NW): the
  // batch's K and V rows are requested together, so a warp waits one memory
  // round trip per batch rather than per key, and the batch's logits share
  // one max update.
  for (int j0 = sp.lo + warp; j0 < sp.hi; j0 += NW * U) {
    float kr[U][PER], vr[U][PER];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + u * NW;
      // key j comes from the cache, or is the appended token (key number cached_hi);
      // a cache row past the cache's rows reads as zero
      const bool fresh = sp.has_new && j == sp.cached_hi;
      if (j < sp.hi && (fresh || a.kv_rows < 0 || sp.off + j < a.kv_rows)) {
        const size_t base = fresh ? new_base : ((size_t)(sp.off + j) * a.h_kv + g) * D + lane * PER;
        const float* ksrc = fresh ? static_cast<const float*>(a.k_new) : kp;
        const float* vsrc = fresh ? static_cast<const float*>(a.v_new) : vp;
        if constexpr (PER == 4) {
          const float4 k4 = __ldg(reinterpret_cast<const float4*>(ksrc + base));
          const float4 v4 = __ldg(reinterpret_cast<const float4*>(vsrc + base));
          kr[u][0] = k4.x; kr[u][1] = k4.y; kr[u][2] = k4.z; kr[u][3] = k4.w;
          vr[u][0] = v4.x; vr[u][1] = v4.y; vr[u][2] = v4.z; vr[u][3] = v4.w;
        } else {
          const float2 k2 = __ldg(reinterpret_cast<const float2*>(ksrc + base));
          const float2 v2 = __ldg(reinterpret_cast<const float2*>(vsrc + base));
          kr[u][0] = k2.x; kr[u][1] = k2.y;
          vr[u][0] = v2.x; vr[u][1] = v2.y;
        }
      } else {
#pragma unroll
        for (int e = 0; e < PER; ++e) kr[u][e] = vr[u][e] = 0.f;
      }
    }
#pragma unroll
    for (int hh = 0; hh < HB; ++hh) {
      if (hb * HB + hh >= a.G) break;
      float s[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < PER; ++e) part = fmaf(qr[hh][e], kr[u][e], part);
        s[u] = part;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int u = 0; u < U; ++u) s[u] += __shfl_xor_sync(kFull, s[u], o);
      float mb = -INFINITY;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        s[u] = (j0 + u * NW < sp.hi) ? s[u] * a.scale_log2 : -INFINITY;
        mb = fmaxf(mb, s[u]);
      }
      // key j0 is in the range, so the batch max is finite
      const float m_new = fmaxf(m_run[hh], mb);
      const float alpha = exp2f(m_run[hh] - m_new);  // 0 on the first batch
      float psum = 0.f;
#pragma unroll
      for (int e = 0; e < PER; ++e) o_acc[hh][e] *= alpha;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float p = exp2f(s[u] - m_new);  // 0 past the range
        psum += p;
#pragma unroll
        for (int e = 0; e < PER; ++e) o_acc[hh][e] = fmaf(p, vr[u][e], o_acc[hh][e]);
      }
      l_run[hh] = fmaf(l_run[hh], alpha, psum);
      m_run[hh] = m_new;
    }
  }

  if (sp.has_new && hb == 0 && warp == 0 &&  // write the appended token's row
      in_bounds(sp.off + sp.cached_hi, (long long)a.B * a.cap, kSiteAppend)) {
    const size_t dst = ((size_t)(sp.off + sp.cached_hi) * a.h_kv + g) * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const_cast<float*>(kp)[dst + e] = static_cast<const float*>(a.k_new)[new_base + e];
      const_cast<float*>(vp)[dst + e] = static_cast<const float*>(a.v_new)[new_base + e];
    }
  }

#pragma unroll
  for (int hh = 0; hh < HB; ++hh) {
    if (lane == 0) {
      sm_m[warp * HB + hh] = m_run[hh];
      sm_l[warp * HB + hh] = l_run[hh];
    }
#pragma unroll
    for (int e = 0; e < PER; ++e) sm_o[(warp * HB + hh) * D + lane * PER + e] = o_acc[hh][e];
  }
  __syncthreads();
  emit_split_triplet<NW, HB, D>(sm_m, sm_l, sm_o, a, b, g, hb, slot);
  if (MODE == kFused) fused_finish<NW, HB, D>(a, b, g, hb, sp.n_active, &sm_flag);
}

}  // namespace gqa
