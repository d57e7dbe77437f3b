// Per-group correction sums of a block's input rows for the integer-code
// decode GEMM (see decode_gemm.cu): for routed row p and group g,
// corr[p][16g .. 16g+15] = (-XP_hi, -XP_lo, -X_hi, -X_lo, 0 x 12) in fp16 with
// XP = sum_k (P_k / 1024) x_pk and X = sum_k x_pk, each the fp16 value of the
// fp32 sum followed by the fp16 value of its remainder. One warp per
// (routed row, group), four such items per round with their loads in flight
// together; the warp's lanes reduce in a fixed butterfly order.
#pragma once
#include "kernels.h"
#include "decode_frag.cuh"

namespace moeq {

__device__ __forceinline__ void act_corr_rows(const CorrArgs& a, int slot, int cta, int ncta) {
  if (slot >= *a.n_active) return;
  const int e = a.active[slot];
  const BlockDesc& d = a.experts[e].blk[a.block];
  if (d.fmt != FMT_INT) return;
  const int n_e = a.counts[e], prow0 = a.poffsets[e];
  const int G = d.group, NG = a.K / G, bits = d.bits;
  const int per = G / 32;  // codes per lane: 2 (one u32 load) or 4 (one u64 load)
  const int nw = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long items = (long long)n_e * NG;
  const long long stride = (long long)ncta * nw;
  constexpr int U = 4;  // items per round: their loads are in flight together
  for (long long it0 = (long long)cta * nw + warp; it0 < items; it0 += U * stride) {
    float xs[U], xp[U];
    long long prow[U];
    int grp[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long it = it0 + u * stride;
      xs[u] = xp[u] = 0.f;
      prow[u] = -1;
      if (it >= items) continue;
      prow[u] = prow0 + it / NG;
      grp[u] = (int)(it % NG);
      const int k0 = grp[u] * G + lane * per;
      const __half* x = a.act + prow[u] * a.lda + k0;
      alignas(8) __half v[4];
      if (per == 4) {
        *reinterpret_cast<uint2*>(v) = *reinterpret_cast<const uint2*>(x);
      } else {
        *reinterpret_cast<uint32_t*>(v) = *reinterpret_cast<const uint32_t*>(x);
      }
      for (int j = 0; j < per; ++j) {
        const float f = __half2float(v[j]);
        xs[u] += f;
        xp[u] = fmaf(int_pfac(bits, (k0 + j) & 63), f, xp[u]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int u = 0; u < U; ++u) {
        xs[u] += __shfl_xor_sync(0xffffffffu, xs[u], o);
        xp[u] += __shfl_xor_sync(0xffffffffu, xp[u], o);
      }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (prow[u] < 0 || lane >= 8) continue;
      uint32_t val = 0u;
      if (lane < 2) {
        const float t = lane == 0 ? -xp[u] : -xs[u];
        if (!(fabsf(t) < 65504.f)) atomicOr(a.status, ST_RANGE);
        const __half hi = __float2half_rn(t);
        const __half lo = __float2half_rn(t - __half2float(hi));
        const __half2 hv = __halves2half2(hi, lo);
        val = *reinterpret_cast<const uint32_t*>(&hv);
      }
      reinterpret_cast<uint32_t*>(a.corr + prow[u] * a.ldc + 16 * grp[u])[lane] = val;
    }
  }
}

}  // namespace moeq
