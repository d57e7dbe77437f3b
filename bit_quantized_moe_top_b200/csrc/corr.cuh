// Per-chunk correction sums of a block's input rows for the integer-code
// decode GEMM (see decode_gemm.cu): for routed row p and 64-column chunk c of
// group g = c / cpg (cpg = g / 64 chunks per group),
//   corr[p][16g + 4(c % cpg) .. +3] = (-XP_hi, -XP_lo, -X_hi, -X_lo)
// in fp16 with XP = sum_k (P_k / 1024) x_pk and X = sum_k x_pk over the chunk,
// each the fp16 value of the fp32 sum followed by the fp16 value of its
// remainder; the other slots of a group stay zero. One warp per (routed row,
// chunk), two columns per lane, four such items per round with their loads in
// flight together; the lanes reduce in a fixed butterfly order.
#pragma once
#include "kernels.h"
#include "decode_frag.cuh"

namespace moeq {

// the fp16 pair (value, remainder) of -t; flags sums beyond fp16's range
__device__ __forceinline__ uint32_t corr_pair(float t, unsigned* status) {
  t = -t;
  if (!(fabsf(t) < 65504.f)) atomicOr(status, ST_RANGE);
  const __half hi = __float2half_rn(t);
  const __half lo = __float2half_rn(t - __half2float(hi));
  const __half2 hv = __halves2half2(hi, lo);
  return *reinterpret_cast<const uint32_t*>(&hv);
}

__device__ __forceinline__ void act_corr_rows(const CorrArgs& a, int slot, int cta, int ncta) {
  if (slot >= *a.n_active) return;
  const int e = a.active[slot];
  const BlockDesc& d = a.experts[e].blk[a.block];
  if (d.fmt != FMT_INT) return;
  const int n_e = a.counts[e], prow0 = a.poffsets[e];
  const int KC = a.K / 64, cpg = d.group / 64, bits = d.bits;
  const int nw = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long items = (long long)n_e * KC;
  const long long stride = (long long)ncta * nw;
  constexpr int U = 4;  // items per round: their loads are in flight together
  const float f0 = int_pfac(bits, 2 * lane), f1 = int_pfac(bits, 2 * lane + 1);
  for (long long it0 = (long long)cta * nw + warp; it0 < items; it0 += U * stride) {
    float xs[U], xp[U];
    long long prow[U];
    int chunk[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long it = it0 + u * stride;
      xs[u] = xp[u] = 0.f;
      prow[u] = -1;
      if (it >= items) continue;
      prow[u] = prow0 + it / KC;
      chunk[u] = (int)(it % KC);
      const __half2 v = *reinterpret_cast<const __half2*>(a.act + prow[u] * a.lda + 64 * chunk[u] + 2 * lane);
      const float x0 = __low2float(v), x1 = __high2float(v);
      xs[u] = x0 + x1;
      xp[u] = fmaf(f1, x1, f0 * x0);
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
      if (prow[u] < 0 || lane >= 2) continue;
      const int g = chunk[u] / cpg, c = chunk[u] % cpg;
      reinterpret_cast<uint32_t*>(a.corr + prow[u] * a.ldc + 16 * g + 4 * c)[lane] =
          corr_pair(lane == 0 ? xp[u] : xs[u], a.status);
    }
  }
}

}  // namespace moeq
