// Per-group correction sums of a block's input rows for the integer-code
// decode GEMM (see decode_gemm.cu): for routed row p and group g,
// corr[p][16g .. 16g+15] = (-XP_hi, -XP_lo, -X_hi, -X_lo, 0 x 12) in fp16 with
// XP = sum_k (P_k / 1024) x_pk and X = sum_k x_pk, each the fp16 value of the
// fp32 sum followed by the fp16 value of its remainder. One warp per
// (routed row, group); the warp's lanes reduce in a fixed butterfly order.
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
  const int per = G / 32;  // codes per lane: 2 or 4
  const int nw = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long items = (long long)n_e * NG;
  for (long long it = (long long)cta * nw + warp; it < items; it += (long long)ncta * nw) {
    const long long p = prow0 + it / NG;
    const int g = (int)(it % NG);
    const int k0 = g * G + lane * per;
    const __half* x = a.act + p * a.lda + k0;
    float xs = 0.f, xp = 0.f;
    for (int j = 0; j < per; ++j) {
      const float v = __half2float(x[j]);
      xs += v;
      xp = fmaf(int_pfac(bits, (k0 + j) & 63), v, xp);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      xs += __shfl_xor_sync(0xffffffffu, xs, o);
      xp += __shfl_xor_sync(0xffffffffu, xp, o);
    }
    if (lane < 8) {
      uint32_t val = 0u;
      if (lane < 2) {
        const float t = lane == 0 ? -xp : -xs;
        if (!(fabsf(t) < 65504.f)) atomicOr(a.status, ST_RANGE);
        const __half hi = __float2half_rn(t);
        const __half lo = __float2half_rn(t - __half2float(hi));
        const __half2 hv = __halves2half2(hi, lo);
        val = *reinterpret_cast<const uint32_t*>(&hv);
      }
      reinterpret_cast<uint32_t*>(a.corr + p * a.ldc + 16 * g)[lane] = val;
    }
  }
}

}  // namespace moeq
