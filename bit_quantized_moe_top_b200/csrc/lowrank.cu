// Low-rank compensator down-projection and the weighted combine.
//
// lowrank_kernel: U = V A^T for every expert's routed rows (V = the block's
// input activations, A = the compensator's [r, K] factor), split over K across
// CTAs; each CTA writes an fp32 partial and the last CTA of an expert (atomic
// ticket) sums the partials in a fixed order and stores U as fp16 into the
// activation columns [K, K + r) that the expert GEMM reads as extra K
// (MiLo abstract: per-expert low-rank compensators of the quantisation
// residual).
//
// combine_kernel: y_t = sum_j w[t, j] * o_(t, j), slots in a fixed order, the
// K-split partials of o summed first; bf16 out.
#include "kernels.h"

namespace moeq {

constexpr int kLrWarps = 8;
constexpr int kLrNT = 4;  // n8 token tiles per pass

__global__ void __launch_bounds__(256) lowrank_kernel(LowrankArgs a) {
  __shared__ float red[4 * kLrNT * 32 * 4];
  __shared__ int is_last;
  const int slot = blockIdx.y;
  if (slot >= *a.n_active) return;
  const int e = a.active[slot];
  const int n_e = a.counts[e];
  const BlockDesc& dd = a.experts[e].blk[a.block];
  const int r = dd.rank;
  if (r <= 0 || n_e <= 0) return;
  const uint4* afrag = dd.afrag;
  const int RF = r / 16;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int ks = blockIdx.x;
  const int S16 = a.K / 16;
  const int s0 = (int)((long long)S16 * ks / a.KS), s1 = (int)((long long)S16 * (ks + 1) / a.KS);
  const int prow0 = a.poffsets[e];
  const int ntiles = (n_e + 7) >> 3;
  const uint4* act4 = reinterpret_cast<const uint4*>(a.act);
  for (int pb = 0; pb < ntiles; pb += kLrNT) {
    const int np = min(kLrNT, ntiles - pb);
    float acc[4][kLrNT][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int t = 0; t < kLrNT; ++t)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[i][t][q] = 0.f;
    for (int S = s0 + warp; S < s1; S += kLrWarps) {
      uint32_t b0[kLrNT], b1[kLrNT];
#pragma unroll
      for (int t = 0; t < kLrNT; ++t) {
        b0[t] = b1[t] = 0;
        if (t < np) {
          const long long n0 = prow0 + 8LL * (pb + t);
          if (a.act_layout == ACT_FRAG) {
            const uint4 v = act4[act_frag_u4(n0 >> 3, S >> 1, a.nt8cap, lane)];
            b0[t] = (S & 1) ? v.z : v.x;
            b1[t] = (S & 1) ? v.w : v.y;
          } else {
            const uint32_t* row = reinterpret_cast<const uint32_t*>(a.act + (n0 + g) * a.Kpad + 16 * S);
            b0[t] = row[c];
            b1[t] = row[c + 4];
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (i >= RF) break;
        const uint4 v = afrag[((long long)i * S16 + S) * 32 + lane];
        const uint32_t av[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int t = 0; t < kLrNT; ++t)
          if (t < np) mma_16816(acc[i][t], av, b0[t], b1[t]);
      }
    }
    // fixed-order reduction over warps
    for (int i = threadIdx.x; i < 4 * kLrNT * 32 * 4; i += blockDim.x) red[i] = 0.f;
    __syncthreads();
    for (int w = 0; w < kLrWarps; ++w) {
      if (warp == w) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int t = 0; t < kLrNT; ++t)
#pragma unroll
            for (int q = 0; q < 4; ++q) red[((i * kLrNT + t) * 32 + lane) * 4 + q] += acc[i][t][q];
      }
      __syncthreads();
    }
    // CTA partial -> part[ks][prow][j]
    for (int idx = threadIdx.x; idx < RF * kLrNT * 32 * 4; idx += blockDim.x) {
      const int q = idx & 3, ln = (idx >> 2) & 31, t = (idx >> 7) % kLrNT, i = (idx >> 7) / kLrNT;
      if (t >= np) continue;
      const int n = 8 * (pb + t) + 2 * (ln & 3) + (q & 1);
      if (n >= n_e) continue;
      const int j = 16 * i + (ln >> 2) + 8 * (q >> 1);
      a.part[ks * a.part_ks_stride + (long long)(prow0 + n) * kMaxRank + j] = red[idx];
    }
    __syncthreads();
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(a.sem + e, 1) == a.KS - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  for (int idx = threadIdx.x; idx < n_e * r; idx += blockDim.x) {
    const int n = idx / r, j = idx % r;
    float s = 0.f;
    for (int k2 = 0; k2 < a.KS; ++k2) s += __ldcg(a.part + k2 * a.part_ks_stride + (long long)(prow0 + n) * kMaxRank + j);
    const __half hv = __float2half_rn(s);
    if (a.act_layout == ACT_FRAG) a.act[act_frag_index(prow0 + n, a.K + j, a.nt8cap)] = hv;
    else a.act[(long long)(prow0 + n) * a.Kpad + a.K + j] = hv;
  }
  if (threadIdx.x == 0) a.sem[e] = 0;
}

__global__ void __launch_bounds__(256) combine_kernel(CombineArgs a) {
  const int t = blockIdx.x;
  float wt[kMaxTopK];
  long long pr[kMaxTopK];
  for (int j = 0; j < a.k; ++j) {
    wt[j] = a.w[(long long)t * a.k + j];
    pr[j] = a.pinv[(long long)t * a.k + j];
  }
  for (int k = threadIdx.x * 4; k < a.K; k += blockDim.x * 4) {
    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < a.k; ++j) {
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s = 0; s < a.KS; ++s) {
        const float4 v = *reinterpret_cast<const float4*>(a.O + s * a.ks_stride + pr[j] * a.K + k);
        o.x += v.x; o.y += v.y; o.z += v.z; o.w += v.w;
      }
      y.x += wt[j] * o.x; y.y += wt[j] * o.y; y.z += wt[j] * o.z; y.w += wt[j] * o.w;
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(y.x, y.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(y.z, y.w);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&lo);
    pk.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(a.Y + (long long)t * a.K + k) = pk;
  }
}

cudaError_t launch_lowrank(const LowrankArgs& a, int grid_y, cudaStream_t st, int* launches) {
  dim3 grid(a.KS, grid_y);
  lowrank_kernel<<<grid, kLrWarps * 32, 0, st>>>(a);
  if (launches) ++*launches;
  return cudaGetLastError();
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st, int* launches) {
  combine_kernel<<<a.T, 256, 0, st>>>(a);
  if (launches) ++*launches;
  return cudaGetLastError();
}

}  // namespace moeq
