// Low-rank compensator down-projection and the weighted combine.
//
// lowrank_kernel: U = V A^T for every expert's routed rows (V = the block's
// input activations, A = the compensator's [r, K] factor), stored as fp16
// into the activation columns [K, K + r) that the expert GEMM reads as extra
// K (MiLo abstract: per-expert low-rank compensators of the quantisation
// residual). Small batches split K across CTAs (fixed-order sum of partials).
//
// combine_kernel: y_t = sum_j w[t, j] * o_(t, j), slots in a fixed order, the
// K-split partials of o summed first; bf16 out.
#include "kernels.h"
#include "common.cuh"

namespace moeq {

constexpr int kLrWarps = 4;    // each warp: 16 routed rows (tokens) x all r columns
constexpr int kLrRows = 16 * kLrWarps;
constexpr int kCombineThreads = 128;

// K steps [s0, s1) of one warp's 16 rows x 16 RF columns: a few steps per
// round with every load of the round issued before its MMAs (fewer steps per
// round at larger ranks, to keep the registers in bounds)
template <int RF>
__device__ __forceinline__ void lr_kloop(const uint32_t* act32, const uint4* afrag, long long ra, long long ldw, int S16,
                                         int s0, int s1, int c, int lane, float (&acc)[8][4]) {
  constexpr int kB = RF <= 2 ? 4 : 2;
  const long long rb = ra + 8;
  for (int S0 = s0; S0 < s1; S0 += kB) {
    uint32_t av[kB][4];
    uint4 v[kB][RF];
#pragma unroll
    for (int q = 0; q < kB; ++q) {
      const int S = min(S0 + q, s1 - 1);  // (a clamped step is loaded and not used)
      av[q][0] = act32[ra * ldw + 8 * S + c];
      av[q][1] = act32[rb * ldw + 8 * S + c];
      av[q][2] = act32[ra * ldw + 8 * S + c + 4];
      av[q][3] = act32[rb * ldw + 8 * S + c + 4];
#pragma unroll
      for (int i = 0; i < RF; ++i) v[q][i] = afrag[((long long)i * S16 + S) * 32 + lane];
    }
#pragma unroll
    for (int q = 0; q < kB; ++q) {
      if (S0 + q >= s1) break;
#pragma unroll
      for (int i = 0; i < RF; ++i) {
        mma_16816(acc[2 * i], av[q], v[q][i].x, v[q][i].z);
        mma_16816(acc[2 * i + 1], av[q], v[q][i].y, v[q][i].w);
      }
    }
  }
}

// grid: (KS x token tiles of 64 rows, expert slots). Tokens are the MMA's M:
// a warp's A fragments are 16 routed rows of the activations, its B
// fragments come straight from the factor's dense fragments (two n8 tiles per
// uint4). A tile with few rows (small decode batches) spreads its K range over
// the CTA's warps instead of its rows, so every warp keeps loads in flight;
// the warps' partial products meet in shared memory and are summed in a fixed
// order. With KS == 1 the result is written directly; otherwise each CTA
// writes an fp32 partial and the last CTA of a (expert, token tile) sums the
// partials in a fixed order.
__global__ void __launch_bounds__(kLrWarps * 32, 7) lowrank_kernel(LowrankArgs a) {
  __shared__ int is_last;
  __shared__ float red[kLrWarps][16][kMaxRank + 1];
  pdl_wait();
  pdl_trigger();
  const int slot = blockIdx.y;
  if (slot >= *a.n_active) return;
  const int e = a.active[slot];
  const int n_e = a.counts[e];
  const int ks = blockIdx.x % a.KS, tile = blockIdx.x / a.KS;
  const int nrows = min(kLrRows, n_e - tile * kLrRows);
  if (nrows <= 0) return;
  const BlockDesc& dd = a.experts[e].blk[a.block];
  const int r = dd.rank;
  if (r <= 0 || dd.tq_span > 0) return;  // 2D-tiled shared compensators have their own kernels
  const uint4* afrag = dd.afrag;
  const int RF = r / 16;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  // warps along K: 4 for one 16-row sub-tile, 2 for two, 1 otherwise
  const int wk = nrows <= 16 ? 4 : nrows <= 32 ? 2 : 1;
  const int rsub = warp / wk, kw = warp % wk;
  const int S16 = a.K / 16;
  const int c0 = (int)((long long)S16 * ks / a.KS), c1 = (int)((long long)S16 * (ks + 1) / a.KS);
  const int s0 = c0 + (c1 - c0) * kw / wk, s1 = c0 + (c1 - c0) * (kw + 1) / wk;
  const int prow0 = a.poffsets[e];
  const int rbase = tile * kLrRows + rsub * 16;  // first row (within the expert) of this warp
  const uint32_t* act32 = reinterpret_cast<const uint32_t*>(a.act);
  float acc[8][4];
#pragma unroll
  for (int t = 0; t < 8; ++t)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[t][q] = 0.f;
  if (rbase < n_e) {
    // rows past the expert's count read the padded slack rows of the buffer
    const long long ra = prow0 + rbase + g;  // row of a0a1/a4a5 (a2a3/a6a7: 8 rows later)
    switch (RF) {
      case 1: lr_kloop<1>(act32, afrag, ra, a.Kpad >> 1, S16, s0, s1, c, lane, acc); break;
      case 2: lr_kloop<2>(act32, afrag, ra, a.Kpad >> 1, S16, s0, s1, c, lane, acc); break;
      case 3: lr_kloop<3>(act32, afrag, ra, a.Kpad >> 1, S16, s0, s1, c, lane, acc); break;
      default: lr_kloop<4>(act32, afrag, ra, a.Kpad >> 1, S16, s0, s1, c, lane, acc); break;
    }
  }
  // acc[t][q]: row g + 8*(q>>1) of the sub-tile, column j = 8t + 2c + (q&1)
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    if (t >= 2 * RF) break;
#pragma unroll
    for (int q = 0; q < 4; ++q) red[warp][g + 8 * (q >> 1)][8 * t + 2 * c + (q & 1)] = acc[t][q];
  }
  __syncthreads();
  auto store_u = [&](int n, int j, float v) {
    // only the first comp_top_n routing slots of a token are compensated
    if (a.comp_top_n > 0 && a.pslot[prow0 + n] >= a.comp_top_n) v = 0.f;
    a.act[(long long)(prow0 + n) * a.Kpad + a.K + j] = __float2half_rn(v);
  };
  // the CTA's value for tile row i, column j: the K-warps' partials in order
  auto cta_value = [&](int i, int j) {
    const int sub = i >> 4;
    float v = 0.f;
    for (int w = 0; w < wk; ++w) v += red[sub * wk + w][i & 15][j];
    return v;
  };
  if (a.KS == 1) {
    for (int idx = threadIdx.x; idx < nrows * r; idx += blockDim.x) {
      const int i = idx / r, j = idx % r;
      store_u(tile * kLrRows + i, j, cta_value(i, j));
    }
    return;
  }
  for (int idx = threadIdx.x; idx < nrows * r; idx += blockDim.x) {
    const int i = idx / r, j = idx % r;
    a.part[ks * a.part_ks_stride + (long long)(prow0 + tile * kLrRows + i) * kMaxRank + j] = cta_value(i, j);
  }
  __threadfence();
  __syncthreads();
  int* sem = a.sem + (long long)e * a.sem_stride + tile;
  if (threadIdx.x == 0) is_last = (atomicAdd(sem, 1) == a.KS - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  for (int idx = threadIdx.x; idx < nrows * r; idx += blockDim.x) {
    const int n = tile * kLrRows + idx / r, j = idx % r;
    const float* pp = a.part + (long long)(prow0 + n) * kMaxRank + j;
    // the partials in split order, eight loads in flight at a time
    float sum = 0.f;
    for (int k0 = 0; k0 < a.KS; k0 += 8) {
      float pv[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) pv[q] = k0 + q < a.KS ? __ldcg(pp + (long long)(k0 + q) * a.part_ks_stride) : 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q) sum += pv[q];
    }
    store_u(n, j, sum);
  }
  if (threadIdx.x == 0) *sem = 0;
}

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(CombineArgs a) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  float wt[kMaxTopK];
  long long pr[kMaxTopK];
  for (int j = 0; j < a.k; ++j) {
    wt[j] = a.w[(long long)t * a.k + j];
    pr[j] = a.pinv[(long long)t * a.k + j];
  }
  // this CTA's slice of the token's K columns, 4 per thread
  for (int k = (blockIdx.y * blockDim.x + threadIdx.x) * 4; k < a.K; k += gridDim.y * blockDim.x * 4) {
    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < a.k; ++j) {
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
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
  dim3 grid(a.KS * a.tiles, grid_y);
  const cudaError_t err = launch_kernel(lowrank_kernel, grid, dim3(kLrWarps * 32), 0, st, true, a);
  if (launches) ++*launches;
  return err;
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st, int* launches) {
  const int ky = (a.K + 4 * kCombineThreads - 1) / (4 * kCombineThreads);
  const cudaError_t err = launch_kernel(combine_kernel, dim3(a.T, ky), dim3(kCombineThreads), 0, st, true, a);
  if (launches) ++*launches;
  return err;
}

}  // namespace moeq
