// 2D-tiled shared low-rank compensators (TileQ: Efficient Low-Rank
// Quantization of Mixture-of-Experts with 2D Tiling, abstract: factors shared
// across the input and output dimensions of the experts, and the experts'
// low-rank terms evaluated together in one pass).
//
// Expert e's compensator of one block type on tile (p, q) is U_p C[e,p,q] V_q,
// with U_p and V_q shared by every expert. The input-side projection is
// therefore shared too: tileq_z_kernel computes z_q = V_q x once per source
// row (once per token for W1, whose input is the same for all of a token's
// experts; once per routed row for W2). tileq_u_kernel then forms, for every
// routed row and row tile p, u_p = sum_q C[e,p,q] z_q and writes it into the
// activation columns after Kin. The quantised GEMM's compensator stage
// multiplies those columns by U_p (its B operand, shared by all experts), so
// U_p never runs as a separate pass.
//
// Both are small GEMMs on the mma.sync tensor path. z: [sources, Kin] x
// [Kin, r] per column tile (the tile's K range split over four warps, partial
// sums added in a fixed order). u: per (row tile, expert) [rows, Q r] x
// [Q r, r], with z rounded to fp16 as the A operand and the fp16 cores as B.
#include "kernels.h"

namespace moeq {

namespace {
constexpr int kZWarps = 4;

__device__ __forceinline__ void mma_16816_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
}  // namespace

// grid (Q, ceil(sources / (16 MT))), kZWarps warps: warp w covers the w-th
// quarter of column tile q's K range for the CTA's 16 MT source rows (MT
// m-tiles share each load of V).
template <int MODE, int MT>
__global__ void __launch_bounds__(kZWarps * 32) tileq_z_kernel(const TileqArgs a) {
  __shared__ float red[kZWarps][16 * MT][33];
  pdl_wait();
  pdl_trigger();
  const int q = blockIdx.x;
  const int nsrc = MODE == 0 ? a.T : a.T * a.k;
  const int s0 = blockIdx.y * 16 * MT;
  if (s0 >= nsrc) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int NT = a.r / 8;  // n-tiles of 8 outputs
  // fragment rows g and g + 8 of each m-tile (clamped: rows past the end
  // load a valid row and are not stored)
  const uint32_t* ra[MT];
  const uint32_t* rb[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    const int sa = min(s0 + 16 * m + g, nsrc - 1), sb = min(s0 + 16 * m + g + 8, nsrc - 1);
    if constexpr (MODE == 0) {
      ra[m] = reinterpret_cast<const uint32_t*>(a.x + (long long)sa * a.Kin);
      rb[m] = reinterpret_cast<const uint32_t*>(a.x + (long long)sb * a.Kin);
    } else {
      ra[m] = reinterpret_cast<const uint32_t*>(a.act + (long long)a.pinv[sa] * a.lda);
      rb[m] = reinterpret_cast<const uint32_t*>(a.act + (long long)a.pinv[sb] * a.lda);
    }
  }
  const uint32_t* v32 = reinterpret_cast<const uint32_t*>(a.v);
  const int ldv = a.Kin / 2;  // V row pitch in u32
  const int steps = a.tile_k / 16;
  const int k0 = q * a.tile_k;
  const int st0 = steps * warp / kZWarps, st1 = steps * (warp + 1) / kZWarps;
  float acc[MT][4][4];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[m][t][i] = 0.f;
#pragma unroll 4
  for (int sidx = st0; sidx < st1; ++sidx) {
    const int kw = (k0 + 16 * sidx) / 2 + c;  // u32 column of elements k0 + 16 sidx + 2c
    uint32_t bv[4][2];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      // B[k][n] = V[n][k]: the pair (k, k+1) of output n = 8t + g is one u32 of V's row
      const uint32_t* vr = v32 + (long long)(8 * min(t, NT - 1) + g) * ldv;
      bv[t][0] = vr[kw];
      bv[t][1] = vr[kw + 4];
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      uint32_t av[4];
      av[0] = ra[m][kw];
      av[1] = rb[m][kw];
      av[2] = ra[m][kw + 4];
      av[3] = rb[m][kw + 4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        if (t < NT) {
          if constexpr (MODE == 0) {
            mma_16816_bf16(acc[m][t], av, bv[t][0], bv[t][1]);
          } else {
            mma_16816(acc[m][t], av, bv[t][0], bv[t][1]);
          }
        }
      }
    }
  }
  // acc[m][t][i]: row 16m + g + 8 (i >> 1), output 8t + 2c + (i & 1)
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int t = 0; t < 4; ++t)
      if (t < NT)
#pragma unroll
        for (int i = 0; i < 4; ++i) red[warp][16 * m + g + 8 * (i >> 1)][8 * t + 2 * c + (i & 1)] = acc[m][t][i];
  __syncthreads();
  for (int idx = threadIdx.x; idx < 16 * MT * a.r; idx += blockDim.x) {
    const int i = idx / a.r, j = idx % a.r, s = s0 + i;
    if (s >= nsrc) continue;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kZWarps; ++w) v += red[w][i][j];
    a.z[((long long)s * a.Q + q) * a.r + j] = v;
  }
}

// u_p = Z C_p^T per (row tile p, expert e) as a small GEMM on the mma.sync
// path: rows = the expert's routed rows, K = Q r (z of all column tiles, fp16),
// N = r. Large batches (SPLITK false): grid (P, active experts,
// ceil(max rows per expert / (64 MT))), four warps each owning MT m-tiles of
// 16 routed rows. Small batches (SPLITK true, MT = 1): grid (P, active
// experts, ceil(max rows per expert / 16)), the four warps split K for the
// CTA's 16 rows and their partials are added in a fixed order.
template <int MT, bool SPLITK>
__global__ void __launch_bounds__(128) tileq_u_kernel(const TileqArgs a) {
  __shared__ float red[SPLITK ? 4 : 1][16][33];
  pdl_wait();
  pdl_trigger();
  const int p = blockIdx.x;
  const int slot = blockIdx.y;
  if (slot >= *a.n_active) return;
  const int e = a.active[slot];
  const int n_e = a.counts[e];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = SPLITK ? blockIdx.z * 16 : (blockIdx.z * 4 + warp) * 16 * MT;
  if (r0 >= n_e) return;  // uniform over the CTA when SPLITK (its only block-level synchronisation)
  const int g = lane >> 2, c = lane & 3;
  const int R = a.r, NT = R / 8;
  long long prow[MT][2];
  int jslot[MT][2];
  const float* zr[MT][2];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = min(r0 + 16 * m + g + 8 * h, n_e - 1);
      prow[m][h] = a.poffsets[e] + i;
      const int t = a.ptok[prow[m][h]];
      jslot[m][h] = a.pslot[prow[m][h]];
      const long long src = a.mode == 0 ? t : (long long)t * a.k + jslot[m][h];
      zr[m][h] = a.z + src * a.Q * R;
    }
  // B[k][n] = C[q][n][j] for k = q r + j: the pair (j, j+1) of output n is one u32 of the core's row n
  const uint32_t* c32 = reinterpret_cast<const uint32_t*>(a.c16) + ((long long)e * a.P + p) * a.Q * R * R / 2;
  float acc[MT][4][4];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[m][t][i] = 0.f;
  const int ksteps = a.Q * R / 16;
  const int kk0 = SPLITK ? ksteps * warp / 4 : 0, kk1 = SPLITK ? ksteps * (warp + 1) / 4 : ksteps;
#pragma unroll 2
  for (int kk = kk0; kk < kk1; ++kk) {
    const int k0 = 16 * kk;
    const int q = k0 / R, j0 = k0 % R;  // a 16-wide step never crosses a column tile (R = 16 or 32)
    uint32_t bv[4][2];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int n = 8 * min(t, NT - 1) + g;
      const uint32_t* cr = c32 + ((long long)q * R + n) * R / 2;
      bv[t][0] = cr[(j0 + 2 * c) / 2];
      bv[t][1] = cr[(j0 + 2 * c + 8) / 2];
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float2 x0 = *reinterpret_cast<const float2*>(zr[m][0] + k0 + 2 * c);
      const float2 x1 = *reinterpret_cast<const float2*>(zr[m][1] + k0 + 2 * c);
      const float2 x2 = *reinterpret_cast<const float2*>(zr[m][0] + k0 + 2 * c + 8);
      const float2 x3 = *reinterpret_cast<const float2*>(zr[m][1] + k0 + 2 * c + 8);
      uint32_t av[4];
      av[0] = pack_half2(x0.x, x0.y);
      av[1] = pack_half2(x1.x, x1.y);
      av[2] = pack_half2(x2.x, x2.y);
      av[3] = pack_half2(x3.x, x3.y);
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if (t < NT) mma_16816(acc[m][t], av, bv[t][0], bv[t][1]);
    }
  }
  // W1: gate tile j and up tile P/2 + j sit side by side (2r columns per j),
  // matching the interleaved gate/up rows of one 128-row block
  const int hp = a.P / 2;
  const int col = a.mode == 0 ? (p < hp ? p * 2 * R : (p - hp) * 2 * R + R) : p * R;
  // acc[m][t][i]: row 16m + g + 8 (i >> 1), output 8t + 2c + (i & 1)
  if constexpr (SPLITK) {
#pragma unroll
    for (int t = 0; t < 4; ++t)
      if (t < NT)
#pragma unroll
        for (int i = 0; i < 4; ++i) red[warp][g + 8 * (i >> 1)][8 * t + 2 * c + (i & 1)] = acc[0][t][i];
    __syncthreads();
    if (warp != 0) return;
#pragma unroll
    for (int t = 0; t < 4; ++t)
      if (t < NT)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int rr = g + 8 * (i >> 1), cc = 8 * t + 2 * c + (i & 1);
          acc[0][t][i] = red[0][rr][cc] + red[1][rr][cc] + red[2][rr][cc] + red[3][rr][cc];
        }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (r0 + 16 * m + g + 8 * h >= n_e) continue;
      const bool off = a.comp_top_n > 0 && jslot[m][h] >= a.comp_top_n;
      uint32_t* dst = reinterpret_cast<uint32_t*>(a.act + prow[m][h] * a.lda + a.Kin + col);
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if (t < NT)
          dst[(8 * t + 2 * c) / 2] = off ? 0u : pack_half2(acc[m][t][2 * h], acc[m][t][2 * h + 1]);
    }
}

cudaError_t launch_tileq(const TileqArgs& a, int grid_y, cudaStream_t st, int* launches) {
  const int nsrc = a.mode == 0 ? a.T : a.T * a.k;
  const bool big = nsrc >= 512;
  const int mt = big ? 4 : 1;
  const int zy = (nsrc + 16 * mt - 1) / (16 * mt);
  const dim3 zg(a.Q, zy);
  const dim3 zb(kZWarps * 32);
  cudaError_t err;
  if (a.mode == 0)
    err = big ? launch_kernel(tileq_z_kernel<0, 4>, zg, zb, 0, st, true, a)
              : launch_kernel(tileq_z_kernel<0, 1>, zg, zb, 0, st, true, a);
  else
    err = big ? launch_kernel(tileq_z_kernel<1, 4>, zg, zb, 0, st, true, a)
              : launch_kernel(tileq_z_kernel<1, 1>, zg, zb, 0, st, true, a);
  if (err != cudaSuccess) return err;
  if (launches) ++*launches;
  // an expert has at most one routed row per token; large batches give each
  // warp four m-tiles so one load of the cores serves 64 rows
  const bool many = (long long)a.T * a.k >= 1024;
  const int rows_cta = many ? 256 : 16;
  const dim3 ug(a.P, grid_y, (a.T + rows_cta - 1) / rows_cta);
  err = many ? launch_kernel(tileq_u_kernel<4, false>, ug, dim3(128), 0, st, true, a)
             : launch_kernel(tileq_u_kernel<1, true>, ug, dim3(128), 0, st, true, a);
  if (err == cudaSuccess && launches) ++*launches;
  return err;
}

}  // namespace moeq
