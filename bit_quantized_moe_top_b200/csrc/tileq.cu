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
// z: a small GEMM [sources, Kin] x [Kin, r] per column tile on the mma.sync
// tensor path (16 source rows per CTA, the tile's K range split over four
// warps, partial sums added in a fixed order). u: per (row tile, expert,
// 16 routed rows) one CTA stages the expert's cores of that row tile in
// shared memory, lanes own output components, fp32 FMA.
#include "kernels.h"

namespace moeq {

namespace {
constexpr int kZWarps = 4;
constexpr int kUQChunk = 8;  // column tiles of cores staged per round (8 x 32 x 32 bf16 = 16 KiB)

__device__ __forceinline__ void mma_16816_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
}  // namespace

// grid (Q, ceil(sources / 16)), kZWarps warps: warp w covers the w-th quarter
// of column tile q's K range for the CTA's 16 source rows.
template <int MODE>
__global__ void __launch_bounds__(kZWarps * 32) tileq_z_kernel(const TileqArgs a) {
  __shared__ float red[kZWarps][16][33];
  pdl_wait();
  pdl_trigger();
  const int q = blockIdx.x;
  const int nsrc = MODE == 0 ? a.T : a.T * a.k;
  const int s0 = blockIdx.y * 16;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int NT = a.r / 8;  // n-tiles of 8 outputs
  // the fragment rows g and g + 8 of the CTA's 16 sources (clamped: rows past
  // the end load a valid row and are not stored)
  const int sa = min(s0 + g, nsrc - 1), sb = min(s0 + g + 8, nsrc - 1);
  const uint32_t* ra;
  const uint32_t* rb;
  if constexpr (MODE == 0) {
    ra = reinterpret_cast<const uint32_t*>(a.x + (long long)sa * a.Kin);
    rb = reinterpret_cast<const uint32_t*>(a.x + (long long)sb * a.Kin);
  } else {
    ra = reinterpret_cast<const uint32_t*>(a.act + (long long)a.pinv[sa] * a.lda);
    rb = reinterpret_cast<const uint32_t*>(a.act + (long long)a.pinv[sb] * a.lda);
  }
  const uint32_t* v32 = reinterpret_cast<const uint32_t*>(a.v);
  const int ldv = a.Kin / 2;  // V row pitch in u32
  const int steps = a.tile_k / 16;
  const int k0 = q * a.tile_k;
  const int st0 = steps * warp / kZWarps, st1 = steps * (warp + 1) / kZWarps;
  float acc[4][4];
#pragma unroll
  for (int t = 0; t < 4; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[t][i] = 0.f;
#pragma unroll 2
  for (int sidx = st0; sidx < st1; ++sidx) {
    const int kw = (k0 + 16 * sidx) / 2 + c;  // u32 column of elements k0 + 16 sidx + 2c
    uint32_t av[4];
    av[0] = ra[kw];
    av[1] = rb[kw];
    av[2] = ra[kw + 4];
    av[3] = rb[kw + 4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      if (t < NT) {
        // B[k][n] = V[n][k]: the pair (k, k+1) of output n = 8t + g is one u32 of V's row
        const uint32_t* vr = v32 + (long long)(8 * t + g) * ldv;
        if constexpr (MODE == 0) {
          mma_16816_bf16(acc[t], av, vr[kw], vr[kw + 4]);
        } else {
          mma_16816(acc[t], av, vr[kw], vr[kw + 4]);
        }
      }
    }
  }
  // acc[t][i]: row g + 8 (i >> 1), output 8t + 2c + (i & 1)
#pragma unroll
  for (int t = 0; t < 4; ++t)
    if (t < NT)
#pragma unroll
      for (int i = 0; i < 4; ++i) red[warp][g + 8 * (i >> 1)][8 * t + 2 * c + (i & 1)] = acc[t][i];
  __syncthreads();
  for (int idx = threadIdx.x; idx < 16 * a.r; idx += blockDim.x) {
    const int i = idx / a.r, j = idx % a.r, s = s0 + i;
    if (s >= nsrc) continue;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kZWarps; ++w) v += red[w][i][j];
    a.z[((long long)s * a.Q + q) * a.r + j] = v;
  }
}

// grid (P, active experts, ceil(max rows per expert / 16)), 8 warps: warp w
// handles routed rows 2w and 2w + 1 of the CTA's 16 rows of expert e.
__global__ void __launch_bounds__(256) tileq_u_kernel(const TileqArgs a) {
  __shared__ __align__(16) __nv_bfloat16 cs[kUQChunk * 32 * 32];
  pdl_wait();
  pdl_trigger();
  const int p = blockIdx.x;
  const int slot = blockIdx.y;
  if (slot >= *a.n_active) return;
  const int e = a.active[slot];
  const int n_e = a.counts[e];
  const int r0 = blockIdx.z * 16;
  if (r0 >= n_e) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int R = a.r;
  const int i0 = r0 + 2 * warp, i1 = i0 + 1;
  const bool v0 = i0 < n_e, v1 = i1 < n_e;
  const long long pr0 = a.poffsets[e] + min(i0, n_e - 1), pr1 = a.poffsets[e] + min(i1, n_e - 1);
  const int t0 = a.ptok[pr0], t1 = a.ptok[pr1];
  const int j0 = a.pslot[pr0], j1 = a.pslot[pr1];
  const long long src0 = a.mode == 0 ? t0 : (long long)t0 * a.k + j0;
  const long long src1 = a.mode == 0 ? t1 : (long long)t1 * a.k + j1;
  const float* z0 = a.z + src0 * a.Q * R;
  const float* z1 = a.z + src1 * a.Q * R;
  const __nv_bfloat16* cg = a.ct + ((long long)e * a.P + p) * a.Q * R * R;
  float acc0 = 0.f, acc1 = 0.f;
  for (int qb = 0; qb < a.Q; qb += kUQChunk) {
    const int nq = min(kUQChunk, a.Q - qb);
    __syncthreads();
    const int n16 = nq * R * R / 8;  // uint4 units
    const uint4* src = reinterpret_cast<const uint4*>(cg + (long long)qb * R * R);
    for (int i = threadIdx.x; i < n16; i += blockDim.x) reinterpret_cast<uint4*>(cs)[i] = src[i];
    __syncthreads();
    if (lane < R) {
      for (int q = 0; q < nq; ++q) {
        const float* za = z0 + (qb + q) * R;
        const float* zb = z1 + (qb + q) * R;
#pragma unroll 8
        for (int j = 0; j < R; ++j) {
          const float cv = __bfloat162float(cs[(q * R + j) * R + lane]);
          acc0 = fmaf(cv, za[j], acc0);
          acc1 = fmaf(cv, zb[j], acc1);
        }
      }
    }
  }
  if (lane >= R) return;
  if (a.comp_top_n > 0) {
    if (j0 >= a.comp_top_n) acc0 = 0.f;
    if (j1 >= a.comp_top_n) acc1 = 0.f;
  }
  // W1: gate tile j and up tile P/2 + j sit side by side (2r columns per j),
  // matching the interleaved gate/up rows of one 128-row block
  const int hp = a.P / 2;
  const int col = a.mode == 0 ? (p < hp ? p * 2 * R : (p - hp) * 2 * R + R) : p * R;
  if (v0) a.act[pr0 * a.lda + a.Kin + col + lane] = __float2half_rn(acc0);
  if (v1) a.act[pr1 * a.lda + a.Kin + col + lane] = __float2half_rn(acc1);
}

cudaError_t launch_tileq(const TileqArgs& a, int grid_y, cudaStream_t st, int* launches) {
  const int nsrc = a.mode == 0 ? a.T : a.T * a.k;
  const dim3 zg(a.Q, (nsrc + 15) / 16);
  cudaError_t err = a.mode == 0 ? launch_kernel(tileq_z_kernel<0>, zg, dim3(kZWarps * 32), 0, st, true, a)
                                : launch_kernel(tileq_z_kernel<1>, zg, dim3(kZWarps * 32), 0, st, true, a);
  if (err != cudaSuccess) return err;
  if (launches) ++*launches;
  // an expert has at most one routed row per token
  err = launch_kernel(tileq_u_kernel, dim3(a.P, grid_y, (a.T + 15) / 16), dim3(256), 0, st, true, a);
  if (err == cudaSuccess && launches) ++*launches;
  return err;
}

}  // namespace moeq
