// Routing: top-k softmax per token, per-expert histogram, exclusive scan and a
// stable token permutation (expert-major, token-ascending), plus the gather of
// routed token rows into the activation layout of the expert GEMMs.
//
// Top-k per token follows the routing of the Bandwidth-Efficient Adaptive
// Mixture-of-Experts via Low-Rank Compensation page (abstract: each token has
// k routed experts, of which the Top-n get compensation). Selection compares
// the fp32 logits exactly, ties to the lower expert index; the weights are the
// softmax over the selected logits (or the full softmax, by flag).
#include <algorithm>

#include "kernels.h"

namespace moeq {

constexpr int kRouteTokensPerCta = 16;
constexpr int kRouteThreads = 256;

__device__ __forceinline__ bool better(float a, int ia, float b, int ib) {
  return a > b || (a == b && ia < ib);
}

// grid: ceil(T/16) CTAs of 256 threads (8 warps, 2 tokens each).
// The last CTA to finish (atomic ticket) scans the block histograms.
__global__ void __launch_bounds__(kRouteThreads) route_topk_kernel(RouteArgs a) {
  __shared__ int hist[kMaxExperts];
  __shared__ int seg[kMaxExperts > kRouteThreads ? kMaxExperts : kRouteThreads];  // per-(expert, segment) sums
  __shared__ int is_last;
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * kRouteTokensPerCta;
  for (int tt = warp; tt < kRouteTokensPerCta; tt += 8) {
    const int t = t0 + tt;
    if (t >= a.T) break;
    const float* row = a.logits + (long long)t * a.E;
    float v[8];
    unsigned taken = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      v[i] = e < a.E ? row[e] : -INFINITY;
    }
    float lsel[kMaxTopK];
    int isel[kMaxTopK];
    for (int j = 0; j < a.k; ++j) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        if (e < a.E && !((taken >> i) & 1u) && (bi == 0x7fffffff || better(v[i], e, bv, bi))) {
          bv = v[i];
          bi = e;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (oi != 0x7fffffff && (bi == 0x7fffffff || better(ov, oi, bv, bi))) {
          bv = ov;
          bi = oi;
        }
      }
      lsel[j] = bv;
      isel[j] = bi;
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    }
    // softmax weights
    const float m = lsel[0];
    float den = 0.f;
    if (a.renorm) {
      for (int j = 0; j < a.k; ++j) den += expf(lsel[j] - m);
    } else {
      float part = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        if (e < a.E) part += expf(v[i] - m);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      den = part;
    }
    if (lane < a.k) {
      int myi = isel[0];
      float myl = lsel[0];
      for (int j = 1; j < a.k; ++j)
        if (j == lane) {
          myi = isel[j];
          myl = lsel[j];
        }
      if (myi < 0 || myi >= a.E) {
        atomicOr(a.status, ST_ROUTE);
        myi = 0;
      }
      a.idx[(long long)t * a.k + lane] = myi;
      a.w[(long long)t * a.k + lane] = expf(myl - m) / den;
      atomicAdd(&hist[myi], 1);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) a.block_counts[(long long)blockIdx.x * a.E + e] = hist[e];
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(a.ticket, 1) == (int)gridDim.x - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // ---- last CTA: totals, offsets, padded offsets, per-block bases, active list.
  // Thread (e, s) owns a contiguous segment of the token blocks of expert e
  // (S segments per expert), so long block lists are summed in parallel.
  const int nb = gridDim.x;
  const int S = a.E >= kRouteThreads ? 1 : kRouteThreads / a.E;
  const int bpseg = (nb + S - 1) / S;
  for (int t = threadIdx.x; t < a.E * S; t += blockDim.x) {
    const int e = t / S, sg = t % S;
    const int b0 = min(nb, sg * bpseg), b1 = min(nb, b0 + bpseg);
    int sum = 0;
#pragma unroll 4
    for (int b = b0; b < b1; ++b) sum += __ldcg(a.block_counts + (long long)b * a.E + e);
    seg[t] = sum;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
    int tot = 0;
    for (int sg = 0; sg < S; ++sg) {
      const int v = seg[e * S + sg];
      seg[e * S + sg] = tot;  // exclusive prefix over the expert's segments
      tot += v;
    }
    hist[e] = tot;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int off = 0, poff = 0, na = 0;
    for (int e = 0; e < a.E; ++e) {
      const int c = hist[e];
      a.counts[e] = c;
      a.offsets[e] = off;
      a.poffsets[e] = poff;
      if (c > 0) a.active[na++] = e;
      off += c;
      poff += (c + 7) & ~7;
    }
    a.offsets[a.E] = off;
    a.poffsets[a.E] = poff;
    a.n_active[0] = na;
    *a.ticket = 0;
  }
  __syncthreads();
  for (int t = threadIdx.x; t < a.E * S; t += blockDim.x) {
    const int e = t / S, sg = t % S;
    const int b0 = min(nb, sg * bpseg), b1 = min(nb, b0 + bpseg);
    int run = a.offsets[e] + seg[t], prun = a.poffsets[e] + seg[t];
    for (int b = b0; b < b1; ++b) {
      const long long i = (long long)b * a.E + e;
      const int c = __ldcg(a.block_counts + i);
      a.block_base[i] = run;
      a.pblock_base[i] = prun;
      run += c;
      prun += c;
    }
  }
}

// grid: (token blocks of route_topk, K slices). Ranks within the block come
// from per-expert token bitmasks; slice 0 writes perm/inv_pos; every CTA
// gathers its K slice of the block's routed rows (bf16 -> fp16) into the
// row-major fp16 activation buffer.
__global__ void __launch_bounds__(kRouteThreads) route_permute_kernel(RouteArgs a) {
  __shared__ unsigned mask[kMaxExperts];
  __shared__ int prow_s[kRouteTokensPerCta * kMaxTopK];
  pdl_wait();
  pdl_trigger();
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) mask[e] = 0u;
  __syncthreads();
  const int t0 = blockIdx.x * kRouteTokensPerCta;
  const int nt = min(kRouteTokensPerCta, a.T - t0);
  for (int i = threadIdx.x; i < nt * a.k; i += blockDim.x) {
    const int tt = i / a.k;
    const int e = a.idx[(long long)(t0 + tt) * a.k + (i % a.k)];
    atomicOr(&mask[e], 1u << tt);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nt * a.k; i += blockDim.x) {
    const int tt = i / a.k, j = i % a.k;
    const int t = t0 + tt;
    const int e = a.idx[(long long)t * a.k + j];
    const int rank = __popc(mask[e] & ((1u << tt) - 1u));
    const long long bi = (long long)blockIdx.x * a.E + e;
    const int ppos = a.pblock_base[bi] + rank;
    prow_s[i] = ppos;
    if (blockIdx.y == 0) {
      a.pslot[ppos] = j;
      a.ptok[ppos] = t;
      const int pos = a.block_base[bi] + rank;
      a.perm_token[pos] = t;
      a.inv_pos[(long long)t * a.k + j] = pos;
      a.pinv[(long long)t * a.k + j] = ppos;
    }
  }
  __syncthreads();
  // gather of this CTA's K slice
  const int Kq = a.K;
  const int ks0 = (int)((long long)Kq * blockIdx.y / gridDim.y), ks1 = (int)((long long)Kq * (blockIdx.y + 1) / gridDim.y);
  {
    // one item = 8 consecutive elements of a routed row
    const int k80 = ks0 / 8, nk8 = ks1 / 8 - k80;
    const int items = nt * a.k * nk8;
    for (int it = threadIdx.x; it < items; it += blockDim.x) {
      const int k8 = k80 + it % nk8;
      const int i = it / nk8;
      const int t = t0 + i / a.k;
      const long long prow = prow_s[i];
      const uint4 raw = *reinterpret_cast<const uint4*>(a.X + (long long)t * Kq + 8 * k8);
      const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&raw);
      uint32_t v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) v[q] = pack_half2(__bfloat162float(b[q].x), __bfloat162float(b[q].y));
      *reinterpret_cast<uint4*>(reinterpret_cast<__half*>(a.act) + prow * a.Kpad + 8 * k8) =
          make_uint4(v[0], v[1], v[2], v[3]);
    }
  }
}

cudaError_t launch_route_topk(const RouteArgs& a, cudaStream_t st, int* launches) {
  const int nb = (a.T + kRouteTokensPerCta - 1) / kRouteTokensPerCta;
  // first kernel of a forward: normally serialized after whatever the stream ran before
  const cudaError_t err = launch_kernel(route_topk_kernel, dim3(nb), dim3(kRouteThreads), 0, st, false, a);
  if (launches) ++*launches;
  return err;
}

cudaError_t launch_route_permute(const RouteArgs& a, cudaStream_t st, int* launches) {
  const int nb = (a.T + kRouteTokensPerCta - 1) / kRouteTokensPerCta;
  // K slices of the gather: enough CTAs to fill the GPU, each slice at least
  // 256 columns wide, and always at least one (K = 128 gives one slice)
  const int gs = std::max(1, std::min(296 / nb, a.K / 256));
  const cudaError_t err = launch_kernel(route_permute_kernel, dim3(nb, gs), dim3(kRouteThreads), 0, st, true, a);
  if (launches) ++*launches;
  return err;
}

int route_num_blocks(int T) { return (T + kRouteTokensPerCta - 1) / kRouteTokensPerCta; }

}  // namespace moeq
