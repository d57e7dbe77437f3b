// Routing: top-k softmax per token, per-expert histogram, exclusive scan and a
// stable token permutation (expert-major, token-ascending), plus the gather of
// routed token rows into the activation layout of the expert GEMMs.
//
// Top-k per token follows the routing of the Bandwidth-Efficient Adaptive
// Mixture-of-Experts via Low-Rank Compensation page (abstract: each token has
// k routed experts, of which the Top-n get compensation). Selection compares
// the fp32 logits exactly, ties to the lower expert index; the weights are the
// softmax over the selected logits (or the full softmax, by flag).
//
// route_fused_kernel does all of it in one launch: phase A (top-k and the
// histogram of each 16-token block), the scan by the CTA that finishes phase
// A last, which then publishes a flag, and phase B (ranks, permutation and
// the gather of one (token block, K slice) item at a time) once the flag is
// seen. Its CTAs wait for one another, so the grid is at most one CTA per SM
// and every wait is bounded. route_topk_kernel is phase A plus the scan alone
// (the allocation-free routing entry point).
#include <algorithm>

#include "kernels.h"
#include "common.cuh"

namespace moeq {

constexpr int kRouteTokensPerCta = 16;
constexpr int kRouteThreads = 256;

__device__ __forceinline__ bool better(float a, int ia, float b, int ib) {
  return a > b || (a == b && ia < ib);
}

// Top-k of the tokens of block b (8 warps, 2 tokens each): idx, w to global
// memory, the block's expert histogram into hist (shared, zeroed by the caller).
__device__ void topk_block(const RouteArgs& a, int b, int* hist) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t0 = b * kRouteTokensPerCta;
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
}

// The scan, by the CTA that finished phase A last: totals, offsets, padded
// offsets, the active list and the per-block bases. Thread (e, s) owns a
// contiguous segment of the token blocks of expert e (S segments per
// expert), so long block lists are summed in parallel.
__device__ void scan_blocks(const RouteArgs& a, int nb, int* hist, int* seg) {
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
  // offsets and padded offsets, kept in shared memory for the bases below
  __shared__ int off_s[kMaxExperts + 1], poff_s[kMaxExperts + 1];
  if (threadIdx.x == 0) {
    int off = 0, poff = 0, na = 0;
    for (int e = 0; e < a.E; ++e) {
      const int c = hist[e];
      off_s[e] = off;
      poff_s[e] = poff;
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
    int run = off_s[e] + seg[t], prun = poff_s[e] + seg[t];
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

// grid: ceil(T/16) CTAs of 256 threads. The last CTA to finish (atomic
// ticket) scans the block histograms.
__global__ void __launch_bounds__(kRouteThreads) route_topk_kernel(RouteArgs a) {
  __shared__ int hist[kMaxExperts];
  __shared__ int seg[kMaxExperts > kRouteThreads ? kMaxExperts : kRouteThreads];
  __shared__ int is_last;
  pdl_wait();
  pdl_trigger();
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  topk_block(a, blockIdx.x, hist);
  __syncthreads();
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) a.block_counts[(long long)blockIdx.x * a.E + e] = hist[e];
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(a.ticket, 1) == (int)gridDim.x - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  scan_blocks(a, gridDim.x, hist, seg);
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;\n" ::"l"(p), "r"(v) : "memory");
}

// Phase B item: ranks of block b's routed pairs from per-expert token
// bitmasks, the permutation (slice 0 only), and the gather of chunks
// [c0, c1) of the block's routed rows (bf16 -> fp16).
__device__ void permute_item(const RouteArgs& a, int b, int ks, unsigned* mask, int* prow_s) {
  const int t0 = b * kRouteTokensPerCta;
  const int nt = min(kRouteTokensPerCta, a.T - t0);
  const int rows = nt * a.k;
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) mask[e] = 0u;
  __syncthreads();
  for (int i = threadIdx.x; i < rows; i += blockDim.x) {
    const int tt = i / a.k;
    const int e = __ldcg(a.idx + (long long)(t0 + tt) * a.k + (i % a.k));
    atomicOr(&mask[e], 1u << tt);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < rows; i += blockDim.x) {
    const int tt = i / a.k, j = i % a.k;
    const int t = t0 + tt;
    const int e = __ldcg(a.idx + (long long)t * a.k + j);
    const int rank = __popc(mask[e] & ((1u << tt) - 1u));
    const long long bi = (long long)b * a.E + e;
    const int ppos = __ldcg(a.pblock_base + bi) + rank;
    prow_s[i] = ppos;
    if (ks == 0) {
      a.pslot[ppos] = j;
      a.ptok[ppos] = t;
      const int pos = __ldcg(a.block_base + bi) + rank;
      a.perm_token[pos] = t;
      a.inv_pos[(long long)t * a.k + j] = pos;
      a.pinv[(long long)t * a.k + j] = ppos;
    }
  }
  __syncthreads();
  // gather: one 8-lane group per (row, chunk), 8 columns per lane
  const int KC = a.K / 64;
  const int c0 = (int)((long long)KC * ks / a.gs), c1 = (int)((long long)KC * (ks + 1) / a.gs);
  const int nch = c1 - c0;
  const int total = rows * nch * 8;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // eight rounds' loads are issued before their stores: a CTA (one per SM)
  // then keeps 32 KiB of the gather in flight
  constexpr int kU = 8;
  for (int base0 = warp * 32; base0 < total; base0 += kU * blockDim.x) {
    uint4 raw[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int it = base0 + u * blockDim.x + lane;
      if (it < total) {
        const int pc = it >> 3;
        const int i = pc / nch, c = c0 + pc % nch;
        raw[u] = *reinterpret_cast<const uint4*>(a.X + (long long)(t0 + i / a.k) * a.K + 64 * c + 8 * (it & 7));
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int it = base0 + u * blockDim.x + lane;
      const bool valid = it < total;  // 8-lane groups are all valid or all not (total is a multiple of 8)
      const int q8 = it & 7, pc = it >> 3;
      const int i = valid ? pc / nch : 0, c = c0 + (valid ? pc % nch : 0);
      const long long prow = prow_s[i];
      if (valid) {
        const __nv_bfloat162* bv = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
        uint32_t v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) v[q] = pack_half2(__bfloat162float(bv[q].x), __bfloat162float(bv[q].y));
        *reinterpret_cast<uint4*>(reinterpret_cast<__half*>(a.act) + prow * a.Kpad + 64 * c + 8 * q8) =
            make_uint4(v[0], v[1], v[2], v[3]);
      }
    }
  }
  __syncthreads();
}

// grid: at most one CTA per SM (the CTAs wait for one another), 256 threads.
__global__ void __launch_bounds__(kRouteThreads) route_fused_kernel(RouteArgs a) {
  __shared__ int hist[kMaxExperts];
  __shared__ int seg[kMaxExperts > kRouteThreads ? kMaxExperts : kRouteThreads];
  __shared__ unsigned mask[kMaxExperts];
  __shared__ int prow_s[kRouteTokensPerCta * kMaxTopK];
  __shared__ int is_last, go;
  pdl_wait();
  pdl_trigger();
  // ---- phase A: top-k and block histograms
  for (int b = blockIdx.x; b < a.nb; b += gridDim.x) {
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    topk_block(a, b, hist);
    __syncthreads();
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) a.block_counts[(long long)b * a.E + e] = hist[e];
    __syncthreads();
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(a.ticket, 1) == (int)gridDim.x - 1);
  __syncthreads();
  if (is_last) {
    __threadfence();
    scan_blocks(a, a.nb, hist, seg);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) st_release_gpu(a.flag, (int)a.epoch);
  }
  // ---- every CTA waits for the scan (bounded)
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned long long t0 = clock_cycles();
    while (ld_acquire_gpu(a.flag) != (int)a.epoch) {
      if ((clock_cycles() - t0) / 2 >= a.wait_ns) {
        atomicOr(a.status, ST_TIMEOUT);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    go = ok;
  }
  __syncthreads();
  if (!go) return;
  // ---- phase B: permutation, gather
  for (int item = blockIdx.x; item < a.nb * a.gs; item += gridDim.x)
    permute_item(a, item / a.gs, item % a.gs, mask, prow_s);
}

int route_num_blocks(int T) { return (T + kRouteTokensPerCta - 1) / kRouteTokensPerCta; }

int route_gather_slices(int T, int K) {
  // K slices of the gather: enough items to spread over the GPU, each slice
  // at least four 64-column chunks, and always at least one
  const int nb = route_num_blocks(T);
  return std::max(1, std::min(296 / nb, K / 256));
}

cudaError_t launch_route_topk(const RouteArgs& a, cudaStream_t st, int* launches) {
  const int nb = route_num_blocks(a.T);
  // first kernel of a forward: normally serialized after whatever the stream ran before
  const cudaError_t err = launch_kernel(route_topk_kernel, dim3(nb), dim3(kRouteThreads), 0, st, false, a);
  if (launches) ++*launches;
  return err;
}

cudaError_t launch_route_fused(const RouteArgs& a, int num_sms, cudaStream_t st, int* launches) {
  // every CTA must be resident at once: at most one per SM. Programmatic
  // launch: the CTAs may be placed while the stream's previous kernel (the
  // last forward's combine) drains; they write nothing before pdl_wait()
  const int grid = std::max(1, std::min(num_sms, a.nb * a.gs));
  const cudaError_t err = launch_kernel(route_fused_kernel, dim3(grid), dim3(kRouteThreads), 0, st, true, a);
  if (launches) ++*launches;
  return err;
}

}  // namespace moeq
