// Grouped expert GEMM for small per-expert batches (the decode path).
//
// The layer's matmuls stream weights: every byte of packed codes is read once
// per token pass, so this kernel is bound by HBM bandwidth and by the ALU work
// of unpacking. Each CTA owns 256 weight rows of one expert (8 consumer warps
// x 2 row fragments of 16) and a range of 128-wide K chunks. A producer warp
// moves, per chunk, the 16 row fragments' packed codes (one contiguous range
// in the chunk-major layout), their scales and the expert's activation
// fragments into a 4-stage shared-memory ring with TMA bulk copies (no
// multicast) tracked by mbarriers. Consumer warps unpack and dequantise codes
// in registers straight into mma.m16n8k16 A fragments (weights = M, tokens =
// N = 8 per fragment) and accumulate in fp32. The rank-r compensator enters as
// r extra K columns: the B factor as dense fp16 A fragments against the U = A x
// columns stored after the activations' K (MiLo abstract: low-rank
// compensators of the quantised experts; TileQ abstract: low-rank expert
// terms in the same pass as the quantised GEMM).
//
// Epilogues: SwiGLU of the gate/up pair each thread holds (W1, writes the fp16
// activation fragments of the down projection), or fp32 partial outputs per
// K split (W2, summed by the combine kernel in a fixed order).
#include "kernels.h"
#include "decode_frag.cuh"

namespace moeq {

constexpr int kCWarps = 8;                       // consumer warps
constexpr int kThreads = (kCWarps + 1) * 32;     // + one producer warp
constexpr int kRF = 2;                           // row fragments per consumer warp
constexpr int kFragsPerCta = kCWarps * kRF;      // 16
constexpr int kRowsPerCta = kFragsPerCta * 16;   // 256
constexpr int kStages = 8;
constexpr int kSzBytesPerGroup = kFragsPerCta * 64;  // 16 fragments x 8 lane groups x uint2

__host__ __device__ inline int wbytes_of(int maxbits) { return kFragsPerCta * (maxbits >= 16 ? 4096 : 256 * maxbits); }
__host__ __device__ inline int stage_bytes_of(int nt, int maxbits) {
  return nt * 2048 + wbytes_of(maxbits) + 2 * kSzBytesPerGroup;
}
// as many stages as fit in shared memory (at most kStages, at least 2)
__host__ __device__ inline int stages_of(int nt, int maxbits) {
  const int n = (232448 - 1024) / stage_bytes_of(nt, maxbits);
  return n > kStages ? kStages : (n < 2 ? 2 : n);
}

// Lane words of one row fragment's chunk, from the stage's weight area.
template <int FMT, int BITS>
__device__ __forceinline__ void load_words(const uint8_t* wst, int rl, int lane, uint32_t (&w)[8]) {
  if constexpr (FMT == FMT_INT && BITS == 4) {
    const uint4* p = reinterpret_cast<const uint4*>(wst + rl * 1024);
    const uint4 v0 = p[lane], v1 = p[32 + lane];
    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
    w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
  } else if constexpr (FMT == FMT_INT) {
    const uint8_t* ws = wst + rl * (256 * BITS);
    const uint4 v0 = reinterpret_cast<const uint4*>(ws)[lane];
    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
    if constexpr (BITS == 3) {
      const uint2 h = reinterpret_cast<const uint2*>(ws + 512)[lane];
      w[4] = h.x; w[5] = h.y;
    }
  } else if constexpr (FMT == FMT_BITPLANE) {
#pragma unroll
    for (int p = 0; p < BITS; ++p) {
      const uint2 v = reinterpret_cast<const uint2*>(wst + p * (kFragsPerCta * 256) + rl * 256)[lane];
      w[2 * p] = v.x; w[2 * p + 1] = v.y;
    }
  }
}

// One 128-wide K chunk for the warp's kRF row fragments and NP token tiles
// (NP is the exact number of live tiles: no predicated MMAs).
template <int NP, int NT, int FMT, int BITS, int GROUP>
__device__ __forceinline__ void chunk_compute(const uint8_t* base, int wbytes, int warp, int lane,
                                              const LutRegs& lut, float (&acc)[kRF][NT][4]) {
  const int g = lane >> 2;
  const uint4* as = reinterpret_cast<const uint4*>(base);
  const uint8_t* wst = base + NT * 2048;
  const uint8_t* sst = wst + wbytes;
  uint32_t w[kRF][8];
#pragma unroll
  for (int r = 0; r < kRF; ++r) load_words<FMT, BITS>(wst, warp * kRF + r, lane, w[r]);
  uint32_t sA[kRF], nA[kRF], sB[kRF], nB[kRF];
  uint4 bq[NP];
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    if ((s & 1) == 0) {
#pragma unroll
      for (int t = 0; t < NP; ++t) bq[t] = as[t * 128 + (s >> 1) * 32 + lane];
    }
#pragma unroll
    for (int r = 0; r < kRF; ++r) {
      uint32_t av[4];
      if constexpr (FMT == FMT_INT) {
        if ((16 * s) % GROUP == 0) {
          const int gs = (16 * s) / GROUP;
          const uint2 z2 =
              *reinterpret_cast<const uint2*>(sst + gs * kSzBytesPerGroup + (warp * kRF + r) * 64 + g * 8);
          sA[r] = prmt(z2.x, z2.x, 0x1010u); nA[r] = prmt(z2.x, z2.x, 0x3232u);
          sB[r] = prmt(z2.y, z2.y, 0x1010u); nB[r] = prmt(z2.y, z2.y, 0x3232u);
        }
        uint32_t q[4];
        int_codes<BITS>(w[r], s, q);
        av[0] = hfma2u(q[0], sA[r], nA[r]);
        av[1] = hfma2u(q[1], sB[r], nB[r]);
        av[2] = hfma2u(q[2], sA[r], nA[r]);
        av[3] = hfma2u(q[3], sB[r], nB[r]);
      } else if constexpr (FMT == FMT_BITPLANE) {
        lut_decode<BITS>(plane_codes<BITS>(w[r], s), lut, av);
      } else {
        const uint4 v = reinterpret_cast<const uint4*>(wst + (warp * kRF + r) * 4096)[s * 32 + lane];
        av[0] = v.x; av[1] = v.y; av[2] = v.z; av[3] = v.w;
      }
#pragma unroll
      for (int t = 0; t < NP; ++t)
        mma_16816(acc[r][t], av, (s & 1) ? bq[t].z : bq[t].x, (s & 1) ? bq[t].w : bq[t].y);
    }
  }
}

// rank-r compensator columns: B factor fragments against the U columns
template <int NP, int NT>
__device__ __forceinline__ void ext_compute(const GemmArgs& a, const BlockDesc& d, int rfw, long long tile0,
                                            int lane, float (&acc)[kRF][NT][4]) {
  const int RS = d.rank / 16;
  for (int rs = 0; rs < RS; ++rs) {
    const int kk2 = (a.K >> 5) + (rs >> 1);
    uint32_t b0[NP], b1[NP];
#pragma unroll
    for (int t = 0; t < NP; ++t) {
      const uint4 v = a.act[act_frag_u4(tile0 + t, kk2, a.nt8cap, lane)];
      b0[t] = (rs & 1) ? v.z : v.x;
      b1[t] = (rs & 1) ? v.w : v.y;
    }
#pragma unroll
    for (int r = 0; r < kRF; ++r) {
      const uint4 bv = d.bfrag[((long long)(rfw + r) * RS + rs) * 32 + lane];
      const uint32_t av[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int t = 0; t < NP; ++t) mma_16816(acc[r][t], av, b0[t], b1[t]);
    }
  }
}

#define MOEQ_DISPATCH_NP(NPV, CALL)                                        \
  switch (NPV) {                                                           \
    case 1: { constexpr int NP_ = 1; CALL; } break;                        \
    case 2: if constexpr (NT >= 2) { constexpr int NP_ = 2; CALL; } break; \
    case 3: if constexpr (NT >= 3) { constexpr int NP_ = 3; CALL; } break; \
    case 4: if constexpr (NT >= 4) { constexpr int NP_ = 4; CALL; } break; \
    case 5: if constexpr (NT >= 5) { constexpr int NP_ = 5; CALL; } break; \
    case 6: if constexpr (NT >= 6) { constexpr int NP_ = 6; CALL; } break; \
    case 7: if constexpr (NT >= 7) { constexpr int NP_ = 7; CALL; } break; \
    case 8: if constexpr (NT >= 8) { constexpr int NP_ = 8; CALL; } break; \
    default: break;                                                        \
  }

struct TileCtx {
  int n_e, prow0, rt, ks, kc0, nchunks, ntiles;
};

// producer: one elected thread streams every stage of every token pass
template <int NT, int FMT, int BITS, int GROUP>
__device__ __forceinline__ void produce(const GemmArgs& a, const BlockDesc& d, const TileCtx& c, uint8_t* smem,
                                        int nstages, int stage_b, int wbytes, uint32_t bar0,
                                        volatile int* abort_flag) {
  const int MF = a.M / 16;
  const int rf0 = c.rt * kFragsPerCta;
  const int nfr = min(kFragsPerCta, MF - rf0);
  constexpr int CB = (FMT == FMT_DENSE) ? 4096 : 256 * BITS;
  constexpr int GPC = (FMT == FMT_INT) ? (kChunkK / GROUP) : 0;
  int it = 0;
  for (int pb = 0; pb < c.ntiles && !*abort_flag; pb += NT) {
    const int np = min(NT, c.ntiles - pb);
    const long long tile0 = (long long)(c.prow0 >> 3) + pb;
    for (int ci = 0; ci < c.nchunks; ++ci, ++it) {
      const int slot = it % nstages;
      const uint32_t full = bar0 + 8 * slot, empty = bar0 + 8 * (nstages + slot);
      if (*abort_flag || (it >= nstages && !mbar_wait(empty, ((it / nstages) & 1) ^ 1, a.status))) {
        *abort_flag = 1;
        break;
      }
      const int kc = c.kc0 + ci;
      uint8_t* base = smem + slot * stage_b;
      const uint32_t act_bytes = np * 2048;
      const uint32_t w_bytes = (FMT == FMT_BITPLANE ? BITS * 256 : CB) * nfr;
      const uint32_t sz_bytes = GPC * nfr * 64;
      mbar_expect_tx(full, act_bytes + w_bytes + sz_bytes);
      bulk_g2s(smem_u32(base), a.act + act_frag_u4(tile0, kc * 4, a.nt8cap, 0), act_bytes, full);
      uint8_t* wst = base + NT * 2048;
      if constexpr (FMT == FMT_BITPLANE) {
#pragma unroll
        for (int p = 0; p < BITS; ++p)
          bulk_g2s(smem_u32(wst + p * (kFragsPerCta * 256)),
                   d.codes + p * d.plane_stride + ((long long)kc * MF + rf0) * 256, 256 * nfr, full);
      } else {
        bulk_g2s(smem_u32(wst), d.codes + ((long long)kc * MF + rf0) * CB, CB * nfr, full);
      }
      if constexpr (FMT == FMT_INT) {
        uint8_t* sst = wst + wbytes;
#pragma unroll
        for (int gi = 0; gi < GPC; ++gi)
          bulk_g2s(smem_u32(sst + gi * kSzBytesPerGroup), d.sz + ((long long)(kc * GPC + gi) * MF + rf0) * 16,
                   64 * nfr, full);
      }
    }
  }
  // drain: wait (bounded) until every issued stage has landed before the CTA may exit
  // (matters only when a consumer gave up early)
  for (int k = (it > nstages ? it - nstages : 0); k < it; ++k) {
    if (!mbar_wait(bar0 + 8 * (k % nstages), (k / nstages) & 1, a.status)) return;
  }
}

template <int NT, int FMT, int BITS, int GROUP>
__device__ __forceinline__ void consume(const GemmArgs& a, const BlockDesc& d, const TileCtx& c, uint8_t* smem,
                                        int nstages, int stage_b, int wbytes, uint32_t bar0,
                                        volatile int* abort_flag) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, cc = lane & 3;
  const int MF = a.M / 16;
  const int rfw = c.rt * kFragsPerCta + warp * kRF;
  const bool wvalid = rfw + kRF <= MF;  // M % 128 == 0: both fragments valid or both past M
  LutRegs lut;
  if constexpr (FMT == FMT_BITPLANE) lut = load_lut(d.lut, BITS);
  int it = 0;
  for (int pb = 0; pb < c.ntiles; pb += NT) {
    const int np = min(NT, c.ntiles - pb);
    const long long tile0 = (long long)(c.prow0 >> 3) + pb;
    float acc[kRF][NT][4];
#pragma unroll
    for (int r = 0; r < kRF; ++r)
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[r][t][q] = 0.f;
    for (int ci = 0; ci < c.nchunks; ++ci, ++it) {
      const int slot = it % nstages;
      const uint32_t full = bar0 + 8 * slot, empty = bar0 + 8 * (nstages + slot);
      if (*abort_flag || !mbar_wait(full, (it / nstages) & 1, a.status)) {
        *abort_flag = 1;
        return;
      }
      if (wvalid) {
        const uint8_t* base = smem + slot * stage_b;
        MOEQ_DISPATCH_NP(np, (chunk_compute<NP_, NT, FMT, BITS, GROUP>(base, wbytes, warp, lane, lut, acc)))
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty);
    }
    if (!wvalid) continue;
    if (c.ks == 0 && d.rank > 0) {
      MOEQ_DISPATCH_NP(np, (ext_compute<NP_, NT>(a, d, rfw, tile0, lane, acc)))
    }
#pragma unroll
    for (int r = 0; r < kRF; ++r) {
      const int rf = rfw + r;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        if (t >= np) continue;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int n = (pb + t) * 8 + 2 * cc + h;
          if (n >= c.n_e) continue;
          if (a.mode == MODE_SWIGLU) {
            const float gate = acc[r][t][h], up = acc[r][t][2 + h];
            const float z = gate / (1.f + expf(-gate)) * up;
            a.zout[act_frag_index(c.prow0 + n, 8 * rf + g, a.nt8cap)] = __float2half_rn(z);
          } else {
            float* o = a.out + c.ks * a.out_ks_stride + (long long)(c.prow0 + n) * a.M + 16 * rf + g;
            o[0] = acc[r][t][h];
            o[8] = acc[r][t][2 + h];
          }
        }
      }
    }
  }
}

template <int NT, int FMT, int BITS, int GROUP>
__device__ __forceinline__ void run_tile(const GemmArgs& a, const BlockDesc& d, const TileCtx& c, uint8_t* smem,
                                         int nstages, int stage_b, int wbytes, uint32_t bar0,
                                         volatile int* abort_flag) {
  if (threadIdx.x >= kCWarps * 32) {
    if (threadIdx.x == kCWarps * 32)
      produce<NT, FMT, BITS, GROUP>(a, d, c, smem, nstages, stage_b, wbytes, bar0, abort_flag);
  } else {
    consume<NT, FMT, BITS, GROUP>(a, d, c, smem, nstages, stage_b, wbytes, bar0, abort_flag);
  }
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1) decode_gemm_kernel(GemmArgs a, int nstages, int stage_b, int wbytes) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) unsigned long long bars[2 * kStages];
  __shared__ int abort_flag;
  const int slot = blockIdx.y;
  if (slot >= *a.n_active) return;
  const int e = a.active[slot];
  TileCtx c;
  c.n_e = a.counts[e];
  if (c.n_e <= 0) return;
  c.prow0 = a.poffsets[e];
  c.rt = blockIdx.x / a.KS;
  c.ks = blockIdx.x % a.KS;
  const int KC = a.K / kChunkK;
  c.kc0 = (int)((long long)KC * c.ks / a.KS);
  c.nchunks = (int)((long long)KC * (c.ks + 1) / a.KS) - c.kc0;
  c.ntiles = (c.n_e + 7) >> 3;
  const BlockDesc d = a.experts[e].blk[a.block];
  const uint32_t bar0 = smem_u32(bars);
  if (threadIdx.x == 0) {
    for (int i = 0; i < nstages; ++i) {
      mbar_init(bar0 + 8 * i, 1);                    // full: producer arrival + tx bytes
      mbar_init(bar0 + 8 * (nstages + i), kCWarps);  // empty: one arrival per consumer warp
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* ab = &abort_flag;
  if (d.fmt == FMT_INT) {
    switch (d.bits * 1000 + d.group) {
      case 2064: run_tile<NT, FMT_INT, 2, 64>(a, d, c, smem, nstages, stage_b, wbytes, bar0, ab); return;
      case 2128: run_tile<NT, FMT_INT, 2, 128>(a, d, c, smem, nstages, stage_b, wbytes, bar0, ab); return;
      case 3064: run_tile<NT, FMT_INT, 3, 64>(a, d, c, smem, nstages, stage_b, wbytes, bar0, ab); return;
      case 3128: run_tile<NT, FMT_INT, 3, 128>(a, d, c, smem, nstages, stage_b, wbytes, bar0, ab); return;
      case 4064: run_tile<NT, FMT_INT, 4, 64>(a, d, c, smem, nstages, stage_b, wbytes, bar0, ab); return;
      case 4128: run_tile<NT, FMT_INT, 4, 128>(a, d, c, smem, nstages, stage_b, wbytes, bar0, ab); return;
      default: break;
    }
  } else if (d.fmt == FMT_BITPLANE) {
    switch (d.bits) {
      case 2: run_tile<NT, FMT_BITPLANE, 2, 0>(a, d, c, smem, nstages, stage_b, wbytes, bar0, ab); return;
      case 3: run_tile<NT, FMT_BITPLANE, 3, 0>(a, d, c, smem, nstages, stage_b, wbytes, bar0, ab); return;
      case 4: run_tile<NT, FMT_BITPLANE, 4, 0>(a, d, c, smem, nstages, stage_b, wbytes, bar0, ab); return;
      default: break;
    }
  } else if (d.fmt == FMT_DENSE) {
    run_tile<NT, FMT_DENSE, 16, 0>(a, d, c, smem, nstages, stage_b, wbytes, bar0, ab);
    return;
  }
  if (threadIdx.x == 0) atomicOr(a.status, ST_BOUNDS);
}

int decode_rows_per_cta() { return kRowsPerCta; }

size_t decode_smem_bytes(int nt, int maxbits) { return (size_t)stages_of(nt, maxbits) * stage_bytes_of(nt, maxbits); }

template <int NT>
static cudaError_t launch_nt(const GemmArgs& a, int maxbits, int grid_y, cudaStream_t st) {
  const int stage_b = stage_bytes_of(NT, maxbits);
  const int nstages = stages_of(NT, maxbits);
  const size_t smem = (size_t)nstages * stage_b;
  cudaError_t err = cudaFuncSetAttribute(decode_gemm_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  const int row_tiles = (a.M + kRowsPerCta - 1) / kRowsPerCta;
  dim3 grid(row_tiles * a.KS, grid_y);
  decode_gemm_kernel<NT><<<grid, kThreads, smem, st>>>(a, nstages, stage_b, wbytes_of(maxbits));
  return cudaGetLastError();
}

cudaError_t launch_decode_gemm(const GemmArgs& a, int nt_max, int maxbits, int grid_y, cudaStream_t st,
                               int* launches) {
  if (launches) ++*launches;
  if (nt_max <= 1) return launch_nt<1>(a, maxbits, grid_y, st);
  if (nt_max <= 2) return launch_nt<2>(a, maxbits, grid_y, st);
  if (nt_max <= 4) return launch_nt<4>(a, maxbits, grid_y, st);
  return launch_nt<8>(a, maxbits, grid_y, st);
}

}  // namespace moeq
