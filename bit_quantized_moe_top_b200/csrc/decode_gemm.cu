// Grouped expert GEMM for small per-expert batches (the decode path).
//
// The layer's matmuls are weight-streaming: every byte of packed codes is
// read once per token pass, so this kernel is bound by HBM bandwidth. Each CTA
// owns 256 weight rows of one expert (8 warps x 2 row fragments of 16) and a
// range of K chunks; packed codes, scales and the expert's routed activation
// rows move global -> shared with a 4-stage cp.async pipeline (16-byte
// coalesced copies); each warp unpacks and dequantises its codes in registers
// straight into mma.m16n8k16 A fragments (weights = M, tokens = N = 8 per
// fragment) and accumulates in fp32. The rank-r compensator enters as r extra
// K columns: the B factor as dense fp16 A fragments against the U = A x
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

constexpr int kWarps = 8;
constexpr int kRF = 2;
constexpr int kRowsPerCta = kWarps * kRF * 16;
constexpr int kSzBytesPerRf = 2 * 64;  // <= 2 scale groups per chunk (group >= 64)

__host__ __device__ inline int stage_bytes_of(int nt, int maxbits) {
  const int cb = maxbits >= 16 ? 4096 : 256 * maxbits;
  return nt * 2048 + kWarps * kRF * (cb + kSzBytesPerRf);
}
__host__ __device__ inline int stages_of(int maxbits) { return maxbits >= 16 ? 2 : 4; }

// Lane words of one row fragment's chunk, from shared memory.
template <int FMT, int BITS>
__device__ __forceinline__ void load_words(const uint8_t* ws, int lane, uint32_t (&w)[8]) {
  if constexpr (FMT == FMT_INT && BITS == 4) {
    const uint4 v0 = reinterpret_cast<const uint4*>(ws)[lane];
    const uint4 v1 = reinterpret_cast<const uint4*>(ws)[32 + lane];
    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
    w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
  } else if constexpr (FMT == FMT_INT) {
    const uint4 v0 = reinterpret_cast<const uint4*>(ws)[lane];
    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
    if constexpr (BITS == 3) {
      const uint2 h = reinterpret_cast<const uint2*>(ws + 512)[lane];
      w[4] = h.x; w[5] = h.y;
    }
  } else if constexpr (FMT == FMT_BITPLANE) {
#pragma unroll
    for (int p = 0; p < BITS; ++p) {
      const uint2 v = reinterpret_cast<const uint2*>(ws + p * 256)[lane];
      w[2 * p] = v.x; w[2 * p + 1] = v.y;
    }
  }
}

// One 128-wide K chunk for the warp's kRF row fragments and NP token tiles
// (NP is the exact number of live tiles: no predicated MMAs).
template <int NP, int NT, int FMT, int BITS, int GROUP>
__device__ __forceinline__ void chunk_compute(const uint8_t* base, int warp, int lane, int wbytes_rf,
                                              const LutRegs& lut, float (&acc)[kRF][NT][4]) {
  const int g = lane >> 2;
  const uint4* as = reinterpret_cast<const uint4*>(base);
  uint32_t w[kRF][8];
  const uint32_t* ssz[kRF];
#pragma unroll
  for (int r = 0; r < kRF; ++r) {
    const uint8_t* ws = base + NT * 2048 + (warp * kRF + r) * wbytes_rf;
    ssz[r] = reinterpret_cast<const uint32_t*>(base + NT * 2048 + kWarps * kRF * wbytes_rf +
                                               (warp * kRF + r) * kSzBytesPerRf);
    load_words<FMT, BITS>(ws, lane, w[r]);
  }
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
          const uint2 z2 = *reinterpret_cast<const uint2*>(ssz[r] + (gs * 8 + g) * 2);
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
        const uint8_t* ws = base + NT * 2048 + (warp * kRF + r) * wbytes_rf;
        const uint4 v = reinterpret_cast<const uint4*>(ws)[s * 32 + lane];
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
                                            long long kblk, int lane, float (&acc)[kRF][NT][4]) {
  const int RS = d.rank / 16;
  for (int rs = 0; rs < RS; ++rs) {
    const long long kk = (a.K >> 5) + (rs >> 1);
    uint32_t b0[NP], b1[NP];
#pragma unroll
    for (int t = 0; t < NP; ++t) {
      const uint4 v = a.act[((tile0 + t) * kblk + kk) * 32 + lane];
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

#define MOEQ_DISPATCH_NP(NPV, CALL)                 \
  switch (NPV) {                                    \
    case 1: { constexpr int NP_ = 1; CALL; } break; \
    case 2: if constexpr (NT >= 2) { constexpr int NP_ = 2; CALL; } break; \
    case 3: if constexpr (NT >= 3) { constexpr int NP_ = 3; CALL; } break; \
    case 4: if constexpr (NT >= 4) { constexpr int NP_ = 4; CALL; } break; \
    case 5: if constexpr (NT >= 5) { constexpr int NP_ = 5; CALL; } break; \
    case 6: if constexpr (NT >= 6) { constexpr int NP_ = 6; CALL; } break; \
    case 7: if constexpr (NT >= 7) { constexpr int NP_ = 7; CALL; } break; \
    case 8: if constexpr (NT >= 8) { constexpr int NP_ = 8; CALL; } break; \
    default: break;                                 \
  }

template <int NT, int FMT, int BITS, int GROUP>
__device__ __forceinline__ void run_tile(const GemmArgs& a, const BlockDesc& d, uint8_t* smem, int nstages,
                                         int stage_b, int wbytes_rf, int n_e, int prow0, int rt, int ks) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int MF = a.M / 16;
  const int KC = a.K / kChunkK;
  const int kc0 = (int)((long long)KC * ks / a.KS), kc1 = (int)((long long)KC * (ks + 1) / a.KS);
  const int nchunks = kc1 - kc0;
  const int rfw = rt * (kWarps * kRF) + warp * kRF;
  const bool wvalid = rfw + kRF <= MF;  // M % 128 == 0: a warp's fragments are all valid or all past M
  const int ntiles = (n_e + 7) >> 3;
  const long long kblk = a.Kpad_in >> 5;
  constexpr int CB = (FMT == FMT_DENSE) ? 4096 : 256 * BITS;
  constexpr int GPC = (FMT == FMT_INT) ? (kChunkK / GROUP) : 1;
  const int G = (FMT == FMT_INT) ? a.K / GROUP : 1;

  LutRegs lut;
  if constexpr (FMT == FMT_BITPLANE) lut = load_lut(d.lut, BITS);

  for (int pb = 0; pb < ntiles; pb += NT) {
    const int np = min(NT, ntiles - pb);
    const long long tile0 = (long long)(prow0 >> 3) + pb;
    float acc[kRF][NT][4];
#pragma unroll
    for (int r = 0; r < kRF; ++r)
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[r][t][q] = 0.f;

    auto load_stage = [&](int kc, int st) {
      uint8_t* base = smem + st * stage_b;
      uint4* as = reinterpret_cast<uint4*>(base);
      for (int i = threadIdx.x; i < np * 128; i += blockDim.x) {
        const int t = i >> 7, p = i & 127;
        cp_async16(as + t * 128 + p, a.act + ((tile0 + t) * kblk + kc * 4) * 32 + p);
      }
      if (wvalid) {
#pragma unroll
        for (int r = 0; r < kRF; ++r) {
          const int rf = rfw + r;
          uint8_t* ws = base + NT * 2048 + (warp * kRF + r) * wbytes_rf;
          if constexpr (FMT == FMT_BITPLANE) {
            for (int pc = lane; pc < 16 * BITS; pc += 32)
              cp_async16(ws + pc * 16, d.codes + (pc >> 4) * d.plane_stride + ((long long)rf * KC + kc) * 256 +
                                           (pc & 15) * 16);
          } else {
            const uint8_t* src = d.codes + ((long long)rf * KC + kc) * CB;
            for (int pc = lane; pc < CB / 16; pc += 32) cp_async16(ws + pc * 16, src + pc * 16);
          }
          if constexpr (FMT == FMT_INT) {
            uint8_t* ss = base + NT * 2048 + kWarps * kRF * wbytes_rf + (warp * kRF + r) * kSzBytesPerRf;
            const uint8_t* src = reinterpret_cast<const uint8_t*>(d.sz + ((long long)rf * G + kc * GPC) * 16);
            if (lane < GPC * 4) cp_async16(ss + lane * 16, src + lane * 16);
          }
        }
      }
    };

    for (int i = 0; i < nstages - 1; ++i) {
      if (i < nchunks) load_stage(kc0 + i, i);
      cp_async_commit();
    }
    for (int ci = 0; ci < nchunks; ++ci) {
      if (nstages == 4) cp_async_wait<2>();
      else cp_async_wait<0>();
      __syncthreads();
      {
        const int nc = ci + nstages - 1;
        if (nc < nchunks) load_stage(kc0 + nc, nc % nstages);
        cp_async_commit();
      }
      if (wvalid) {
        const uint8_t* base = smem + (ci % nstages) * stage_b;
        MOEQ_DISPATCH_NP(np, (chunk_compute<NP_, NT, FMT, BITS, GROUP>(base, warp, lane, wbytes_rf, lut, acc)))
      }
    }
    cp_async_wait<0>();
    __syncthreads();

    if (ks == 0 && d.rank > 0 && wvalid) {
      MOEQ_DISPATCH_NP(np, (ext_compute<NP_, NT>(a, d, rfw, tile0, kblk, lane, acc)))
    }

    // epilogue
    if (wvalid) {
#pragma unroll
      for (int r = 0; r < kRF; ++r) {
        const int rf = rfw + r;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          if (t >= np) continue;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int n = (pb + t) * 8 + 2 * c + h;
            if (n >= n_e) continue;
            if (a.mode == MODE_SWIGLU) {
              const float gate = acc[r][t][h], up = acc[r][t][2 + h];
              const float z = gate / (1.f + expf(-gate)) * up;
              a.zout[act_frag_index(prow0 + n, 8 * rf + g, a.Kpad_out)] = __float2half_rn(z);
            } else {
              float* o = a.out + ks * a.out_ks_stride + (long long)(prow0 + n) * a.M + 16 * rf + g;
              o[0] = acc[r][t][h];
              o[8] = acc[r][t][2 + h];
            }
          }
        }
      }
    }
  }
}

template <int NT>
__global__ void __launch_bounds__(256) decode_gemm_kernel(GemmArgs a, int nstages, int stage_b, int wbytes_rf) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int slot = blockIdx.y;
  if (slot >= *a.n_active) return;
  const int e = a.active[slot];
  const int n_e = a.counts[e];
  if (n_e <= 0) return;
  const int prow0 = a.poffsets[e];
  const BlockDesc d = a.experts[e].blk[a.block];
  const int rt = blockIdx.x / a.KS, ks = blockIdx.x % a.KS;
  if (d.fmt == FMT_INT) {
    const int key = d.bits * 1000 + d.group;
    switch (key) {
      case 2064: run_tile<NT, FMT_INT, 2, 64>(a, d, smem, nstages, stage_b, wbytes_rf, n_e, prow0, rt, ks); return;
      case 2128: run_tile<NT, FMT_INT, 2, 128>(a, d, smem, nstages, stage_b, wbytes_rf, n_e, prow0, rt, ks); return;
      case 3064: run_tile<NT, FMT_INT, 3, 64>(a, d, smem, nstages, stage_b, wbytes_rf, n_e, prow0, rt, ks); return;
      case 3128: run_tile<NT, FMT_INT, 3, 128>(a, d, smem, nstages, stage_b, wbytes_rf, n_e, prow0, rt, ks); return;
      case 4064: run_tile<NT, FMT_INT, 4, 64>(a, d, smem, nstages, stage_b, wbytes_rf, n_e, prow0, rt, ks); return;
      case 4128: run_tile<NT, FMT_INT, 4, 128>(a, d, smem, nstages, stage_b, wbytes_rf, n_e, prow0, rt, ks); return;
      default: break;
    }
  } else if (d.fmt == FMT_BITPLANE) {
    switch (d.bits) {
      case 2: run_tile<NT, FMT_BITPLANE, 2, 0>(a, d, smem, nstages, stage_b, wbytes_rf, n_e, prow0, rt, ks); return;
      case 3: run_tile<NT, FMT_BITPLANE, 3, 0>(a, d, smem, nstages, stage_b, wbytes_rf, n_e, prow0, rt, ks); return;
      case 4: run_tile<NT, FMT_BITPLANE, 4, 0>(a, d, smem, nstages, stage_b, wbytes_rf, n_e, prow0, rt, ks); return;
      default: break;
    }
  } else if (d.fmt == FMT_DENSE) {
    run_tile<NT, FMT_DENSE, 16, 0>(a, d, smem, nstages, stage_b, wbytes_rf, n_e, prow0, rt, ks);
    return;
  }
  if (threadIdx.x == 0) atomicOr(a.status, ST_BOUNDS);
}

int decode_rows_per_cta() { return kRowsPerCta; }

size_t decode_smem_bytes(int nt, int maxbits) {
  return (size_t)stages_of(maxbits) * stage_bytes_of(nt, maxbits);
}

template <int NT>
static cudaError_t launch_nt(const GemmArgs& a, int maxbits, int grid_y, cudaStream_t st) {
  const int stage_b = stage_bytes_of(NT, maxbits);
  const int nstages = stages_of(maxbits);
  const int wbytes_rf = maxbits >= 16 ? 4096 : 256 * maxbits;
  const size_t smem = (size_t)nstages * stage_b;
  cudaError_t err = cudaFuncSetAttribute(decode_gemm_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  const int row_tiles = (a.M + kRowsPerCta - 1) / kRowsPerCta;
  dim3 grid(row_tiles * a.KS, grid_y);
  decode_gemm_kernel<NT><<<grid, kWarps * 32, smem, st>>>(a, nstages, stage_b, wbytes_rf);
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
