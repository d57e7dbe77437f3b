// Grouped expert GEMM for small per-expert batches (the decode path), on the
// 5th-generation tensor cores with the dequantised weights in TMEM.
//
// The decode matmuls stream weights: every packed code is read once per
// token pass, so the kernel is bound by HBM bandwidth and by the ALU work of
// unpacking. One CTA owns 128 weight rows of one expert (one row per TMEM
// lane) and a range of 64-wide K chunks:
//   warp 4     producer: per chunk, the 128 rows' packed codes (one contiguous
//              block), their scales, and the expert's routed activation rows
//              (TMA 2-D boxes of 16 rows, 128-byte swizzle, no multicast);
//   warps 0-3  one thread per weight row unpacks and dequantises the row's 64
//              codes in registers to fp16 and stores them into a TMEM buffer
//              (tcgen05.st) that is the A operand of the MMA;
//   warp 5     allocates TMEM and issues tcgen05.mma kind::f16 with A from
//              TMEM (M = 128 weight rows), B = activations from shared memory
//              (N = tokens, 16..128), D accumulated in TMEM.
// No accumulator lives in registers, so several CTAs share an SM. The rank-r
// compensator is one more 64-wide stage: the B factor's row values as A
// against the U = A x columns stored after the activations' K (MiLo abstract:
// low-rank compensators of the quantised experts; TileQ abstract: low-rank
// terms in the same pass as the quantised GEMM).
//
// Epilogues (warps 0-3, tcgen05.ld): SwiGLU of the gate/up rows 8 lanes apart
// (W1, fp16 rows of the down projection's input), or fp32 partial outputs per
// K split (W2, summed by the combine kernel in a fixed order). Every wait is
// bounded; a timeout sets the status word and the CTA unwinds.
#include "kernels.h"
#include "decode_frag.cuh"
#include "tc.cuh"

namespace moeq {
namespace dk {

constexpr int kThreads = 192;
constexpr int kRows = 128;
constexpr int kStages = 4;
constexpr int kABufs = 2;
constexpr int kActBox = 16;  // rows per TMA box

__host__ __device__ inline int code_bytes(int maxbits) { return maxbits >= 16 ? 16384 : 4096; }
__host__ __device__ inline int stage_bytes(int ntok, int maxbits) {
  const int b = ntok * 128 + code_bytes(maxbits) + 512;
  return (b + 1023) & ~1023;
}
__host__ __device__ inline int tmem_cols(int ntok) {
  const int need = ntok + kABufs * 32;
  return need <= 32 ? 32 : need <= 64 ? 64 : need <= 128 ? 128 : need <= 256 ? 256 : 512;
}

struct Ctx {
  int n_e, prow0, rb, ks, kc0, nmain, next, npass, cbytes;
};

template <int NTOK, int FMT, int BITS, int GROUP>
__device__ void producer(const DecodeArgs& a, const BlockDesc& d, const Ctx& c, uint8_t* sm, int stage_b,
                         uint32_t bars, volatile int* abort_flag) {
  const uint32_t full = bars, empty = bars + 8 * kStages;
  const int RB = a.M / kRows;
  constexpr int kBlk = (FMT == FMT_DENSE) ? 16384 : 128 * 8 * BITS;  // bytes of one code block (per plane: 1 KiB)
  int it = 0, issued = 0;
  for (int p = 0; p < c.npass && !*abort_flag; ++p) {
    const int n_pass = min(NTOK, c.n_e - p * NTOK);
    const int nbox = (n_pass + kActBox - 1) / kActBox;
    for (int i = 0; i < c.nmain + c.next; ++i, ++it) {
      const int slot = it % kStages;
      if (*abort_flag || (it >= kStages && !mbar_wait(empty + 8 * slot, ((it / kStages) & 1) ^ 1, a.status))) {
        *abort_flag = 1;
        break;
      }
      uint8_t* st = sm + slot * stage_b;
      const bool main = i < c.nmain;
      const int kc = c.kc0 + i;
      uint32_t bytes = nbox * kActBox * 128;
      if (main) bytes += kBlk + (FMT == FMT_INT ? 512 : 0);
      mbar_expect_tx(full + 8 * slot, bytes);
      const int kx = main ? kc * 64 : a.K;
      for (int b = 0; b < nbox; ++b)
        tma_load_2d(smem_u32(st + b * kActBox * 128), &a.tmap_act, kx, c.prow0 + p * NTOK + b * kActBox,
                    full + 8 * slot);
      if (main) {
        uint8_t* cs = st + NTOK * 128;
        const long long bidx = (long long)kc * RB + c.rb;
        if constexpr (FMT == FMT_BITPLANE) {
#pragma unroll
          for (int q = 0; q < BITS; ++q)
            bulk_g2s(smem_u32(cs + q * 1024), d.codes + q * d.plane_stride + bidx * 1024, 1024, full + 8 * slot);
        } else {
          bulk_g2s(smem_u32(cs), d.codes + bidx * kBlk, kBlk, full + 8 * slot);
        }
        if constexpr (FMT == FMT_INT)
          bulk_g2s(smem_u32(cs + c.cbytes), d.sz + (long long)(kc * 64 / GROUP) * a.M + c.rb * kRows, 512,
                   full + 8 * slot);
      }
      ++issued;
    }
  }
  // drain: every issued stage must land before the CTA may exit
  for (int k = max(0, issued - kStages); k < issued; ++k)
    if (!mbar_wait(full + 8 * (k % kStages), (k / kStages) & 1, a.status)) break;
}

template <int NTOK>
__device__ void mma_issuer(const DecodeArgs& a, const Ctx& c, uint8_t* sm, int stage_b, uint32_t bars,
                           uint32_t tmem, volatile int* abort_flag) {
  const uint32_t full = bars, empty = bars + 8 * kStages;
  const uint32_t afull = bars + 16 * kStages, aempty = afull + 8 * kABufs;
  const uint32_t accfull = aempty + 8 * kABufs, dfree = accfull + 8;
  int it = 0;
  for (int p = 0; p < c.npass; ++p) {
    const int n_pass = min(NTOK, c.n_e - p * NTOK);
    const int npad = (n_pass + 15) & ~15;
    const uint32_t idesc = idesc_f16(128, npad);
    if (p > 0 && !mbar_wait(dfree, (p - 1) & 1, a.status)) {  // previous pass's epilogue is done with D
      *abort_flag = 1;
      break;
    }
    bool ok = true;
    for (int i = 0; i < c.nmain + c.next; ++i, ++it) {
      const int slot = it % kStages, buf = it % kABufs;
      if (*abort_flag || !mbar_wait(full + 8 * slot, (it / kStages) & 1, a.status) ||
          !mbar_wait(afull + 8 * buf, (it / kABufs) & 1, a.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t bt = smem_u32(sm + slot * stage_b);
#pragma unroll
      for (int k16 = 0; k16 < 4; ++k16)
        mma_f16_ts(tmem, tmem + NTOK + buf * 32 + k16 * 8, sw128_desc(bt + k16 * 32), idesc, (i > 0 || k16 > 0));
      mma_commit(empty + 8 * slot);
      mma_commit(aempty + 8 * buf);
    }
    mma_commit(accfull);
    if (!ok) {
      *abort_flag = 1;
      break;
    }
  }
}

template <int NTOK, int FMT, int BITS>
__device__ void dequant_epilogue(const DecodeArgs& a, const BlockDesc& d, const Ctx& c, uint8_t* sm, int stage_b,
                                 uint32_t bars, uint32_t tmem, volatile int* abort_flag) {
  const uint32_t full = bars, empty = bars + 8 * kStages;
  const uint32_t afull = bars + 16 * kStages, aempty = afull + 8 * kABufs;
  const uint32_t accfull = aempty + 8 * kABufs, dfree = accfull + 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = threadIdx.x;       // 0..127 = TMEM lane
  const int R = c.rb * kRows + row;  // internal row of the block
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  LutRegs lut;
  if constexpr (FMT == FMT_BITPLANE) lut = load_lut(d.lut, BITS);
  const int RS2 = d.rank / 2;  // compensator column pairs
  int it = 0;
  for (int p = 0; p < c.npass; ++p) {
    const int n_pass = min(NTOK, c.n_e - p * NTOK);
    const int npad = (n_pass + 15) & ~15;
    for (int i = 0; i < c.nmain + c.next; ++i, ++it) {
      const int slot = it % kStages, buf = it % kABufs;
      if (*abort_flag || !mbar_wait(full + 8 * slot, (it / kStages) & 1, a.status) ||
          !mbar_wait(aempty + 8 * buf, ((it / kABufs) & 1) ^ 1, a.status)) {
        *abort_flag = 1;
        return;
      }
      uint32_t v[32];
      if (i < c.nmain) {
        const uint8_t* cs = sm + slot * stage_b + NTOK * 128;
        if constexpr (FMT == FMT_DENSE) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint4 x = reinterpret_cast<const uint4*>(cs + q * 2048)[row];
            v[4 * q] = x.x; v[4 * q + 1] = x.y; v[4 * q + 2] = x.z; v[4 * q + 3] = x.w;
          }
        } else {
          uint32_t w[8];
          uint32_t sz = 0;
          if constexpr (FMT == FMT_INT) {
            load_row_words_int(cs, row, BITS, w);
            sz = reinterpret_cast<const uint32_t*>(cs + c.cbytes)[row];
          } else {
            load_row_planes<BITS>(cs, 1024, row, w);
          }
          decode_row64<FMT, BITS>(w, sz, lut, v);
        }
      } else {
        // compensator stage: the row's B values (pairs), zero past the rank
#pragma unroll
        for (int q = 0; q < 32; ++q) v[q] = q < RS2 ? d.brow[(long long)q * a.M + R] : 0u;
      }
      tmem_st32(tmem + lane_base + NTOK + buf * 32, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(afull + 8 * buf);
        mbar_arrive(empty + 8 * slot);
      }
    }
    // ---- epilogue of pass p
    if (!mbar_wait(accfull, p & 1, a.status)) {
      *abort_flag = 1;
      return;
    }
    tc_fence_after();
    const int tok0 = p * NTOK;
    for (int cb = 0; cb < npad / 16; ++cb) {
      uint32_t acc[16];
      tmem_ld16(tmem + lane_base + cb * 16, acc);
      if (a.mode == MODE_SWIGLU) {
        // gate rows are lanes 16f..16f+7 of each 16-row group, up rows 8 lanes later
        float up[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) up[t] = __shfl_down_sync(0xffffffffu, __uint_as_float(acc[t]), 8);
        if ((R & 15) < 8) {
          const int col = 8 * (R >> 4) + (R & 7);
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const int n = cb * 16 + t;
            if (n < n_pass) {
              const float gt = __uint_as_float(acc[t]);
              a.zout[(long long)(c.prow0 + tok0 + n) * a.ldz + col] = __float2half_rn(gt / (1.f + expf(-gt)) * up[t]);
            }
          }
        }
      } else {
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const int n = cb * 16 + t;
          if (n < n_pass)
            a.out[c.ks * a.out_ks_stride + (long long)(c.prow0 + tok0 + n) * a.M + R] = __uint_as_float(acc[t]);
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(dfree);
  }
}

}  // namespace dk

template <int NTOK, int FMT, int BITS, int GROUP>
__device__ void decode_tile(const DecodeArgs& a, const BlockDesc& d, const dk::Ctx& c, uint8_t* sm, int stage_b,
                            uint32_t bars, uint32_t tmem, volatile int* ab) {
  const int warp = threadIdx.x >> 5;
  if (warp < 4) {
    dk::dequant_epilogue<NTOK, FMT, BITS>(a, d, c, sm, stage_b, bars, tmem, ab);
  } else if (warp == 4) {
    if ((threadIdx.x & 31) == 0) dk::producer<NTOK, FMT, BITS, GROUP>(a, d, c, sm, stage_b, bars, ab);
  } else {
    if ((threadIdx.x & 31) == 0) dk::mma_issuer<NTOK>(a, c, sm, stage_b, bars, tmem, ab);
  }
}

template <int NTOK>
__global__ void __launch_bounds__(dk::kThreads, 1) decode_gemm_kernel(const __grid_constant__ DecodeArgs a,
                                                                        int stage_b, int cbytes) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) unsigned long long bars[2 * dk::kStages + 2 * dk::kABufs + 2];
  __shared__ int abort_flag;
  __shared__ uint32_t tmem_slot;
  const int slot = blockIdx.y;
  if (slot >= *a.n_active) return;
  const int e = a.active[slot];
  dk::Ctx c;
  c.n_e = a.counts[e];
  if (c.n_e <= 0) return;
  c.prow0 = a.poffsets[e];
  c.rb = blockIdx.x / a.KS;
  c.ks = blockIdx.x % a.KS;
  const int KC = a.K / 64;
  c.kc0 = (int)((long long)KC * c.ks / a.KS);
  c.nmain = (int)((long long)KC * (c.ks + 1) / a.KS) - c.kc0;
  const BlockDesc d = a.experts[e].blk[a.block];
  c.next = (c.ks == 0 && d.rank > 0) ? 1 : 0;
  c.npass = (c.n_e + NTOK - 1) / NTOK;
  c.cbytes = cbytes;
  const uint32_t b0 = smem_u32(bars);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int i = 0; i < dk::kStages; ++i) {
      mbar_init(b0 + 8 * i, 1);                  // full: producer arrival + tx bytes
      mbar_init(b0 + 8 * (dk::kStages + i), 5);  // empty: 4 dequant warps + MMA commit
    }
    for (int i = 0; i < dk::kABufs; ++i) {
      mbar_init(b0 + 8 * (2 * dk::kStages + i), 4);               // A buffer written (4 warps)
      mbar_init(b0 + 8 * (2 * dk::kStages + dk::kABufs + i), 1);  // A buffer free (MMA commit)
    }
    mbar_init(b0 + 8 * (2 * dk::kStages + 2 * dk::kABufs), 1);      // accumulator complete
    mbar_init(b0 + 8 * (2 * dk::kStages + 2 * dk::kABufs + 1), 4);  // accumulator drained
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) tmem_alloc(smem_u32(&tmem_slot), dk::tmem_cols(NTOK));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int* ab = &abort_flag;
  bool ran = true;
  if (d.fmt == FMT_INT) {
    switch (d.bits * 1000 + d.group) {
      case 2064: decode_tile<NTOK, FMT_INT, 2, 64>(a, d, c, sm, stage_b, b0, tmem, ab); break;
      case 2128: decode_tile<NTOK, FMT_INT, 2, 128>(a, d, c, sm, stage_b, b0, tmem, ab); break;
      case 3064: decode_tile<NTOK, FMT_INT, 3, 64>(a, d, c, sm, stage_b, b0, tmem, ab); break;
      case 3128: decode_tile<NTOK, FMT_INT, 3, 128>(a, d, c, sm, stage_b, b0, tmem, ab); break;
      case 4064: decode_tile<NTOK, FMT_INT, 4, 64>(a, d, c, sm, stage_b, b0, tmem, ab); break;
      case 4128: decode_tile<NTOK, FMT_INT, 4, 128>(a, d, c, sm, stage_b, b0, tmem, ab); break;
      default: ran = false; break;
    }
  } else if (d.fmt == FMT_BITPLANE) {
    switch (d.bits) {
      case 2: decode_tile<NTOK, FMT_BITPLANE, 2, 64>(a, d, c, sm, stage_b, b0, tmem, ab); break;
      case 3: decode_tile<NTOK, FMT_BITPLANE, 3, 64>(a, d, c, sm, stage_b, b0, tmem, ab); break;
      case 4: decode_tile<NTOK, FMT_BITPLANE, 4, 64>(a, d, c, sm, stage_b, b0, tmem, ab); break;
      default: ran = false; break;
    }
  } else if (d.fmt == FMT_DENSE) {
    decode_tile<NTOK, FMT_DENSE, 16, 64>(a, d, c, sm, stage_b, b0, tmem, ab);
  } else {
    ran = false;
  }
  if (!ran && threadIdx.x == 0) atomicOr(a.status, ST_BOUNDS);
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, dk::tmem_cols(NTOK));
  }
}

int decode_rows_per_cta() { return dk::kRows; }

template <int NTOK>
static cudaError_t launch_ntok(const DecodeArgs& a, int maxbits, int grid_y, cudaStream_t st) {
  const int stage_b = dk::stage_bytes(NTOK, maxbits);
  const size_t smem = (size_t)dk::kStages * stage_b + 1024;
  cudaError_t err = cudaFuncSetAttribute(decode_gemm_kernel<NTOK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid((a.M / dk::kRows) * a.KS, grid_y);
  decode_gemm_kernel<NTOK><<<grid, dk::kThreads, smem, st>>>(a, stage_b, dk::code_bytes(maxbits));
  return cudaGetLastError();
}

cudaError_t launch_decode_gemm(const DecodeArgs& a, int ntok, int maxbits, int grid_y, cudaStream_t st,
                               int* launches) {
  if (launches) ++*launches;
  if (ntok <= 16) return launch_ntok<16>(a, maxbits, grid_y, st);
  if (ntok <= 32) return launch_ntok<32>(a, maxbits, grid_y, st);
  if (ntok <= 64) return launch_ntok<64>(a, maxbits, grid_y, st);
  return launch_ntok<128>(a, maxbits, grid_y, st);
}

}  // namespace moeq
