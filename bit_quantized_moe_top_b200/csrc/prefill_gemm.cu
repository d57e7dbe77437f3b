// Grouped expert GEMM for large per-expert batches (the prefill path), on the
// 5th-generation tensor cores.
//
// One CTA computes, for one expert, 256 weight rows (16 row fragments of the
// chunk-major code layout) against up to 256 routed tokens (two 128-row
// tiles), over the whole K plus the compensator columns. Warp roles:
//   warp 0     TMA producer: activation tiles (2-D tensor map, 128-byte
//              swizzle, no multicast) and packed code chunks + scales (bulk
//              copies);
//   warp 1     allocates 512 TMEM columns and (one thread) issues
//              tcgen05.mma kind::f16, M=128 (tokens) x N=256 (weight rows) x
//              K=16, accumulating both token tiles in TMEM;
//   warps 2-9  dequantise codes into fp16 weight tiles in shared memory, laid
//              out K-major with the 128-byte swizzle the MMA descriptor reads,
//              then run the epilogue (TMEM -> registers -> SwiGLU -> fp16
//              rows of the down projection's input, or fp32 output rows).
// The rank-r compensator is one more 64-wide K stage: the B factor (dense
// fp16) against the U = A x columns stored after the activations' K
// (MiLo abstract: low-rank compensators of the quantised experts).
// Every wait is bounded; on a timeout the CTA sets the status word, drains its
// copies, frees its TMEM and returns.
#include <cuda.h>

#include "kernels.h"
#include "decode_frag.cuh"
#include "tc.cuh"

namespace moeq {

namespace pf {

constexpr int kThreads = 320;      // 10 warps
constexpr int kDqWarps = 8;        // dequant / epilogue warps (2..9)
constexpr int kBN = 256;           // weight rows per CTA
constexpr int kFr = kBN / 16;      // row fragments per CTA
constexpr int kBK = 64;            // K per stage (one 128-byte swizzle atom of fp16)
constexpr int kTileM = 128;        // tokens per accumulator
constexpr int kSA = 3, kSB = 2, kSC = 3;
constexpr int kATile = kTileM * kBK * 2;       // 16 KiB
constexpr int kASlot = 2 * kATile;             // 32 KiB
constexpr int kBSlot = kBN * kBK * 2;          // 32 KiB
constexpr int kCSlot = 2 * 4096 + 1024;        // two 128-row code blocks (<= 4 bits) + scales, 9 KiB
constexpr int kSmemA = 0;
constexpr int kSmemB = kSmemA + kSA * kASlot;
constexpr int kSmemC = kSmemB + kSB * kBSlot;
constexpr int kSmemBar = kSmemC + kSC * kCSlot;
constexpr int kNumBars = 2 * kSA + 2 * kSB + 2 * kSC + 1;
constexpr int kSmemTotal = kSmemBar + kNumBars * 8 + 16;
constexpr int kSmemAlloc = kSmemTotal + 1024;  // slack to align the base to 1024 B

constexpr uint32_t kIdesc = idesc_f16(kTileM, kBN);

struct Ctx {
  int e, n_e, prow0, rt, pair, ntile_live, nk;  // nk: 64-wide stages incl. the compensator stage
  int KC;
};

template <int FMT, int BITS, int GROUP>
__device__ void producer(const PrefillArgs& a, const BlockDesc& d, const Ctx& c, uint8_t* sm, uint32_t bars,
                         volatile int* abort_flag) {
  const uint32_t a_full = bars, a_empty = bars + 8 * kSA;
  const uint32_t c_full = bars + 8 * (2 * kSA + 2 * kSB), c_empty = c_full + 8 * kSC;
  const int RB = a.M / 128;
  const int rb0 = c.rt * 2;
  const int nrb = min(2, RB - rb0);
  constexpr int kBlk = 128 * 8 * BITS;  // bytes of one 128-row code block (per plane: 1 KiB)
  const int row0 = c.prow0 + c.pair * 2 * kTileM;
  int issued_a = 0, issued_c = 0;
  for (int i = 0; i < c.nk && !*abort_flag; ++i) {
    // code blocks + scales of stage i (main K only)
    if (i < c.KC) {
      const int slot = i % kSC;
      if (i >= kSC && !mbar_wait(c_empty + 8 * slot, ((i / kSC) & 1) ^ 1, a.status, a.wait_ns)) {
        *abort_flag = 1;
        break;
      }
      uint8_t* cs = sm + kSmemC + slot * kCSlot;
      const long long bidx = (long long)i * RB + rb0;
      const uint32_t wb = (FMT == FMT_BITPLANE ? BITS * 1024 : kBlk) * nrb;
      mbar_expect_tx(c_full + 8 * slot, wb + (FMT == FMT_INT ? 512 * nrb : 0));
      if constexpr (FMT == FMT_BITPLANE) {
#pragma unroll
        for (int p = 0; p < BITS; ++p)
          bulk_g2s(smem_u32(cs + p * 2048), d.plane[p] + bidx * 1024, 1024 * nrb, c_full + 8 * slot);
      } else {
        bulk_g2s(smem_u32(cs), d.codes + bidx * kBlk, kBlk * nrb, c_full + 8 * slot);
      }
      if constexpr (FMT == FMT_INT)
        bulk_g2s(smem_u32(cs + 8192), d.sz + (long long)(i * 64 / GROUP) * a.M + rb0 * 128, 512 * nrb,
                 c_full + 8 * slot);
      ++issued_c;
    }
    // activation tiles of stage i
    {
      const int slot = i % kSA;
      if (i >= kSA && !mbar_wait(a_empty + 8 * slot, ((i / kSA) & 1) ^ 1, a.status, a.wait_ns)) {
        *abort_flag = 1;
        break;
      }
      mbar_expect_tx(a_full + 8 * slot, c.ntile_live * kATile);
      // the compensator stage (i == KC) reads the row tile's columns after K
      const int kx = i < c.KC ? i * kBK : a.K + comp_col_offset(d, rb0);
      for (int t = 0; t < c.ntile_live; ++t)
        tma_load_2d(smem_u32(sm + kSmemA + slot * kASlot + t * kATile), &a.tmap_act, kx, row0 + t * kTileM,
                    a_full + 8 * slot);
      ++issued_a;
    }
  }
  // drain: every issued copy must land before the CTA may exit
  for (int k = max(0, issued_a - kSA); k < issued_a; ++k)
    if (!mbar_wait(a_full + 8 * (k % kSA), (k / kSA) & 1, a.status, kDrainLimitNs)) break;
  for (int k = max(0, issued_c - kSC); k < issued_c; ++k)
    if (!mbar_wait(c_full + 8 * (k % kSC), (k / kSC) & 1, a.status, kDrainLimitNs)) break;
}

__device__ void mma_issuer(const Ctx& c, uint8_t* sm, uint32_t bars, uint32_t tmem, unsigned* status,
                           unsigned long long wait_ns, volatile int* abort_flag) {
  const uint32_t a_full = bars, a_empty = bars + 8 * kSA;
  const uint32_t b_full = bars + 8 * 2 * kSA, b_empty = b_full + 8 * kSB;
  const uint32_t acc_full = bars + 8 * (2 * kSA + 2 * kSB + 2 * kSC);
  for (int i = 0; i < c.nk; ++i) {
    const int sa = i % kSA, sb = i % kSB;
    if (*abort_flag || !mbar_wait(a_full + 8 * sa, (i / kSA) & 1, status, wait_ns) ||
        !mbar_wait(b_full + 8 * sb, (i / kSB) & 1, status, wait_ns)) {
      *abort_flag = 1;
      break;
    }
    tc_fence_after();
    const uint32_t abase = smem_u32(sm + kSmemA + sa * kASlot);
    const uint32_t bbase = smem_u32(sm + kSmemB + sb * kBSlot);
#pragma unroll
    for (int k16 = 0; k16 < kBK / 16; ++k16) {
      const uint64_t bdesc = sw128_desc(bbase + k16 * 32);
      for (int t = 0; t < c.ntile_live; ++t)
        mma_f16_ss(tmem + t * kBN, sw128_desc(abase + t * kATile + k16 * 32), bdesc, kIdesc, (i > 0 || k16 > 0));
    }
    mma_commit(a_empty + 8 * sa);
    mma_commit(b_empty + 8 * sb);
  }
  mma_commit(acc_full);
  // every issued MMA completes before the CTA frees its TMEM, also when the
  // epilogue gave up and will not wait for the accumulators
  mbar_wait(acc_full, 0, status, kDrainLimitNs);
}

template <int FMT, int BITS, int GROUP>
__device__ void dequant_and_epilogue(const PrefillArgs& a, const BlockDesc& d, const Ctx& c, uint8_t* sm,
                                     uint32_t bars, uint32_t tmem, volatile int* abort_flag) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int dw = warp - 2;               // 0..7
  const int t = threadIdx.x - 64;        // weight row of the tile, 0..255
  const uint32_t b_full = bars + 8 * 2 * kSA, b_empty = b_full + 8 * kSB;
  const uint32_t c_full = bars + 8 * (2 * kSA + 2 * kSB), c_empty = c_full + 8 * kSC;
  const uint32_t acc_full = bars + 8 * (2 * kSA + 2 * kSB + 2 * kSC);
  const int RB = a.M / 128;
  const int rb = c.rt * 2 + (t >> 7);    // this thread's 128-row block
  const bool rvalid = rb < RB;
  const int R = c.rt * kBN + t;          // internal row
  const int nfr = min(kFr, a.M / 16 - c.rt * kFr);
  constexpr int kBlk = 128 * 8 * BITS;
  LutRegs lut;
  if constexpr (FMT == FMT_BITPLANE) lut = load_lut(d.lut, BITS);
  const int RS2 = d.rank / 2;
  bool ok = true;
  for (int i = 0; i < c.nk && ok; ++i) {
    const int sb = i % kSB;
    if (*abort_flag || !mbar_wait(b_empty + 8 * sb, ((i / kSB) & 1) ^ 1, a.status, a.wait_ns)) {
      ok = false;
      break;
    }
    uint8_t* bt = sm + kSmemB + sb * kBSlot;
    uint32_t v[32];
    if (i < c.KC) {
      const int cs_slot = i % kSC;
      if (!mbar_wait(c_full + 8 * cs_slot, (i / kSC) & 1, a.status, a.wait_ns)) {
        ok = false;
        break;
      }
      const uint8_t* cs = sm + kSmemC + cs_slot * kCSlot;
      if (rvalid) {
        if constexpr (FMT == FMT_INT) {
          decode_row64<FMT, BITS>(cs + (t >> 7) * kBlk, 0, t & 127, reinterpret_cast<const uint32_t*>(cs + 8192)[t],
                                  lut, v);
        } else {
          decode_row64<FMT, BITS>(cs + (t >> 7) * 1024, 2048, t & 127, 0u, lut, v);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 32; ++q) v[q] = 0u;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(c_empty + 8 * cs_slot);
    } else {
      // compensator stage: the row's B values (pairs), zero past the rank
#pragma unroll
      for (int q = 0; q < 32; ++q) v[q] = (rvalid && q < RS2) ? d.brow[(long long)q * a.M + R] : 0u;
    }
#pragma unroll
    for (int s8 = 0; s8 < 8; ++s8)
      *reinterpret_cast<uint4*>(bt + sw128_off(t, 8 * s8)) = make_uint4(v[4 * s8], v[4 * s8 + 1], v[4 * s8 + 2], v[4 * s8 + 3]);
    fence_proxy_async();
    __syncwarp();
    if (lane == 0) mbar_arrive(b_full + 8 * sb);
  }
  if (!ok) {
    *abort_flag = 1;
    return;
  }
  const int rf0 = c.rt * kFr;
  // ---- epilogue
  if (!mbar_wait(acc_full, 0, a.status, a.wait_ns)) {
    *abort_flag = 1;
    return;
  }
  tc_fence_after();
  const int quarter = warp & 3;        // TMEM lanes 32*quarter .. +31
  const int chalf = dw >> 2;           // column half handled by this warp
  (void)nfr;
  for (int t = 0; t < c.ntile_live; ++t) {
    const int n = c.pair * 2 * kTileM + t * kTileM + quarter * 32 + lane;  // token within the expert
    const bool live = n < c.n_e;
    const long long prow = (long long)c.prow0 + n;
#pragma unroll 1
    for (int f = chalf * 8; f < chalf * 8 + 8; ++f) {
      uint32_t v[16];
      tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + t * kBN + f * 16, v);
      if (!live || f >= nfr) continue;
      const int rf = rf0 + f;
      if (a.mode == MODE_SWIGLU) {
        uint32_t z[4];
#pragma unroll
        for (int i2 = 0; i2 < 4; ++i2) {
          const float g0 = __uint_as_float(v[2 * i2]), g1 = __uint_as_float(v[2 * i2 + 1]);
          const float u0 = __uint_as_float(v[8 + 2 * i2]), u1 = __uint_as_float(v[8 + 2 * i2 + 1]);
          z[i2] = pack_half2(g0 / (1.f + expf(-g0)) * u0, g1 / (1.f + expf(-g1)) * u1);
        }
        *reinterpret_cast<uint4*>(a.zout + prow * a.ldz + 8 * rf) = make_uint4(z[0], z[1], z[2], z[3]);
      } else {
        float4* o = reinterpret_cast<float4*>(a.out + prow * a.M + 16 * rf);
#pragma unroll
        for (int i2 = 0; i2 < 4; ++i2)
          o[i2] = make_float4(__uint_as_float(v[4 * i2]), __uint_as_float(v[4 * i2 + 1]),
                              __uint_as_float(v[4 * i2 + 2]), __uint_as_float(v[4 * i2 + 3]));
      }
    }
  }
}

}  // namespace pf

template <int FMT, int BITS, int GROUP>
__device__ void prefill_tile(const PrefillArgs& a, const BlockDesc& d, const pf::Ctx& c, uint8_t* sm, uint32_t bars,
                             uint32_t tmem, volatile int* ab) {
  const int warp = threadIdx.x >> 5;
  if (warp == 0) {
    if ((threadIdx.x & 31) == 0) pf::producer<FMT, BITS, GROUP>(a, d, c, sm, bars, ab);
  } else if (warp == 1) {
    if ((threadIdx.x & 31) == 0) pf::mma_issuer(c, sm, bars, tmem, a.status, a.wait_ns, ab);
  } else {
    pf::dequant_and_epilogue<FMT, BITS, GROUP>(a, d, c, sm, bars, tmem, ab);
  }
}

__global__ void __launch_bounds__(pf::kThreads, 1) prefill_gemm_kernel(const __grid_constant__ PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, as an offset into the shared array (the compiler
  // then keeps the shared address space and emits shared-memory loads)
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ int abort_flag;
  __shared__ uint32_t tmem_slot;
  pdl_wait();
  pdl_trigger();
  const int slot = blockIdx.z;
  if (slot >= *a.n_active) return;
  pf::Ctx c;
  c.e = a.active[slot];
  c.n_e = a.counts[c.e];
  c.pair = blockIdx.y;
  if (c.pair * 2 * pf::kTileM >= c.n_e) return;
  c.ntile_live = (c.n_e - c.pair * 2 * pf::kTileM) > pf::kTileM ? 2 : 1;
  c.prow0 = a.poffsets[c.e];
  c.rt = blockIdx.x;
  c.KC = a.K / pf::kBK;
  const BlockDesc d = a.experts[c.e].blk[a.block];
  c.nk = a.K / pf::kBK + (d.rank > 0 ? 1 : 0);
  const uint32_t bars = smem_u32(sm + pf::kSmemBar);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int i = 0; i < pf::kSA; ++i) {
      mbar_init(bars + 8 * i, 1);               // a_full
      mbar_init(bars + 8 * (pf::kSA + i), 1);   // a_empty (MMA commit)
    }
    for (int i = 0; i < pf::kSB; ++i) {
      mbar_init(bars + 8 * (2 * pf::kSA + i), pf::kDqWarps);    // b_full
      mbar_init(bars + 8 * (2 * pf::kSA + pf::kSB + i), 1);     // b_empty (MMA commit)
    }
    for (int i = 0; i < pf::kSC; ++i) {
      mbar_init(bars + 8 * (2 * pf::kSA + 2 * pf::kSB + i), 1);                     // c_full
      mbar_init(bars + 8 * (2 * pf::kSA + 2 * pf::kSB + pf::kSC + i), pf::kDqWarps);  // c_empty
    }
    mbar_init(bars + 8 * (2 * pf::kSA + 2 * pf::kSB + 2 * pf::kSC), 1);  // acc_full
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(&tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int* ab = &abort_flag;
  bool ran = true;
  if (d.fmt == FMT_INT) {
    switch (d.bits * 1000 + d.group) {
      case 2064: prefill_tile<FMT_INT, 2, 64>(a, d, c, sm, bars, tmem, ab); break;
      case 2128: prefill_tile<FMT_INT, 2, 128>(a, d, c, sm, bars, tmem, ab); break;
      case 3064: prefill_tile<FMT_INT, 3, 64>(a, d, c, sm, bars, tmem, ab); break;
      case 3128: prefill_tile<FMT_INT, 3, 128>(a, d, c, sm, bars, tmem, ab); break;
      case 4064: prefill_tile<FMT_INT, 4, 64>(a, d, c, sm, bars, tmem, ab); break;
      case 4128: prefill_tile<FMT_INT, 4, 128>(a, d, c, sm, bars, tmem, ab); break;
      default: ran = false; break;
    }
  } else if (d.fmt == FMT_BITPLANE) {
    switch (d.bits) {
      case 2: prefill_tile<FMT_BITPLANE, 2, 0>(a, d, c, sm, bars, tmem, ab); break;
      case 3: prefill_tile<FMT_BITPLANE, 3, 0>(a, d, c, sm, bars, tmem, ab); break;
      case 4: prefill_tile<FMT_BITPLANE, 4, 0>(a, d, c, sm, bars, tmem, ab); break;
      default: ran = false; break;
    }
  } else {
    ran = false;
  }
  if (!ran && threadIdx.x == 0) atomicOr(a.status, ST_BOUNDS);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_prefill_gemm(const PrefillArgs& a, int grid_y, int grid_z, cudaStream_t st, int* launches) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(prefill_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         pf::kSmemAlloc);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int row_tiles = (a.M + pf::kBN - 1) / pf::kBN;
  cudaError_t err = launch_kernel(prefill_gemm_kernel, dim3(row_tiles, grid_y, grid_z), dim3(pf::kThreads),
                                  (size_t)pf::kSmemAlloc, st, true, a);
  if (launches) ++*launches;
  return err;
}

int prefill_smem_bytes() { return pf::kSmemAlloc; }

}  // namespace moeq
