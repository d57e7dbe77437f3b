// Grouped expert GEMM for small per-expert batches (the decode path), on the
// 5th-generation tensor cores with the unpacked weights in TMEM.
//
// The decode matmuls stream weights: every packed code is read once per
// token pass, so the kernel is bound by HBM bandwidth and by the instruction
// work of unpacking. A CTA owns 128 weight rows of one expert (one row per
// TMEM lane) and a group-aligned range of 64-wide K chunks; CTAs are
// persistent and walk the (expert, row block, K split, token pass) tiles.
//   warp 8     producer: per chunk, the 128 rows' packed codes (one contiguous
//              block), at a group's first chunk the group's scale/zero pairs,
//              and the expert's routed activation rows (TMA 2-D boxes of 16
//              rows, no multicast);
//   warps 0-3  unpack: one thread per weight row turns the row's 64 codes into
//              32 fp16 pairs of dequantised weights in registers and stores
//              them into a TMEM buffer, the MMA's A operand;
//   warp 9     allocates TMEM and issues tcgen05.mma kind::f16 with A from
//              TMEM (M = 128 weight rows), B = activations from shared memory
//              (N = tokens, 16 or 32), D in TMEM;
//   warps 4-7  epilogue: the accumulator into fp32 registers; at the end of
//              the tile SwiGLU or fp32 output rows.
// Every hand-off is an mbarrier; a warp's work per chunk is kept to a few
// dozen instructions (ring positions advance incrementally, waits have an
// inlined fast path), since that instruction stream, not the tensor core,
// sets the pace.
//
// Integer codes are dequantised in registers: the exponent-bias unpack gives
// the exact fp16 values P_k + q_k (a small integer offset by a per-position
// power of two), one fp16 subtraction removes P_k exactly and one fp16 FMA
// per pair forms (q - z) s with the group's (s, -z s). Every format then
// stores fp16 weights as A, and one accumulator covers the tile's whole K
// range (this measured faster than per-group accumulators of raw codes with a
// correction MMA per group: fewer MMAs, no per-group accumulator hand-off).
//
// The rank-r compensator is one more 64-wide stage (its own accumulator,
// scale 1): the B factor's row values as A against the U = A x columns stored
// after the activations' K (MiLo abstract: low-rank compensators of the
// quantised experts; TileQ abstract: low-rank terms in the same pass as the
// quantised GEMM).
//
// Outputs: SwiGLU of the gate/up rows 8 lanes apart (W1, fp16 rows of the
// down projection's input), or fp32 partial outputs per K split (W2, summed
// by the combine kernel in a fixed order). Every wait is bounded; a timeout
// sets the status word and the CTA unwinds.
#include <algorithm>

#include "kernels.h"
#include "decode_frag.cuh"
#include "tc.cuh"

namespace moeq {
namespace dk {

constexpr int kDqWarps = 4;
constexpr int kEpWarps = 4;
constexpr int kProdWarp = kDqWarps + kEpWarps, kMmaWarp = kProdWarp + 1;
constexpr int kThreads = 32 * (kMmaWarp + 1);
constexpr int kRows = 128;
constexpr int kMaxStages = 16;  // stage ring depth: as many as about 100 KiB of shared memory hold
constexpr int kSub = 2;         // 64-wide chunks per barrier round (step)
constexpr int kA = 2;           // TMEM A buffers, one per step
constexpr int kAcc = 3;         // TMEM accumulators (a tile's main K range, its compensator stage)
constexpr int kACols = 32;      // per chunk: 32 columns of fp16 weight pairs
constexpr int kAStep = kSub * kACols;
constexpr int kABase = 96;      // accumulators at [0, kAcc * NTOK), A buffers at [96, 256)
constexpr int kTmemCols = 256;
constexpr int kActBox = 16;     // rows per TMA box
static_assert(kABase + kA * kAStep <= kTmemCols, "TMEM rings exceed the allocation");
static_assert(kAcc * 32 <= kABase, "accumulators overlap the A buffers");

// barrier slots (8 bytes each)
constexpr int kBarFull = 0, kBarEmpty = kMaxStages, kBarAFull = 2 * kMaxStages, kBarAEmpty = kBarAFull + kA,
              kBarAccFull = kBarAEmpty + kA, kBarAccFree = kBarAccFull + kAcc, kBarDone = kBarAccFree + kAcc,
              kNumBars = kBarDone + 1;

// code block bytes of a 128-row x 64-k chunk at the largest bitwidth of the block's experts
__host__ __device__ inline int code_bytes(int maxbits) { return maxbits >= 16 ? 16384 : 1024 * maxbits; }
// one chunk's part of a stage: [act NTOK x 128 B][codes][scales 512 B];
// a stage holds kSub of them (one step)
__host__ __device__ inline int sub_stage_bytes(int ntok, int maxbits) {
  const int b = ntok * 128 + code_bytes(maxbits) + 512;
  return (b + 1023) & ~1023;
}
__host__ __device__ inline int stage_bytes(int ntok, int maxbits) { return kSub * sub_stage_bytes(ntok, maxbits); }

// position in a ring of n slots with the phase parity of the current lap
struct RingPos {
  int idx = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ void next(int n) {
    if (++idx == n) {
      idx = 0;
      ph ^= 1u;
    }
  }
};

struct Ctx {
  int n_e, prow0, rb, ks, kc0, nmain, next;
  int tok0;  // first token (within the expert) of this tile's pass of up to NTOK tokens
  // the part of the tile this CTA runs: chunks [ib, ie) of the tile's nmain
  // main chunks and its compensator stage (a whole number of steps); a tile
  // split between two CTAs has a head part (this CTA finishes the tile after
  // adding the other CTA's partial sums) and a tail part (written as partial
  // sums for the head's CTA)
  int ib, ie;
  int head_wait, tail_write;
};

// per-role ring positions, kept across tiles
struct Pos {
  RingPos st;   // stage ring (one stage per step of kSub chunks)
  RingPos rel;  // stage to release (unpack warps: kA steps behind st)
  RingPos ab;   // A buffer ring (one buffer per step)
  RingPos acc;  // accumulator ring (one per group)
  int steps = 0;
};

// group position of chunk i of a tile: first / last chunk of its accumulator group
template <int FMT, int GROUP>
__device__ __forceinline__ void group_pos(const Ctx& c, int i, bool& first, bool& last) {
  if (i >= c.nmain) {
    first = last = true;  // compensator stage
  } else {
    first = i == c.ib;
    last = i == min(c.ie, c.nmain) - 1;
  }
}

template <int NTOK, int FMT, int BITS, int GROUP>
__device__ void producer(const DecodeArgs& a, const BlockDesc& d, const Ctx& c, uint8_t* sm, int stage_b, int cbytes,
                         uint32_t bars, Pos& ps, volatile int* abort_flag) {
  const uint32_t full = bars + 8 * kBarFull, empty = bars + 8 * kBarEmpty;
  const int RB = a.M / kRows;
  constexpr int kBlk = (FMT == FMT_DENSE) ? 16384 : 128 * 8 * BITS;  // bytes of one code block (per plane: 1 KiB)
  const int n_pass = min(NTOK, c.n_e - c.tok0);
  const int nbox = (n_pass + kActBox - 1) / kActBox;
  const int row0 = c.prow0 + c.tok0;
  const uint8_t* codes = (FMT == FMT_BITPLANE) ? d.plane[0] : d.codes;
  const int sub_b = stage_b / kSub;
  const int n = c.ie;
  // the whole warp runs the loop (warp-uniform values); one lane issues the copies
  for (int i0 = c.ib; i0 < n; i0 += kSub, ps.st.next(a.nstages)) {
    if (!__all_sync(0xffffffffu, !*abort_flag && mbar_wait_fast(empty + 8 * ps.st.idx, ps.st.ph ^ 1u, a.status, a.wait_ns))) {
      *abort_flag = 1;
      return;
    }
    const uint32_t fb = full + 8 * ps.st.idx;
    const int nsub = min(kSub, n - i0);
    uint32_t bytes = 0;
    for (int u = 0; u < nsub; ++u) {
      bool first, last;
      group_pos<FMT, GROUP>(c, i0 + u, first, last);
      const bool main = i0 + u < c.nmain;
      bytes += nbox * kActBox * 128;
      if (main) bytes += (FMT == FMT_BITPLANE ? BITS * 1024 : kBlk);
      if (FMT == FMT_INT && main && ((c.kc0 + i0 + u) * 64) % GROUP == 0) bytes += 512;
    }
    if (elect_one()) {
      mbar_expect_tx(fb, bytes);
      for (int u = 0; u < nsub; ++u) {
        const int i = i0 + u;
        bool first, last;
        group_pos<FMT, GROUP>(c, i, first, last);
        const uint32_t st = smem_u32(sm) + ps.st.idx * stage_b + u * sub_b;
        const bool main = i < c.nmain;
        const int kc = c.kc0 + i;
        const bool gfirst = FMT == FMT_INT && main && ((c.kc0 + i) * 64) % GROUP == 0;
        const int kx = main ? kc * 64 : a.K + comp_col_offset(d, c.rb);
        const uint32_t cs = st + NTOK * 128;
        const long long bidx = (long long)kc * RB + c.rb;
        const int g = kc * 64 / GROUP;
        for (int b = 0; b < nbox; ++b) tma_load_2d(st + b * kActBox * 128, &a.tmap_act, kx, row0 + b * kActBox, fb);
        if (main) {
          if constexpr (FMT == FMT_BITPLANE) {
#pragma unroll
            for (int q = 0; q < BITS; ++q) bulk_g2s(cs + q * 1024, d.plane[q] + bidx * 1024, 1024, fb);
          } else {
            bulk_g2s(cs, codes + bidx * kBlk, kBlk, fb);
          }
          if (gfirst) bulk_g2s(cs + cbytes, d.sz + (long long)g * a.M + c.rb * kRows, 512, fb);
        }
      }
    }
    __syncwarp();
  }
}

template <int NTOK, int FMT, int GROUP>
__device__ void mma_issuer(const DecodeArgs& a, const Ctx& c, uint8_t* sm, int stage_b, uint32_t bars, uint32_t tmem,
                           Pos& ps, volatile int* abort_flag) {
  const uint32_t full = bars + 8 * kBarFull;
  const uint32_t afull = bars + 8 * kBarAFull, aempty = bars + 8 * kBarAEmpty;
  const uint32_t accfull = bars + 8 * kBarAccFull, accfree = bars + 8 * kBarAccFree;
  const int n_pass = min(NTOK, c.n_e - c.tok0);
  const uint32_t idesc = idesc_f16(128, (n_pass + 15) & ~15);
  const uint32_t sm0 = smem_u32(sm);
  const int sub_b = stage_b / kSub;
  const int n = c.ie;
  for (int i0 = c.ib; i0 < n; i0 += kSub) {
    const bool ok = !*abort_flag && mbar_wait_fast(full + 8 * ps.st.idx, ps.st.ph, a.status, a.wait_ns) &&
                    mbar_wait_fast(afull + 8 * ps.ab.idx, ps.ab.ph, a.status, a.wait_ns);
    if (!__all_sync(0xffffffffu, ok)) {
      *abort_flag = 1;
      return;
    }
    tc_fence_after();
    const int nsub = min(kSub, n - i0);
    for (int u = 0; u < nsub; ++u) {
      const int i = i0 + u;
      bool first, last;
      group_pos<FMT, GROUP>(c, i, first, last);
      if (first) {
        if (!__all_sync(0xffffffffu,
                        !*abort_flag && mbar_wait_fast(accfree + 8 * ps.acc.idx, ps.acc.ph ^ 1u, a.status, a.wait_ns))) {
          *abort_flag = 1;
          return;
        }
        tc_fence_after();
      }
      const uint32_t bt = sm0 + ps.st.idx * stage_b + u * sub_b;
      const uint32_t acc = tmem + ps.acc.idx * NTOK;
      const uint32_t ta = tmem + kABase + ps.ab.idx * kAStep + u * kACols;
      const uint64_t dact = sw128_desc(bt);
      // the whole warp runs the loop (warp-uniform values); one lane issues
      if (elect_one()) {
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16)
          mma_f16_ts(acc, ta + k16 * 8, dact + 2 * k16, idesc, (!first || k16 > 0) ? 1 : 0);
        if (last) mma_commit(accfull + 8 * ps.acc.idx);
      }
      __syncwarp();
      if (last) ps.acc.next(kAcc);
    }
    // the step's A buffer and stage are read once all its MMAs complete
    if (elect_one()) mma_commit(aempty + 8 * ps.ab.idx);
    __syncwarp();
    ps.st.next(a.nstages);
    ps.ab.next(kA);
  }
}

template <int NTOK, int FMT, int BITS, int GROUP>
__device__ void unpack(const DecodeArgs& a, const BlockDesc& d, const Ctx& c, uint8_t* sm, int stage_b, int cbytes,
                       uint32_t bars, uint32_t tmem, Pos& ps, volatile int* abort_flag) {
  const uint32_t full = bars + 8 * kBarFull, empty = bars + 8 * kBarEmpty;
  const uint32_t afull = bars + 8 * kBarAFull, aempty = bars + 8 * kBarAEmpty;
  const int lane = threadIdx.x & 31;
  const int row = threadIdx.x;  // 0..127 = TMEM lane
  const uint32_t lane_base = (uint32_t)(row & ~31) << 16;
  LutRegs lut;
  if constexpr (FMT == FMT_BITPLANE) lut = load_lut(d.lut, BITS);
  const int RS2 = d.rank / 2;  // compensator column pairs
  const int R = c.rb * kRows + row;
  const int sub_b = stage_b / kSub;
  uint32_t dq_s2 = 0u, dq_n2 = 0u;  // the current group's (s, s) and (-z s, -z s)
  const int n = c.ie;
  for (int i0 = c.ib; i0 < n; i0 += kSub) {
    // warp-uniform waits: every lane reaches the .sync.aligned TMEM stores
    const bool ok = !*abort_flag && mbar_wait_fast(full + 8 * ps.st.idx, ps.st.ph, a.status, a.wait_ns) &&
                    mbar_wait_fast(aempty + 8 * ps.ab.idx, ps.ab.ph ^ 1u, a.status, a.wait_ns);
    if (!__all_sync(0xffffffffu, ok)) {
      *abort_flag = 1;
      return;
    }
    // the MMAs of step (this - kA) are complete: its stage (codes read by
    // these warps, activations read by the MMAs) may be refilled
    if (ps.steps >= kA) {
      if (lane == 0) mbar_arrive(empty + 8 * ps.rel.idx);
      ps.rel.next(a.nstages);
    }
    const int nsub = min(kSub, n - i0);
    for (int u = 0; u < nsub; ++u) {
      const int i = i0 + u;
      bool first, last;
      group_pos<FMT, GROUP>(c, i, first, last);
      const uint32_t ta = tmem + lane_base + kABase + ps.ab.idx * kAStep + u * kACols;
      uint32_t v[32];
      if (i < c.nmain) {
        const uint8_t* cs = sm + ps.st.idx * stage_b + u * sub_b + NTOK * 128;
        if constexpr (FMT == FMT_INT) {
          if (((c.kc0 + i) * 64) % GROUP == 0) {
            const uint32_t sz = lds_u32(smem_u32(cs + cbytes) + 4 * row);
            dq_s2 = prmt(sz, sz, 0x1010u);
            dq_n2 = hmul2u(hneg2u(prmt(sz, sz, 0x3232u)), dq_s2);
          }
          const uint32_t blk = smem_u32(cs);
          uint32_t w0[4], w1[4], r0[16], r1[16];
          lds_half_words_int<BITS>(blk, row, 0, w0);
          lds_half_words_int<BITS>(blk, row, 1, w1);
          int_raw_half<BITS>(w0, r0);
          int_raw_half<BITS>(w1, r1);
          uint32_t d0[16], d1[16];
          int_dequant_half<BITS>(r0, dq_s2, dq_n2, d0);
          int_dequant_half<BITS>(r1, dq_s2, dq_n2, d1);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            v[j] = d0[j];
            v[16 + j] = d1[j];
          }
        } else if constexpr (FMT == FMT_BITPLANE) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t pw[4], r16[16];
            load_half_planes<BITS>(cs, 1024, row, h, pw);
            lut_half<BITS>(pw, lut, r16);
#pragma unroll
            for (int j = 0; j < 16; ++j) v[16 * h + j] = r16[j];
          }
        } else {
#pragma unroll
          for (int qd = 0; qd < 8; ++qd) {
            const uint4 x = reinterpret_cast<const uint4*>(cs + qd * 2048)[row];
            v[4 * qd] = x.x; v[4 * qd + 1] = x.y; v[4 * qd + 2] = x.z; v[4 * qd + 3] = x.w;
          }
        }
      } else {
        // compensator stage: the row's B values (pairs), zero past the rank
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = j < RS2 ? d.brow[(long long)j * a.M + R] : 0u;
      }
      tmem_st32(ta, v);  // includes the wait for the store
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(afull + 8 * ps.ab.idx);
    ps.st.next(a.nstages);
    ps.ab.next(kA);
    ++ps.steps;
  }
}

template <int NTOK, int FMT, int GROUP>
__device__ void epilogue(const DecodeArgs& a, const BlockDesc& d, const Ctx& c, uint32_t bars, uint32_t tmem,
                         Pos& ps, volatile int* abort_flag) {
  const uint32_t accfull = bars + 8 * kBarAccFull, accfree = bars + 8 * kBarAccFree;
  const int lane = threadIdx.x & 31;
  const int row = threadIdx.x - 32 * kDqWarps;  // 0..127 = TMEM lane
  const uint32_t lane_base = (uint32_t)(row & ~31) << 16;
  const int R = c.rb * kRows + row;
  // the part's accumulators: one over its main chunks [ib, min(ie, nmain)),
  // then the compensator's if ie > nmain (both added with weight 1)
  const int nacc = (min(c.ie, c.nmain) > c.ib ? 1 : 0) + (c.ie > c.nmain ? 1 : 0);
  float y[NTOK];
#pragma unroll
  for (int t = 0; t < NTOK; ++t) y[t] = 0.f;
  for (int gi = 0; gi < nacc; ++gi) {
    if (!__all_sync(0xffffffffu, !*abort_flag && mbar_wait_fast(accfull + 8 * ps.acc.idx, ps.acc.ph, a.status, a.wait_ns))) {
      *abort_flag = 1;
      return;
    }
    tc_fence_after();
    uint32_t v[NTOK];
    tmem_ld<NTOK>(tmem + lane_base + ps.acc.idx * NTOK, v);
#pragma unroll
    for (int t = 0; t < NTOK; ++t) y[t] += __uint_as_float(v[t]);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(accfree + 8 * ps.acc.idx);
    ps.acc.next(kAcc);
  }
  // ---- a tile split between two CTAs: the tail part's sums go to the head's
  // CTA, which adds them before the outputs (fixed order: head + tail)
  if (c.tail_write) {
    float* part = a.sk_part + (long long)blockIdx.x * (kRows * 32) + row * NTOK;
#pragma unroll
    for (int t = 0; t < NTOK; t += 4) *reinterpret_cast<float4*>(part + t) = make_float4(y[t], y[t + 1], y[t + 2], y[t + 3]);
    __threadfence();
    named_bar_sync(1, 32 * kEpWarps);
    if (row == 0) st_release_gpu_u32(a.sk_flag + blockIdx.x, a.sk_epoch);
    return;
  }
  if (c.head_wait) {
    const unsigned* flag = a.sk_flag + blockIdx.x + 1;
    if (row == 0) {
      const unsigned long long t0 = clock_cycles();
      while (ld_acquire_gpu_u32(flag) != a.sk_epoch) {
        if ((clock_cycles() - t0) / 2 >= a.wait_ns) {
          atomicOr(a.status, ST_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        __nanosleep(32);
      }
    }
    named_bar_sync(1, 32 * kEpWarps);
    if (*abort_flag) return;
    const float* other = a.sk_part + (long long)(blockIdx.x + 1) * (kRows * 32) + row * NTOK;  // the next CTA's slot
#pragma unroll
    for (int t = 0; t < NTOK; t += 4) {
      const float4 o = __ldcg(reinterpret_cast<const float4*>(other + t));
      y[t] += o.x;
      y[t + 1] += o.y;
      y[t + 2] += o.z;
      y[t + 3] += o.w;
    }
  }
  // ---- outputs: tokens tok0 + t
  const int nt = min(NTOK, c.n_e - c.tok0);
  if (a.mode == MODE_SWIGLU) {
    // gate rows are lanes 16f..16f+7 of each 16-row group, up rows 8 lanes later
    float up[NTOK];
#pragma unroll
    for (int t = 0; t < NTOK; ++t) up[t] = __shfl_down_sync(0xffffffffu, y[t], 8);
    if ((R & 15) < 8) {
      const int col = 8 * (R >> 4) + (R & 7);
#pragma unroll
      for (int t = 0; t < NTOK; ++t) {
        if (t < nt) {
          const float gt = y[t];
          a.zout[(long long)(c.prow0 + c.tok0 + t) * a.ldz + col] = __float2half_rn(gt / (1.f + expf(-gt)) * up[t]);
        }
      }
    }
  } else {
#pragma unroll
    for (int t = 0; t < NTOK; ++t)
      if (t < nt) a.out[c.ks * a.out_ks_stride + (long long)(c.prow0 + c.tok0 + t) * a.M + R] = y[t];
  }
}

template <int NTOK, int FMT, int BITS, int GROUP>
__device__ void decode_tile(const DecodeArgs& a, const BlockDesc& d, const Ctx& c, uint8_t* sm, int stage_b,
                            int cbytes, uint32_t bars, uint32_t tmem, Pos& ps, volatile int* ab) {
  const int warp = threadIdx.x >> 5;
  if (warp < kDqWarps) {
    unpack<NTOK, FMT, BITS, GROUP>(a, d, c, sm, stage_b, cbytes, bars, tmem, ps, ab);
  } else if (warp < kProdWarp) {
    epilogue<NTOK, FMT, GROUP>(a, d, c, bars, tmem, ps, ab);
  } else if (warp == kProdWarp) {
    producer<NTOK, FMT, BITS, GROUP>(a, d, c, sm, stage_b, cbytes, bars, ps, ab);
  } else {
    mma_issuer<NTOK, FMT, GROUP>(a, c, sm, stage_b, bars, tmem, ps, ab);
  }
}

}  // namespace dk

template <int NTOK>
__global__ void __launch_bounds__(dk::kThreads, 2) decode_gemm_kernel(const __grid_constant__ DecodeArgs a,
                                                                        int stage_b, int cbytes) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, as an offset into the shared array
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ __align__(8) unsigned long long bars[dk::kNumBars];
  __shared__ int s_pre[kMaxExperts + 1];
  __shared__ int abort_flag;
  __shared__ uint32_t tmem_slot;
  const uint32_t b0 = smem_u32(bars);
  const uint32_t done_bar = b0 + 8 * dk::kBarDone;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int i = 0; i < a.nstages; ++i) {
      mbar_init(b0 + 8 * (dk::kBarFull + i), 1);                  // producer arrival + tx bytes
      mbar_init(b0 + 8 * (dk::kBarEmpty + i), dk::kDqWarps);      // unpack warps, after the stage's MMAs
    }
    for (int i = 0; i < dk::kA; ++i) {
      mbar_init(b0 + 8 * (dk::kBarAFull + i), dk::kDqWarps);      // A buffer written
      mbar_init(b0 + 8 * (dk::kBarAEmpty + i), 1);                // A buffer read (MMA commit)
    }
    for (int i = 0; i < dk::kAcc; ++i) {
      mbar_init(b0 + 8 * (dk::kBarAccFull + i), 1);               // accumulator complete (MMA commit)
      mbar_init(b0 + 8 * (dk::kBarAccFree + i), dk::kEpWarps);    // accumulator read
    }
    mbar_init(done_bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == dk::kMmaWarp) tmem_alloc(smem_u32(&tmem_slot), dk::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // everything above overlaps the previous kernel's tail
  pdl_wait();
  pdl_trigger();
  // Tiles: per active expert slot, (row block, K split, token pass) with the
  // passes of one (row block, K split) adjacent, so that they run at about the
  // same time and share the weight block through L2. s_pre = exclusive prefix
  // of the token passes (ceil(n_e / NTOK)) over the slots.
  const int RB = a.M / dk::kRows;
  const int per = RB * a.KS;
  const int nact = *a.n_active;
  if (warp == 0) {
    const int lane = threadIdx.x & 31;
    constexpr int kPerLane = kMaxExperts / 32;
    int sum = 0;
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) {
      const int sl = kPerLane * lane + j;
      sum += sl < nact ? (a.counts[a.active[sl]] + NTOK - 1) / NTOK : 0;
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int run = incl - sum;
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) {
      const int sl = kPerLane * lane + j;
      s_pre[sl] = run;
      run += sl < nact ? (a.counts[a.active[sl]] + NTOK - 1) / NTOK : 0;
    }
    if (lane == 31) s_pre[kMaxExperts] = incl;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Each CTA takes a contiguous range of the tiles (passes of one row block
  // and K split adjacent: they reuse its weights from L2). With at least one
  // tile per CTA the ranges are cut at step granularity: CTA b covers
  // [total b / G, total (b + 1) / G) in tile units, and a fractional edge
  // splits that tile at step ceil(r n / G) (r = the remainder, n = the tile's
  // steps), which the two CTAs sharing the tile compute alike. The CTA
  // holding the tile's tail runs it first and hands its sums over; the CTA
  // holding the head runs it last and adds them. With fewer tiles than CTAs,
  // whole tiles only.
  const int total = s_pre[nact] * per;
  volatile int* ab = &abort_flag;
  dk::Pos ps;
  const int G = gridDim.x;
  // (only where whole tiles would leave the busiest CTA over 10% above the mean)
  const bool split = !a.mixed && a.sk_part != nullptr && total >= G &&
                     (long long)((total + G - 1) / G) * G * 10 > 11LL * total;
  const long long P0 = (long long)total * blockIdx.x, P1 = P0 + total;
  const int t_first = (int)(P0 / G), t_last = (int)(P1 / G);
  const int r_first = split ? (int)(P0 % G) : 0, r_last = split ? (int)(P1 % G) : 0;
  const int t_stop = r_last > 0 ? t_last + 1 : t_last;
  const int KC = a.K / 64;
  // blocks that differ between experts (bits, format, group, rank) take the
  // tiles round-robin instead: their costs differ, and contiguous ranges
  // would pile one expert's dear tiles onto a few CTAs
  const bool rr = a.mixed != 0;
  for (int tile = rr ? (int)blockIdx.x : t_first; tile < (rr ? total : t_stop) && !*ab; tile += rr ? G : 1) {
    int lo = 0, hi = nact - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] * per <= tile) lo = mid;
      else hi = mid - 1;
    }
    const int slot = lo;
    const int np = s_pre[slot + 1] - s_pre[slot];
    const int local = tile - s_pre[slot] * per;
    const int e = a.active[slot];
    dk::Ctx c;
    c.n_e = a.counts[e];
    c.prow0 = a.poffsets[e];
    c.tok0 = (local % np) * NTOK;
    c.rb = (local / np) / a.KS;
    c.ks = (local / np) % a.KS;
    const BlockDesc& d = a.experts[e].blk[a.block];
    c.next = (c.ks == 0 && d.rank > 0) ? 1 : 0;
    // the K range of split ks (group-aligned for integer codes)
    if (d.fmt == FMT_INT) {
      const int cpg = max(1, d.group / 64), NG = KC / cpg;
      const int g0 = (int)((long long)NG * c.ks / a.KS), g1 = (int)((long long)NG * (c.ks + 1) / a.KS);
      c.kc0 = g0 * cpg;
      c.nmain = (g1 - g0) * cpg;
    } else {
      c.kc0 = (int)((long long)KC * c.ks / a.KS);
      c.nmain = (int)((long long)KC * (c.ks + 1) / a.KS) - c.kc0;
    }
    const int nch = c.nmain + c.next;
    const int nsteps = (nch + dk::kSub - 1) / dk::kSub;
    const int sb = (tile == t_first && r_first > 0) ? (int)(((long long)r_first * nsteps + G - 1) / G) : 0;
    const int se = (tile == t_last && r_last > 0) ? (int)(((long long)r_last * nsteps + G - 1) / G) : nsteps;
    c.ib = sb * dk::kSub;
    c.ie = min(se * dk::kSub, nch);
    c.tail_write = sb > 0 ? 1 : 0;
    c.head_wait = se < nsteps ? 1 : 0;
    if (c.ib >= c.ie) continue;  // nothing of this tile falls to this CTA
    bool ran = true;
    if (d.fmt == FMT_INT) {
      switch (d.bits * 1000 + d.group) {
        case 2064: dk::decode_tile<NTOK, FMT_INT, 2, 64>(a, d, c, sm, stage_b, cbytes, b0, tmem, ps, ab); break;
        case 2128: dk::decode_tile<NTOK, FMT_INT, 2, 128>(a, d, c, sm, stage_b, cbytes, b0, tmem, ps, ab); break;
        case 3064: dk::decode_tile<NTOK, FMT_INT, 3, 64>(a, d, c, sm, stage_b, cbytes, b0, tmem, ps, ab); break;
        case 3128: dk::decode_tile<NTOK, FMT_INT, 3, 128>(a, d, c, sm, stage_b, cbytes, b0, tmem, ps, ab); break;
        case 4064: dk::decode_tile<NTOK, FMT_INT, 4, 64>(a, d, c, sm, stage_b, cbytes, b0, tmem, ps, ab); break;
        case 4128: dk::decode_tile<NTOK, FMT_INT, 4, 128>(a, d, c, sm, stage_b, cbytes, b0, tmem, ps, ab); break;
        default: ran = false; break;
      }
    } else if (d.fmt == FMT_BITPLANE) {
      switch (d.bits) {
        case 2: dk::decode_tile<NTOK, FMT_BITPLANE, 2, 64>(a, d, c, sm, stage_b, cbytes, b0, tmem, ps, ab); break;
        case 3: dk::decode_tile<NTOK, FMT_BITPLANE, 3, 64>(a, d, c, sm, stage_b, cbytes, b0, tmem, ps, ab); break;
        case 4: dk::decode_tile<NTOK, FMT_BITPLANE, 4, 64>(a, d, c, sm, stage_b, cbytes, b0, tmem, ps, ab); break;
        default: ran = false; break;
      }
    } else if (d.fmt == FMT_DENSE) {
      dk::decode_tile<NTOK, FMT_DENSE, 16, 64>(a, d, c, sm, stage_b, cbytes, b0, tmem, ps, ab);
    } else {
      ran = false;
    }
    if (!ran) {
      if (threadIdx.x == 0) atomicOr(a.status, ST_BOUNDS);
      break;
    }
  }
  if (warp == dk::kProdWarp && (threadIdx.x & 31) == 0) {
    // every issued stage must land before the CTA may exit: walk back over
    // the last nstages fills (a slot never filled in that lap tests complete)
    dk::RingPos p = ps.st;
    for (int k = 0; k < a.nstages; ++k) {
      if (p.idx == 0) {
        p.idx = a.nstages - 1;
        p.ph ^= 1u;
      } else {
        --p.idx;
      }
      if (!mbar_wait_fast(b0 + 8 * (dk::kBarFull + p.idx), p.ph, a.status, kDrainLimitNs)) break;
    }
  }
  if (warp == dk::kMmaWarp && (threadIdx.x & 31) == 0) {
    // every issued MMA must complete before TMEM is released
    mma_commit(done_bar);
    mbar_wait(done_bar, 0, a.status, kDrainLimitNs);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == dk::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, dk::kTmemCols);
  }
}

static int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

int decode_rows_per_cta() { return dk::kRows; }
int decode_ctas() { return 2 * num_sms(); }
int device_sms() { return num_sms(); }

template <int NTOK>
static cudaError_t launch_ntok(const DecodeArgs& a, int maxbits, int grid_y, cudaStream_t st) {
  const int stage_b = dk::stage_bytes(NTOK, maxbits);
  // two CTAs per SM (2 x 256 TMEM columns): each takes about 100 KiB of
  // stages (a stage holds one step of kSub chunks), as deep a ring as fits,
  // to keep enough weight bytes in flight (a stage is released kA steps
  // after its own; kA + 2 stages keep the producer ahead, even for the large
  // dense code blocks, which then leave room for one CTA per SM)
  DecodeArgs b = a;
  b.nstages = std::max(dk::kA + 2, std::min(dk::kMaxStages, (100 * 1024 - 1024) / stage_b));
  const size_t smem = (size_t)b.nstages * stage_b + 1024;
  cudaError_t err = cudaFuncSetAttribute(decode_gemm_kernel<NTOK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  // at most rows / NTOK + (one ragged pass per expert) token passes
  const long long passes = std::min<long long>(a.rows / NTOK + grid_y, a.rows);
  const long long tiles = passes * (a.M / dk::kRows) * a.KS;
  const int grid = (int)std::min<long long>(tiles, 2LL * num_sms());
  return launch_kernel(decode_gemm_kernel<NTOK>, dim3(grid), dim3(dk::kThreads), smem, st, true, b, stage_b,
                       dk::code_bytes(maxbits));
}

cudaError_t launch_decode_gemm(const DecodeArgs& a, int ntok, int maxbits, int grid_y, cudaStream_t st,
                               int* launches) {
  if (launches) ++*launches;
  if (ntok <= 16) return launch_ntok<16>(a, maxbits, grid_y, st);
  return launch_ntok<32>(a, maxbits, grid_y, st);
}

}  // namespace moeq
