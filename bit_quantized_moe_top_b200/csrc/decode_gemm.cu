// Grouped expert GEMM for small per-expert batches (the decode path), on the
// 5th-generation tensor cores with the unpacked weights in TMEM.
//
// The decode matmuls stream weights: every packed code is read once per
// token pass, so the kernel is bound by HBM bandwidth as long as the work of
// unpacking and the hand-offs between roles keep up. One CTA per SM owns all
// 512 TMEM columns and, per tile, a pair of 128-row blocks of one expert (one
// weight row per TMEM lane, the two blocks in different columns) over a
// group-aligned range of 64-wide K chunks and one pass of up to NTOK routed
// tokens. CTAs are persistent and walk the (expert, row-block pair, K split,
// token pass) tiles. Roles:
//   warp 8     producer: per chunk, the expert's routed activation rows (TMA
//              2-D boxes of 16 rows, shared by both row blocks), the two
//              blocks' packed codes (one contiguous bulk copy) and, at a
//              group's first chunk, the routed rows' correction columns and
//              the group's scale/zero pairs; a ring of ~16 chunk stages;
//   warps 0-7  unpack + epilogue: warp w owns row block w / 4 and TMEM lanes
//              32 (w % 4) .. +31; per chunk a thread turns its row's 64 codes
//              into 32 fp16 pairs and stores them into a TMEM A buffer (one
//              tcgen05.st); after finishing group g it reads the accumulators
//              of group g - 2 (long complete by then) and adds s * acc into
//              fp32 registers, the scale s having come from the stage with
//              the codes; at the end of the tile it writes SwiGLU or fp32
//              output rows;
//   warp 9     allocates TMEM and issues tcgen05.mma kind::f16 with A from
//              TMEM (M = 128 weight rows per block), B = activations from
//              shared memory (N = tokens, rounded to 16), D in TMEM.
// Every hand-off is an mbarrier; rings: ~16 stages (smem), 4 A buffers and 3
// accumulator sets (TMEM).
//
// Integer codes are not dequantised per weight. The A operand holds the raw
// fp16 values P_k + q_k of the exponent-bias unpack (exact small integers
// offset by a per-position power of two), and each quantisation group g gets
// its own accumulator:
//   acc_g = sum_{k in g} (P_k + q_k) x_k + 1024 (-XP_g) + z_g (-X_g)
//         = sum_{k in g} (q_k - z_g) x_k,
// the two extra terms being one more K = 16 MMA step per group whose A
// columns are (1024, 1024, z_g, z_g) once per 64-wide chunk of the group and
// whose B columns are the routed row's precomputed chunk sums
// XP_c = sum (P_k/1024) x_k and X_c = sum x_k, each split into fp16 value +
// fp16 remainder (XP_g, X_g are the sums of the group's chunks). The epilogue of a group is
// y += s_g * acc_g. Per pair of weights this leaves one or two logic ops and
// no fp16 arithmetic. Bit-plane (LUT) and dense blocks store their fp16
// weight values as A and use one accumulator for the whole K range.
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
// sets the status word and the CTA unwinds after draining its own copies and
// MMAs.
#include <algorithm>

#include "kernels.h"
#include "decode_frag.cuh"
#include "tc.cuh"
#include "corr.cuh"

namespace moeq {
namespace dk {

#ifndef MOE_DECODE_RB
#define MOE_DECODE_RB 2
#endif
constexpr int kRB = MOE_DECODE_RB;            // 128-row blocks per tile (1: two CTAs per SM; 2: one)
constexpr int kCtasPerSm = 2 / kRB;
constexpr int kDqWarps = 4 * kRB;             // unpack + epilogue warps
constexpr int kMmaWarps = kRB;                // one issuing warp per row block: an issuer sustains one
                                              // small-N MMA per ~58 cycles, whatever its N up to 64
constexpr int kProdWarp = kDqWarps, kMmaWarp = kDqWarps + 1;
constexpr int kThreads = 32 * (kMmaWarp + kMmaWarps);
constexpr int kRows = 128;
constexpr int kMaxStages = 24;
constexpr int kA = 4;                         // TMEM A buffers, one per step (chunk)
constexpr int kAcc = 3;                       // accumulator sets (one per group; a set holds both row blocks)
constexpr int kLag = 2;                       // group g's accumulators are read after group g + kLag is unpacked
constexpr int kACols = 40;                    // per row block and chunk: 32 code columns + 8 correction columns
constexpr int kAStep = kRB * kACols;
constexpr int kAccBase = kA * kAStep;         // accumulators after the A buffers
constexpr int kTmemCols = 256 * kRB;
constexpr int kActBox = 16;                   // rows per TMA box
constexpr int kSmemBudget = 200 * 1024 / kCtasPerSm;  // stage ring
constexpr uint32_t kOne1024 = 0x64006400u;    // fp16 pair (1024, 1024)
static_assert(kLag < kAcc, "the accumulator ring must outrun the epilogue lag");
static_assert(kAccBase + kAcc * kRB * 32 <= kTmemCols, "TMEM rings exceed the allocation");

// barrier slots (8 bytes each)
constexpr int kBarFull = 0, kBarEmpty = kMaxStages, kBarAFull = 2 * kMaxStages, kBarAEmpty = kBarAFull + kA,
              kBarAccFull = kBarAEmpty + kA, kBarAccFree = kBarAccFull + kAcc, kBarDone = kBarAccFree + kAcc,
              kNumBars = kBarDone + 1;

// code bytes of one 128-row x 64-k block at the largest bitwidth of the block's experts
__host__ __device__ inline int code_bytes(int maxbits) { return maxbits >= 16 ? 16384 : 1024 * maxbits; }
// one stage (one chunk of both row blocks):
// [act NTOK x 128 B][corr NTOK x 32 B][codes kRB x cbytes][scales kRB x 512 B]
__host__ __device__ inline int stage_bytes(int ntok, int maxbits) {
  const int b = ntok * 160 + kRB * code_bytes(maxbits) + kRB * 512;
  return (b + 1023) & ~1023;
}

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
  int n_e, prow0, rb0, nrb, ks, kc0, nmain, next;  // row blocks rb0 .. rb0 + nrb - 1
  int tok0;  // first token (within the expert) of this tile's pass of up to NTOK tokens
};

// per-role ring positions, kept across tiles
struct Pos {
  RingPos st;   // stage ring (one stage per chunk)
  RingPos rel;  // stage to release (unpack warps: kA steps behind st)
  RingPos ab;   // A buffer ring
  RingPos acc;  // accumulator ring (one set per group)
  int steps = 0;
};

// group position of chunk i of a tile: first / last chunk of its accumulator group
template <int FMT, int GROUP>
__device__ __forceinline__ void group_pos(const Ctx& c, int i, bool& first, bool& last) {
  if (i >= c.nmain) {
    first = last = true;  // compensator stage
  } else if (FMT == FMT_INT) {
    constexpr int cpg = GROUP / 64;
    first = (i % cpg) == 0;
    last = (i % cpg) == cpg - 1;
  } else {
    first = i == 0;
    last = i == c.nmain - 1;
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
  const int rb0 = c.rb0;
  const int n = c.nmain + c.next;
  // the whole warp runs the loop (warp-uniform values); one lane issues the copies
  for (int i = 0; i < n; ++i, ps.st.next(a.nstages)) {
    if (!__all_sync(0xffffffffu,
                    !*abort_flag && mbar_wait_fast(empty + 8 * ps.st.idx, ps.st.ph ^ 1u, a.status, a.wait_ns))) {
      *abort_flag = 1;
      return;
    }
    bool first, last;
    group_pos<FMT, GROUP>(c, i, first, last);
    const bool main = i < c.nmain;
    const bool corr = FMT == FMT_INT && main && first;
    uint32_t bytes = nbox * kActBox * 128;
    if (main) bytes += (FMT == FMT_BITPLANE ? BITS * 1024 : kBlk) * c.nrb;
    if (corr) bytes += nbox * kActBox * 32 + 512 * c.nrb;
    if (elect_one()) {
      const uint32_t fb = full + 8 * ps.st.idx;
      const uint32_t st = smem_u32(sm) + ps.st.idx * stage_b;
      const uint32_t cs = st + NTOK * 160;
      const int kc = c.kc0 + i;
      const int kx = main ? kc * 64 : a.K + comp_col_offset(d, rb0);
      const long long bidx = (long long)kc * RB + rb0;
      mbar_expect_tx(fb, bytes);
      for (int b = 0; b < nbox; ++b) tma_load_2d(st + b * kActBox * 128, &a.tmap_act, kx, row0 + b * kActBox, fb);
      if (main) {
        if constexpr (FMT == FMT_BITPLANE) {
          // plane p of both blocks: 2 KiB at cs + p * 2 KiB (block rb at + rb KiB)
#pragma unroll
          for (int q = 0; q < BITS; ++q) bulk_g2s(cs + q * kRB * 1024, d.plane[q] + bidx * 1024, 1024 * c.nrb, fb);
        } else {
          bulk_g2s(cs, d.codes + bidx * kBlk, kBlk * c.nrb, fb);
        }
        if (corr) {
          const int g = kc * 64 / GROUP;
          for (int b = 0; b < nbox; ++b)
            tma_load_2d(st + NTOK * 128 + b * kActBox * 32, &a.tmap_corr, 16 * g, row0 + b * kActBox, fb);
          bulk_g2s(cs + kRB * cbytes, d.sz + (long long)g * a.M + rb0 * kRows, 512 * c.nrb, fb);
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
  const int n = c.nmain + c.next;
  for (int i = 0; i < n; ++i) {
    const bool ok = !*abort_flag && mbar_wait_fast(full + 8 * ps.st.idx, ps.st.ph, a.status, a.wait_ns) &&
                    mbar_wait_fast(afull + 8 * ps.ab.idx, ps.ab.ph, a.status, a.wait_ns);
    if (!__all_sync(0xffffffffu, ok)) {
      *abort_flag = 1;
      return;
    }
    bool first, last;
    group_pos<FMT, GROUP>(c, i, first, last);
    if (first && !__all_sync(0xffffffffu, !*abort_flag && mbar_wait_fast(accfree + 8 * ps.acc.idx, ps.acc.ph ^ 1u,
                                                                          a.status, a.wait_ns))) {
      *abort_flag = 1;
      return;
    }
    tc_fence_after();
    const uint32_t bt = sm0 + ps.st.idx * stage_b;
    const bool corr = FMT == FMT_INT && i < c.nmain && first;
    const uint64_t dact = sw128_desc(bt), dcorr = sw32_desc(bt + NTOK * 128);
    // the whole warp runs the loop (warp-uniform values); one lane issues,
    // for this warp's row block (a warp whose block is absent only commits)
    const int rb = (threadIdx.x >> 5) - kMmaWarp;
    if (elect_one()) {
      if (rb < c.nrb) {
        const uint32_t acc = tmem + kAccBase + (ps.acc.idx * kRB + rb) * NTOK;
        const uint32_t ta = tmem + ps.ab.idx * kAStep + rb * kACols;
        if (corr) mma_f16_ts(acc, ta + 32, dcorr, idesc, 0);
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16)
          mma_f16_ts(acc, ta + k16 * 8, dact + 2 * k16, idesc, (corr || !first || k16 > 0) ? 1 : 0);
      }
      // the chunk's A buffer and stage are read once its MMAs complete
      mma_commit(aempty + 8 * ps.ab.idx);
      if (last) mma_commit(accfull + 8 * ps.acc.idx);
    }
    __syncwarp();
    if (last) ps.acc.next(kAcc);
    ps.st.next(a.nstages);
    ps.ab.next(kA);
  }
}

// One group's accumulators into y: wait until its MMAs completed, read the
// row's NTOK columns, y += scale * acc, hand the accumulator set back.
template <int NTOK>
__device__ __forceinline__ bool epilogue_group(const DecodeArgs& a, uint32_t bars, uint32_t tmem_row, float scale,
                                               float (&y)[NTOK], Pos& ps, volatile int* abort_flag) {
  const uint32_t accfull = bars + 8 * kBarAccFull, accfree = bars + 8 * kBarAccFree;
  if (!__all_sync(0xffffffffu,
                  !*abort_flag && mbar_wait_fast(accfull + 8 * ps.acc.idx, ps.acc.ph, a.status, a.wait_ns))) {
    *abort_flag = 1;
    return false;
  }
  tc_fence_after();
  uint32_t v[NTOK];
  tmem_ld<NTOK>(tmem_row + ps.acc.idx * kRB * NTOK, v);
#pragma unroll
  for (int t = 0; t < NTOK; ++t) y[t] = fmaf(scale, __uint_as_float(v[t]), y[t]);
  tc_fence_before();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(accfree + 8 * ps.acc.idx);
  ps.acc.next(kAcc);
  return true;
}

template <int NTOK, int FMT, int BITS, int GROUP>
__device__ void unpack_epilogue(const DecodeArgs& a, const BlockDesc& d, const Ctx& c, uint8_t* sm, int stage_b,
                                int cbytes, uint32_t bars, uint32_t tmem, Pos& ps, volatile int* abort_flag) {
  const uint32_t full = bars + 8 * kBarFull, empty = bars + 8 * kBarEmpty;
  const uint32_t afull = bars + 8 * kBarAFull, aempty = bars + 8 * kBarAEmpty;
  constexpr int kBlk = (FMT == FMT_DENSE) ? 16384 : 128 * 8 * BITS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rb = warp >> 2;                           // row block of the pair
  const int row = ((warp & 3) << 5) + lane;           // TMEM lane = row within the block
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const bool rvalid = rb < c.nrb;
  const int R = (c.rb0 + rb) * kRows + row;          // internal row of the block
  LutRegs lut;
  if constexpr (FMT == FMT_BITPLANE) lut = load_lut(d.lut, BITS);
  const int RS2 = d.rank / 2;  // compensator column pairs
  const int n = c.nmain + c.next;
  const uint32_t tmem_acc_row = tmem + lane_base + kAccBase + rb * NTOK;
  const uint32_t sm0 = smem_u32(sm);
  float y[NTOK];
#pragma unroll
  for (int t = 0; t < NTOK; ++t) y[t] = 0.f;
  // scales of the last groups unpacked: sh0 = newest
  float s_cur = 1.f, sh0 = 1.f, sh1 = 1.f, sh2 = 1.f;
  int gdone = 0, gepi = 0;
  for (int i = 0; i < n; ++i) {
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
    bool first, last;
    group_pos<FMT, GROUP>(c, i, first, last);
    const uint32_t ta = tmem + lane_base + ps.ab.idx * kAStep + rb * kACols;
    const uint32_t stg = sm0 + ps.st.idx * stage_b;
    uint32_t v[32];
    if (i < c.nmain) {
      const uint32_t cs = stg + NTOK * 160;
      if constexpr (FMT == FMT_INT) {
        if (first) {
          const uint32_t sz = lds_u32(cs + kRB * cbytes + 4 * (rb * kRows + row));
          s_cur = __half2float(__ushort_as_half((uint16_t)(sz & 0xFFFFu)));
          // (1024, 1024), (z, z) against chunk 0's (-XP_hi, -XP_lo), (-X_hi, -X_lo),
          // and for two-chunk groups again against chunk 1's (zeros otherwise:
          // those slots may hold another expert's sums from an earlier forward)
          const uint32_t zz = prmt(sz, sz, 0x3232u);
          const uint32_t cz[4] = {kOne1024, zz, GROUP > 64 ? kOne1024 : 0u, GROUP > 64 ? zz : 0u};
          tmem_st4_nw(ta + 32, cz);
        }
        const uint32_t blk = cs + rb * kBlk;
        uint32_t w0[4], w1[4];
        lds_half_words_int<BITS>(blk, row, 0, w0);
        lds_half_words_int<BITS>(blk, row, 1, w1);
        uint32_t r0[16], r1[16];
        int_raw_half<BITS>(w0, r0);
        int_raw_half<BITS>(w1, r1);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          v[j] = r0[j];
          v[16 + j] = r1[j];
        }
      } else if constexpr (FMT == FMT_BITPLANE) {
        s_cur = 1.f;
        uint32_t p0[4], p1[4];
        lds_half_planes<BITS>(cs + rb * 1024, kRB * 1024, row, 0, p0);
        lds_half_planes<BITS>(cs + rb * 1024, kRB * 1024, row, 1, p1);
        uint32_t r0[16], r1[16];
        lut_half<BITS>(p0, lut, r0);
        lut_half<BITS>(p1, lut, r1);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          v[j] = r0[j];
          v[16 + j] = r1[j];
        }
      } else {
        s_cur = 1.f;
        const uint32_t blk = cs + rb * kBlk;
#pragma unroll
        for (int qd = 0; qd < 8; ++qd) {
          const uint4 x = lds_v4(blk + qd * 2048 + 16 * row);
          v[4 * qd] = x.x; v[4 * qd + 1] = x.y; v[4 * qd + 2] = x.z; v[4 * qd + 3] = x.w;
        }
      }
    } else {
      // compensator stage: the row's B values (pairs), zero past the rank
      s_cur = 1.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = (rvalid && j < RS2) ? d.brow[(long long)j * a.M + R] : 0u;
    }
    tmem_st32(ta, v);  // includes the wait for the store
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(afull + 8 * ps.ab.idx);
    ps.st.next(a.nstages);
    ps.ab.next(kA);
    ++ps.steps;
    if (last) {
      sh2 = sh1;
      sh1 = sh0;
      sh0 = s_cur;
      ++gdone;
      if (gdone - gepi > kLag) {
        // group gdone - 1 - kLag (scale sh2): its MMAs were issued kLag groups ago
        if (!epilogue_group<NTOK>(a, bars, tmem_acc_row, sh2, y, ps, abort_flag)) return;
        ++gepi;
      }
    }
  }
  // the last groups of the tile
  if (gdone - gepi == 2) {
    if (!epilogue_group<NTOK>(a, bars, tmem_acc_row, sh1, y, ps, abort_flag)) return;
    if (!epilogue_group<NTOK>(a, bars, tmem_acc_row, sh0, y, ps, abort_flag)) return;
  } else if (gdone - gepi == 1) {
    if (!epilogue_group<NTOK>(a, bars, tmem_acc_row, sh0, y, ps, abort_flag)) return;
  }
  // ---- outputs: tokens tok0 + t
  const int nt = min(NTOK, c.n_e - c.tok0);
  if (a.mode == MODE_SWIGLU) {
    // gate rows are lanes 16f..16f+7 of each 16-row group, up rows 8 lanes later
    float up[NTOK];
#pragma unroll
    for (int t = 0; t < NTOK; ++t) up[t] = __shfl_down_sync(0xffffffffu, y[t], 8);
    if (rvalid && (R & 15) < 8) {
      const int col = 8 * (R >> 4) + (R & 7);
#pragma unroll
      for (int t = 0; t < NTOK; ++t) {
        if (t < nt) {
          const float gt = y[t];
          a.zout[(long long)(c.prow0 + c.tok0 + t) * a.ldz + col] = __float2half_rn(gt / (1.f + expf(-gt)) * up[t]);
        }
      }
    }
  } else if (rvalid) {
#pragma unroll
    for (int t = 0; t < NTOK; ++t)
      if (t < nt) a.out[c.ks * a.out_ks_stride + (long long)(c.prow0 + c.tok0 + t) * a.M + R] = y[t];
  }
}

template <int NTOK, int FMT, int BITS, int GROUP>
__device__ void decode_tile(const DecodeArgs& a, const BlockDesc& d, const Ctx& c0, uint8_t* sm, int stage_b,
                            int cbytes, uint32_t bars, uint32_t tmem, Pos& ps, volatile int* ab) {
  // group-aligned K range of this split
  Ctx c = c0;
  const int KC = a.K / 64;
  if constexpr (FMT == FMT_INT) {
    constexpr int cpg = GROUP / 64;
    const int NG = KC / cpg;
    const int g0 = (int)((long long)NG * c.ks / a.KS), g1 = (int)((long long)NG * (c.ks + 1) / a.KS);
    c.kc0 = g0 * cpg;
    c.nmain = (g1 - g0) * cpg;
  } else {
    c.kc0 = (int)((long long)KC * c.ks / a.KS);
    c.nmain = (int)((long long)KC * (c.ks + 1) / a.KS) - c.kc0;
  }
  const int warp = threadIdx.x >> 5;
  if (warp < kDqWarps) {
    unpack_epilogue<NTOK, FMT, BITS, GROUP>(a, d, c, sm, stage_b, cbytes, bars, tmem, ps, ab);
  } else if (warp == kProdWarp) {
    producer<NTOK, FMT, BITS, GROUP>(a, d, c, sm, stage_b, cbytes, bars, ps, ab);
  } else {
    mma_issuer<NTOK, FMT, GROUP>(a, c, sm, stage_b, bars, tmem, ps, ab);
  }
}

}  // namespace dk

template <int NTOK>
__global__ void __launch_bounds__(dk::kThreads, dk::kCtasPerSm) decode_gemm_kernel(const __grid_constant__ DecodeArgs a,
                                                                        int stage_b, int cbytes) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, as an offset into the shared array (the compiler
  // then keeps the shared address space and emits shared-memory loads)
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
      mbar_init(b0 + 8 * (dk::kBarAEmpty + i), dk::kMmaWarps);    // A buffer read (MMA commits)
    }
    for (int i = 0; i < dk::kAcc; ++i) {
      mbar_init(b0 + 8 * (dk::kBarAccFull + i), dk::kMmaWarps);   // accumulators complete (MMA commits)
      mbar_init(b0 + 8 * (dk::kBarAccFree + i), dk::kDqWarps);    // accumulators read
    }
    mbar_init(done_bar, dk::kMmaWarps);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == dk::kMmaWarp) tmem_alloc(smem_u32(&tmem_slot), dk::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (warp < dk::kDqWarps) {
    // correction columns of this warp's A buffers: zeros past the four that
    // each group's first chunk writes
    const uint32_t lb = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t cz[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    for (int b = 0; b < dk::kA; ++b)
      tmem_st8_nw(tmem + lb + b * dk::kAStep + (warp >> 2) * dk::kACols + 32, cz);
    tmem_wait_st();
  }
  // everything above overlaps the previous kernel's tail
  pdl_wait();
  pdl_trigger();
  // Work units: per active expert slot, (token pass, K split, row block),
  // row blocks fastest. Each CTA takes a contiguous, balanced range of units
  // and walks it two adjacent row blocks at a time (one where a pair would
  // leave its range, its expert, pass or split, or straddle a 2D-tiled
  // compensator's row tile). s_pre = exclusive prefix of the token passes
  // (ceil(n_e / NTOK)) over the slots.
  const int RB = a.M / dk::kRows;
  const long long per = (long long)RB * a.KS;
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
  const long long units = (long long)s_pre[nact] * per;
  const long long u_end = units * (blockIdx.x + 1) / gridDim.x;
  volatile int* ab = &abort_flag;
  dk::Pos ps;
  for (long long u = units * blockIdx.x / gridDim.x; u < u_end && !*ab;) {
    int lo = 0, hi = nact - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] * per <= u) lo = mid;
      else hi = mid - 1;
    }
    const int slot = lo;
    const long long local = u - s_pre[slot] * per;
    const int e = a.active[slot];
    dk::Ctx c;
    c.n_e = a.counts[e];
    c.prow0 = a.poffsets[e];
    c.rb0 = (int)(local % RB);
    c.ks = (int)((local / RB) % a.KS);
    c.tok0 = (int)(local / per) * NTOK;
    const BlockDesc& d = a.experts[e].blk[a.block];
    c.nrb = (dk::kRB > 1 && u + 1 < u_end && c.rb0 + 1 < RB &&
             comp_col_offset(d, c.rb0) == comp_col_offset(d, c.rb0 + 1)) ? 2 : 1;
    u += c.nrb;
    c.next = (c.ks == 0 && d.rank > 0) ? 1 : 0;
    c.kc0 = c.nmain = 0;
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
  if (warp >= dk::kMmaWarp && (threadIdx.x & 31) == 0) {
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

// ---------------------------------------------------------------------------
// per-group correction sums (one warp per routed row x group)

__global__ void __launch_bounds__(256) act_corr_kernel(const CorrArgs a) {
  pdl_wait();
  pdl_trigger();
  act_corr_rows(a, blockIdx.y, blockIdx.x, gridDim.x);
}

int act_corr_ctas(int rows_per_expert, int K) {
  const long long items = (long long)rows_per_expert * (K / 64);
  return (int)std::max<long long>(1, std::min<long long>((items + 7) / 8, 256));
}

cudaError_t launch_act_corr(const CorrArgs& a, int rows_per_expert, int grid_y, cudaStream_t st, int* launches) {
  const cudaError_t err =
      launch_kernel(act_corr_kernel, dim3(act_corr_ctas(rows_per_expert, a.K), grid_y), dim3(256), 0, st, true, a);
  if (launches) ++*launches;
  return err;
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
int decode_ctas() { return dk::kCtasPerSm * num_sms(); }
int device_sms() { return num_sms(); }

template <int NTOK>
static cudaError_t launch_ntok(const DecodeArgs& a, int maxbits, int grid_y, cudaStream_t st) {
  const int stage_b = dk::stage_bytes(NTOK, maxbits);
  // a stage ring as deep as the CTA's share of about 200 KiB of shared
  // memory per SM holds, so that enough weight bytes are in flight per SM (a
  // stage is released kA chunks after its own; kA + 2 stages keep the
  // producer ahead even for the large dense code blocks)
  DecodeArgs b = a;
  b.nstages = std::max(dk::kA + 2, std::min(dk::kMaxStages, dk::kSmemBudget / stage_b));
  const size_t smem = (size_t)b.nstages * stage_b + 1024;
  cudaError_t err = cudaFuncSetAttribute(decode_gemm_kernel<NTOK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  // at most rows / NTOK + (one ragged pass per expert) token passes
  const long long passes = std::min<long long>(a.rows / NTOK + grid_y, a.rows);
  const long long units = passes * (a.M / dk::kRows) * a.KS;
  const int grid = (int)std::min<long long>(units, (long long)dk::kCtasPerSm * num_sms());
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
