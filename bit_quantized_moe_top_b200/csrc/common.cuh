// Shared device definitions of the quantized MoE layer: internal weight and
// activation layouts, the per-block descriptor, and small PTX helpers.
//
// Internal layouts (all built on the device at weight-load time):
//
//  * Rows of W1 (gate||up, 2N x K) are interleaved per 16-row group: internal
//    row 16f+i is gate row 8f+i for i < 8 and up row 8f+i-8 for i >= 8, so the
//    gate and up values of one SwiGLU column sit 8 rows (8 TMEM lanes) apart.
//  * Codes are stored per 64-wide K chunk kc and 128-row block rb, chunk-major
//    ([kc][rb]), so the rows a CTA streams for one chunk are one contiguous
//    range. Inside a block, row i's 64 codes are two halves of 16 pairs
//    (k = 32h + 2p, 32h + 2p + 1) packed into the words that the decode
//    routines consume (field positions in decode_frag.cuh), stored so that
//    consecutive rows are consecutive 4, 8 or 16-byte units (conflict-free
//    for a thread per row). A block holds 128 * 8 * b bytes (b = bits; 16
//    for dense fp16).
//  * Activations are row-major fp16 [rows, Kpad]: routed rows bucketed per
//    expert, each expert's range padded to a multiple of 8 rows; the rank
//    columns U = A x sit after column K.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

namespace moeq {

constexpr int kChunkK = 128;   // K per code chunk
constexpr int kMaxRank = 64;
constexpr int kMaxTopK = 8;
constexpr int kMaxExperts = 256;

enum : int { FMT_INT = 0, FMT_BITPLANE = 1, FMT_DENSE = 2 };

// device status word bits
enum : unsigned { ST_BOUNDS = 1u, ST_TIMEOUT = 2u, ST_ROUTE = 4u, ST_RANGE = 8u };

// One expert linear block as the kernels see it.
struct BlockDesc {
  const uint8_t* codes;   // code blocks [K/64][M/128][block] (INT / DENSE)
  const uint8_t* plane[4];// BITPLANE: plane p as [K/64][M/128][1 KiB] (null while released to host)
  const uint32_t* sz;     // INT: [K/g][M] half2(s, z), internal row order
  const uint32_t* lut;    // BITPLANE: 28 fp16 as 14 u32
  const uint32_t* brow;   // compensator B as fp16 pairs [r/2][M] (column-pair-major)
  const uint4* afrag;     // compensator A [r, K] as mma A-fragments [r/16][K/16][32] uint4 (fp16)
  int fmt, bits, group, rank;
  int M, K;
  int loaded;
  // 2D-tiled shared compensator (0 = per-expert factors): the compensator
  // activations of internal rows [128 rb, 128 rb + 128) start at column
  // K + (128 rb / tq_span) * tq_cols of the activation rows
  int tq_span, tq_cols;
};

// Column offset, after K, of a 128-row block's compensator activations.
__host__ __device__ __forceinline__ int comp_col_offset(const BlockDesc& d, int rb) {
  return d.tq_span > 0 ? (rb * 128 / d.tq_span) * d.tq_cols : 0;
}

struct ExpertDesc {
  BlockDesc blk[2];
};

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while its predecessor finishes; pdl_wait() blocks
// until every prerequisite grid has completed and its writes are visible (a
// no-op for a normally serialized launch), pdl_trigger() lets the dependent
// grid launch once every CTA of this grid has triggered or exited.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lop3_sel(uint32_t a, uint32_t b, uint32_t m) {
  // (a & m) | (b & ~m)
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xE4;\n" : "=r"(d) : "r"(a), "r"(b), "r"(m));
  return d;
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t m, uint32_t o) {
  // (a & m) | o
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;\n" : "=r"(d) : "r"(a), "r"(m), "r"(o));
  return d;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(s));
  return d;
}

__device__ __forceinline__ uint32_t hsub2u(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t hfma2u(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t hmul2u(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t hneg2u(uint32_t a) { return a ^ 0x80008000u; }

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async8(void* smem, const void* gmem) {
  uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// ---------------------------------------------------------------------------
// layout index helpers (shared by the re-layout kernels and the GEMMs)
// ---------------------------------------------------------------------------

// canonical row of internal row ir of a block (W1 interleaves gate/up per fragment)
__host__ __device__ __forceinline__ int canon_row(int ir, int block, int N) {
  if (block != 0) return ir;
  int f = ir >> 4, i = ir & 15;
  return i < 8 ? 8 * f + i : N + 8 * f + (i - 8);
}

// words per row of one 64-wide chunk (INT: 2*b; dense fp16: 32)
__host__ __device__ __forceinline__ int words_per_row(int fmt, int bits) { return fmt == FMT_DENSE ? 32 : 2 * bits; }
// bytes of one [128-row x 64-k] code block
__host__ __device__ __forceinline__ int block_bytes(int fmt, int bits) { return 128 * 4 * words_per_row(fmt, bits); }

// ---------------------------------------------------------------------------
// mbarrier / bulk-copy helpers (TMA engine, no multicast)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}
// Suspends the thread until the phase completes or ~1 ms passes (suspend-time
// hint), so waiting warps do not spin on the issue slots.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
  return t;
}
// Limit of the waits that drain a CTA's own copies and MMAs before it exits
// (they always complete; the limit only guards against a broken invariant).
constexpr unsigned long long kDrainLimitNs = 2000000000ull;
// Default limit of the hand-off waits between a kernel's roles.
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;

// Non-blocking probe of a phase.
__device__ __forceinline__ bool mbar_probe(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Probe of a phase without a suspend hint: a completed phase returns at once,
// an open one may suspend the thread for a short system-dependent time.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long clock_cycles() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%clock64;\n" : "=l"(t));
  return t;
}
// Limits at least this long may sleep in try_wait; shorter ones poll.
constexpr unsigned long long kSleepLimitNs = 2000000ull;
// Bounded wait: gives up once limit_ns have passed, sets ST_TIMEOUT and
// returns false. Limits far above the suspend hint sleep in try_wait and are
// timed with the global nanosecond timer; shorter ones poll with the
// non-blocking test_wait and are timed in SM clock cycles (two per ns, so at
// most twice the limit at lower clocks), whose resolution, unlike the global
// timer's, also honours limits of a few ns.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned* status,
                                          unsigned long long limit_ns = kDefaultWaitNs) {
  const bool sleep = limit_ns >= kSleepLimitNs;
  if (sleep ? mbar_try_wait(bar, parity) : mbar_probe(bar, parity)) return true;
  const unsigned long long t0 = sleep ? globaltimer_ns() : clock_cycles();
  for (;;) {
    if (sleep ? mbar_try_wait(bar, parity) : mbar_probe(bar, parity)) return true;
    const unsigned long long dt = sleep ? globaltimer_ns() - t0 : (clock_cycles() - t0) / 2;
    if (dt >= limit_ns) {
      atomicOr(status, ST_TIMEOUT);
      return false;
    }
  }
}
// The bounded wait, out of line: only taken when the phase is still open.
static __device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, unsigned* status,
                                                   unsigned long long limit_ns) {
  return mbar_wait(bar, parity, status, limit_ns);
}
// Bounded wait with an inlined fast path (a short limit skips it: the probe
// without a suspend hint could outlast the limit).
__device__ __forceinline__ bool mbar_wait_fast(uint32_t bar, uint32_t parity, unsigned* status,
                                               unsigned long long limit_ns = kDefaultWaitNs) {
  return (limit_ns >= kSleepLimitNs && mbar_test(bar, parity)) || mbar_wait_slow(bar, parity, status, limit_ns);
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ unsigned ld_acquire_gpu_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu_u32(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;\n" ::"l"(p), "r"(v) : "memory");
}
// named barrier id (1..15) over n threads (a multiple of 32)
__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

}  // namespace moeq
