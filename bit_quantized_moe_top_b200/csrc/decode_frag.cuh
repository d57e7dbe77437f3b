// Register-level unpack + dequantisation of packed codes into fp16 pairs.
// One thread owns one weight row; a 64-wide K chunk of that row is 8 "steps"
// of 4 pairs, pair j of step s being the codes at k = 8s+2j and 8s+2j+1.
//
// Integer codes become fp16 through the exponent-bias trick: a b-bit field
// OR-ed into the mantissa of a power of two P whose mantissa ulp is 1 reads as
// P + q exactly; subtracting P gives q exactly; one fp16 FMA with the group's
// scale s and the pre-rounded -z*s gives (q - z) * s with one rounding.
// The field positions inside each 32-bit word are chosen so that no word
// needs more than one shift per step; see the layout notes in common.cuh.
#pragma once
#include "common.cuh"

namespace moeq {

// fp16x2 powers of two whose mantissa ulp is 1 for a field at bit 0, 2, 4, 6
__device__ __forceinline__ uint32_t magic2(int pos) {
  return pos == 0 ? 0x64006400u : pos == 1 ? 0x5C005C00u : pos == 2 ? 0x54005400u : 0x4C004C00u;
}

// ---- integer formats: produce the exact codes q as fp16x2 (q_k, q_k+1) ----

// INT4: word s of the chunk; slot j lives in nibbles j and j+4.
__device__ __forceinline__ void int4_codes(uint32_t w, uint32_t (&q)[4]) {
  const uint32_t w8 = w >> 8;
  q[0] = hsub2u(lop3_and_or(w, 0x000F000Fu, 0x64006400u), 0x64006400u);
  q[1] = hsub2u(lop3_and_or(w, 0x00F000F0u, 0x54005400u), 0x54005400u);
  q[2] = hsub2u(lop3_and_or(w8, 0x000F000Fu, 0x64006400u), 0x64006400u);
  q[3] = hsub2u(lop3_and_or(w8, 0x00F000F0u, 0x54005400u), 0x54005400u);
}

// INT2: word s/2 of the chunk; step parity selects the byte half.
__device__ __forceinline__ void int2_codes(uint32_t w, int s, uint32_t (&q)[4]) {
  const uint32_t b = (s & 1) ? (w >> 8) : w;
  q[0] = hsub2u(lop3_and_or(b, 0x00030003u, 0x64006400u), 0x64006400u);
  q[1] = hsub2u(lop3_and_or(b, 0x000C000Cu, 0x5C005C00u), 0x5C005C00u);
  q[2] = hsub2u(lop3_and_or(b, 0x00300030u, 0x54005400u), 0x54005400u);
  q[3] = hsub2u(lop3_and_or(b, 0x00C000C0u, 0x4C004C00u), 0x4C004C00u);
}

// INT3: low two bits as INT2 (word s/2), the third bit from hi word s/4 after
// the transform (s & 3): identity, >>1, rotate-right 8, rotate-right 9.
__device__ __forceinline__ uint32_t int3_hi_transform(uint32_t h, int t) {
  return t == 0 ? h : t == 1 ? (h >> 1) : t == 2 ? __funnelshift_r(h, h, 8) : __funnelshift_r(h, h, 9);
}
__device__ __forceinline__ void int3_codes(uint32_t lo, uint32_t hi, int s, uint32_t (&q)[4]) {
  const uint32_t b = (s & 1) ? (lo >> 8) : lo;
  const uint32_t t = int3_hi_transform(hi, s & 3);
  q[0] = hsub2u(lop3_and_or(lop3_sel(b, t, 0x00030003u), 0x00070007u, 0x64006400u), 0x64006400u);
  q[1] = hsub2u(lop3_and_or(lop3_sel(b, t, 0x000C000Cu), 0x001C001Cu, 0x5C005C00u), 0x5C005C00u);
  q[2] = hsub2u(lop3_and_or(lop3_sel(b, t, 0x00300030u), 0x00700070u, 0x54005400u), 0x54005400u);
  q[3] = hsub2u(lop3_and_or(lop3_sel(b, t, 0x00C000C0u), 0x01C001C0u, 0x4C004C00u), 0x4C004C00u);
}

// codes of step s (4 fp16x2 pairs) from the row's chunk words (in registers)
//   INT2: w[0..3]   INT3: w[0..3] lo + w[4..5] hi   INT4: w[0..7]
template <int BITS>
__device__ __forceinline__ void int_codes(const uint32_t* w, int s, uint32_t (&q)[4]) {
  if constexpr (BITS == 4) {
    int4_codes(w[s], q);
  } else if constexpr (BITS == 3) {
    int3_codes(w[s >> 1], w[4 + (s >> 2)], s, q);
  } else {
    int2_codes(w[s >> 1], s, q);
  }
}

// ---- bit-plane + LUT: 4-bit layout per plane word: bit 4*(2j+h) + (s&3) of
// word s>>2 is element (step s, slot j, half h).  Codes are built as prmt
// nibble selectors; the LUT is split in a low-byte and a high-byte table. ----

struct LutRegs {
  // low / high bytes of LUT entries 0..7 (a) and 8..15 (b, 4-bit only)
  uint32_t lo_a0, lo_a1, hi_a0, hi_a1, lo_b0, lo_b1, hi_b0, hi_b1;
};

__device__ __forceinline__ LutRegs load_lut(const uint32_t* lut28, int bits) {
  // entries of LUT_b as fp16: lut28 holds LUT_2 (4) | LUT_3 (8) | LUT_4 (16)
  const uint16_t* h = reinterpret_cast<const uint16_t*>(lut28);
  const int off = bits == 2 ? 0 : bits == 3 ? 4 : 12;
  const int n = 1 << bits;
  uint8_t lo[16], hi[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    uint16_t v = i < n ? h[off + i] : (uint16_t)0;
    lo[i] = (uint8_t)(v & 0xFF);
    hi[i] = (uint8_t)(v >> 8);
  }
  auto pk = [](const uint8_t* p) {
    return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
  };
  LutRegs r;
  r.lo_a0 = pk(lo);
  r.lo_a1 = pk(lo + 4);
  r.hi_a0 = pk(hi);
  r.hi_a1 = pk(hi + 4);
  r.lo_b0 = pk(lo + 8);
  r.lo_b1 = pk(lo + 12);
  r.hi_b0 = pk(hi + 8);
  r.hi_b1 = pk(hi + 12);
  return r;
}

// b-bit code nibbles of step s (8 elements: nibble 2j+h) from the plane words
// of word s>>2; bit 3 of every nibble is left 0 (b<=3) or holds the MSB (b=4).
template <int BITS>
__device__ __forceinline__ uint32_t plane_codes(const uint32_t* pw, int s) {
  const int q = s & 3;
  const int w = s >> 2;
  uint32_t c = 0;
#pragma unroll
  for (int p = 0; p < BITS; ++p) {
    const uint32_t bit = (pw[2 * p + w] >> q) & 0x11111111u;
    c |= bit << (BITS - 1 - p);
  }
  return c;
}

// LUT lookup of the 8 codes of step s: out[j] = (LUT[c(j,0)], LUT[c(j,1)])
template <int BITS>
__device__ __forceinline__ void lut_decode(uint32_t codes, const LutRegs& L, uint32_t (&a)[4]) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const uint32_t sel = half ? (codes >> 16) : (codes & 0xFFFFu);
    uint32_t lo, hi;
    if constexpr (BITS == 4) {
      const uint32_t s3 = sel & 0x7777u;
      const uint32_t msb = (sel >> 3) & 0x1111u;
      const uint32_t pick = 0x3210u + (msb << 2);
      lo = prmt(prmt(L.lo_a0, L.lo_a1, s3), prmt(L.lo_b0, L.lo_b1, s3), pick);
      hi = prmt(prmt(L.hi_a0, L.hi_a1, s3), prmt(L.hi_b0, L.hi_b1, s3), pick);
    } else {
      lo = prmt(L.lo_a0, L.lo_a1, sel);
      hi = prmt(L.hi_a0, L.hi_a1, sel);
    }
    a[2 * half + 0] = prmt(lo, hi, 0x5140u);
    a[2 * half + 1] = prmt(lo, hi, 0x7362u);
  }
}

// ---- whole 64-wide chunk of one row ----

// words of row `row` of a [128-row] code block (global or shared memory)
__device__ __forceinline__ void load_row_words_int(const uint8_t* blk, int row, int bits, uint32_t (&w)[8]) {
  const uint4 v0 = reinterpret_cast<const uint4*>(blk)[row];
  w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
  w[4] = w[5] = w[6] = w[7] = 0u;
  if (bits == 4) {
    const uint4 v1 = reinterpret_cast<const uint4*>(blk + 2048)[row];
    w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
  } else if (bits == 3) {
    const uint2 h = reinterpret_cast<const uint2*>(blk + 2048)[row];
    w[4] = h.x; w[5] = h.y;
  }
}

// bit-plane words of row `row`: plane p at blk + p * plane_bytes
template <int BITS>
__device__ __forceinline__ void load_row_planes(const uint8_t* blk, int plane_bytes, int row, uint32_t (&w)[8]) {
#pragma unroll
  for (int p = 0; p < BITS; ++p) {
    const uint2 v = reinterpret_cast<const uint2*>(blk + p * plane_bytes)[row];
    w[2 * p] = v.x; w[2 * p + 1] = v.y;
  }
}

// 32 fp16 pairs (k = 0..63) of one row chunk: out[4s+j] = pair (8s+2j, 8s+2j+1)
// INT: w^ = (q - z) * s with sz = half2(s, -z*s); bit-plane: LUT_b[code].
template <int FMT, int BITS>
__device__ __forceinline__ void decode_row64(const uint32_t (&w)[8], uint32_t sz, const LutRegs& lut,
                                             uint32_t (&out)[32]) {
  if constexpr (FMT == FMT_INT) {
    const uint32_t s2 = prmt(sz, sz, 0x1010u), n2 = prmt(sz, sz, 0x3232u);
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      uint32_t q[4];
      int_codes<BITS>(w, s, q);
#pragma unroll
      for (int j = 0; j < 4; ++j) out[4 * s + j] = hfma2u(q[j], s2, n2);
    }
  } else {
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      uint32_t av[4];
      lut_decode<BITS>(plane_codes<BITS>(w, s), lut, av);
#pragma unroll
      for (int j = 0; j < 4; ++j) out[4 * s + j] = av[j];
    }
  }
}

}  // namespace moeq
