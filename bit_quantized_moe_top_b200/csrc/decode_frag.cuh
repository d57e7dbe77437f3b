// Register-level unpack of packed codes into fp16 pairs.
//
// A 64-wide K chunk of one weight row is two halves of 32 codes; half h is
// 16 pairs, pair i holding the codes at k = 32h + 2i (low 16 bits) and
// k = 32h + 2i + 1 (high 16 bits). One routine decodes one half, so a row's
// chunk can be shared by two threads or walked by one.
//
// Integer codes become fp16 through the exponent-bias trick: a b-bit field
// q OR-ed into the mantissa of a power of two P whose mantissa unit at the
// field's position is 1 reads as P + q exactly. The "raw" value P_i + q is
// where dequantising starts: one fp16 subtraction removes P_i exactly and one
// fp16 FMA applies the group's scale and -z*s. P_i depends only on the pair
// index i (both halves of a word use the same bit position), so each format
// has a fixed table of P_i (int_magic).
//
// Field positions per format (per 16-bit half of a word; P = 2^(10 - pos)):
//   INT4: word s (0..3) holds pairs 4s..4s+3: nibbles 0 and 1 of each byte
//         after a shift of 0 or 8, P = 1024, 64, 1024, 64.
//   INT2: word u (0..1) holds pairs 8u..8u+7: 2-bit fields at 0,2,4,6 after a
//         shift of 0 or 8, P = 1024, 256, 64, 16.
//   INT3: words a, b, c hold pairs 5w..5w+4 as 3-bit fields at 0,3,6 and at
//         9,12 (read after a shift of 6 as 3,6): P = 1024, 128, 16, 128, 16.
//         Pair 15 takes its three bits from bit 15 of a (lsb), b and c.
#pragma once
#include "common.cuh"

namespace moeq {

// ---- integer formats --------------------------------------------------------

template <int BITS>
__host__ __device__ __forceinline__ uint32_t int_magic(int i) {
  if (BITS == 4) return (i & 1) ? 0x54005400u : 0x64006400u;
  if (BITS == 2) {
    const int j = i & 3;
    return j == 0 ? 0x64006400u : j == 1 ? 0x5C005C00u : j == 2 ? 0x54005400u : 0x4C004C00u;
  }
  if (i == 15) return 0x48004800u;
  const int f = i % 5;
  return f == 0 ? 0x64006400u : (f & 1) ? 0x58005800u : 0x4C004C00u;
}

// number of 32-bit code words per half chunk of one row
__host__ __device__ __forceinline__ int int_half_words(int bits) { return bits == 4 ? 4 : bits == 3 ? 3 : 2; }

// raw pairs P_i + q of one half chunk from its code words
//   INT4: w[0..3]   INT3: w[0..2]   INT2: w[0..1]
template <int BITS>
__device__ __forceinline__ void int_raw_half(const uint32_t* w, uint32_t (&r)[16]) {
  if constexpr (BITS == 4) {
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const uint32_t w8 = w[s] >> 8;
      r[4 * s + 0] = lop3_and_or(w[s], 0x000F000Fu, 0x64006400u);
      r[4 * s + 1] = lop3_and_or(w[s], 0x00F000F0u, 0x54005400u);
      r[4 * s + 2] = lop3_and_or(w8, 0x000F000Fu, 0x64006400u);
      r[4 * s + 3] = lop3_and_or(w8, 0x00F000F0u, 0x54005400u);
    }
  } else if constexpr (BITS == 2) {
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const uint32_t b = (s & 1) ? (w[s >> 1] >> 8) : w[s >> 1];
      r[4 * s + 0] = lop3_and_or(b, 0x00030003u, 0x64006400u);
      r[4 * s + 1] = lop3_and_or(b, 0x000C000Cu, 0x5C005C00u);
      r[4 * s + 2] = lop3_and_or(b, 0x00300030u, 0x54005400u);
      r[4 * s + 3] = lop3_and_or(b, 0x00C000C0u, 0x4C004C00u);
    }
  } else {
    uint32_t w6[3];
#pragma unroll
    for (int v = 0; v < 3; ++v) {
      w6[v] = w[v] >> 6;
      r[5 * v + 0] = lop3_and_or(w[v], 0x00070007u, 0x64006400u);
      r[5 * v + 1] = lop3_and_or(w[v], 0x00380038u, 0x58005800u);
      r[5 * v + 2] = lop3_and_or(w[v], 0x01C001C0u, 0x4C004C00u);
      r[5 * v + 3] = lop3_and_or(w6[v], 0x00380038u, 0x58005800u);
      r[5 * v + 4] = lop3_and_or(w6[v], 0x01C001C0u, 0x4C004C00u);
    }
    // pair 15: bit 15 of a -> bit 7, of b -> bit 8, of c -> bit 9 (each half)
    const uint32_t t = lop3_sel(w[0] >> 8, w[1] >> 7, 0x00800080u);
    const uint32_t t2 = lop3_sel(t, w6[2], 0x01800180u);
    r[15] = lop3_and_or(t2, 0x03800380u, 0x48004800u);
  }
}

// (q - z) * s of one half: raw - P exactly, then one fp16 FMA with
// s2 = (s, s) and n2 = (-z*s, -z*s)
template <int BITS>
__device__ __forceinline__ void int_dequant_half(const uint32_t (&raw)[16], uint32_t s2, uint32_t n2,
                                                 uint32_t (&out)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) out[i] = hfma2u(hsub2u(raw[i], int_magic<BITS>(i)), s2, n2);
}

// ---- bit-plane + LUT ---------------------------------------------------------
// Per plane, a half chunk is one 32-bit word: bit 4*(2j+h) + s of it is the
// plane bit of element (step s, slot j, half h), step s = 0..3 covering pairs
// 4s..4s+3. Codes are built as prmt nibble selectors; the LUT is split in a
// low-byte and a high-byte table.

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

// b-bit code nibbles of step s (8 elements: nibble 2j+h) from the half's
// plane words pw[p] (p = 0 is the MSB plane); bit 3 of every nibble is 0
// (b <= 3) or holds the MSB (b = 4).
template <int BITS>
__device__ __forceinline__ uint32_t plane_codes(const uint32_t* pw, int s) {
  uint32_t c = 0;
#pragma unroll
  for (int p = 0; p < BITS; ++p) c |= ((pw[p] >> s) & 0x11111111u) << (BITS - 1 - p);
  return c;
}

// LUT lookup of the 8 codes of one step: a[j] = (LUT[c(j,0)], LUT[c(j,1)])
template <int BITS>
__device__ __forceinline__ void lut_decode(uint32_t codes, const LutRegs& L, uint32_t* a) {
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

// LUT values of one half from its plane words pw[0..BITS-1]
template <int BITS>
__device__ __forceinline__ void lut_half(const uint32_t* pw, const LutRegs& L, uint32_t (&out)[16]) {
#pragma unroll
  for (int s = 0; s < 4; ++s) lut_decode<BITS>(plane_codes<BITS>(pw, s), L, out + 4 * s);
}

// ---- code blocks in memory (global or shared) --------------------------------
// INT4: words 0..3 of all rows ([128] x 16 B), then words 4..7.
// INT2: words 0..3 of all rows ([128] x 16 B).
// INT3: word-major, [6][128] x 4 B.
// BITPLANE: per plane [128] x 8 B (word 0 = half 0), planes plane_bytes apart.

// half h's code words of row `row`
template <int BITS>
__device__ __forceinline__ void load_half_words_int(const uint8_t* blk, int row, int h, uint32_t (&w)[4]) {
  if constexpr (BITS == 4) {
    const uint4 v = reinterpret_cast<const uint4*>(blk + 2048 * h)[row];
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (BITS == 2) {
    const uint2 v = reinterpret_cast<const uint2*>(blk + 16 * row + 8 * h)[0];
    w[0] = v.x; w[1] = v.y; w[2] = w[3] = 0u;
  } else {
    const uint32_t* b32 = reinterpret_cast<const uint32_t*>(blk);
    w[0] = b32[(3 * h + 0) * 128 + row];
    w[1] = b32[(3 * h + 1) * 128 + row];
    w[2] = b32[(3 * h + 2) * 128 + row];
    w[3] = 0u;
  }
}

template <int BITS>
__device__ __forceinline__ void load_half_planes(const uint8_t* blk, int plane_bytes, int row, int h,
                                                 uint32_t (&pw)[4]) {
#pragma unroll
  for (int p = 0; p < 4; ++p)
    pw[p] = p < BITS ? reinterpret_cast<const uint32_t*>(blk + p * plane_bytes)[2 * row + h] : 0u;
}

// ---- the same loads from shared memory, by 32-bit shared address -------------
// (explicit ld.shared, so the hot loops never take the generic-address path)

__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds_v2(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 lds_v4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}

template <int BITS>
__device__ __forceinline__ void lds_half_words_int(uint32_t blk, int row, int h, uint32_t (&w)[4]) {
  if constexpr (BITS == 4) {
    const uint4 v = lds_v4(blk + 2048 * h + 16 * row);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (BITS == 2) {
    const uint2 v = lds_v2(blk + 16 * row + 8 * h);
    w[0] = v.x; w[1] = v.y; w[2] = w[3] = 0u;
  } else {
    w[0] = lds_u32(blk + 4 * ((3 * h + 0) * 128 + row));
    w[1] = lds_u32(blk + 4 * ((3 * h + 1) * 128 + row));
    w[2] = lds_u32(blk + 4 * ((3 * h + 2) * 128 + row));
    w[3] = 0u;
  }
}

template <int BITS>
__device__ __forceinline__ void lds_half_planes(uint32_t blk, int plane_bytes, int row, int h, uint32_t (&pw)[4]) {
#pragma unroll
  for (int p = 0; p < 4; ++p) pw[p] = p < BITS ? lds_u32(blk + p * plane_bytes + 4 * (2 * row + h)) : 0u;
}

// 32 dequantised fp16 pairs (k = 0..63) of one row chunk: out[16h + i] = pair i of half h
// INT: (q - z) * s with sz = half2(s, z); bit-plane: LUT_b[code].
template <int FMT, int BITS>
__device__ __forceinline__ void decode_row64(const uint8_t* blk, int plane_bytes, int row, uint32_t sz,
                                             const LutRegs& lut, uint32_t (&out)[32]) {
  uint32_t s2 = 0, n2 = 0;
  if constexpr (FMT == FMT_INT) {
    s2 = prmt(sz, sz, 0x1010u);
    const uint32_t z2 = prmt(sz, sz, 0x3232u);
    n2 = hmul2u(hneg2u(z2), s2);
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t v[16];
    if constexpr (FMT == FMT_INT) {
      uint32_t w[4], raw[16];
      load_half_words_int<BITS>(blk, row, h, w);
      int_raw_half<BITS>(w, raw);
      int_dequant_half<BITS>(raw, s2, n2, v);
    } else {
      uint32_t pw[4];
      load_half_planes<BITS>(blk, plane_bytes, row, h, pw);
      lut_half<BITS>(pw, lut, v);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) out[16 * h + i] = v[i];
  }
}

}  // namespace moeq
