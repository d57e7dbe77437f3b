// Load-time re-layout of canonical weight formats into the internal
// row-per-thread block layout (see common.cuh), and the debug unpack that runs
// the GEMM kernels' own decode routine and writes the codes back in canonical
// order.
#include "kernels.h"
#include "decode_frag.cuh"

namespace moeq {

__device__ __forceinline__ int read_code(const uint8_t* row, int rowbytes, int bits, int k) {
  const int bit = bits * k;
  const int byte = bit >> 3, sh = bit & 7;
  uint32_t v = row[byte];
  if (byte + 1 < rowbytes) v |= (uint32_t)row[byte + 1] << 8;
  return (int)((v >> sh) & ((1u << bits) - 1u));
}

// Packs the 64 codes c[k] of one row chunk into the words the decode
// routines consume (field positions in decode_frag.cuh): half hh holds pairs
// i = 0..15 of codes (32hh + 2i, 32hh + 2i + 1), the even code in bits 0..15.
__device__ __forceinline__ void pack_int_words(const int (&c)[64], int bits, uint32_t (&w)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = 0u;
  for (int hh = 0; hh < 2; ++hh)
    for (int i = 0; i < 16; ++i)
      for (int h = 0; h < 2; ++h) {
        const uint32_t q = (uint32_t)c[32 * hh + 2 * i + h];
        const int hs = 16 * h;
        if (bits == 4) {
          // word 4hh + i/4: slot j = i%4 at nibble 0/1 of byte 0/1 of the half
          const int j = i & 3;
          w[4 * hh + (i >> 2)] |= q << (hs + 4 * (j & 1) + 8 * (j >> 1));
        } else if (bits == 2) {
          // word 2hh + i/8: step i/4 (parity = byte), 2-bit field i%4
          w[2 * hh + (i >> 3)] |= q << (hs + 8 * ((i >> 2) & 1) + 2 * (i & 3));
        } else if (i < 15) {
          // word 3hh + i/5: fields at bits 0, 3, 6, 9, 12 of the half
          w[3 * hh + i / 5] |= q << (hs + 3 * (i % 5));
        } else {
          // pair 15: bit 0 in word a, bit 1 in word b, bit 2 in word c, at bit 15 of the half
          for (int v = 0; v < 3; ++v) w[3 * hh + v] |= ((q >> v) & 1u) << (hs + 15);
        }
      }
}

// store of one row's words into a [128-row] block (layouts in decode_frag.cuh)
__device__ __forceinline__ void store_row_words(uint8_t* blk, int row, int bits, const uint32_t (&w)[8]) {
  if (bits == 4) {
    reinterpret_cast<uint4*>(blk)[row] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(blk + 2048)[row] = make_uint4(w[4], w[5], w[6], w[7]);
  } else if (bits == 2) {
    reinterpret_cast<uint4*>(blk)[row] = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    for (int v = 0; v < 6; ++v) reinterpret_cast<uint32_t*>(blk)[v * 128 + row] = w[v];
  }
}

// one thread per (chunk kc, internal row)
__global__ void relayout_int_kernel(const uint8_t* __restrict__ canon, uint8_t* __restrict__ out, int M, int K,
                                    int bits, int block, int N) {
  const int KC = K / 64;
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (tid >= (long long)KC * M) return;
  const int row = (int)(tid % M), kc = (int)(tid / M);
  const int crow = canon_row(row, block, N);
  const int rowbytes = K * bits / 8;
  int c[64];
  for (int k = 0; k < 64; ++k) c[k] = read_code(canon + (long long)crow * rowbytes, rowbytes, bits, kc * 64 + k);
  uint32_t w[8];
  pack_int_words(c, bits, w);
  uint8_t* blk = out + ((long long)kc * (M / 128) + row / 128) * block_bytes(FMT_INT, bits);
  store_row_words(blk, row % 128, bits, w);
}

// one thread per (group, internal row): half2(s, z)
__global__ void relayout_sz_kernel(const __half* __restrict__ s, const __half* __restrict__ z,
                                   uint32_t* __restrict__ out, int M, int K, int group, int block, int N) {
  const int G = K / group;
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (tid >= (long long)G * M) return;
  const int row = (int)(tid % M), gi = (int)(tid / M);
  const int crow = canon_row(row, block, N);
  const __half2 v = __halves2half2(s[(long long)crow * G + gi], z[(long long)crow * G + gi]);
  out[(long long)gi * M + row] = *reinterpret_cast<const uint32_t*>(&v);
}

// dense bf16 [M, K] (rows mapped by block/N) -> fp16 blocks: per (kc, rb),
// 8 quads x [128 rows x 16 B], quad q of a row = k 8q..8q+7
__global__ void relayout_dense_kernel(const __nv_bfloat16* __restrict__ src, uint8_t* __restrict__ out, int M, int K,
                                      int block, int N) {
  const int KC = K / 64;
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (tid >= (long long)KC * M) return;
  const int row = (int)(tid % M), kc = (int)(tid / M);
  const int crow = canon_row(row, block, N);
  uint8_t* blk = out + ((long long)kc * (M / 128) + row / 128) * block_bytes(FMT_DENSE, 16);
  for (int q = 0; q < 8; ++q) {
    uint32_t v[4];
    for (int j = 0; j < 4; ++j) {
      const int k = kc * 64 + 8 * q + 2 * j;
      v[j] = pack_half2(__bfloat162float(src[(long long)crow * K + k]), __bfloat162float(src[(long long)crow * K + k + 1]));
    }
    reinterpret_cast<uint4*>(blk + q * 2048)[row % 128] = make_uint4(v[0], v[1], v[2], v[3]);
  }
}

// compensator A [r, K] bf16 -> mma A-fragments [r/16][K/16][32] uint4 (fp16), r a multiple of 16
__global__ void relayout_afrag_kernel(const __nv_bfloat16* __restrict__ src, uint4* __restrict__ out, int r, int K) {
  const int S = K / 16;
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (tid >= (long long)(r / 16) * S * 32) return;
  const int lane = (int)(tid & 31);
  const long long t2 = tid >> 5;
  const int st = (int)(t2 % S), rf = (int)(t2 / S);
  const int g = lane >> 2, c = lane & 3;
  uint32_t v[4];
  for (int j = 0; j < 4; ++j) {
    const int row = 16 * rf + g + 8 * (j & 1);
    const int k = 16 * st + 2 * c + 8 * (j >> 1);
    v[j] = pack_half2(__bfloat162float(src[(long long)row * K + k]), __bfloat162float(src[(long long)row * K + k + 1]));
  }
  out[tid] = make_uint4(v[0], v[1], v[2], v[3]);
}

// compensator B [M, r] bf16 -> fp16 pairs [r/2][M] in internal row order
__global__ void relayout_brow_kernel(const __nv_bfloat16* __restrict__ src, uint32_t* __restrict__ out, int M, int r,
                                     int block, int N) {
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (tid >= (long long)(r / 2) * M) return;
  const int row = (int)(tid % M), cp = (int)(tid / M);
  const int crow = canon_row(row, block, N);
  out[tid] = pack_half2(__bfloat162float(src[(long long)crow * r + 2 * cp]),
                        __bfloat162float(src[(long long)crow * r + 2 * cp + 1]));
}

// bit-planes [4][M][K/32] u32 -> per plane [kc][rb][128 rows x 8 B]
__global__ void relayout_planes_kernel(const uint32_t* __restrict__ canon, PlaneOut out, int M, int K, int block,
                                       int N) {
  const int KC = K / 64, KW = K / 32;
  const long long per_plane = (long long)KC * M;
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (tid >= per_plane * 4) return;
  const int p = (int)(tid / per_plane);
  const long long t = tid % per_plane;
  const int row = (int)(t % M), kc = (int)(t / M);
  const int crow = canon_row(row, block, N);
  uint32_t w[2] = {0u, 0u};
  for (int s = 0; s < 8; ++s)
    for (int j = 0; j < 4; ++j)
      for (int h = 0; h < 2; ++h) {
        const int kk = kc * 64 + 8 * s + 2 * j + h;
        const uint32_t word = canon[((long long)p * M + crow) * KW + (kk >> 5)];
        w[s >> 2] |= ((word >> (kk & 31)) & 1u) << (4 * (2 * j + h) + (s & 3));
      }
  const long long o = (long long)kc * (M / 128) + row / 128;  // block index within the plane
  reinterpret_cast<uint2*>(out.p[p] + o * 1024)[row % 128] = make_uint2(w[0], w[1]);
}

// ---------------------------------------------------------------------------
// debug unpack: the GEMM's decode of each (chunk, row), written back to
// canonical [M, K] order as uint8 codes.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int half_to_int(uint16_t h) { return (int)__half2float(__ushort_as_half(h)); }

template <int BITS>
__device__ void unpack_int_half(const uint8_t* blk, int row, int h, int (&code)[32]) {
  uint32_t w[4], raw[16];
  load_half_words_int<BITS>(blk, row, h, w);
  int_raw_half<BITS>(w, raw);
  for (int i = 0; i < 16; ++i) {
    const uint32_t q = hsub2u(raw[i], int_magic<BITS>(i));
    code[2 * i] = half_to_int((uint16_t)(q & 0xFFFF));
    code[2 * i + 1] = half_to_int((uint16_t)(q >> 16));
  }
}

template <int BITS>
__device__ void unpack_plane_half(const BlockDesc& d, long long bidx, int row, int h, int (&code)[32]) {
  uint32_t pw[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) pw[p] = p < BITS ? reinterpret_cast<const uint32_t*>(d.plane[p] + bidx * 1024)[2 * row + h] : 0u;
  for (int s = 0; s < 4; ++s) {
    const uint32_t nib = plane_codes<BITS>(pw, s);
    for (int j = 0; j < 4; ++j)
      for (int hh = 0; hh < 2; ++hh) code[8 * s + 2 * j + hh] = (int)((nib >> (4 * (2 * j + hh))) & 0xF);
  }
}

__global__ void debug_unpack_kernel(BlockDesc d, uint8_t* __restrict__ out, int block, int N) {
  const int KC = d.K / 64;
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (tid >= (long long)KC * d.M) return;
  const int row = (int)(tid % d.M), kc = (int)(tid / d.M);
  const long long bidx = (long long)kc * (d.M / 128) + row / 128;
  const int crow = canon_row(row, block, N);
  for (int h = 0; h < 2; ++h) {
    int code[32];
    if (d.fmt == FMT_INT) {
      const uint8_t* blk = d.codes + bidx * block_bytes(FMT_INT, d.bits);
      if (d.bits == 4) unpack_int_half<4>(blk, row % 128, h, code);
      else if (d.bits == 3) unpack_int_half<3>(blk, row % 128, h, code);
      else unpack_int_half<2>(blk, row % 128, h, code);
    } else {
      if (d.bits == 4) unpack_plane_half<4>(d, bidx, row % 128, h, code);
      else if (d.bits == 3) unpack_plane_half<3>(d, bidx, row % 128, h, code);
      else unpack_plane_half<2>(d, bidx, row % 128, h, code);
    }
    for (int k = 0; k < 32; ++k) out[(long long)crow * d.K + kc * 64 + 32 * h + k] = (uint8_t)code[k];
  }
}

// ---------------------------------------------------------------------------
static inline unsigned grid_for(long long n, int bs) { return (unsigned)((n + bs - 1) / bs); }

cudaError_t launch_relayout_int(const uint8_t* canon, uint8_t* out, int M, int K, int bits, int block, int N,
                                cudaStream_t st) {
  relayout_int_kernel<<<grid_for((long long)(K / 64) * M, 256), 256, 0, st>>>(canon, out, M, K, bits, block, N);
  return cudaGetLastError();
}
cudaError_t launch_relayout_sz(const __half* s, const __half* z, uint32_t* out, int M, int K, int group, int block,
                               int N, cudaStream_t st) {
  relayout_sz_kernel<<<grid_for((long long)(K / group) * M, 256), 256, 0, st>>>(s, z, out, M, K, group, block, N);
  return cudaGetLastError();
}
cudaError_t launch_relayout_dense(const __nv_bfloat16* src, uint8_t* out, int M, int K, int block, int N,
                                  cudaStream_t st) {
  relayout_dense_kernel<<<grid_for((long long)(K / 64) * M, 256), 256, 0, st>>>(src, out, M, K, block, N);
  return cudaGetLastError();
}
cudaError_t launch_relayout_afrag(const __nv_bfloat16* src, uint4* out, int r, int K, cudaStream_t st) {
  relayout_afrag_kernel<<<grid_for((long long)(r / 16) * (K / 16) * 32, 256), 256, 0, st>>>(src, out, r, K);
  return cudaGetLastError();
}
cudaError_t launch_relayout_brow(const __nv_bfloat16* src, uint32_t* out, int M, int r, int block, int N,
                                 cudaStream_t st) {
  relayout_brow_kernel<<<grid_for((long long)(r / 2) * M, 256), 256, 0, st>>>(src, out, M, r, block, N);
  return cudaGetLastError();
}
cudaError_t launch_relayout_planes(const uint32_t* canon, PlaneOut out, int M, int K, int block, int N,
                                   cudaStream_t st) {
  relayout_planes_kernel<<<grid_for((long long)(K / 64) * M * 4, 256), 256, 0, st>>>(canon, out, M, K, block, N);
  return cudaGetLastError();
}
cudaError_t launch_debug_unpack(const BlockDesc& d, uint8_t* out, int block, int N, cudaStream_t st) {
  debug_unpack_kernel<<<grid_for((long long)(d.K / 64) * d.M, 256), 256, 0, st>>>(d, out, block, N);
  return cudaGetLastError();
}

}  // namespace moeq
