// Load-time re-layout of canonical weight formats into the internal
// fragment-ordered layouts (see common.cuh), and the debug unpack that runs
// the GEMM kernels' own decode routine backwards to canonical order.
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

// one thread per (rf, kc, lane)
__global__ void relayout_int_kernel(const uint8_t* __restrict__ canon, uint8_t* __restrict__ out, int M, int K,
                                    int bits, int block, int N) {
  const int KC = K / kChunkK, MF = M / 16;
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (tid >= (long long)MF * KC * 32) return;
  const int lane = (int)(tid & 31);
  const long long ch = tid >> 5;
  const int kc = (int)(ch % KC), rf = (int)(ch / KC);
  const int rowbytes = K * bits / 8;
  uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int s = 0; s < 8; ++s)
    for (int j = 0; j < 4; ++j)
      for (int h = 0; h < 2; ++h) {
        int r, k;
        frag_elem(lane, s, j, h, r, k);
        const int crow = canon_row(16 * rf + r, block, N);
        const int q = read_code(canon + (long long)crow * rowbytes, rowbytes, bits, kc * kChunkK + k);
        if (bits == 4) {
          w[s] |= (uint32_t)q << (4 * (j + 4 * h));
        } else {
          const int p = 4 * (s & 1) + j;
          const int pos = 2 * (p & 3) + 8 * (p >> 2) + 16 * h;
          w[s >> 1] |= (uint32_t)(q & 3) << pos;
          if (bits == 3) {
            const int t = s & 3;  // transform of hi word s>>2
            const int base = (h ? 18 : 2) + 2 * j;
            const int src = t == 0 ? base : t == 1 ? base + 1 : t == 2 ? (base + 8) & 31 : (base + 9) & 31;
            w[4 + (s >> 2)] |= (uint32_t)(q >> 2) << src;
          }
        }
      }
  uint32_t* chunk = reinterpret_cast<uint32_t*>(out + ((long long)kc * MF + rf) * 256LL * bits);
  if (bits == 4) {
    for (int s = 0; s < 8; ++s) chunk[(s >> 2) * 128 + lane * 4 + (s & 3)] = w[s];
  } else {
    for (int i = 0; i < 4; ++i) chunk[lane * 4 + i] = w[i];
    if (bits == 3) {
      chunk[128 + lane * 2 + 0] = w[4];
      chunk[128 + lane * 2 + 1] = w[5];
    }
  }
}

// one thread per (rf, group, g): half2(s, -z*s) for rows g and g+8
__global__ void relayout_sz_kernel(const __half* __restrict__ s, const __half* __restrict__ z,
                                   uint32_t* __restrict__ out, int M, int K, int group, int block, int N) {
  const int G = K / group, MF = M / 16;
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (tid >= (long long)MF * G * 8) return;
  const int g = (int)(tid & 7);
  const long long t2 = tid >> 3;
  const int gi = (int)(t2 % G), rf = (int)(t2 / G);
  for (int hrow = 0; hrow < 2; ++hrow) {
    const int crow = canon_row(16 * rf + g + 8 * hrow, block, N);
    const float sv = __half2float(s[(long long)crow * G + gi]);
    const float zv = __half2float(z[(long long)crow * G + gi]);
    out[(((long long)gi * MF + rf) * 8 + g) * 2 + hrow] = pack_half2(sv, -zv * sv);
  }
}

// dense bf16 [rows, K] (row map by block/N, or identity when block < 0) ->
// fp16 A fragments [MF][K/16][32] uint4
__global__ void relayout_dense_kernel(const __nv_bfloat16* __restrict__ src, uint4* __restrict__ out, int M, int K,
                                      int block, int N, long long src_ld, int chunked) {
  const int S = K / 16, MF = M / 16;
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (tid >= (long long)MF * S * 32) return;
  const int lane = (int)(tid & 31);
  const long long t2 = tid >> 5;
  const int st = (int)(t2 % S), rf = (int)(t2 / S);
  uint32_t v[4];
  for (int j = 0; j < 4; ++j) {
    float e[2];
    for (int h = 0; h < 2; ++h) {
      int r, k;
      frag_elem(lane, 0, j, h, r, k);
      const int row = 16 * rf + r;
      const int crow = block < 0 ? row : canon_row(row, block, N);
      e[h] = __bfloat162float(src[(long long)crow * src_ld + 16 * st + k]);
    }
    v[j] = pack_half2(e[0], e[1]);
  }
  // chunked: [kc][rf][8 steps][32] (the GEMM weight layout); else [rf][K/16][32]
  const long long o = chunked ? ((((long long)(st >> 3) * MF + rf) * 8 + (st & 7)) * 32 + lane) : tid;
  out[o] = make_uint4(v[0], v[1], v[2], v[3]);
}

// bit-planes [4][M][K/32] u32 -> per plane [MF][KC][32] uint2
__global__ void relayout_planes_kernel(const uint32_t* __restrict__ canon, uint32_t* __restrict__ out, int M, int K,
                                       int block, int N) {
  const int KC = K / kChunkK, MF = M / 16, KW = K / 32;
  const long long per_plane = (long long)MF * KC * 32;
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (tid >= per_plane * 4) return;
  const int p = (int)(tid / per_plane);
  const long long t = tid % per_plane;
  const int lane = (int)(t & 31);
  const long long ch = t >> 5;
  const int kc = (int)(ch % KC), rf = (int)(ch / KC);
  uint32_t w[2] = {0, 0};
  for (int s = 0; s < 8; ++s)
    for (int j = 0; j < 4; ++j)
      for (int h = 0; h < 2; ++h) {
        int r, k;
        frag_elem(lane, s, j, h, r, k);
        const int crow = canon_row(16 * rf + r, block, N);
        const int kk = kc * kChunkK + k;
        const uint32_t word = canon[((long long)p * M + crow) * KW + (kk >> 5)];
        const uint32_t bit = (word >> (kk & 31)) & 1u;
        w[s >> 2] |= bit << (4 * (2 * j + h) + (s & 3));
      }
  const long long o = (((long long)p * KC + kc) * MF + rf) * 32 + lane;
  out[o * 2 + 0] = w[0];
  out[o * 2 + 1] = w[1];
}

// ---------------------------------------------------------------------------
// debug unpack: the GEMM's decode of each (rf, kc, lane), written back to
// canonical [M, K] order as uint8 codes.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int half_to_int(uint16_t h) { return (int)__half2float(__ushort_as_half(h)); }

__global__ void debug_unpack_kernel(BlockDesc d, uint8_t* __restrict__ out, int block, int N) {
  const int KC = d.K / kChunkK, MF = d.M / 16;
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (tid >= (long long)MF * KC * 32) return;
  const int lane = (int)(tid & 31);
  const long long ch = tid >> 5;
  const int kc = (int)(ch % KC), rf = (int)(ch / KC);
  uint32_t w[8];
  if (d.fmt == FMT_INT) {
    const uint32_t* chunk = reinterpret_cast<const uint32_t*>(d.codes + ((long long)kc * MF + rf) * 256LL * d.bits);
    if (d.bits == 4) {
      for (int s = 0; s < 8; ++s) w[s] = chunk[(s >> 2) * 128 + lane * 4 + (s & 3)];
    } else {
      for (int i = 0; i < 4; ++i) w[i] = chunk[lane * 4 + i];
      if (d.bits == 3) {
        w[4] = chunk[128 + lane * 2];
        w[5] = chunk[128 + lane * 2 + 1];
      }
    }
  } else {
    for (int p = 0; p < d.bits; ++p) {
      const uint32_t* pl = reinterpret_cast<const uint32_t*>(d.codes + p * d.plane_stride);
      const long long o = ((long long)kc * MF + rf) * 32 + lane;
      w[2 * p] = pl[o * 2];
      w[2 * p + 1] = pl[o * 2 + 1];
    }
  }
  for (int s = 0; s < 8; ++s) {
    uint32_t q[4];
    uint32_t nib = 0;
    if (d.fmt == FMT_INT) {
      if (d.bits == 4) int_codes<4>(w, s, q);
      else if (d.bits == 3) int_codes<3>(w, s, q);
      else int_codes<2>(w, s, q);
    } else {
      nib = d.bits == 4 ? plane_codes<4>(w, s) : d.bits == 3 ? plane_codes<3>(w, s) : plane_codes<2>(w, s);
    }
    for (int j = 0; j < 4; ++j)
      for (int h = 0; h < 2; ++h) {
        int r, k;
        frag_elem(lane, s, j, h, r, k);
        const int crow = canon_row(16 * rf + r, block, N);
        int code;
        if (d.fmt == FMT_INT) code = half_to_int((uint16_t)(h ? (q[j] >> 16) : (q[j] & 0xFFFF)));
        else code = (int)((nib >> (4 * (2 * j + h))) & 0xF);
        out[(long long)crow * d.K + kc * kChunkK + k] = (uint8_t)code;
      }
  }
}

// ---------------------------------------------------------------------------
static inline unsigned grid_for(long long n, int bs) { return (unsigned)((n + bs - 1) / bs); }

cudaError_t launch_relayout_int(const uint8_t* canon, uint8_t* out, int M, int K, int bits, int block, int N,
                                cudaStream_t st) {
  const long long n = (long long)(M / 16) * (K / kChunkK) * 32;
  relayout_int_kernel<<<grid_for(n, 256), 256, 0, st>>>(canon, out, M, K, bits, block, N);
  return cudaGetLastError();
}
cudaError_t launch_relayout_sz(const __half* s, const __half* z, uint32_t* out, int M, int K, int group, int block,
                               int N, cudaStream_t st) {
  const long long n = (long long)(M / 16) * (K / group) * 8;
  relayout_sz_kernel<<<grid_for(n, 256), 256, 0, st>>>(s, z, out, M, K, group, block, N);
  return cudaGetLastError();
}
cudaError_t launch_relayout_dense(const __nv_bfloat16* src, uint4* out, int M, int K, int block, int N,
                                  long long ld, int chunked, cudaStream_t st) {
  const long long n = (long long)(M / 16) * (K / 16) * 32;
  relayout_dense_kernel<<<grid_for(n, 256), 256, 0, st>>>(src, out, M, K, block, N, ld, chunked);
  return cudaGetLastError();
}
cudaError_t launch_relayout_planes(const uint32_t* canon, uint32_t* out, int M, int K, int block, int N,
                                   cudaStream_t st) {
  const long long n = (long long)(M / 16) * (K / kChunkK) * 32 * 4;
  relayout_planes_kernel<<<grid_for(n, 256), 256, 0, st>>>(canon, out, M, K, block, N);
  return cudaGetLastError();
}
cudaError_t launch_debug_unpack(const BlockDesc& d, uint8_t* out, int block, int N, cudaStream_t st) {
  const long long n = (long long)(d.M / 16) * (d.K / kChunkK) * 32;
  debug_unpack_kernel<<<grid_for(n, 256), 256, 0, st>>>(d, out, block, N);
  return cudaGetLastError();
}

}  // namespace moeq
