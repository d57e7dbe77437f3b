// Internal launch interface between the C-ABI host code and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include "common.cuh"

#include <utility>

namespace moeq {

enum : int { MODE_SWIGLU = 0, MODE_OUT = 1 };

// Kernel launch on `st`, with programmatic stream serialization when `pdl`
// (the kernel then calls pdl_wait() before it reads what earlier kernels wrote).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                 bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

struct RouteArgs {
  const float* logits;        // [T, E]
  const __nv_bfloat16* X;     // [T, K]
  int T, E, k, K, renorm;
  int* idx;                   // [T, k]
  float* w;                   // [T, k]
  int* block_counts;          // [nb, E]
  int* block_base;            // [nb, E]
  int* pblock_base;           // [nb, E]
  int* counts;                // [E]
  int* offsets;               // [E+1]
  int* poffsets;              // [E+1] (8-row padded)
  int* active;                // [E]
  int* n_active;              // [1]
  int* ticket;                // [1], zero between launches
  int* perm_token;            // [T*k]
  int* inv_pos;               // [T, k]
  int* pinv;                  // [T, k] padded row
  int* pslot;                 // [padded rows] routing slot of each routed row
  int* ptok;                  // [padded rows] token of each routed row
  void* act;                  // activation buffer, fp16 row-major [rows, Kpad]
  int Kpad;
  unsigned* status;
  // fused kernel only
  int* flag;                  // [1] set to epoch once the scan is done
  unsigned epoch;             // nonzero, different for every forward of the layer
  int nb, gs;                 // token blocks of 16, K slices of the gather
  unsigned long long wait_ns; // limit of the wait for the scan
};

struct DecodeArgs {
  CUtensorMap tmap_act;       // activations [rows, Kpad] fp16 row-major; box 64 x 16, 128-byte swizzle
  const ExpertDesc* experts;
  int block;                  // 0 = W1, 1 = W2
  const int* active;
  const int* n_active;
  const int* counts;
  const int* poffsets;
  int K;                      // quantised K of the block
  int M;                      // rows of the block
  int mode;
  __half* zout;               // MODE_SWIGLU: output rows (fp16), leading dimension ldz
  long long ldz;
  float* out;                 // MODE_OUT: [KS][prows][M] fp32 partials
  long long out_ks_stride;
  int KS;
  long long rows;             // routed rows of the forward (host-side grid sizing)
  int nstages;                // shared-memory stages of the ring (set by the launcher)
  unsigned long long wait_ns; // limit of the hand-off waits between roles
  unsigned* status;
  // tiles split between two CTAs (null: whole tiles only): per CTA 128 x 32
  // fp32 partial sums and a flag set to sk_epoch once they are written
  float* sk_part;
  unsigned* sk_flag;
  unsigned sk_epoch;          // nonzero, different for every launch of the layer
  int mixed;                  // the experts' blocks differ (bits, format, group or rank): tiles dealt round-robin
};

struct LowrankArgs {
  const ExpertDesc* experts;
  int block;
  const int* active;
  const int* n_active;
  const int* counts;
  const int* poffsets;
  __half* act;                // activation buffer, fp16 row-major; reads [0,K), writes columns [K, K+r)
  int Kpad;
  int K;
  int KS;                     // K splits
  int tiles;                  // token tiles of 64 rows per expert covered by the grid
  float* part;                // [KS][prows][64]
  long long part_ks_stride;
  int* sem;                   // [E][sem_stride], zero between launches
  long long sem_stride;
  const int* pslot;           // routing slot of each padded row
  int comp_top_n;             // > 0: rows in slots >= comp_top_n get U = 0 (no compensation)
  unsigned* status;
};

// 2D-tiled shared compensator of one block type (TileQ abstract): z = V_q x
// per source row and column tile, then u_p = sum_q C[e, p, q] z_q per routed
// row and row tile, written as fp16 into the activation columns after Kin.
struct TileqArgs {
  int mode;                   // 0: W1 (sources = tokens, rows of x, bf16); 1: W2 (sources = routed pairs t*k+j, rows of act, fp16)
  const __nv_bfloat16* x;     // mode 0: layer input [T, Kin]
  __half* act;                // activation buffer, fp16 row-major, leading dimension lda
  long long lda;
  const int* pinv;            // [T, k] padded row of (t, j)
  const int* ptok;            // [padded rows] token of each routed row
  const int* pslot;           // [padded rows] routing slot of each routed row
  const int* active;          // experts with rows, n_active of them
  const int* n_active;
  const int* counts;          // [E] routed rows per expert
  const int* poffsets;        // [E+1] first padded row per expert
  int T, k;
  int Kin;                    // input features of the block
  int r;                      // rank, 16 or 32
  int tile_k, Q;              // column tiles
  int P;                      // row tiles; mode 0: tiles < P/2 are gate tiles, the rest up tiles
  const void* v;              // V [r][Kin] row-major, bf16 (mode 0) or fp16 (mode 1): the MMA's B operand
  const __half* c16;          // cores [E][P][Q][r (output i)][r (input j)], fp16
  float* z;                   // [sources][Q][r]
  int comp_top_n;             // > 0: routed rows in slots >= comp_top_n get u = 0
};

struct PrefillArgs {
  CUtensorMap tmap_act;       // activations [rows, Kpad] fp16 row-major; box 64 x 128, 128-byte swizzle
  const ExpertDesc* experts;
  int block;
  const int* active;
  const int* n_active;
  const int* counts;
  const int* poffsets;
  int K;                      // quantised K of the block
  int M;                      // rows of the block
  int mode;
  __half* zout;               // MODE_SWIGLU: output rows (fp16), leading dimension ldz
  long long ldz;
  float* out;                 // MODE_OUT: [prows][M] fp32
  unsigned long long wait_ns; // limit of the hand-off waits between roles
  unsigned* status;
};

struct CombineArgs {
  const float* O;             // [KS][prows][K]
  long long ks_stride;
  int KS;
  const float* w;             // [T, k]
  const int* pinv;            // [T, k]
  int T, k, K;
  __nv_bfloat16* Y;           // [T, K]
};

cudaError_t launch_relayout_int(const uint8_t* canon, uint8_t* out, int M, int K, int bits, int block, int N,
                                cudaStream_t st);
cudaError_t launch_relayout_sz(const __half* s, const __half* z, uint32_t* out, int M, int K, int group, int block,
                               int N, cudaStream_t st);
cudaError_t launch_relayout_dense(const __nv_bfloat16* src, uint8_t* out, int M, int K, int block, int N,
                                  cudaStream_t st);
cudaError_t launch_relayout_afrag(const __nv_bfloat16* src, uint4* out, int r, int K, cudaStream_t st);
cudaError_t launch_relayout_brow(const __nv_bfloat16* src, uint32_t* out, int M, int r, int block, int N,
                                 cudaStream_t st);
struct PlaneOut {
  uint8_t* p[4];  // the four plane buffers, [K/64][M/128][1 KiB] each
};
cudaError_t launch_relayout_planes(const uint32_t* canon, PlaneOut out, int M, int K, int block, int N,
                                   cudaStream_t st);
cudaError_t launch_debug_unpack(const BlockDesc& d, uint8_t* out, int block, int N, cudaStream_t st);

cudaError_t launch_route_topk(const RouteArgs& a, cudaStream_t st, int* launches);
cudaError_t launch_route_fused(const RouteArgs& a, int num_sms, cudaStream_t st, int* launches);
int route_num_blocks(int T);
int route_gather_slices(int T, int K);
int device_sms();

int decode_rows_per_cta();
int decode_ctas();
cudaError_t launch_decode_gemm(const DecodeArgs& a, int ntok, int maxbits, int grid_y, cudaStream_t st,
                               int* launches);
cudaError_t launch_lowrank(const LowrankArgs& a, int grid_y, cudaStream_t st, int* launches);
cudaError_t launch_tileq(const TileqArgs& a, int grid_y, cudaStream_t st, int* launches);
cudaError_t launch_prefill_gemm(const PrefillArgs& a, int grid_y, int grid_z, cudaStream_t st, int* launches);
int prefill_smem_bytes();
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st, int* launches);

}  // namespace moeq
