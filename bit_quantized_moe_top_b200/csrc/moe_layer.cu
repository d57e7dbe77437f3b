// C ABI of the quantized MoE expert layer: ownership, validation, weight
// loading (device re-layout) and the launch sequence of one forward pass.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <vector>

#include <cudaTypedefs.h>

#include "../../include/moe_layer.h"
#include "kernels.h"

using namespace moeq;

namespace {

struct DevBuf {
  void* p = nullptr;
  size_t n = 0;
};

// allocation-failure injection for the error-path tests (host side only)
int g_alloc_count = 0;
int fail_alloc_at() {
  const char* s = std::getenv("MOE_TEST_FAIL_ALLOC_AT");
  return s ? std::atoi(s) : -1;
}

moe_status_t dalloc(DevBuf& b, size_t n) {
  const int at = fail_alloc_at();
  ++g_alloc_count;
  if (at >= 0 && g_alloc_count == at) return MOE_ERR_OOM;
  if (n == 0) n = 16;
  if (cudaMalloc(&b.p, n) != cudaSuccess) {
    cudaGetLastError();
    b.p = nullptr;
    return MOE_ERR_OOM;
  }
  b.n = n;
  return MOE_OK;
}
void dfree(DevBuf& b) {
  if (b.p) cudaFree(b.p);
  b.p = nullptr;
  b.n = 0;
}

// Bit-plane pages of one block: each plane is its own stream-ordered device
// allocation so it can be released to (and restored from) pinned host memory.
struct PlaneStore {
  void* dev[4] = {nullptr, nullptr, nullptr, nullptr};
  void* host[4] = {nullptr, nullptr, nullptr, nullptr};  // pinned copies of released planes (kept as a cache)
  size_t bytes = 0;                                     // bytes of one plane
  int resident = 0;                                     // planes 0..resident-1 are (or are being made) resident
  cudaEvent_t reload = nullptr;                         // completion of the last reload's copies
  bool reload_pending = false;
};

struct BlockStore {
  DevBuf codes, sz, lut, afrag, brow;
  PlaneStore planes;
};

void free_planes(PlaneStore& ps) {
  for (int p = 0; p < 4; ++p) {
    if (ps.dev[p]) cudaFree(ps.dev[p]);
    if (ps.host[p]) cudaFreeHost(ps.host[p]);
    ps.dev[p] = ps.host[p] = nullptr;
  }
  if (ps.reload) cudaEventDestroy(ps.reload);
  ps.reload = nullptr;
  ps.reload_pending = false;
  ps.resident = 0;
  ps.bytes = 0;
}

}  // namespace

struct moe_layer {
  int E = 0, K = 0, N = 0, max_tokens = 0, max_top_k = 0;
  unsigned flags = 0;
  int path = MOE_PATH_AUTO;
  std::vector<moe_expert_desc_t> descs;
  std::vector<ExpertDesc> hdesc;
  std::vector<BlockStore> store;  // [E * 2]
  DevBuf d_experts;
  // workspace
  int rmax_pad = 0, Kpad_x = 0, Kpad_z = 0;
  long long rows_pad_max = 0, nt8cap = 0;
  int nb_max = 0, ks2_max = 1, kslr_max = 1;
  long long sem_stride = 0;
  DevBuf idx, w, counts, offsets, poffsets, active, n_active, ticket, perm, inv_pos, pinv, pslot, ptok, flag;
  unsigned route_epoch = 0;  // value the routing kernel's scan publishes in `flag` (never 0)
  int comp_top_n = 0;
  unsigned long long wait_ns = kDefaultWaitNs;  // hand-off wait limit of the GEMM kernels
  // 2D-tiled shared compensators, per block type (0 = W1, 1 = W2)
  struct Tileq {
    bool on = false;
    int r = 0, tile_m = 0, tile_k = 0, P = 0, Q = 0, cols = 0, span = 0;
    DevBuf brow, v, ct, z;  // v: V [r][Kin] in the z MMA's operand type (W1 bf16, W2 fp16); ct: cores, fp16
  } tq[2];
  DevBuf block_counts, block_base, pblock_base, sem, status;
  DevBuf xact, zact, obuf, part;
  DevBuf sk_part, sk_flag;  // decode GEMM tiles split between two CTAs: partial sums, flags
  unsigned sk_epoch = 0;
  DevBuf hx, hl, hy;  // device buffers for forward_host
  CUtensorMap tmap_x, tmap_z;    // activation buffers, 128-row boxes (prefill GEMMs)
  CUtensorMap tmap_xd, tmap_zd;  // activation buffers, 16-row boxes (decode GEMMs)
  bool have_tmaps = false;
  int last_T = 0, last_k = 0, last_launches = 0;
  cudaStream_t last_stream = nullptr;
  cudaEvent_t fwd_done = nullptr;  // recorded at the end of every forward (page release orders after it)
  // profiling: events around each launch of the last forward (1), or around
  // the gate/up expert GEMM alone (2: the other launches keep their overlap)
  int profiling = 0;
  bool prof_open = false;
  std::vector<cudaEvent_t> events;
  std::vector<const char*> prof_names;
  int prof_count = -1;
};

static bool ensure_events(moe_layer_t* L, size_t n) {
  while (L->events.size() < n) {
    cudaEvent_t ev;
    if (cudaEventCreate(&ev) != cudaSuccess) return false;
    L->events.push_back(ev);
  }
  return true;
}
static bool is_gate_up_gemm(const char* name) { return std::strstr(name, "gemm_w1") != nullptr; }
// records an event before a kernel (profiling only)
static void prof_mark(moe_layer_t* L, cudaStream_t st, const char* name) {
  if (!L->profiling) return;
  if (L->profiling == 2) {
    // level 2: one event before the gate/up GEMM and one after it
    if (L->prof_open) {
      cudaEventRecord(L->events[1], st);
      L->prof_open = false;
    }
    if (is_gate_up_gemm(name) && ensure_events(L, 2)) {
      cudaEventRecord(L->events[0], st);
      L->prof_names.assign(1, name);
      L->prof_open = true;
    }
    return;
  }
  const size_t i = L->prof_names.size();
  if (!ensure_events(L, i + 2)) return;
  cudaEventRecord(L->events[i], st);
  L->prof_names.push_back(name);
}
static void prof_end(moe_layer_t* L, cudaStream_t st) {
  if (!L->profiling) return;
  if (L->profiling == 2) {
    if (L->prof_open) {
      cudaEventRecord(L->events[1], st);
      L->prof_open = false;
    }
    L->prof_count = (int)L->prof_names.size();
    return;
  }
  const size_t i = L->prof_names.size();
  if (L->events.size() > i) cudaEventRecord(L->events[i], st);
  L->prof_count = (int)i;
}

static moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// 2-D tensor map over a row-major fp16 [rows, cols] buffer: box 64 columns x
// box_rows rows, 128-byte swizzle, zero fill outside the buffer.
static bool encode_map(CUtensorMap* map, void* base, int cols, long long rows, int box_cols, int box_rows,
                       CUtensorMapSwizzle swz) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !p)
      return false;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// activation rows: boxes of 64 columns (128 B, 128-byte swizzle)
static bool encode_act_map(CUtensorMap* map, void* base, int cols, long long rows, int box_rows) {
  return encode_map(map, base, cols, rows, 64, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

static bool valid_desc(const moe_expert_desc_t& d, int K, int N) {
  if (d.rank < 0 || d.rank > kMaxRank) return false;
  if (d.format == MOE_FMT_INT_ASYM) {
    for (int b = 0; b < 2; ++b)
      if (d.bits[b] < 2 || d.bits[b] > 4) return false;
    if (d.group_size != 64 && d.group_size != 128) return false;
    if (K % d.group_size || N % d.group_size) return false;
    return true;
  }
  if (d.format == MOE_FMT_BITPLANE_LUT) {
    for (int b = 0; b < 2; ++b)
      if (d.bits[b] < 2 || d.bits[b] > 4) return false;
    return true;
  }
  if (d.format == MOE_FMT_DENSE16) return d.bits[0] == 16 && d.bits[1] == 16;
  return false;
}

static void free_block(BlockStore& s) {
  free_planes(s.planes);
  dfree(s.codes);
  dfree(s.sz);
  dfree(s.lut);
  dfree(s.afrag);
  dfree(s.brow);
}

extern "C" {

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_OOM: return "device allocation failed";
    case MOE_ERR_NOT_LOADED: return "expert weights not loaded";
    case MOE_ERR_UNSUPPORTED: return "unsupported";
    case MOE_ERR_BITS_UNAVAILABLE: return "bitwidth not available";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_CHECK: return "device-side check failed";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_TOO_LARGE: return "request exceeds a fixed capacity";
  }
  return "unknown status";
}

void moe_layer_destroy(moe_layer_t* L) {
  if (!L) return;
  for (auto& s : L->store) free_block(s);
  for (auto& t : L->tq) {
    dfree(t.brow);
    dfree(t.v);
    dfree(t.ct);
    dfree(t.z);
  }
  DevBuf* bufs[] = {&L->d_experts, &L->idx, &L->w, &L->counts, &L->offsets, &L->poffsets, &L->active,
                    &L->n_active, &L->ticket, &L->flag, &L->perm, &L->inv_pos, &L->pinv, &L->pslot, &L->ptok, &L->block_counts,
                    &L->block_base, &L->pblock_base, &L->sem, &L->status, &L->xact, &L->zact, &L->obuf,
                    &L->part, &L->hx, &L->hl, &L->hy, &L->sk_part, &L->sk_flag};
  for (DevBuf* b : bufs) dfree(*b);
  for (cudaEvent_t ev : L->events) cudaEventDestroy(ev);
  if (L->fwd_done) cudaEventDestroy(L->fwd_done);
  delete L;
}

moe_status_t moe_layer_create(int E, int K, int N, int max_tokens, int max_top_k, const moe_expert_desc_t* descs,
                              unsigned flags, moe_layer_t** out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (!descs || E < 1 || E > kMaxExperts || K < 128 || N < 128 || K % 128 || N % 128 || max_tokens < 1 ||
      max_top_k < 1 || max_top_k > kMaxTopK || max_top_k > E || (flags & ~(MOE_FLAG_NO_TOPK_RENORM | MOE_FLAG_DETERMINISTIC)))
    return MOE_ERR_INVALID_ARG;
  int rmax = 0;
  for (int e = 0; e < E; ++e) {
    if (!valid_desc(descs[e], K, N)) return MOE_ERR_INVALID_ARG;
    const int rp = (descs[e].rank + 15) / 16 * 16;
    rmax = rp > rmax ? rp : rmax;
  }
  g_alloc_count = 0;
  moe_layer_t* L = new moe_layer_t();
  L->E = E;
  L->K = K;
  L->N = N;
  L->max_tokens = max_tokens;
  L->max_top_k = max_top_k;
  L->flags = flags;
  L->descs.assign(descs, descs + E);
  L->hdesc.assign(E, ExpertDesc{});
  L->store.resize(2 * E);
  for (int e = 0; e < E; ++e)
    for (int b = 0; b < 2; ++b) {
      BlockDesc& d = L->hdesc[e].blk[b];
      std::memset(&d, 0, sizeof(d));
      d.fmt = descs[e].format == MOE_FMT_INT_ASYM ? FMT_INT : descs[e].format == MOE_FMT_BITPLANE_LUT ? FMT_BITPLANE : FMT_DENSE;
      d.bits = descs[e].bits[b];
      d.group = descs[e].group_size;
      d.rank = (descs[e].rank + 15) / 16 * 16;  // kernels take the rank in k16 steps
      d.M = b == 0 ? 2 * N : K;
      d.K = b == 0 ? K : N;
      d.loaded = 0;
    }
  L->rmax_pad = (rmax + 31) / 32 * 32;
  L->Kpad_x = K + L->rmax_pad;
  L->Kpad_z = N + L->rmax_pad;
  const long long rows = (long long)max_tokens * max_top_k;
  // padded rows of all experts, plus 16 rows of slack: 16-row fragments that
  // start inside the last expert may read (and never store) past its end
  L->rows_pad_max = (rows + 7LL * E + 7) / 8 * 8 + 16;
  L->nt8cap = L->rows_pad_max / 8;
  L->nb_max = route_num_blocks(max_tokens);
  L->ks2_max = 16;
  L->kslr_max = 32;
  // split-K partial outputs (ks2 > 1) are used only when T*k <= 1024
  const long long small_rows = std::min<long long>(L->rows_pad_max, (1024 + 7LL * E + 7) / 8 * 8);
  const long long o_elems = std::max<long long>(L->rows_pad_max, (long long)L->ks2_max * small_rows);
  moe_status_t st = MOE_OK;
  auto A = [&](DevBuf& b, size_t n) {
    if (st == MOE_OK) st = dalloc(b, n);
  };
  A(L->d_experts, sizeof(ExpertDesc) * E);
  A(L->idx, sizeof(int) * rows);
  A(L->w, sizeof(float) * rows);
  A(L->counts, sizeof(int) * E);
  A(L->offsets, sizeof(int) * (E + 1));
  A(L->poffsets, sizeof(int) * (E + 1));
  A(L->active, sizeof(int) * E);
  A(L->n_active, sizeof(int));
  A(L->ticket, sizeof(int));
  A(L->flag, sizeof(int));
  A(L->perm, sizeof(int) * rows);
  A(L->inv_pos, sizeof(int) * rows);
  A(L->pinv, sizeof(int) * rows);
  A(L->pslot, sizeof(int) * (size_t)L->rows_pad_max);
  A(L->ptok, sizeof(int) * (size_t)L->rows_pad_max);
  A(L->block_counts, sizeof(int) * (size_t)L->nb_max * E);
  A(L->block_base, sizeof(int) * (size_t)L->nb_max * E);
  A(L->pblock_base, sizeof(int) * (size_t)L->nb_max * E);
  L->sem_stride = (max_tokens + 63) / 64 + 1;
  A(L->sem, sizeof(int) * E * L->sem_stride);
  A(L->status, sizeof(unsigned));
  A(L->xact, sizeof(__half) * (size_t)L->rows_pad_max * L->Kpad_x);
  A(L->zact, sizeof(__half) * (size_t)L->rows_pad_max * L->Kpad_z);
  A(L->obuf, sizeof(float) * (size_t)o_elems * K);
  A(L->part, sizeof(float) * (size_t)L->kslr_max * L->rows_pad_max * kMaxRank);
  A(L->sk_part, sizeof(float) * (size_t)decode_ctas() * decode_rows_per_cta() * 32);
  A(L->sk_flag, sizeof(unsigned) * (size_t)decode_ctas());
  A(L->hx, sizeof(__nv_bfloat16) * (size_t)max_tokens * K);
  A(L->hl, sizeof(float) * (size_t)max_tokens * E);
  A(L->hy, sizeof(__nv_bfloat16) * (size_t)max_tokens * K);
  if (st != MOE_OK) {
    moe_layer_destroy(L);
    return st;
  }
  cudaError_t ce = cudaSuccess;
  DevBuf* zero[] = {&L->ticket, &L->flag, &L->sem, &L->status, &L->xact, &L->zact, &L->n_active, &L->counts,
                    &L->sk_flag};
  for (DevBuf* b : zero)
    if (ce == cudaSuccess) ce = cudaMemset(b->p, 0, b->n);
  if (ce == cudaSuccess)
    ce = cudaMemcpy(L->d_experts.p, L->hdesc.data(), sizeof(ExpertDesc) * E, cudaMemcpyHostToDevice);
  if (ce == cudaSuccess) ce = cudaEventCreateWithFlags(&L->fwd_done, cudaEventDisableTiming);
  if (ce == cudaSuccess) ce = cudaDeviceSynchronize();
  if (ce != cudaSuccess) {
    moe_layer_destroy(L);
    return MOE_ERR_CUDA;
  }
  L->have_tmaps = encode_act_map(&L->tmap_x, L->xact.p, L->Kpad_x, L->rows_pad_max, 128) &&
                  encode_act_map(&L->tmap_z, L->zact.p, L->Kpad_z, L->rows_pad_max, 128) &&
                  encode_act_map(&L->tmap_xd, L->xact.p, L->Kpad_x, L->rows_pad_max, 16) &&
                  encode_act_map(&L->tmap_zd, L->zact.p, L->Kpad_z, L->rows_pad_max, 16);
  if (!L->have_tmaps) {
    moe_layer_destroy(L);
    return MOE_ERR_CUDA;
  }
  *out = L;
  return MOE_OK;
}

// the device copy of an expert's descriptor: its own blocks, with a block
// type's shared 2D-tiled compensator in place of the expert's factors
static ExpertDesc device_desc(const moe_layer_t* L, int e) {
  ExpertDesc x = L->hdesc[e];
  for (int b = 0; b < 2; ++b) {
    BlockDesc& d = x.blk[b];
    const auto& t = L->tq[b];
    d.tq_span = d.tq_cols = 0;
    if (!t.on) continue;
    d.rank = t.cols;
    d.brow = static_cast<const uint32_t*>(t.brow.p);
    d.afrag = nullptr;
    d.tq_span = t.span;
    d.tq_cols = t.cols;
  }
  return x;
}

static moe_status_t upload_desc(moe_layer_t* L, int e) {
  const ExpertDesc x = device_desc(L, e);
  return cuda_status(
      cudaMemcpy(static_cast<ExpertDesc*>(L->d_experts.p) + e, &x, sizeof(ExpertDesc), cudaMemcpyHostToDevice));
}

// device copy of a caller buffer (host or device); owned by `tmp`
static moe_status_t stage_in(DevBuf& tmp, const void* src, size_t n, int ptr_kind, const void** dev) {
  if (ptr_kind == 1) {
    *dev = src;
    return MOE_OK;
  }
  moe_status_t st = dalloc(tmp, n);
  if (st != MOE_OK) return st;
  if (cudaMemcpy(tmp.p, src, n, cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
  *dev = tmp.p;
  return MOE_OK;
}

moe_status_t moe_layer_set_expert_weights(moe_layer_t* L, int e, int block, const void* codes, const void* scales,
                                          const void* zeros_or_lut, const void* Af, const void* Bf, int ptr_kind) {
  if (!L || e < 0 || e >= L->E || block < 0 || block > 1 || !codes || (ptr_kind != 0 && ptr_kind != 1))
    return MOE_ERR_INVALID_ARG;
  BlockDesc& d = L->hdesc[e].blk[block];
  const int M = d.M, Kin = d.K, r = d.rank;
  if (d.fmt == FMT_INT && (!scales || !zeros_or_lut)) return MOE_ERR_INVALID_ARG;
  if (d.fmt == FMT_BITPLANE && !zeros_or_lut) return MOE_ERR_INVALID_ARG;
  if (r > 0 && (!Af || !Bf)) return MOE_ERR_INVALID_ARG;
  BlockStore& S = L->store[2 * e + block];
  free_block(S);
  d.loaded = 0;
  g_alloc_count = 0;  // allocation-failure injection counts this call's allocations
  moe_status_t st = MOE_OK;
  DevBuf t1, t2, t3, t4, t5;
  const int RB = M / 128, KC = Kin / 64;
  cudaStream_t s0 = 0;
  cudaError_t ce = cudaSuccess;
  const void* dc = nullptr;
  if (d.fmt == FMT_INT) {
    const size_t nbytes = (size_t)M * Kin * d.bits / 8;
    const size_t nsz = (size_t)M * (Kin / d.group) * sizeof(__half);
    const void *ds = nullptr, *dz = nullptr;
    st = stage_in(t1, codes, nbytes, ptr_kind, &dc);
    if (st == MOE_OK) st = stage_in(t2, scales, nsz, ptr_kind, &ds);
    if (st == MOE_OK) st = stage_in(t3, zeros_or_lut, nsz, ptr_kind, &dz);
    if (st == MOE_OK) st = dalloc(S.codes, (size_t)KC * RB * block_bytes(FMT_INT, d.bits));
    if (st == MOE_OK) st = dalloc(S.sz, (size_t)(Kin / d.group) * M * sizeof(uint32_t));
    if (st == MOE_OK) {
      ce = launch_relayout_int(static_cast<const uint8_t*>(dc), static_cast<uint8_t*>(S.codes.p), M, Kin, d.bits,
                               block, L->N, s0);
      if (ce == cudaSuccess)
        ce = launch_relayout_sz(static_cast<const __half*>(ds), static_cast<const __half*>(dz),
                                static_cast<uint32_t*>(S.sz.p), M, Kin, d.group, block, L->N, s0);
    }
  } else if (d.fmt == FMT_BITPLANE) {
    const size_t nbytes = (size_t)4 * M * (Kin / 32) * sizeof(uint32_t);
    const void* dl = nullptr;
    st = stage_in(t1, codes, nbytes, ptr_kind, &dc);
    if (st == MOE_OK) st = stage_in(t3, zeros_or_lut, 28 * sizeof(__half), ptr_kind, &dl);
    PlaneStore& ps = S.planes;
    ps.bytes = (size_t)KC * RB * 1024;
    PlaneOut po;
    for (int p = 0; p < 4 && st == MOE_OK; ++p) {
      const int at = fail_alloc_at();
      ++g_alloc_count;
      if ((at >= 0 && g_alloc_count == at) || cudaMallocAsync(&ps.dev[p], ps.bytes, s0) != cudaSuccess) {
        cudaGetLastError();
        ps.dev[p] = nullptr;
        st = MOE_ERR_OOM;
      }
      po.p[p] = static_cast<uint8_t*>(ps.dev[p]);
    }
    ps.resident = st == MOE_OK ? 4 : 0;
    if (st == MOE_OK) st = dalloc(S.lut, 28 * sizeof(__half));
    if (st == MOE_OK) {
      ce = launch_relayout_planes(static_cast<const uint32_t*>(dc), po, M, Kin, block, L->N, s0);
      if (ce == cudaSuccess) ce = cudaMemcpy(S.lut.p, dl, 28 * sizeof(__half), cudaMemcpyDeviceToDevice);
    }
  } else {
    const size_t nbytes = (size_t)M * Kin * sizeof(__nv_bfloat16);
    st = stage_in(t1, codes, nbytes, ptr_kind, &dc);
    if (st == MOE_OK) st = dalloc(S.codes, nbytes);
    if (st == MOE_OK)
      ce = launch_relayout_dense(static_cast<const __nv_bfloat16*>(dc), static_cast<uint8_t*>(S.codes.p), M, Kin,
                                 block, L->N, s0);
  }
  if (st == MOE_OK && ce == cudaSuccess && r > 0) {
    // factors padded with zeros to the k16 rank r (caller rank r0 <= r)
    const int r0 = L->descs[e].rank;
    const size_t es = sizeof(__nv_bfloat16);
    const void *da = nullptr, *db = nullptr;
    st = dalloc(t4, (size_t)r * Kin * es);
    if (st == MOE_OK) st = dalloc(t5, (size_t)M * r * es);
    if (st == MOE_OK) {
      const cudaMemcpyKind kind = ptr_kind == 1 ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
      ce = cudaMemset(t4.p, 0, t4.n);
      if (ce == cudaSuccess) ce = cudaMemset(t5.p, 0, t5.n);
      if (ce == cudaSuccess) ce = cudaMemcpy(t4.p, Af, (size_t)r0 * Kin * es, kind);
      if (ce == cudaSuccess) ce = cudaMemcpy2D(t5.p, r * es, Bf, r0 * es, r0 * es, M, kind);
      da = t4.p;
      db = t5.p;
    }
    if (st == MOE_OK) st = dalloc(S.afrag, (size_t)r * Kin * sizeof(__half));
    if (st == MOE_OK) st = dalloc(S.brow, (size_t)M * r * sizeof(__half));
    if (st == MOE_OK && ce == cudaSuccess) {
      ce = launch_relayout_afrag(static_cast<const __nv_bfloat16*>(da), static_cast<uint4*>(S.afrag.p), r, Kin, s0);
      if (ce == cudaSuccess)
        ce = launch_relayout_brow(static_cast<const __nv_bfloat16*>(db), static_cast<uint32_t*>(S.brow.p), M, r, block,
                                  L->N, s0);
    }
  }
  if (st == MOE_OK && ce == cudaSuccess) ce = cudaDeviceSynchronize();
  dfree(t1);
  dfree(t2);
  dfree(t3);
  dfree(t4);
  dfree(t5);
  if (st == MOE_OK && ce != cudaSuccess) st = MOE_ERR_CUDA;
  if (st != MOE_OK) {
    free_block(S);
    upload_desc(L, e);
    return st;
  }
  d.codes = static_cast<const uint8_t*>(S.codes.p);
  d.sz = static_cast<const uint32_t*>(S.sz.p);
  d.lut = static_cast<const uint32_t*>(S.lut.p);
  d.afrag = static_cast<const uint4*>(S.afrag.p);
  d.brow = static_cast<const uint32_t*>(S.brow.p);
  for (int p = 0; p < 4; ++p) d.plane[p] = static_cast<const uint8_t*>(S.planes.dev[p]);
  d.loaded = 1;
  return upload_desc(L, e);
}

moe_status_t moe_layer_set_bits(moe_layer_t* L, int e, int block, int bits) {
  if (!L || e < 0 || e >= L->E || block < -1 || block > 1) return MOE_ERR_INVALID_ARG;
  const int b0 = block < 0 ? 0 : block, b1 = block < 0 ? 1 : block;
  const int fmt = L->hdesc[e].blk[b0].fmt;
  if (fmt == FMT_DENSE) return MOE_ERR_UNSUPPORTED;
  if (bits > 4) return MOE_ERR_BITS_UNAVAILABLE;
  if (bits < 2) return MOE_ERR_INVALID_ARG;
  if (fmt == FMT_BITPLANE) {
    // a bitwidth needs its planes resident; a pending reload completes first
    for (int b = b0; b <= b1; ++b) {
      PlaneStore& ps = L->store[2 * e + b].planes;
      if (!L->hdesc[e].blk[b].loaded) continue;
      if (bits > ps.resident) return MOE_ERR_BITS_UNAVAILABLE;
      if (ps.reload_pending) {
        if (cudaEventSynchronize(ps.reload) != cudaSuccess) return MOE_ERR_CUDA;
        ps.reload_pending = false;
      }
    }
  }
  for (int b = b0; b <= b1; ++b) {
    BlockDesc& d = L->hdesc[e].blk[b];
    if (d.bits == bits) continue;
    d.bits = bits;
    L->descs[e].bits[b] = bits;
    if (fmt == FMT_INT) {
      free_block(L->store[2 * e + b]);
      d.loaded = 0;
      d.codes = nullptr;
      d.sz = nullptr;
      d.afrag = nullptr;
      d.brow = nullptr;
    }
  }
  return upload_desc(L, e);
}

moe_status_t moe_layer_release_planes(moe_layer_t* L, int e, int block, int keep, void* stream) {
  if (!L || e < 0 || e >= L->E || block < 0 || block > 1 || keep < 2 || keep > 4) return MOE_ERR_INVALID_ARG;
  BlockDesc& d = L->hdesc[e].blk[block];
  if (d.fmt != FMT_BITPLANE) return MOE_ERR_UNSUPPORTED;
  if (!d.loaded) return MOE_ERR_NOT_LOADED;
  if (keep < d.bits) return MOE_ERR_INVALID_ARG;  // lower the committed bitwidth first
  PlaneStore& ps = L->store[2 * e + block].planes;
  if (keep >= ps.resident) return MOE_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // after every forward issued so far (they may still read these planes)
  cudaError_t ce = cudaStreamWaitEvent(st, L->fwd_done, 0);
  if (ce == cudaSuccess && ps.reload_pending) ce = cudaStreamWaitEvent(st, ps.reload, 0);
  for (int p = keep; p < ps.resident && ce == cudaSuccess; ++p) {
    if (!ps.host[p]) {
      if (cudaMallocHost(&ps.host[p], ps.bytes) != cudaSuccess) {
        cudaGetLastError();
        ps.host[p] = nullptr;
        return MOE_ERR_OOM;
      }
      ce = cudaMemcpyAsync(ps.host[p], ps.dev[p], ps.bytes, cudaMemcpyDeviceToHost, st);
    }
    if (ce == cudaSuccess) ce = cudaFreeAsync(ps.dev[p], st);
    if (ce == cudaSuccess) {
      ps.dev[p] = nullptr;
      d.plane[p] = nullptr;
    }
  }
  if (ce != cudaSuccess) return MOE_ERR_CUDA;
  ps.resident = keep;
  return upload_desc(L, e);
}

moe_status_t moe_layer_reload_planes(moe_layer_t* L, int e, int block, int planes, void* stream) {
  if (!L || e < 0 || e >= L->E || block < 0 || block > 1 || planes < 2 || planes > 4) return MOE_ERR_INVALID_ARG;
  BlockDesc& d = L->hdesc[e].blk[block];
  if (d.fmt != FMT_BITPLANE) return MOE_ERR_UNSUPPORTED;
  if (!d.loaded) return MOE_ERR_NOT_LOADED;
  PlaneStore& ps = L->store[2 * e + block].planes;
  if (planes <= ps.resident) return MOE_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t ce = cudaSuccess;
  if (!ps.reload) ce = cudaEventCreateWithFlags(&ps.reload, cudaEventDisableTiming);
  for (int p = ps.resident; p < planes && ce == cudaSuccess; ++p) {
    if (!ps.host[p]) return MOE_ERR_BITS_UNAVAILABLE;
    ce = cudaMallocAsync(&ps.dev[p], ps.bytes, st);
    if (ce != cudaSuccess) {
      cudaGetLastError();
      ps.dev[p] = nullptr;
      return MOE_ERR_OOM;
    }
    ce = cudaMemcpyAsync(ps.dev[p], ps.host[p], ps.bytes, cudaMemcpyHostToDevice, st);
    d.plane[p] = static_cast<const uint8_t*>(ps.dev[p]);
    ps.resident = p + 1;
  }
  if (ce == cudaSuccess) ce = cudaEventRecord(ps.reload, st);
  if (ce != cudaSuccess) return MOE_ERR_CUDA;
  ps.reload_pending = true;
  return upload_desc(L, e);
}

moe_status_t moe_layer_page_state(moe_layer_t* L, int e, int block, int* committed_bits, int* resident_planes,
                                  int* host_planes) {
  if (!L || e < 0 || e >= L->E || block < 0 || block > 1) return MOE_ERR_INVALID_ARG;
  const BlockDesc& d = L->hdesc[e].blk[block];
  const PlaneStore& ps = L->store[2 * e + block].planes;
  int nh = 0;
  for (int p = 0; p < 4; ++p) nh += ps.host[p] ? 1 : 0;
  if (committed_bits) *committed_bits = d.bits;
  if (resident_planes) *resident_planes = d.fmt == FMT_BITPLANE ? ps.resident : (d.loaded ? d.bits : 0);
  if (host_planes) *host_planes = nh;
  return MOE_OK;
}

moe_status_t moe_layer_set_wait_limit(moe_layer_t* L, unsigned long long limit_ns) {
  if (!L) return MOE_ERR_INVALID_ARG;
  L->wait_ns = limit_ns == 0 ? kDefaultWaitNs : limit_ns;
  return MOE_OK;
}

moe_status_t moe_layer_set_comp_top_n(moe_layer_t* L, int n) {
  if (!L || n < 0 || n > L->max_top_k) return MOE_ERR_INVALID_ARG;
  L->comp_top_n = n;
  return MOE_OK;
}

// Grows the activation buffers to Kin + wx / Kin + wz columns after the
// inputs (wx, wz: compensator columns of W1 / W2), re-encoding their tensor
// maps. Synchronous; no forward may be in flight.
static moe_status_t grow_act(moe_layer_t* L, int wx, int wz) {
  const int kx = std::max(L->Kpad_x, L->K + (wx + 31) / 32 * 32);
  const int kz = std::max(L->Kpad_z, L->N + (wz + 31) / 32 * 32);
  if (kx == L->Kpad_x && kz == L->Kpad_z) return MOE_OK;
  DevBuf nx, nz;
  moe_status_t st = dalloc(nx, sizeof(__half) * (size_t)L->rows_pad_max * kx);
  if (st == MOE_OK) st = dalloc(nz, sizeof(__half) * (size_t)L->rows_pad_max * kz);
  cudaError_t ce = cudaSuccess;
  if (st == MOE_OK) ce = cudaMemset(nx.p, 0, nx.n);
  if (st == MOE_OK && ce == cudaSuccess) ce = cudaMemset(nz.p, 0, nz.n);
  if (st == MOE_OK && ce == cudaSuccess) ce = cudaDeviceSynchronize();
  CUtensorMap mx, mz, mxd, mzd;
  const bool maps = st == MOE_OK && ce == cudaSuccess && encode_act_map(&mx, nx.p, kx, L->rows_pad_max, 128) &&
                    encode_act_map(&mz, nz.p, kz, L->rows_pad_max, 128) &&
                    encode_act_map(&mxd, nx.p, kx, L->rows_pad_max, 16) &&
                    encode_act_map(&mzd, nz.p, kz, L->rows_pad_max, 16);
  if (!maps) {
    dfree(nx);
    dfree(nz);
    return st != MOE_OK ? st : MOE_ERR_CUDA;
  }
  dfree(L->xact);
  dfree(L->zact);
  L->xact = nx;
  L->zact = nz;
  L->Kpad_x = kx;
  L->Kpad_z = kz;
  L->tmap_x = mx;
  L->tmap_z = mz;
  L->tmap_xd = mxd;
  L->tmap_zd = mzd;
  return MOE_OK;
}

static void free_tileq(moe_layer_t::Tileq& t) {
  dfree(t.brow);
  dfree(t.v);
  dfree(t.ct);
  dfree(t.z);
  t.on = false;
}

moe_status_t moe_layer_set_tileq(moe_layer_t* L, int block, int rank, int tile_m, int tile_k, const void* U,
                                 const void* V, const void* cores, int ptr_kind) {
  if (!L || block < 0 || block > 1 || (rank != 16 && rank != 32) || !U || !V || !cores ||
      (ptr_kind != 0 && ptr_kind != 1))
    return MOE_ERR_INVALID_ARG;
  const int K = L->K, N = L->N, E = L->E;
  const int M = block == 0 ? 2 * N : K, Kin = block == 0 ? K : N, half = block == 0 ? N : K;
  if (tile_m < 256 || tile_m % 256 || half % tile_m || tile_k < 256 || tile_k % 256 || Kin % tile_k)
    return MOE_ERR_INVALID_ARG;
  const int r = rank, P = M / tile_m, Q = Kin / tile_k, cols = block == 0 ? 2 * r : r;
  const size_t nU = (size_t)M * r, nV = (size_t)r * Kin, nC = (size_t)E * P * Q * r * r;
  std::vector<uint16_t> hU(nU), hV(nV), hC(nC);
  auto fetch = [&](std::vector<uint16_t>& h, const void* src) {
    if (ptr_kind == 0) {
      std::memcpy(h.data(), src, h.size() * sizeof(uint16_t));
      return cudaSuccess;
    }
    return cudaMemcpy(h.data(), src, h.size() * sizeof(uint16_t), cudaMemcpyDeviceToHost);
  };
  cudaError_t ce = fetch(hU, U);
  if (ce == cudaSuccess) ce = fetch(hV, V);
  if (ce == cudaSuccess) ce = fetch(hC, cores);
  if (ce != cudaSuccess) return MOE_ERR_CUDA;
  // B operand of the compensator stage: W1 gate rows take the first r
  // columns (their gate tile's u), up rows the next r (their up tile's u)
  std::vector<uint16_t> hB((size_t)M * cols, 0);
  for (int m = 0; m < M; ++m)
    for (int c = 0; c < r; ++c) hB[(size_t)m * cols + (block == 0 && m >= N ? r : 0) + c] = hU[(size_t)m * r + c];
  // fp16 operands where the MMA's other side is fp16: V of W2 (its z MMA
  // multiplies fp16 rows of Z) and every core (the u MMA multiplies fp16 z);
  // bf16 -> fp16 is exact for values in fp16's normal range
  auto to_half = [](std::vector<uint16_t>& v) {
    for (auto& x : v) {
      const uint32_t f = (uint32_t)x << 16;
      float fv;
      std::memcpy(&fv, &f, sizeof(fv));
      const __half h = __float2half_rn(fv);
      std::memcpy(&x, &h, sizeof(x));
    }
  };
  if (block == 1) to_half(hV);
  to_half(hC);
  const long long src_rows = block == 0 ? L->max_tokens : (long long)L->max_tokens * L->max_top_k;
  moe_layer_t::Tileq t;
  DevBuf tmpB;
  moe_status_t st = dalloc(t.brow, (size_t)(cols / 2) * M * sizeof(uint32_t));
  if (st == MOE_OK) st = dalloc(tmpB, hB.size() * sizeof(uint16_t));
  if (st == MOE_OK) st = dalloc(t.v, nV * sizeof(uint16_t));
  if (st == MOE_OK) st = dalloc(t.ct, nC * sizeof(uint16_t));
  if (st == MOE_OK) st = dalloc(t.z, (size_t)src_rows * Q * r * sizeof(float));
  if (st == MOE_OK) {
    ce = cudaMemcpy(tmpB.p, hB.data(), hB.size() * sizeof(uint16_t), cudaMemcpyHostToDevice);
    if (ce == cudaSuccess)
      ce = launch_relayout_brow(static_cast<const __nv_bfloat16*>(tmpB.p), static_cast<uint32_t*>(t.brow.p), M,
                                cols, block, N, nullptr);
    if (ce == cudaSuccess) ce = cudaMemcpy(t.v.p, hV.data(), nV * sizeof(uint16_t), cudaMemcpyHostToDevice);
    if (ce == cudaSuccess) ce = cudaMemcpy(t.ct.p, hC.data(), nC * sizeof(uint16_t), cudaMemcpyHostToDevice);
    if (ce == cudaSuccess) ce = cudaDeviceSynchronize();
    if (ce != cudaSuccess) st = MOE_ERR_CUDA;
  }
  dfree(tmpB);
  if (st == MOE_OK) {
    const auto& o = L->tq[1 - block];
    const int w_this = P * r, w_other = o.on ? o.P * o.r : 0;
    st = grow_act(L, block == 0 ? w_this : w_other, block == 0 ? w_other : w_this);
  }
  if (st != MOE_OK) {
    free_tileq(t);
    return st;
  }
  free_tileq(L->tq[block]);
  t.on = true;
  t.r = r;
  t.tile_m = tile_m;
  t.tile_k = tile_k;
  t.P = P;
  t.Q = Q;
  t.cols = cols;
  t.span = block == 0 ? 2 * tile_m : tile_m;  // internal rows per tile (W1 interleaves gate and up rows)
  L->tq[block] = t;
  for (int e = 0; e < E && st == MOE_OK; ++e) st = upload_desc(L, e);
  return st;
}

moe_status_t moe_layer_clear_tileq(moe_layer_t* L, int block) {
  if (!L || block < 0 || block > 1) return MOE_ERR_INVALID_ARG;
  if (!L->tq[block].on) return MOE_OK;
  if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  free_tileq(L->tq[block]);
  moe_status_t st = MOE_OK;
  for (int e = 0; e < L->E && st == MOE_OK; ++e) st = upload_desc(L, e);
  return st;
}

moe_status_t moe_layer_set_path(moe_layer_t* L, int path) {
  if (!L || path < MOE_PATH_AUTO || path > MOE_PATH_PREFILL) return MOE_ERR_INVALID_ARG;
  L->path = path;
  return MOE_OK;
}

int moe_layer_last_launch_count(const moe_layer_t* L) { return L ? L->last_launches : 0; }

moe_status_t moe_layer_set_profiling(moe_layer_t* L, int enable) {
  if (!L || enable < 0 || enable > 2) return MOE_ERR_INVALID_ARG;
  L->profiling = enable;
  L->prof_open = false;
  L->prof_count = -1;
  return MOE_OK;
}

int moe_layer_kernel_times(moe_layer_t* L, const char** names, float* ms, int cap) {
  if (!L || L->prof_count < 0) return -1;
  if (cudaStreamSynchronize(L->last_stream) != cudaSuccess) return -1;
  const int n = L->prof_count;
  for (int i = 0; i < n && i < cap; ++i) {
    if (names) names[i] = L->prof_names[i];
    if (ms) {
      float t = 0.f;
      cudaEventElapsedTime(&t, L->events[i], L->events[i + 1]);
      ms[i] = t;
    }
  }
  return n;
}

moe_status_t moe_layer_forward(moe_layer_t* L, const void* X, const float* logits, int T, int top_k, void* Y,
                               void* stream) {
  if (!L || !X || !logits || !Y || T < 1 || T > L->max_tokens || top_k < 1 || top_k > L->max_top_k)
    return MOE_ERR_INVALID_ARG;
  for (int e = 0; e < L->E; ++e)
    if (!L->hdesc[e].blk[0].loaded || !L->hdesc[e].blk[1].loaded) return MOE_ERR_NOT_LOADED;
  bool any_dense = false;
  for (int e = 0; e < L->E; ++e) any_dense |= L->hdesc[e].blk[0].fmt == FMT_DENSE;
  int path = L->path;
  if (path == MOE_PATH_AUTO)
    path = ((long long)T * top_k >= 64LL * L->E && !any_dense && L->have_tmaps) ? MOE_PATH_PREFILL : MOE_PATH_DECODE;
  if (path == MOE_PATH_PREFILL && (any_dense || !L->have_tmaps)) return MOE_ERR_UNSUPPORTED;
  const bool prefill = path == MOE_PATH_PREFILL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int E = L->E, K = L->K, N = L->N;
  int maxbits[2] = {0, 0}, rmax = 0;
  bool uniform[2] = {true, true};
  for (int e = 1; e < E; ++e)
    for (int b = 0; b < 2; ++b) {
      const BlockDesc& x = L->hdesc[e].blk[b];
      const BlockDesc& y = L->hdesc[0].blk[b];
      uniform[b] = uniform[b] && x.fmt == y.fmt && x.bits == y.bits && x.group == y.group && x.rank == y.rank;
    }
  for (int e = 0; e < E; ++e) {
    for (int b = 0; b < 2; ++b) {
      const int bb = L->hdesc[e].blk[b].bits;
      maxbits[b] = bb > maxbits[b] ? bb : maxbits[b];
    }
    rmax = L->hdesc[e].blk[0].rank > rmax ? L->hdesc[e].blk[0].rank : rmax;
  }
  const long long rows = (long long)T * top_k;
  const int grid_y = (int)std::min<long long>(E, rows);
  int launches = 0;
  cudaError_t ce = cudaSuccess;

  RouteArgs ra{};
  ra.logits = logits;
  ra.X = static_cast<const __nv_bfloat16*>(X);
  ra.T = T;
  ra.E = E;
  ra.k = top_k;
  ra.K = K;
  ra.renorm = (L->flags & MOE_FLAG_NO_TOPK_RENORM) ? 0 : 1;
  ra.idx = static_cast<int*>(L->idx.p);
  ra.w = static_cast<float*>(L->w.p);
  ra.block_counts = static_cast<int*>(L->block_counts.p);
  ra.block_base = static_cast<int*>(L->block_base.p);
  ra.pblock_base = static_cast<int*>(L->pblock_base.p);
  ra.counts = static_cast<int*>(L->counts.p);
  ra.offsets = static_cast<int*>(L->offsets.p);
  ra.poffsets = static_cast<int*>(L->poffsets.p);
  ra.active = static_cast<int*>(L->active.p);
  ra.n_active = static_cast<int*>(L->n_active.p);
  ra.ticket = static_cast<int*>(L->ticket.p);
  ra.perm_token = static_cast<int*>(L->perm.p);
  ra.inv_pos = static_cast<int*>(L->inv_pos.p);
  ra.pinv = static_cast<int*>(L->pinv.p);
  ra.pslot = static_cast<int*>(L->pslot.p);
  ra.ptok = static_cast<int*>(L->ptok.p);
  ra.act = L->xact.p;
  ra.Kpad = L->Kpad_x;
  ra.status = static_cast<unsigned*>(L->status.p);
  const ExpertDesc* dexp = static_cast<const ExpertDesc*>(L->d_experts.p);
  if (++L->route_epoch == 0) L->route_epoch = 1;
  ra.flag = static_cast<int*>(L->flag.p);
  ra.epoch = L->route_epoch;
  ra.nb = route_num_blocks(T);
  ra.gs = route_gather_slices(T, K);
  ra.wait_ns = L->wait_ns;
  L->prof_names.clear();
  prof_mark(L, st, "route");
  ce = launch_route_fused(ra, device_sms(), st, &launches);

  const long long prows = (rows + 7LL * E + 7) / 8 * 8;
  // the low-rank down-projection U = V A^T of a block's routed rows
  auto lowrank = [&](int block, __half* act, int Kpad, int Kin) {
    if (ce != cudaSuccess || rmax == 0) return;
    LowrankArgs la{};
    la.experts = dexp;
    la.block = block;
    la.active = ra.active;
    la.n_active = ra.n_active;
    la.counts = ra.counts;
    la.poffsets = ra.poffsets;
    la.act = act;
    la.Kpad = Kpad;
    la.K = Kin;
    // token tiles of 64 rows per expert; split K only while the grid is small
    la.tiles = (int)std::min<long long>((T + 63) / 64, (rows + 63) / 64);
    // about eight CTAs per SM: rows / 64 tiles plus the experts' ragged tails
    const long long ctas = (rows + 63) / 64 + grid_y / 2;
    int ks = (int)std::max<long long>(1, (1184 + ctas - 1) / std::max<long long>(1, ctas));
    ks = std::max(1, std::min(ks, std::min(L->kslr_max, Kin / 256)));
    la.KS = ks;
    la.sem_stride = L->sem_stride;
    la.pslot = ra.pslot;
    la.comp_top_n = L->comp_top_n;
    la.part = static_cast<float*>(L->part.p);
    la.part_ks_stride = (long long)L->rows_pad_max * kMaxRank;
    la.sem = static_cast<int*>(L->sem.p);
    la.status = ra.status;
    prof_mark(L, st, block == 0 ? "lowrank_w1" : "lowrank_w2");
    ce = launch_lowrank(la, grid_y, st, &launches);
  };
  // a block type's shared 2D-tiled compensator: z = V x, u = C z
  auto tileq = [&](int block) {
    const auto& t = L->tq[block];
    if (ce != cudaSuccess || !t.on) return;
    TileqArgs ta{};
    ta.mode = block;
    ta.x = static_cast<const __nv_bfloat16*>(X);
    ta.act = static_cast<__half*>(block == 0 ? L->xact.p : L->zact.p);
    ta.lda = block == 0 ? L->Kpad_x : L->Kpad_z;
    ta.pinv = ra.pinv;
    ta.ptok = ra.ptok;
    ta.pslot = ra.pslot;
    ta.active = ra.active;
    ta.n_active = ra.n_active;
    ta.counts = ra.counts;
    ta.poffsets = ra.poffsets;
    ta.T = T;
    ta.k = top_k;
    ta.Kin = block == 0 ? K : N;
    ta.r = t.r;
    ta.tile_k = t.tile_k;
    ta.Q = t.Q;
    ta.P = t.P;
    ta.v = t.v.p;
    ta.c16 = static_cast<const __half*>(t.ct.p);
    ta.z = static_cast<float*>(t.z.p);
    ta.comp_top_n = L->comp_top_n;
    prof_mark(L, st, block == 0 ? "tileq_w1" : "tileq_w2");
    ce = launch_tileq(ta, grid_y, st, &launches);
  };
  // W1 side compensator U1 = X A1^T
  lowrank(0, static_cast<__half*>(L->xact.p), L->Kpad_x, K);
  tileq(0);
  int ks2 = 1;
  if (prefill) {
    // tcgen05 path: one launch per block, CTAs over (row tile, 256-token pair, expert)
    const int pairs = (T + 255) / 256;
    auto prefill_gemm = [&](int block, const CUtensorMap& map, int Kin, int M, int mode) {
      if (ce != cudaSuccess) return;
      PrefillArgs pa;
      std::memset(&pa, 0, sizeof(pa));
      pa.tmap_act = map;
      pa.experts = dexp;
      pa.block = block;
      pa.active = ra.active;
      pa.n_active = ra.n_active;
      pa.counts = ra.counts;
      pa.poffsets = ra.poffsets;
      pa.K = Kin;
      pa.M = M;
      pa.mode = mode;
      pa.zout = static_cast<__half*>(L->zact.p);
      pa.ldz = L->Kpad_z;
      pa.out = static_cast<float*>(L->obuf.p);
      pa.wait_ns = L->wait_ns;
      pa.status = ra.status;
      prof_mark(L, st, block == 0 ? "prefill_gemm_w1_swiglu" : "prefill_gemm_w2");
      ce = launch_prefill_gemm(pa, pairs, grid_y, st, &launches);
    };
    prefill_gemm(0, L->tmap_x, K, 2 * N, MODE_SWIGLU);
    lowrank(1, static_cast<__half*>(L->zact.p), L->Kpad_z, N);
    tileq(1);
    prefill_gemm(1, L->tmap_z, N, K, MODE_OUT);
  } else {
    // tokens per pass: cover the expected per-expert batch (mean + 3 sd);
    // larger batches take more passes
    const double avg = (double)rows / E;
    const int want = (int)std::ceil(avg + 3.0 * std::sqrt(avg) + 1.0);
    // (larger batches take more passes, run as separate tiles that share the weights through L2)
    const int ntok = std::min(T, want) <= 16 ? 16 : 32;
    auto decode_gemm = [&](int block, const CUtensorMap& map, int Kin, int M, int mode, int KS) {
      if (ce != cudaSuccess) return;
      DecodeArgs da;
      std::memset(&da, 0, sizeof(da));
      da.tmap_act = map;
      da.experts = dexp;
      da.block = block;
      da.active = ra.active;
      da.n_active = ra.n_active;
      da.counts = ra.counts;
      da.poffsets = ra.poffsets;
      da.K = Kin;
      da.M = M;
      da.mode = mode;
      da.zout = static_cast<__half*>(L->zact.p);
      da.ldz = L->Kpad_z;
      da.out = static_cast<float*>(L->obuf.p);
      da.out_ks_stride = prows * K;
      da.KS = KS;
      da.rows = rows;
      da.wait_ns = L->wait_ns;
      da.status = ra.status;
      // tiles split between CTAs only where every expert's block has the same
      // format, bits, group and rank (steps of one cost); with mixed blocks
      // the split measured slower than whole tiles
      da.sk_part = uniform[block] ? static_cast<float*>(L->sk_part.p) : nullptr;
      da.mixed = uniform[block] ? 0 : 1;
      da.sk_flag = static_cast<unsigned*>(L->sk_flag.p);
      if (++L->sk_epoch == 0) L->sk_epoch = 1;
      da.sk_epoch = L->sk_epoch;
      prof_mark(L, st, block == 0 ? "decode_gemm_w1_swiglu" : "decode_gemm_w2");
      ce = launch_decode_gemm(da, ntok, maxbits[block], grid_y, st, &launches);
    };
    decode_gemm(0, L->tmap_xd, K, 2 * N, MODE_SWIGLU, 1);
    lowrank(1, static_cast<__half*>(L->zact.p), L->Kpad_z, N);
    tileq(1);
    // split the down projection's K (fixed-order sum of the partials in the
    // combine); splits at least 256 columns wide, and at least one split.
    // With tiles split between CTAs, only until there are at least as many
    // tiles as CTAs (from there the kernel balances the shares at step
    // granularity); otherwise where that shortens the busiest CTA's share:
    // each CTA takes ceil(units / CTAs) units of 128 rows x (N / 64 / KS)
    // chunks, plus about 3 chunks of pipeline fill per unit
    const long long units1 = (long long)(K / decode_rows_per_cta()) * grid_y;
    const int ctas = decode_ctas(), kmax = std::max(1, std::min(L->ks2_max, N / 256));
    if (uniform[1]) {
      while (units1 * ks2 < ctas && ks2 < kmax) ++ks2;
    } else {
      double best = 0.0;
      for (int ks = 1; ks <= kmax; ++ks) {
        const double t = (double)((units1 * ks + ctas - 1) / ctas) * ((double)N / 64.0 / ks + 3.0);
        if (ks == 1 || t < best * 0.98) {
          best = t;
          ks2 = ks;
        }
      }
    }
    if (rows > 1024) ks2 = 1;
    decode_gemm(1, L->tmap_zd, N, K, MODE_OUT, ks2);
  }
  if (ce == cudaSuccess) {
    CombineArgs ca{};
    ca.O = static_cast<const float*>(L->obuf.p);
    ca.ks_stride = prows * K;
    ca.KS = ks2;
    ca.w = ra.w;
    ca.pinv = ra.pinv;
    ca.T = T;
    ca.k = top_k;
    ca.K = K;
    ca.Y = static_cast<__nv_bfloat16*>(Y);
    prof_mark(L, st, "combine");
    ce = launch_combine(ca, st, &launches);
  }
  prof_end(L, st);
  cudaEventRecord(L->fwd_done, st);
  L->last_T = T;
  L->last_k = top_k;
  L->last_launches = launches;
  L->last_stream = st;
  return cuda_status(ce);
}

moe_status_t moe_layer_forward_host(moe_layer_t* L, const void* Xh, const float* Lh, int T, int top_k, void* Yh,
                                    void* stream) {
  if (!L || !Xh || !Lh || !Yh || T < 1 || T > L->max_tokens) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t xb = (size_t)T * L->K * sizeof(__nv_bfloat16), lb = (size_t)T * L->E * sizeof(float);
  cudaError_t ce = cudaMemcpyAsync(L->hx.p, Xh, xb, cudaMemcpyHostToDevice, st);
  if (ce == cudaSuccess) ce = cudaMemcpyAsync(L->hl.p, Lh, lb, cudaMemcpyHostToDevice, st);
  if (ce != cudaSuccess) return MOE_ERR_CUDA;
  moe_status_t s = moe_layer_forward(L, L->hx.p, static_cast<const float*>(L->hl.p), T, top_k, L->hy.p, stream);
  if (s != MOE_OK) return s;
  ce = cudaMemcpyAsync(Yh, L->hy.p, xb, cudaMemcpyDeviceToHost, st);
  if (ce == cudaSuccess) ce = cudaStreamSynchronize(st);
  return cuda_status(ce);
}

moe_status_t moe_layer_get_routing(moe_layer_t* L, int* idx, float* w, int* counts, int* offsets, int* perm_token,
                                   int* inv_pos) {
  if (!L || L->last_T == 0) return MOE_ERR_INVALID_ARG;
  const size_t tk = (size_t)L->last_T * L->last_k;
  cudaError_t ce = cudaStreamSynchronize(L->last_stream);
  auto cp = [&](void* dst, const DevBuf& src, size_t n) {
    if (dst && ce == cudaSuccess) ce = cudaMemcpy(dst, src.p, n, cudaMemcpyDeviceToDevice);
  };
  cp(idx, L->idx, tk * sizeof(int));
  cp(w, L->w, tk * sizeof(float));
  cp(counts, L->counts, L->E * sizeof(int));
  cp(offsets, L->offsets, (L->E + 1) * sizeof(int));
  cp(perm_token, L->perm, tk * sizeof(int));
  cp(inv_pos, L->inv_pos, tk * sizeof(int));
  return cuda_status(ce);
}

moe_status_t moe_layer_debug_unpack(moe_layer_t* L, int e, int block, unsigned char* out) {
  if (!L || e < 0 || e >= L->E || block < 0 || block > 1 || !out) return MOE_ERR_INVALID_ARG;
  const BlockDesc& d = L->hdesc[e].blk[block];
  if (!d.loaded) return MOE_ERR_NOT_LOADED;
  if (d.fmt == FMT_DENSE) return MOE_ERR_UNSUPPORTED;
  cudaError_t ce = launch_debug_unpack(d, out, block, L->N, 0);
  if (ce == cudaSuccess) ce = cudaDeviceSynchronize();
  return cuda_status(ce);
}

moe_status_t moe_layer_sync_status(moe_layer_t* L) {
  if (!L) return MOE_ERR_INVALID_ARG;
  cudaError_t ce = cudaStreamSynchronize(L->last_stream);
  if (ce == cudaSuccess) ce = cudaGetLastError();
  if (ce != cudaSuccess) return MOE_ERR_CUDA;
  unsigned word = 0;
  ce = cudaMemcpy(&word, L->status.p, sizeof(unsigned), cudaMemcpyDeviceToHost);
  if (ce != cudaSuccess) return MOE_ERR_CUDA;
  if (word) {
    cudaMemset(L->status.p, 0, sizeof(unsigned));
    return (word & ST_TIMEOUT) ? MOE_ERR_TIMEOUT : MOE_ERR_DEVICE_CHECK;
  }
  return MOE_OK;
}

}  // extern "C"
