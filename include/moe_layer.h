/*
 * moe_layer.h - C ABI of the B200 quantized Mixture-of-Experts expert layer.
 *
 * The layer computes, for tokens X [T, K] and router logits [T, E]:
 *
 *   top-k routing      idx[t, 0..k-1] = the k largest logits of token t
 *                      (descending, ties to the lower expert index);
 *                      w[t, j] = softmax over the k selected logits
 *                      (Bandwidth-Efficient Adaptive Mixture-of-Experts via
 *                      Low-Rank Compensation, abstract: per-token Top-n of the
 *                      k routed experts presumes this routing);
 *   bucketing          routed (t, j) pairs grouped per expert, expert-major,
 *                      token-ascending;
 *   per expert e       h = W1^_e x + B1_e (A1_e x)      (W1 = [gate; up], 2N x K)
 *                      z = silu(h[0:N]) * h[N:2N]
 *                      o = W2^_e z + B2_e (A2_e z)      (W2 = down, K x N)
 *                      where W^ is the dequantised weight and B A the rank-r_e
 *                      low-rank compensator of the quantisation residual
 *                      (MiLo: Efficient Quantized MoE Inference with Mixture of
 *                      Low-Rank Compensators, abstract);
 *   combine            y_t = sum_j w[t, j] * o_(t, j).
 *
 * Weight formats (per expert linear block, the "weight page" of PagedWeight:
 * Efficient MoE LLM Serving with Dynamic Quality-Aware Weight Quantization,
 * "What carries the argument"):
 *
 *   MOE_FMT_INT_ASYM     b in {2,3,4}; w^ = (q - z) * s, one fp16 scale s and one
 *                        fp16 zero z per group of g consecutive elements along K.
 *                        codes: uint8 [M, K*b/8], each row a little-endian
 *                        bit-stream, code k at bits [b*k, b*k+b);
 *                        scales, zeros: fp16 [M, K/g] row-major.
 *   MOE_FMT_BITPLANE_LUT 4 stored bit-planes, bitwidth b in {2,3,4} chosen at run
 *                        time (PagedWeight, Figure 3 caption: subsets of
 *                        bit-planes give the effective bitwidths; one LUT of
 *                        bitwidth-specific centroids per quantised tensor).
 *                        codes: uint32 [4, M, K/32]; plane 0 = most significant
 *                        bit; bit i of word w of a row is element 32*w + i; the
 *                        b-bit code is the top b planes; w^ = LUT_b[code].
 *                        zeros_or_lut: fp16 [28] = LUT_2 (4) | LUT_3 (8) | LUT_4 (16).
 *   MOE_FMT_DENSE16      codes: bf16 [M, K] row-major (bits = 16).
 *
 * Compensator factors per block: A bf16 [r, K_in], B bf16 [M_out, r], r = the
 * expert's rank (0 disables the term). A block type may instead carry 2D-tiled
 * factors shared by all experts (moe_layer_set_tileq below).
 *
 * Calls: moe_layer_create / _destroy; moe_layer_set_expert_weights;
 * moe_layer_set_bits; the weight-page calls moe_layer_release_planes /
 * _reload_planes / _page_state; moe_layer_set_tileq / _clear_tileq;
 * moe_layer_set_comp_top_n; moe_layer_set_path; moe_layer_set_wait_limit;
 * moe_layer_forward /
 * _forward_host; test and timing hooks (moe_layer_get_routing,
 * moe_layer_debug_unpack, moe_layer_sync_status, moe_layer_last_launch_count,
 * moe_layer_set_profiling, moe_layer_kernel_times); moe_route_topk_noalloc;
 * the host-only planner moe_plan_reduce / moe_plan_restore; moe_status_string.
 *
 * Conventions.
 *   - Every call returns a moe_status_t; nothing aborts or throws across the ABI.
 *   - The layer owns its device copies of the weights and its workspace (sized
 *     at create from max_tokens and max_top_k). The caller owns X, logits and Y.
 *   - moe_layer_forward is asynchronous on the given CUDA stream; device-side
 *     errors surface at moe_layer_sync_status or at the next call.
 *   - One layer is used from one stream at a time.
 *   - Arithmetic: fp16 tensor-core operands (X, the SwiGLU output and the
 *     compensator terms are rounded to fp16, the tiled compensators' inner
 *     projections and cores too, and the dequantised weights (q - z) * s on
 *     both paths), fp32 accumulation, bf16 output. |X|, |z| and |z * s| must
 *     stay below 65504.
 */
#ifndef MOE_LAYER_H
#define MOE_LAYER_H

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,      /* bad pointer, shape, index or flag */
  MOE_ERR_OOM = 2,              /* a device allocation failed */
  MOE_ERR_NOT_LOADED = 3,       /* forward before every expert's weights were set */
  MOE_ERR_UNSUPPORTED = 4,      /* valid request this build does not implement */
  MOE_ERR_BITS_UNAVAILABLE = 5, /* set_bits asks for planes that are not stored */
  MOE_ERR_CUDA = 6,             /* a CUDA runtime call failed */
  MOE_ERR_DEVICE_CHECK = 7,     /* a kernel's own check failed (status word) */
  MOE_ERR_TIMEOUT = 8,          /* a bounded device-side wait gave up */
  MOE_ERR_TOO_LARGE = 9         /* request exceeds a fixed capacity (moe_route_topk_noalloc) */
} moe_status_t;

typedef enum {
  MOE_FMT_INT_ASYM = 0,
  MOE_FMT_BITPLANE_LUT = 1,
  MOE_FMT_DENSE16 = 2
} moe_format_t;

/* Per-expert descriptor. bits[0] is W1's (gate||up) bitwidth, bits[1] W2's.
 * INT_ASYM: bits in {2,3,4}, group_size in {64,128} dividing d_model and d_ff.
 * BITPLANE_LUT: bits in {2,3,4} (the planes read), group_size ignored.
 * DENSE16: bits = 16. rank: 0..64 (0 disables the compensator; a rank that is
 * not a multiple of 16 is zero-padded to one internally). */
typedef struct {
  int bits[2];
  moe_format_t format;
  int group_size;
  int rank;
} moe_expert_desc_t;

typedef struct moe_layer moe_layer_t; /* opaque */

/* flags for moe_layer_create */
#define MOE_FLAG_NO_TOPK_RENORM 1u /* w[t, j] = full-softmax probability of the selected expert */
#define MOE_FLAG_DETERMINISTIC 2u  /* bitwise-repeatable results; always the case here (no floating-point
                                      atomics: split sums are added in a fixed order), so the flag is
                                      accepted and changes nothing */

/* paths for moe_layer_set_path */
#define MOE_PATH_AUTO 0    /* by T: decode kernels for small batches, prefill kernels above */
#define MOE_PATH_DECODE 1  /* weight-streaming tcgen05 grouped GEMM, unpacked codes in TMEM */
#define MOE_PATH_PREFILL 2 /* TMA + shared-memory dequant + tcgen05/TMEM grouped GEMM */

/* Create a layer on the current CUDA device from per-expert descriptors: each
 * expert's linear blocks carry their own bitwidth (MxMoE abstract: bitwidths
 * chosen per linear block and per expert, mixed-precision) and each expert its
 * own compensator rank (MiLo abstract: per-expert low-rank compensators of the
 * quantisation residual, the rank adapted per expert; a rank of 0 leaves the
 * expert uncompensated).
 * d_model and d_ff: multiples of 128. num_experts <= 256, max_top_k <= 8 and
 * <= num_experts, max_tokens >= 1. descs: [num_experts], copied.
 * Weights start unset (forward returns MOE_ERR_NOT_LOADED until every expert's
 * two blocks are set). On failure *out is NULL. */
moe_status_t moe_layer_create(int num_experts, int d_model, int d_ff, int max_tokens, int max_top_k,
                              const moe_expert_desc_t* descs, unsigned flags, moe_layer_t** out);

/* Load one weight page of one expert (PagedWeight, "What carries the
 * argument": the unit of weight storage and movement is one linear block of
 * one expert, identified by layer, expert and block type): block 0 = W1
 * gate||up [2*d_ff, d_model], 1 = W2 down [d_model, d_ff], from the canonical
 * layouts above, together with the block's compensator factors (MiLo abstract). ptr_kind 0 = host pointers,
 * 1 = device pointers. The data are copied and re-laid out on the device (the
 * caller keeps ownership). scales is used by INT_ASYM only; zeros_or_lut holds
 * the zeros (INT_ASYM) or the 28-entry LUT (BITPLANE_LUT). A and B may be NULL
 * only if the expert's rank is 0. Synchronous. */
moe_status_t moe_layer_set_expert_weights(moe_layer_t* layer, int expert, int block, const void* codes,
                                          const void* scales, const void* zeros_or_lut, const void* A,
                                          const void* B, int ptr_kind);

/* Commit a new bitwidth for (expert, block); block = -1 applies to both.
 * BITPLANE_LUT: 2 <= bits <= 4 (bits > 4: MOE_ERR_BITS_UNAVAILABLE); only the
 * descriptor changes, no weight bytes move (PagedWeight, Figure 4: a lower
 * committed bitwidth reads fewer planes). INT_ASYM: the codes cannot be
 * truncated; the block's descriptor changes and its weights must be set again
 * before the next forward (MOE_ERR_NOT_LOADED until then). DENSE16:
 * MOE_ERR_UNSUPPORTED. Must not be called while a forward is in flight. */
moe_status_t moe_layer_set_bits(moe_layer_t* layer, int expert, int block, int bits);

/* ---- Weight-page movement (BITPLANE_LUT blocks) ----
 * PagedWeight ("What carries the argument"; Figure 4, asynchronous page
 * movement): a weight page is one bit-plane of an expert linear block. Each
 * plane is its own stream-ordered device allocation; released planes move to
 * pinned host memory that the layer owns (and keeps as a cache until the
 * block's weights are set again or the layer is destroyed).
 *
 * moe_layer_release_planes: keep planes 0..keep-1 on the device and release
 * planes keep..3. Requires committed bits <= keep (lower them with
 * moe_layer_set_bits first; 2 <= keep <= 4). On `cuda_stream`, after every
 * forward issued so far: each released plane is copied to host (unless a host
 * copy is already cached) and its device memory is freed. Asynchronous.
 * moe_layer_reload_planes: make planes 0..planes-1 resident again: allocates
 * and copies the missing planes back from host on `cuda_stream`
 * (asynchronous). A later moe_layer_set_bits that needs them waits for these
 * copies before it commits (the pages' rule: reload, then commit the higher
 * bitwidth). moe_layer_set_bits with more bits than resident planes returns
 * MOE_ERR_BITS_UNAVAILABLE. Other formats: MOE_ERR_UNSUPPORTED.
 * moe_layer_page_state: committed bits, resident planes and host-cached planes
 * of (expert, block); any output may be NULL. */
moe_status_t moe_layer_release_planes(moe_layer_t* layer, int expert, int block, int keep, void* cuda_stream);
moe_status_t moe_layer_reload_planes(moe_layer_t* layer, int expert, int block, int planes, void* cuda_stream);
moe_status_t moe_layer_page_state(moe_layer_t* layer, int expert, int block, int* committed_bits,
                                  int* resident_planes, int* host_planes);

/* Router-guided compensation: with n > 0, only the first n routing slots of
 * each token (its n highest-logit experts) get the low-rank compensator; the
 * other slots run on the quantised weights alone (Bandwidth-Efficient
 * Adaptive Mixture-of-Experts via Low-Rank Compensation, abstract: Top-n
 * (n < k) compensation per token). n = 0 (default) compensates every slot.
 * 0 <= n <= max_top_k, else MOE_ERR_INVALID_ARG. */
moe_status_t moe_layer_set_comp_top_n(moe_layer_t* layer, int n);

/* ---- 2D-tiled shared compensators ----
 * TileQ: Efficient Low-Rank Quantization of Mixture-of-Experts with 2D Tiling
 * (abstract: low-rank factors shared across the input and output dimensions
 * of the experts through 2D tiling; the experts' low-rank terms computed in
 * one pass). Reading (the page states no formula): one block type of all
 * experts is cut into P x Q tiles of tile_m rows x tile_k columns; row tile p
 * has an output factor U_p shared by all column tiles and experts, column tile
 * q an input factor V_q shared by all row tiles and experts, and expert e an
 * r x r core per tile; expert e's compensator on tile (p, q) is
 * U_p * C[e][p][q] * V_q. It replaces every expert's own (A, B) pair of that
 * block type (their rank in the descriptors is then ignored for it).
 *
 * moe_layer_set_tileq: block 0 = W1 (M = 2*d_ff rows [gate; up], K_in =
 * d_model), 1 = W2 (M = d_model, K_in = d_ff). All inputs bf16, row-major:
 *   U     [M, rank]              rows p*tile_m .. are U_p
 *   V     [rank, K_in]           columns q*tile_k .. are V_q
 *   cores [E][P][Q][rank][rank]  P = M / tile_m, Q = K_in / tile_k;
 *                                core[e][p][q][i][j] multiplies (V_q x)_j
 *                                into component i of U_p's input.
 * rank 16 or 32; tile_m a multiple of 256 that divides d_ff for W1 (the gate
 * and up halves are tiled separately) or d_model for W2; tile_k a multiple of
 * 256 dividing K_in. ptr_kind 0 = host pointers, 1 = device pointers; the data
 * are copied (the caller keeps ownership). Synchronous; must not be called
 * while a forward is in flight (it may grow the layer's activation buffers).
 * Errors: MOE_ERR_INVALID_ARG for a bad shape, rank or pointer, MOE_ERR_OOM,
 * MOE_ERR_CUDA. The forward then computes z_q = V_q x once per token (W1) or
 * per routed row (W2), u_p = sum_q core[e][p][q] z_q per routed row, and adds
 * U_p u_p inside the quantised GEMM's compensator stage.
 * moe_layer_clear_tileq: back to the experts' own compensators (no-op if the
 * block type has none). Synchronous. */
moe_status_t moe_layer_set_tileq(moe_layer_t* layer, int block, int rank, int tile_m, int tile_k, const void* U,
                                 const void* V, const void* cores, int ptr_kind);
moe_status_t moe_layer_clear_tileq(moe_layer_t* layer, int block);

/* Limit, in nanoseconds, of the bounded waits by which the roles of one GEMM
 * kernel (copy engine, unpack, MMA, epilogue) hand work to each other; 0
 * restores the default of 2 s. A wait that runs out sets the device status
 * word (moe_layer_sync_status then returns MOE_ERR_TIMEOUT), and the CTA
 * drains its own copies and tensor-core operations, frees its tensor memory
 * and returns; the forward's output is then undefined, and the layer stays
 * usable. A limit shorter than a hand-off takes (a few ns) makes every
 * forward give up: that is how the timeout path is tested without any fault.
 * Drains are bounded separately (2 s). Takes effect at the next forward. */
moe_status_t moe_layer_set_wait_limit(moe_layer_t* layer, unsigned long long limit_ns);

/* Choose the kernel path (MOE_PATH_*). */
moe_status_t moe_layer_set_path(moe_layer_t* layer, int path);

/* Forward pass of the quantised MoE expert layer, the computation stated at
 * the top of this header: top-k routing and per-expert bucketing
 * (Bandwidth-Efficient Adaptive Mixture-of-Experts via Low-Rank Compensation,
 * abstract), each routed token through its expert's dequantised SwiGLU FFN
 * plus the low-rank compensator of both linear blocks (MiLo abstract; the
 * fused mixed-precision expert kernel of PagedWeight, "What carries the
 * argument"), outputs combined by router weight.
 * X: bf16 [T, d_model] device; router_logits: fp32 [T, E] device;
 * Y: bf16 [T, d_model] device, caller-allocated. 1 <= T <= max_tokens,
 * 1 <= top_k <= max_top_k. cuda_stream: a cudaStream_t (NULL = legacy stream).
 * Asynchronous. */
moe_status_t moe_layer_forward(moe_layer_t* layer, const void* X, const float* router_logits, int T,
                               int top_k, void* Y, void* cuda_stream);

/* The same forward with HOST buffers: copies X and the logits to the device
 * into layer-owned device buffers (pass pinned host memory for asynchronous
 * copies), runs moe_layer_forward and copies Y
 * back; returns after the stream has synchronised. */
moe_status_t moe_layer_forward_host(moe_layer_t* layer, const void* X_host, const float* logits_host, int T,
                                    int top_k, void* Y_host, void* cuda_stream);

/* Routing of the last forward, copied into caller DEVICE buffers (any may be
 * NULL): idx int32 [T, k], w fp32 [T, k], counts int32 [E], offsets int32
 * [E+1], perm_token int32 [T*k], inv_pos int32 [T, k]. Synchronous. */
moe_status_t moe_layer_get_routing(moe_layer_t* layer, int* idx, float* w, int* counts, int* offsets,
                                   int* perm_token, int* inv_pos);

/* Test hook: the codes of (expert, block) unpacked by the same device routine
 * the GEMM kernels use, as uint8 [M, K] in canonical row order into a caller
 * DEVICE buffer (INT_ASYM: q; BITPLANE_LUT: the code at the committed bits).
 * Synchronous. */
moe_status_t moe_layer_debug_unpack(moe_layer_t* layer, int expert, int block, unsigned char* codes_out);

/* Synchronise the layer's last stream; return the device status word (bounds
 * and wait checks) or the pending CUDA error, and clear the status word. */
moe_status_t moe_layer_sync_status(moe_layer_t* layer);

/* Number of kernels the last moe_layer_forward launched. */
int moe_layer_last_launch_count(const moe_layer_t* layer);

/* Profiling. enable = 1: every forward records a CUDA event on its stream
 * before and after each kernel it launches. enable = 2: only the gate/up
 * expert GEMM (decode or prefill) is bracketed, so that the other launches keep
 * their programmatic overlap. enable = 0: off. Other values: MOE_ERR_INVALID_ARG. */
moe_status_t moe_layer_set_profiling(moe_layer_t* layer, int enable);

/* Durations in ms of the kernels of the last profiled forward, in launch order:
 * names[i] (static strings) and ms[i] for i < min(count, cap). Synchronises the
 * stream. Returns the count, or -1 if nothing was profiled. */
int moe_layer_kernel_times(moe_layer_t* layer, const char** names, float* ms, int cap);

/* Routing without any device allocation. The pages have no counterpart of
 * this call; it exists for callers that cannot allocate device memory: a
 * plugin or extension whose host framework owns all device memory, or a
 * serving loop that must not pay the implicit device-wide synchronisation of
 * cudaMalloc/cudaFree. It runs the layer's top-k routing kernel (the same
 * selection and weights as moe_layer_forward) with its scratch in a fixed
 * 196 KiB array that is part of the library image on every GPU that loads the
 * library, kept until the process exits.
 *   logits: fp32 [T, E] device. Outputs (device, caller-allocated): idx int32
 *   [T, top_k], w fp32 [T, top_k], counts int32 [E], offsets int32 [E+1].
 *   flags: 0 or MOE_FLAG_NO_TOPK_RENORM. Asynchronous on cuda_stream.
 *   Capacity: ceil(T / 16) * E <= 16384 (e.g. T <= 4096 at E = 64, T <= 1024 at
 *   E = 256); larger requests return MOE_ERR_TOO_LARGE before any launch.
 * The first call on a device looks up the array's device address (with that
 * device current); make that first call before any stream capture. Every call
 * shares the one array and clears the words that must start at zero, so calls
 * whose kernels overlap on the GPU (concurrent streams or threads) race and
 * must be serialised by the caller. Calls no allocating routine. The routing
 * kernel's own device-side check (an out-of-range selection, which only a NaN
 * logit row can cause) writes a status word inside the shared array that no
 * call reads back: this call does not report device-side checks, only launch
 * errors (MOE_ERR_CUDA) and argument errors. */
moe_status_t moe_route_topk_noalloc(const float* router_logits, int T, int E, int top_k, unsigned flags, int* idx,
                                    float* w, int* counts, int* offsets, void* cuda_stream);

/* ---- Bitwidth planner (host only) ----
 * PagedWeight ("What carries the argument"): under memory pressure the planner
 * lowers the bitwidths of expert linear blocks ("weight pages") greedily,
 * taking the actions with the lowest predicted damage per released byte until
 * the byte target is met; the predicted damage of an action is
 * d = max(eps, mu * g * eta): g the block's offline sensitivity for that
 * bitwidth transition, mu the multiplier of its routing-mass bucket, eta its
 * exponentiated prompt residual. One action drops one bit-plane (b -> b-1) of
 * one block; floors and per-plan depth caps bound the actions (the pages'
 * bitwidth floor stages and depth caps). Reading where the pages are silent:
 * equal damage per byte goes to the lower block index, and a block's next
 * action becomes a candidate only after its previous one was taken. */
typedef struct {
  int committed_bits;    /* q_i: current bitwidth, 2..4 */
  int floor_bits;        /* lowest bitwidth a plan may assign, 2..committed_bits */
  int max_steps;         /* depth cap: planes one plan may drop (reduce) or restore (restore), >= 0 */
  long long plane_bytes; /* device bytes one bit-plane of the block occupies, > 0 */
  float sensitivity[5];  /* g_i^b for the transition b -> b-1, indices 3 and 4 (others unused) */
  float routing_mult;    /* mu of the block's routing-mass bucket, >= 0 */
  float prompt_factor;   /* eta_i, >= 0 */
} moe_plan_block_t;

/* Reduction plan: releases at least bytes_target bytes if the floors and caps
 * allow. new_bits [n] receives each block's planned bitwidth, *bytes_released
 * the bytes the plan frees. MOE_OK when the target is met, MOE_ERR_TOO_LARGE
 * when every allowed action was taken and the target is still not met (the
 * plan is still written), MOE_ERR_INVALID_ARG for bad arguments. */
moe_status_t moe_plan_reduce(const moe_plan_block_t* blocks, int n, long long bytes_target, float eps,
                             int* new_bits, long long* bytes_released);

/* Restore plan (pressure released, PagedWeight Figure 4: pages are reloaded
 * before a higher bitwidth is committed): undoes reductions, the action whose
 * undo removes the most damage per byte first, up to max_bits[i] per block and
 * while the restored bytes stay within bytes_budget. An action b-1 -> b costs
 * plane_bytes and removes the damage of the transition b -> b-1. new_bits,
 * *bytes_used as above; MOE_OK or MOE_ERR_INVALID_ARG. */
moe_status_t moe_plan_restore(const moe_plan_block_t* blocks, int n, const int* max_bits, long long bytes_budget,
                              float eps, int* new_bits, long long* bytes_used);

const char* moe_status_string(moe_status_t status);

/* Free everything the layer owns. NULL is a no-op. */
void moe_layer_destroy(moe_layer_t* layer);

#ifdef __cplusplus
}
#endif
#endif /* MOE_LAYER_H */
