/*
 * moe.h -- C ABI of the B200 routed-expert MoE layer (libmoe.so).
 *
 * The layer is the routed-expert MoE forward described in the FreeToken
 * write-ups: each token picks k of E experts (freetoken.wiki, "FreeToken 753b
 * model", section "FreeToken 753b Model Explained"), the experts live in a
 * GPU expert cache that follows router demand with LRU eviction (same page,
 * mechanism table, "Global LRU expert cache"), missed experts are either
 * filled over PCIe or computed on the CPU, and the two shares of partial sums
 * are added without approximation (explainx.ai hardware guide, section
 * "Decode: decide whether to move an expert or compute where it lives";
 * ainewsfeed.tech, third paragraph).
 *
 * Conventions for every call
 *   - Ownership: the caller allocates every device buffer, the pinned host
 *     pool and every output; no call allocates device memory.  The only
 *     library-owned object is the host-side cache handle (moe_cache).
 *   - Asynchrony: calls that take a cudaStream_t validate their arguments
 *     synchronously, enqueue kernels or copies on that stream and return.
 *     Results are ready when the stream reaches that point.
 *   - Errors: every call returns moe_status.  MOE_OK = success.  On failure
 *     nothing was enqueued, and moe_last_error() (per thread) describes it.
 *     Kernels that detect a bad index at run time (an expert id or slot out of
 *     range) skip the access and record MOE_ERR_DEVICE in the caller's
 *     dev_status word (first error wins); moe_check_status() reads it.
 *     No kernel traps, and no call throws across the ABI.
 *   - Pointers marked "device" must be device memory of the current device;
 *     float/bf16 tensors and byte pools must be 16-byte aligned; int32 arrays
 *     4-byte aligned.
 *   - Index conventions: T tokens, E experts, k experts per token, d hidden
 *     size, I SwiGLU intermediate size; pair p = t*k + j is the j-th choice
 *     of token t; "sorted position" q is the index of a pair after grouping
 *     pairs by expert.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* bad size, null or misaligned pointer, bad id */
  MOE_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement */
  MOE_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
  MOE_ERR_CAPACITY = 4,     /* not enough cache slots, workspace or scratch */
  MOE_ERR_TIMEOUT = 5,      /* a bounded device-side wait ran out */
  MOE_ERR_DEVICE = 6        /* a kernel reported an out-of-range index */
} moe_status;

/* Expert weight formats (explainx.ai hardware guide: NVFP4 routed experts;
 * freetoken.wiki: NVFP4 or MXFP4 builds; fervorai.dev, "What to know before
 * you commit": NVFP4, MXFP4, FP8 and BF16).  Bit layouts: BF16; MXFP4 = E2M1
 * values with one E8M0 scale per 32 elements (OCP MX v1.0); NVFP4 = E2M1
 * values with one E4M3 scale per 16 elements and one fp32 scale per matrix. */
typedef enum moe_wfmt { MOE_W_BF16 = 0, MOE_W_MXFP4 = 1, MOE_W_NVFP4 = 2 } moe_wfmt;

/* Layer shape.  Limits: 1 <= E <= 1024; d and I multiples of 8 (BF16),
 * 32 (MXFP4) or 128 (NVFP4); d, I <= 16384. */
typedef struct moe_shape { int32_t E, d, I, fmt; } moe_shape;

/* moe_expert_ffn flags. */
enum {
  /* Quantise x and the SwiGLU output to NVFP4 (unit tensor scale, one E4M3
   * scale per 16 elements, round-to-nearest-even) before the two products and
   * run them on the FP4 tensor cores.  Requires MOE_W_NVFP4.  Without this
   * flag NVFP4 weights run on the CUDA-core path with the activations kept in
   * bf16/fp32 (BF16 and MXFP4 weights never quantise the activations). */
  MOE_FFN_ACT_NVFP4 = 1
};

/* Version of this ABI (bumped on any signature change). */
int moe_abi_version(void);

/* Testing aid, no counterpart in the pages: every wait of the tensor-core
 * kernels (a pipeline stage, a token-row stage, an accumulator) is bounded;
 * when the limit passes, the CTA records MOE_ERR_TIMEOUT in the status word,
 * stops issuing, drains the copies and MMAs it issued (those drains keep the
 * 2 s bound), frees its tensor memory and returns, so the context stays
 * usable.  This sets the limit for kernels launched afterwards by any thread
 * (ns; 0 restores the default 2 s) and returns the previous one; tests use a
 * few ns to make that path run. */
uint64_t moe_set_wait_limit_ns(uint64_t ns);

/* Testing aid, no counterpart in the pages: while on (nonzero), the
 * tensor-core kernels launched afterwards make CTA 0's epilogue first wait on
 * a barrier that nothing arrives on, so that wait runs out after the limit
 * above and the abort path runs: the call's status word then holds
 * MOE_ERR_TIMEOUT and its outputs are incomplete.  Returns the previous
 * setting.  Nothing faults or hangs: the wait is bounded like every other. */
int moe_set_test_stall(int on);

/* Message of the last failed call on this thread ("" if none). */
const char* moe_last_error(void);

/* ------------------------------------------------------------------------ */
/* Expert blobs.  An expert's weights are stored as one contiguous blob in a
 * device-final layout, identical in the pinned host pool and in a GPU cache
 * slot, so a cache fill is a single copy (futuresignalnews.com, mechanism 3:
 * experts are read into their final host layout and pinned; explainx.ai
 * hardware guide: the FTW layout).  The layout is private to the library. */

/* Bytes of one expert blob (a multiple of 256), or 0 if the shape is invalid.
 * Slot s of a pool starts at pool + s * moe_expert_blob_bytes(shape). */
size_t moe_expert_blob_bytes(moe_shape s);

/* Host-only: build the blob of one expert from canonical row-major tensors.
 *   BF16 : wg, wu = bf16 [I][d]; wd = bf16 [d][I]; sg/su/sd/tensor_scales NULL.
 *   MXFP4: wg, wu = [I][d/2] bytes, wd = [d][I/2] bytes (element 2i in the low
 *          nibble); sg, su = [I][d/32], sd = [d][I/32] E8M0 bytes.
 *   NVFP4: codes as MXFP4; sg, su = [I][d/16], sd = [d][I/16] E4M3 bytes;
 *          tensor_scales = 3 floats (gate, up, down).
 * blob_out: host buffer of moe_expert_blob_bytes(s) bytes.  No CUDA call. */
moe_status moe_pack_expert(moe_shape s, const void* wg, const void* wu, const void* wd,
                           const uint8_t* sg, const uint8_t* su, const uint8_t* sd,
                           const float* tensor_scales, void* blob_out);

/* ------------------------------------------------------------------------ */
/* Step 1 -- top-k expert selection (freetoken.wiki, "FreeToken 753b Model
 * Explained": a token routes through 6 of 256 experts; explainx.ai, "Decode":
 * expert choice per token).  The router is not modified (ainewsfeed.tech,
 * third paragraph): gates are the softmax of the k selected logits.
 *   logits: device fp32 [T][E], finite.
 *   idx:    device int32 [T][k]: the k largest logits of each row, ordered by
 *           logit descending then expert index ascending (ties, including
 *           -0.0 vs +0.0, go to the lower index).
 *   gate:   device fp32 [T][k]: exp(l_j - l_0) / sum_i exp(l_i - l_0).
 * Limits: 1 <= k <= min(E, 32), E <= 1024, T >= 0 (T = 0 enqueues nothing). */
moe_status moe_route_topk(const float* logits, int T, int E, int k,
                          int32_t* idx, float* gate, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Step 2 -- permutation of token-expert pairs by expert, so each expert's
 * FFN runs once per step on all the tokens routed to it (ainewsfeed.tech,
 * second paragraph: many tokens of a layer route to nearly the whole expert
 * set).  A stable counting sort of the pairs p = t*k + j by idx[t][j]:
 *   offsets:  device int32 [E+1], offsets[e] = number of pairs with expert < e.
 *   perm:     device int32 [T*k], perm[q] = pair at sorted position q; pairs of
 *             one expert appear in ascending p.
 *   inv_perm: device int32 [T*k], inv_perm[perm[q]] = q.
 *   scratch:  device buffer of at least moe_permute_scratch_bytes(T, k, E)
 *             bytes (may be NULL when that is 0); contents need no setup.
 *   dev_status: device int32 word or NULL; an idx value outside [0, E) is
 *             recorded there as MOE_ERR_DEVICE and its pair is dropped. */
size_t moe_permute_scratch_bytes(int T, int k, int E);
moe_status moe_permute(const int32_t* idx, int T, int k, int E,
                       int32_t* offsets, int32_t* perm, int32_t* inv_perm,
                       void* scratch, size_t scratch_bytes, int32_t* dev_status,
                       cudaStream_t stream);

/* moe_permute_noalloc -- the same permutation as moe_permute, for callers
 * that cannot allocate device memory: for example a caller embedded in a host
 * engine that has already reserved the device's memory for its own pool (a
 * separate cudaMalloc there can fail, or stall the engine), or a caller on a
 * latency-critical path that cannot afford an allocation call.  It takes no
 * scratch argument and makes no allocation of any kind; its scratch is a
 * fixed array of MOE_PERMUTE_NOALLOC_MAX_SCRATCH bytes compiled into the
 * library, which every device that loads the library holds until the process
 * exits.  The paper has no counterpart to this call.
 *   Limits: moe_permute_scratch_bytes(T, k, E) <= MOE_PERMUTE_NOALLOC_MAX_SCRATCH
 *     (e.g. T*k <= 65536 pairs at E = 1024, <= 262144 at E = 256); larger
 *     problems return MOE_ERR_CAPACITY with nothing enqueued.
 *   Set-up: the first call on a device (with that device current) looks up
 *     the array's device address once; make that first call before any
 *     stream capture.
 *   Sharing: every call on a device uses the same array, which keeps the last
 *     call's contents (the kernels overwrite every entry they read, so nothing
 *     has to start at zero).  Calls that overlap on the GPU -- on different
 *     streams, or from several host threads without ordering -- race on it.
 *   Arguments, outputs and errors are those of moe_permute. */
#define MOE_PERMUTE_NOALLOC_MAX_SCRATCH 262144
moe_status moe_permute_noalloc(const int32_t* idx, int T, int k, int E,
                               int32_t* offsets, int32_t* perm, int32_t* inv_perm,
                               int32_t* dev_status, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Step 3 -- grouped SwiGLU expert FFN over the expert cache.  For every
 * expert e with slot_of_expert[e] >= 0 and every pair at sorted position q in
 * [offsets[e], offsets[e+1]) with token t = perm[q] / k:
 *     h = W_g x_t,  u = W_u x_t,  a = silu(h) * u,  y_q = W_d a
 * with the weights read from the blob at slot_pool + slot * blob_bytes.
 * Experts with slot -1 are not evaluated here: their pairs are computed
 * elsewhere (the host share of the misses; explainx.ai, "Decode").
 *   x:      device bf16 [T][d].
 *   offsets, perm: from moe_permute.  slot_of_expert: device int32 [E].
 *   slot_pool: device, n_slots blobs.
 *   Output, one of:
 *     y_perm != NULL: y_perm[q][:] = y_q (fp32 [T*k][d], unweighted); rows of
 *                     skipped experts are left untouched.  Not available with
 *                     MOE_FFN_ACT_NVFP4.
 *     y_perm == NULL: out[t][:] += gate[t][j] * y_q (fp32 [T][d]) for p = t*k+j,
 *                     accumulated with atomic adds; the caller initialises out
 *                     (zeros, or the host partial).
 *   flags: 0 or MOE_FFN_ACT_NVFP4.
 *   workspace: device, 256-byte aligned, >= moe_expert_ffn_workspace_bytes(s,
 *              T, k, flags); its contents need no initialisation.
 *   dev_status: device int32 word or NULL.  Kernels record the first error
 *              there (read it with moe_check_status after the stream):
 *              MOE_ERR_DEVICE   a slot or expert index out of range;
 *              MOE_ERR_TIMEOUT  a bounded wait on the copy pipeline ran out.
 *              (The MXFP4 tensor-core path applies the E8M0 scales in the
 *              tensor core and takes the activations as E4M3 terms under E8M0
 *              scales of their own: no range limit beyond fp32's.)
 * Paths (chosen from the shape, the same results up to rounding order):
 *   BF16 with d, I multiples of 256 and MXFP4 with d, I multiples of 256: the
 *   tcgen05 decode GEMVs over the tile layouts of moe_pack_expert (gate/up
 *   and down in one cooperative launch or in two launches: see
 *   moe_expert_ffn_launches); other BF16/MXFP4 shapes and NVFP4 without
 *   MOE_FFN_ACT_NVFP4: CUDA cores; MOE_FFN_ACT_NVFP4: the tcgen05 FP4 GEMMs
 *   (d, I multiples of 256), on single CTAs (128 x 128 tiles) when
 *   T*k <= 128*E, else on CTA pairs (256 x 224 tiles); the environment
 *   variable MOE_PREFILL_TILES=cta|pair, read at every call, forces one.  The
 *   workspace size covers both.
 * Limits: T*k <= 1<<24. */
size_t moe_expert_ffn_workspace_bytes(moe_shape s, int T, int k, int flags);

/* Number of kernels one moe_expert_ffn call with these arguments launches on
 * its stream (for launch accounting; no device work).  The tcgen05 decode
 * GEMVs run gate/up and down in one cooperative launch or in two launches:
 * the default is chosen per weight format and T from measurements, and the
 * environment variable MOE_DECODE_SCHEDULE=one|two, read once per process,
 * fixes it.  Returns 0 for invalid arguments or T == 0. */
int moe_expert_ffn_launches(moe_shape s, int T, int k, int flags);
moe_status moe_expert_ffn(moe_shape s, const void* x, int T, int k,
                          const int32_t* offsets, const int32_t* perm,
                          const int32_t* slot_of_expert, const void* slot_pool, int n_slots,
                          const float* gate, float* y_perm, float* out, int flags,
                          void* workspace, size_t ws_bytes, int32_t* dev_status,
                          cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Step 4 -- gate-weighted combine with the exact merge of partial sums
 * computed elsewhere (explainx.ai hardware guide, "Decode": CPU and GPU
 * partial results are merged exactly; ainewsfeed.tech, third paragraph).
 *   out[t][c] = sum_{j=0..k-1, slot_of_expert[idx[t][j]] >= 0}
 *                   gate[t][j] * y_perm[inv_perm[t*k+j]][c]
 *               + host_partial[t][c]            (if host_partial != NULL)
 * summed in that order in fp32.  y_perm fp32 [T*k][d]; idx, gate [T][k];
 * inv_perm [T*k]; slot_of_expert [E] (NULL: every expert counts);
 * host_partial fp32 [T][d] or NULL; out fp32 [T][d] (may alias host_partial).
 * E bounds the expert ids looked up in slot_of_expert (an id outside [0, E)
 * or an inv_perm entry outside [0, T*k) drops that term).
 * All device pointers.  d must be a multiple of 4. */
moe_status moe_combine_merge(const float* y_perm, const int32_t* idx, const float* gate,
                             const int32_t* inv_perm, const int32_t* slot_of_expert,
                             const float* host_partial, int T, int k, int d, int E, float* out,
                             cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* A whole layer call in one entry point: moe_route_topk -> moe_permute ->
 * moe_expert_ffn -> moe_combine_merge, all enqueued on `stream`; with
 * MOE_FFN_ACT_NVFP4, out is first set to host_partial (or zero) and the FFN
 * adds the combine into it (y_perm is then unused and may be NULL).  Every
 * buffer is the one the individual call takes, with the same meaning,
 * layout, ownership and errors; the results are those of the four calls.
 * It exists for the host cost of a decode step: one call instead of four.
 * The arguments of all four steps are checked first: a call rejected by a
 * check (MOE_ERR_INVALID_ARG, MOE_ERR_CAPACITY) enqueues nothing.  After
 * that, a step that fails at launch (MOE_ERR_CUDA, or a device-dependent
 * limit) returns its status and nothing after it is enqueued. */
moe_status moe_layer_forward(moe_shape s, const float* logits, const void* x, int T, int k,
                             int32_t* idx, float* gate, int32_t* offsets, int32_t* perm,
                             int32_t* inv_perm, void* scratch, size_t scratch_bytes,
                             const int32_t* slot_of_expert, const void* slot_pool, int n_slots,
                             float* y_perm, int flags, void* workspace, size_t ws_bytes,
                             const float* host_partial, float* out, int32_t* dev_status,
                             cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* The q split of a decode step's cache misses (host only, no device call):
 * each missed expert is either filled into the GPU cache over PCIe or run on
 * the host, and the two partial sums merge exactly in moe_combine_merge
 * (explainx.ai hardware guide, "Decode: decide whether to move an expert or
 * compute where it lives"; futuresignalnews.com article, "Bandwidth-Adaptive
 * Execution (The q* Policy)").
 *   misses: host int32 [m], distinct expert ids in [0, E).
 *   tokens_per_expert: host int32 [E], the step's routed tokens per expert.
 *   q in [0, 1]: fill floor(q*m + 0.5) misses.  q < 0: the q* policy, which
 *     fills floor(m*bw_pcie/(bw_pcie + bw_host) + 0.5) misses so that the
 *     fills (over PCIe) and the host computation (through host memory), each
 *     moving one blob per expert, take the same time; bw_pcie and bw_host
 *     are the profiled bandwidths in any one unit.
 *   The misses with the most routed tokens are filled (ties: lower id).
 *   filled, host: host int32 [m] each, receive the two sets in ascending id;
 *   *n_filled + *n_host = m.
 * Errors: MOE_ERR_INVALID_ARG for an id out of range or listed twice, q > 1,
 * or q < 0 without positive finite bandwidths. */
moe_status moe_split_misses(const int32_t* misses, int m, const int32_t* tokens_per_expert, int E, double q,
                            double bw_pcie, double bw_host, int32_t* filled, int32_t* n_filled,
                            int32_t* host, int32_t* n_host);

/* ------------------------------------------------------------------------ */
/* Step 5 -- the GPU expert cache: LRU residency of expert blobs in device
 * slots, filled from a pinned host pool (freetoken.wiki mechanism table:
 * "Global LRU expert cache"; explainx.ai hardware guide: experts are copied
 * over PCIe into the GPU cache and kept; the host pool is the source of
 * truth; futuresignalnews.com mechanism 3: a cold cache serves the first
 * request).  The handle keeps the bookkeeping on the host:
 * expert_of_slot[S], last_used[S], slot_of_expert[E].
 *
 * moe_cache_create: slot_pool (device, n_slots blobs), host_pool (pinned host,
 *   E blobs in expert order), slot_of_expert_dev (device int32 [E]; this call
 *   does not write it -- the caller sets it to -1 before the first fill).  A
 *   handle made with slot_pool, host_pool and slot_of_expert_dev all NULL only
 *   plans (no CUDA call is ever made by it).
 * moe_cache_fill: makes the experts of `experts` (n ids, any order, duplicates
 *   ignored) resident for step `step`.  Distinct ids are handled in ascending
 *   order: a resident expert has its last_used set to `step` (a hit); a
 *   missing one takes the lowest free slot, else the slot with the smallest
 *   last_used (ties: lowest slot) whose expert is neither in `experts` nor in
 *   `protect` (the other experts of this step, e.g. the host-computed ones).
 *   For each fill it enqueues on `side`: a wait on `reads_done` (if non-NULL;
 *   recorded after the last kernel of the previous step that reads the pool
 *   OR the slot table -- moe_combine_merge reads the table, so on the unfused
 *   path it is the combine, not the FFN), the blob copy host -> slot with
 *   cudaMemcpyAsync, and one kernel that writes the slot-table changes
 *   (evicted expert -> -1, new expert -> slot); then records `fill_done` (if
 *   non-NULL).  fills (host int32 [n][3] or NULL) receives
 *   (expert, slot, evicted expert or -1) per fill; *n_fills their count.
 *   If there are not enough evictable slots, MOE_ERR_CAPACITY is returned
 *   and the cache state is unchanged.  If enqueueing fails (MOE_ERR_CUDA),
 *   the host bookkeeping is unchanged but a copy may already have reached a
 *   victim slot whose table entry was not rewritten: the handle then refuses
 *   every later fill with MOE_ERR_CUDA; recreate the cache (and its slot
 *   table) before the next FFN call. */
typedef struct moe_cache moe_cache;
moe_status moe_cache_create(moe_shape s, int n_slots, void* slot_pool, const void* host_pool,
                            int32_t* slot_of_expert_dev, moe_cache** out);
moe_status moe_cache_fill(moe_cache* c, const int32_t* experts, int n, int step,
                          const int32_t* protect, int n_protect,
                          cudaStream_t side, cudaEvent_t reads_done, cudaEvent_t fill_done,
                          int32_t* fills, int32_t* n_fills);
/* Copies of the host bookkeeping (any pointer may be NULL): slot_of_expert
 * [L*E] (entry l*E + e: the slot of expert e of layer l, or -1),
 * expert_of_slot [S] (the key l*E + e each slot holds, or -1), last_used [S].
 * With one layer these are slot_of_expert [E] and expert ids. */
moe_status moe_cache_query(const moe_cache* c, int32_t* slot_of_expert,
                           int32_t* expert_of_slot, int32_t* last_used);

/* One cache shared by n_layers MoE layers of the same shape: the global LRU
 * of the pages (freetoken.wiki "FreeToken 753b model", mechanism table,
 * "Global LRU expert cache": cache decisions are shared across MoE layers).
 * Residency is kept over keys (layer, expert) = l*E + e in one slot pool of
 * n_slots blobs; every layer has its own host pool (host_pools[l], E blobs in
 * expert order, pinned) and its own device slot table (slot_tables_dev[l],
 * int32 [E], set to -1 by the caller before the first fill), which that
 * layer's moe_expert_ffn and moe_combine_merge read.  All pointers NULL:
 * a plan-only handle (no CUDA call).  moe_cache_create is this call with one
 * layer.  Errors: MOE_ERR_INVALID_ARG. */
moe_status moe_cache_create_layers(moe_shape s, int n_layers, int n_slots, void* slot_pool,
                                   const void* const* host_pools, int32_t* const* slot_tables_dev,
                                   moe_cache** out);

/* moe_cache_fill for layer `layer` of a shared cache: the experts of this
 * layer's step become resident; a victim may belong to any layer (least
 * recent last_used over the whole pool, ties to the lowest slot, never a key
 * of this layer in `experts` or `protect`).  `step` is the caller's clock,
 * increasing across layers and steps (e.g. token step * n_layers + layer);
 * `reads_done` must follow the last kernel of any layer that read the pool or
 * a slot table.  fills: (expert of this layer, slot, evicted key or -1).
 * moe_cache_fill is this call with layer 0. */
moe_status moe_cache_fill_layer(moe_cache* c, int layer, const int32_t* experts, int n, int step,
                                const int32_t* protect, int n_protect, cudaStream_t side,
                                cudaEvent_t reads_done, cudaEvent_t fill_done, int32_t* fills,
                                int32_t* n_fills);

/* Elastic resize at a safe point (futuresignalnews.com, mechanism 3 "Elastic
 * Memory Management": the GPU expert cache is rebuilt under a new VRAM budget
 * at a safe scheduler point, without reloading the host pool): the cache gets
 * new_n_slots slots in new_slot_pool (device, 256-byte aligned,
 * new_n_slots blobs; it may be the current pool when new_n_slots does not
 * exceed the current count).  The min(residents, new_n_slots) residents with
 * the latest last_used (ties: lower slot first) are kept, keep their
 * last_used, and move to slots 0, 1, ... in their old slot order; the others
 * are evicted.  On `stream`, after a wait on `reads_done` (the last kernel
 * that read the pool or a slot table): device-to-device copies of the kept
 * blobs that move, then the slot-table updates of every layer.  No host-pool
 * copy is made.  The old pool may be freed once the stream has passed this
 * point.  kept: host int32 [min(S, new_n_slots)][2] or NULL, receives (key,
 * old slot) per new slot; *n_kept their count.  Plan-only handles: no CUDA
 * call, new_slot_pool ignored.  Errors: MOE_ERR_INVALID_ARG (growing in
 * place, bad pool), MOE_ERR_CUDA (the handle then refuses further calls). */
moe_status moe_cache_resize(moe_cache* c, int new_n_slots, void* new_slot_pool, cudaStream_t stream,
                            cudaEvent_t reads_done, int32_t* kept, int32_t* n_kept);
moe_status moe_cache_destroy(moe_cache* c);

/* ------------------------------------------------------------------------ */
/* The host share of a split step (host only, no device call): the SwiGLU FFN
 * of the experts the q split leaves on the host, run on the CPU cores against
 * their blobs in the host pool, concurrently with the fills of the GPU share
 * (explainx.ai hardware guide, "Decode: decide whether to move an expert or
 * compute where it lives"; freetoken.wiki "FreeToken 753b model", mechanism
 * table, "Bandwidth-adaptive execution").
 *   host_pool: E blobs in expert order (as for moe_cache_create), any host
 *     memory (pinned or not).
 *   experts: n_experts ids in [0, E) (duplicates ignored; an expert no token
 *     selected costs nothing).
 *   x: host bf16 [T][d]; idx: host int32 [T][k]; gate: host fp32 [T][k] (the
 *     step's routing, e.g. copied back from moe_route_topk).
 *   out: host fp32 [T][d], overwritten with sum over pairs (t, j) whose expert
 *     is listed of gate[t][j] * SwiGLU_{idx[t][j]}(x[t]) -- the host_partial
 *     of moe_combine_merge.  fp32 arithmetic.
 *   n_threads: worker threads (<= 0: one per hardware thread); the call
 *     blocks until the sum is done.  Calls from several threads run one at a
 *     time.
 * Errors: MOE_ERR_INVALID_ARG for a bad shape, id or null pointer. */
moe_status moe_host_expert_ffn(moe_shape s, const void* host_pool, const int32_t* experts, int n_experts,
                               const void* x, const int32_t* idx, const float* gate, int T, int k, float* out,
                               int n_threads);

/* The two bandwidths the q* split balances, measured on this machine
 * (freetoken.wiki "FreeToken 753b model", "Measure System Bandwidth"):
 *   *h2d_gbs: pinned host -> device copy rate of whole blobs: n_blobs
 *     cudaMemcpyAsync copies from host_pool into dev_buf (device, 256-byte
 *     aligned, >= one blob; blobs cycle through its dev_bytes) on `stream`,
 *     timed with CUDA events after one warm-up copy.  dev_buf NULL: skipped
 *     (0).  The call synchronises the stream.
 *   *host_gbs: the host expert kernel's weight bytes per second over the
 *     first n_blobs experts of host_pool (one token each, n_threads threads,
 *     after one warm-up expert).
 * GB = 1e9 bytes.  Errors: MOE_ERR_INVALID_ARG, MOE_ERR_CUDA. */
moe_status moe_profile_bandwidth(moe_shape s, const void* host_pool, int n_blobs, void* dev_buf,
                                 size_t dev_bytes, int n_threads, cudaStream_t stream, double* h2d_gbs,
                                 double* host_gbs);

/* ------------------------------------------------------------------------ */
/* Synchronises `stream`, reads the device status word written by kernels,
 * resets it to 0 and returns it as a moe_status (MOE_OK if it was 0). */
moe_status moe_check_status(int32_t* dev_status, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
