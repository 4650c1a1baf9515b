/*
 * bca.h -- block-causal attention with cross-step prefix K/V reuse, sm_100a.
 *
 * C ABI of libbca.so.  Plain pointers and sizes only; no framework types.
 *
 * The method (cited by page title and section):
 *  - "Qwen-Image-2.1 + vLLM-Omni day-0" (thakicloud.com), "What is Qwen-Image-2.1":
 *    the single-stream DiT uses block-causal attention.  The sequence is split
 *    into ordered blocks (text prompt, reference images 1..k, target latents);
 *    block b attends to blocks 0..b, with full attention inside a block.
 *  - same page, "Serving architecture: the cross-step prefix KV cache": since the
 *    prefix blocks never see the target, their K/V from the first denoising step
 *    are exact for every later step, so they are stored once and reused; the cache
 *    is rebuilt for every new request, so nothing leaks between requests.
 *  - "Qwen/Qwen-Image-2.1" (recipes.vllm.ai), "Prefix KV cache": reuse is exact;
 *    the cache may be stored in FP8 -- "fp8_v" quantises V only, "fp8" K too.
 *  - same page, "Online serving": requests at the same KV-cache phase are batched
 *    together (--step-execution --max-num-seqs 8).
 *
 * Conventions common to every call:
 *  - Element types: activations are bf16; softmax and accumulation are fp32.
 *  - Activation layout ("THD"): [tokens, heads, head_dim], head_dim contiguous,
 *    token rows heads*head_dim elements apart unless a stride is given.
 *  - Cache layout: per (request, layer) slot, K and V each [heads, cap_tokens,
 *    head_dim]; bf16, or OFP8 E4M3 codes (1 byte) with one fp32 scale per head.
 *  - All device memory is owned by the caller (including the optional
 *    bca_step_attend workspace).  The library allocates no device memory; it keeps
 *    only host-side state (a driver entry point, per-device attributes).
 *  - Calls enqueue work on `stream` and return at once.  Argument and state
 *    errors are reported synchronously, before anything is launched, and then
 *    nothing is written.  A failed launch returns BCA_ERR_CUDA.
 *  - Every device-side wait is bounded.  When a bound expires the kernel stores
 *    BCA_ERR_DEVICE_TIMEOUT into *dev_status (if dev_status is not NULL), drains
 *    and returns; the host reads *dev_status after synchronising.
 *  - Supported now: head_dim == 128, heads in [1, 256], device pointers 16-byte
 *    aligned, finite inputs.  (An e4m3 quantiser that meets a non-finite value
 *    writes BCA_ERR_NONFINITE into *dev_status; that head's codes and scale are
 *    then meaningless.)
 *  - A softmax scale is passed in (1/sqrt(head_dim) for the DiT).
 */
#ifndef BCA_H_
#define BCA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BCA_OK = 0,
  BCA_ERR_INVALID_ARG = 1,    /* a pointer, size, stride or offset is invalid      */
  BCA_ERR_UNSUPPORTED = 2,    /* valid but not implemented (e.g. head_dim != 128)  */
  BCA_ERR_CAPACITY = 3,       /* prefix longer than the slot's cap_tokens          */
  BCA_ERR_STATE = 4,          /* slot not filled for the current request (epoch 0) */
  BCA_ERR_CUDA = 5,           /* a CUDA runtime/driver call or a launch failed     */
  BCA_ERR_DEVICE_TIMEOUT = 6, /* a bounded device-side wait expired                */
  BCA_ERR_NONFINITE = 7       /* an e4m3 quantiser met Inf or NaN (via dev_status) */
} bca_status;

/* Cache element type, mirroring the recipe's prefix_kv_cache_dtype values. */
typedef enum {
  BCA_KV_BF16 = 0,   /* K and V bf16                      ("bf16", default)  */
  BCA_KV_FP8_V = 1,  /* K bf16, V e4m3 + per-head scale   ("fp8_v")          */
  BCA_KV_FP8_KV = 2  /* K and V e4m3 + per-head scales    ("fp8")            */
} bca_kv_dtype;

/* Maximum number of blocks in one prefill sequence and of requests in one
 * cached-step call. */
#define BCA_MAX_BLOCKS 64
#define BCA_MAX_BATCH 64

/* One (request, layer) prefix K/V cache slot.  The struct lives in host memory
 * and is owned by the caller; the buffers it points to are device memory owned
 * by the caller.
 *   k, v      : [num_heads, cap_tokens, head_dim]; bf16, or e4m3 bytes when the
 *               dtype quantises that tensor.
 *   k_scale,
 *   v_scale   : device fp32 [num_heads]; read/written only for e4m3 tensors
 *               (may be NULL otherwise).  Dequantised value = fp32(decode(code) * scale).
 *   n_tokens  : prefix rows currently stored (set by bca_kv_store / bca_prefill).
 *   epoch     : 0 = empty.  Storing stamps the caller's (non-zero) request epoch;
 *               a new request stores again with a new epoch (per-request rebuild).
 * Use bca_kv_slot_init to carve a slot from one caller allocation. */
typedef struct bca_kv_slot {
  void* k;
  void* v;
  float* k_scale;
  float* v_scale;
  int32_t cap_tokens;
  int32_t n_tokens;
  int32_t num_heads;
  int32_t head_dim;
  int32_t dtype; /* bca_kv_dtype */
  uint32_t epoch;
} bca_kv_slot;

/* Bytes of one device allocation that bca_kv_slot_init can carve into a slot
 * (K, V and both scale arrays, each 256-byte aligned).  Returns 0 for invalid
 * sizes. */
size_t bca_kv_slot_bytes(int32_t cap_tokens, int32_t num_heads, int32_t head_dim,
                         bca_kv_dtype dtype);

/* Fill *slot with pointers into `base` (device, 256-byte aligned, at least
 * bca_kv_slot_bytes(...) bytes) and mark it empty (n_tokens = 0, epoch = 0).
 * Host-only; touches no device memory.
 * Errors: BCA_ERR_INVALID_ARG (NULL, misaligned base or invalid sizes). */
bca_status bca_kv_slot_init(bca_kv_slot* slot, void* base, int32_t cap_tokens,
                            int32_t num_heads, int32_t head_dim, bca_kv_dtype dtype);

/* Store prefix K/V rows [0, n_prefix) of one request/layer into `slot`, in the
 * slot's dtype (the cache layout step of the method; "Prefix KV cache" on the
 * recipe page for the FP8 modes).
 *   k, v            : device bf16, token t / head h at element t*row_stride + h*head_dim.
 *   n_prefix        : 0 <= n_prefix <= slot->cap_tokens (else BCA_ERR_CAPACITY).
 *   row_stride_elems: elements between consecutive token rows (>= heads*head_dim,
 *                     multiple of 8).
 *   epoch           : non-zero request epoch stamped into the slot.
 * For an e4m3 tensor: amax = max |x| over the n_prefix rows of each head,
 * scale = fp32(amax)/448 (1 when amax == 0), code = e4m3 RNE-satfinite of the
 * correctly rounded fp32 quotient x/scale.  Rows [n_prefix, cap) are not written.
 * One kernel launch (HBM-bound; a head's encode pass re-reads its rows on the same
 * CTAs right after its absmax pass, interleaved with the next head's absmax pass,
 * so that rows still in L2 come from there).
 * Host side effects (at enqueue): slot->n_tokens = n_prefix, slot->epoch = epoch.
 * dev_status: nullable device int32, see the conventions above (a non-finite value
 * in an e4m3 tensor: BCA_ERR_NONFINITE). */
bca_status bca_kv_store(const void* k, const void* v, int32_t n_prefix,
                        int32_t row_stride_elems, bca_kv_slot* slot, uint32_t epoch,
                        int32_t* dev_status, void* stream);

/* One request's part of bca_kv_store_batch: the arguments of bca_kv_store. */
typedef struct bca_kv_store_item {
  const void* k;
  const void* v;
  int32_t n_prefix;
  int32_t row_stride_elems;
  bca_kv_slot* slot;
} bca_kv_store_item;

/* bca_kv_store for n_items (1..BCA_MAX_BATCH) requests of a same-phase batch in one
 * kernel launch ("Online serving" on the recipe page batches requests at the same
 * phase; their prefix stores are one call here).  Every item is checked as
 * bca_kv_store checks its arguments before anything is launched; the slots must be
 * distinct (else BCA_ERR_INVALID_ARG).  Each slot is stamped with `epoch`. */
bca_status bca_kv_store_batch(const bca_kv_store_item* items, int32_t n_items, uint32_t epoch,
                              int32_t* dev_status, void* stream);

/* Step 1 (prefill) of one request at one layer: block-causal attention over the
 * whole sequence ("What is Qwen-Image-2.1" and "Serving architecture: the
 * cross-step prefix KV cache" on the thakicloud page).
 *   q, k, v, o   : device bf16 [seq_len, heads, 128]; o is written.
 *   block_offsets: HOST int32[n_blocks + 1], 0 = off[0] < off[1] < ... <
 *                  off[n_blocks] = seq_len; row i attends to keys [0, end of its block).
 *   n_blocks     : 1..BCA_MAX_BLOCKS.  The last block is the target.
 *   slot         : nullable.  When given, rows [0, off[n_blocks-1]) (every block
 *                  but the target) of k and v are stored into it exactly as
 *                  bca_kv_store does, stamped with `epoch` (non-zero).
 * o and q/k/v must not overlap. */
bca_status bca_prefill(const void* q, const void* k, const void* v, void* o, int32_t seq_len,
                       const int32_t* block_offsets, int32_t n_blocks, int32_t heads,
                       int32_t head_dim, float scale, bca_kv_slot* slot, uint32_t epoch,
                       int32_t* dev_status, void* stream);

/* bca_prefill with the optional workspace of bca_step_attend (256-byte aligned,
 * caller-owned, NULL = none; see bca_step_workspace_bytes).  With it the kernel's
 * schedule balances uneven block-causal work: Q-tile pairs are taken heaviest first
 * (a pair's work is the number of keys its last block allows), the last partial
 * round of the heavy pairs is split along the keys into chunks merged by a second
 * kernel, and the light pairs (e.g. the text rows) fill in after them.  Results
 * equal bca_prefill's up to the order of the fp32 sums.  Calls sharing a
 * workspace must not overlap. */
bca_status bca_prefill_ws(const void* q, const void* k, const void* v, void* o, int32_t seq_len,
                          const int32_t* block_offsets, int32_t n_blocks, int32_t heads,
                          int32_t head_dim, float scale, bca_kv_slot* slot, uint32_t epoch,
                          void* workspace, size_t workspace_bytes, int32_t* dev_status,
                          void* stream);

/* Steps 2..N of a batch of requests at the same phase: every target row of
 * request r attends to [slot r's cached prefix rows ; request r's own target
 * rows], with no mask (the target is the last block, so it sees everything).
 *   q_t, k_t, v_t, o_t: device bf16, packed target rows of all requests,
 *                      [sum_r T_r, heads, 128]; request r owns rows
 *                      [cu_target[r], cu_target[r+1]).
 *   cu_target        : HOST int32[n_req + 1], cu_target[0] = 0, non-decreasing.
 *   slots            : HOST array of n_req slots; each filled (epoch != 0) with
 *                      num_heads == heads, head_dim == 128, and all the same dtype.
 *   n_req            : 1..BCA_MAX_BATCH.
 *   workspace,
 *   workspace_bytes  : optional device scratch (256-byte aligned, caller-owned;
 *                      NULL = none); see bca_step_workspace_bytes.  Its contents
 *                      are overwritten; calls sharing a workspace must not overlap.
 * For e4m3 tensors the per-head scales are folded in: K's into the softmax scale,
 * V's into the P of the cached keys.  A request with T_r == 0 is skipped.
 * Errors: BCA_ERR_STATE for an empty slot, BCA_ERR_UNSUPPORTED for mixed dtypes. */
bca_status bca_step_attend(const void* q_t, const void* k_t, const void* v_t, void* o_t,
                           const int32_t* cu_target, const bca_kv_slot* slots, int32_t n_req,
                           int32_t heads, int32_t head_dim, float scale, void* workspace,
                           size_t workspace_bytes, int32_t* dev_status, void* stream);

/* The cached step of bca_step_attend with e4m3 Q against e4m3 cached keys (all
 * slots BCA_KV_FP8_KV).  Each request's target Q rows are first quantised per head
 * with the cache's own rule (scale = absmax / 448, codes = e4m3_rn_satfinite(q /
 * scale); "Qwen/Qwen-Image-2.1" vLLM recipe, "Prefix KV cache", applied to Q), and
 * the scores against cached keys are those of the e4m3 Q with the e4m3 K, read by
 * the tensor cores as stored (tcgen05.mma kind::f8f6f4); the scale of Q joins K's
 * in the softmax scale.  Scores against the request's own keys use the bf16 Q, and
 * P and V are as in bca_step_attend (V codes expanded exactly to bf16, P bf16).
 *   q8_scratch,
 *   q8_scratch_bytes : device scratch, 256-byte aligned, caller-owned, at least
 *                      bca_step_q8_scratch_bytes(cu_target[n_req], n_req, heads).
 *                      After the call it holds the Q codes [heads, rows, 128] at
 *                      offset 0 and the fp32 scales [n_req][heads] (by request
 *                      index; not written for requests without rows) at offset
 *                      round_up(heads * rows * 128, 256); calls sharing it must
 *                      not overlap.  The quantisation is one launch of the store
 *                      kernel (as bca_kv_store); a non-finite Q value writes
 *                      BCA_ERR_NONFINITE into *dev_status.
 * Other arguments, results and errors: as bca_step_attend, plus
 * BCA_ERR_UNSUPPORTED if the slots are not BCA_KV_FP8_KV, BCA_ERR_INVALID_ARG for a
 * NULL or misaligned scratch and BCA_ERR_CAPACITY for a small one. */
bca_status bca_step_attend_q8(const void* q_t, const void* k_t, const void* v_t, void* o_t,
                              const int32_t* cu_target, const bca_kv_slot* slots, int32_t n_req,
                              int32_t heads, int32_t head_dim, float scale, void* workspace,
                              size_t workspace_bytes, void* q8_scratch, size_t q8_scratch_bytes,
                              int32_t* dev_status, void* stream);

/* The cached step of bca_step_attend over e4m3 slots ("fp8_v" or "fp8"), with each
 * e4m3 cache tensor a request reads first expanded, once per call, into a bf16 copy
 * in dq_scratch (one HBM-bound kernel: read 1 byte, write 2 per value; exact, the
 * per-head scale is not applied) -- instead of every CTA that visits a cached tile
 * converting it in shared memory (a tile is visited by each of the request's
 * Q-tile pairs, 16 for a 4096-row target).  The attention then reads bf16 tiles
 * and folds the scales in as bca_step_attend does, so the result equals
 * bca_step_attend's on the same slots bit for bit.  The slots keep their e4m3
 * bytes: the expansion is transient, one layer's worth at a time.
 *   dq_scratch,
 *   dq_scratch_bytes : device, 256-byte aligned, caller-owned, at least
 *                      bca_step_dq_scratch_bytes(slots, n_req); calls sharing it
 *                      must not overlap.
 * Other arguments, results and errors: as bca_step_attend, plus
 * BCA_ERR_UNSUPPORTED for bf16 slots (nothing to expand) or a slot whose
 * n_tokens x heads reaches 2^29, BCA_ERR_INVALID_ARG for a NULL or misaligned
 * scratch, BCA_ERR_CAPACITY for a small one. */
bca_status bca_step_attend_dq(const void* q_t, const void* k_t, const void* v_t, void* o_t,
                              const int32_t* cu_target, const bca_kv_slot* slots, int32_t n_req,
                              int32_t heads, int32_t head_dim, float scale, void* workspace,
                              size_t workspace_bytes, void* dq_scratch, size_t dq_scratch_bytes,
                              int32_t* dev_status, void* stream);

/* Bytes of bca_step_attend_dq's scratch for these slots (their n_tokens and dtypes):
 * per request, a bf16 [heads, n_tokens, 128] tensor for each of its e4m3 K and V,
 * each 256-byte aligned.  0 for invalid arguments. */
size_t bca_step_dq_scratch_bytes(const bca_kv_slot* slots, int32_t n_req);

/* Bytes of bca_step_attend_q8's scratch for `rows` packed target rows of n_req
 * requests (0 for arguments out of range). */
size_t bca_step_q8_scratch_bytes(int64_t rows, int32_t n_req, int32_t heads);

/* Bytes of the optional bca_step_attend (and bca_prefill_ws) workspace that lets
 * the kernel split the last partial round of work along the keys (so that every SM
 * finishes at the same time) for the current device: one chunk of 256 rows x
 * (128 + 2) fp32 per SM.  Without it (workspace NULL or too small for any chunk)
 * nothing is split. */
size_t bca_step_workspace_bytes(void);

/* bca_step_attend for callers that cannot allocate device memory -- for example a
 * serving process whose device memory is owned by another allocator, or one that
 * reserves its whole memory budget at start-up and allows no allocation after it.
 * The pages have no counterpart to this call; it is a library convenience.
 * Same arguments and results as bca_step_attend without the workspace: the split
 * chunks go to a scratch array that lives in the library itself (a file-scope
 * device array of 160 chunks = 21.3 MB, held on every GPU that loads the library
 * until the process exits).  The call allocates nothing.
 *  - The first call on a device looks up the array's device address (once per
 *    device, with that device current); make that first call before any stream
 *    capture.  The address is kept for the life of the process: do not go on
 *    using the library on a device after cudaDeviceReset (the kept address would
 *    no longer be valid).
 *  - Every call shares the one array and it keeps the previous call's contents.
 *    Nothing in it needs to start at zero: each call writes every chunk it reads.
 *    Calls that overlap on the GPU (other streams, other threads) race on it.
 *  - Errors: as bca_step_attend; BCA_ERR_CAPACITY if the device has more SMs than
 *    the array has chunks (a split schedule can use one chunk per SM). */
bca_status bca_step_attend_noalloc(const void* q_t, const void* k_t, const void* v_t, void* o_t,
                                   const int32_t* cu_target, const bca_kv_slot* slots,
                                   int32_t n_req, int32_t heads, int32_t head_dim, float scale,
                                   int32_t* dev_status, void* stream);

/* ---- Q/K normalisation + rotary embedding ------------------------------------
 * "SGLang-Diffusion stöder Qwen-Image-2.1 på dag noll" (orcarouter.ai), section
 * "Siffrorna, och vad de inte säger": a Q/K-norm change is among the steps around
 * the DiT's attention.  The pages give no formula; the plain reading (RMS norm over
 * the head dimension with one learned weight vector per tensor, then the rotary
 * position embedding of consecutive channel pairs) is computed here, in one pass
 * over each tensor, in place, for x in {q, k} ([rows, heads, 128] bf16):
 *   r          = 1 / sqrt(mean_c x[t,h,c]^2 + eps)
 *   y_c        = x[t,h,c] * r * gamma_x[c]
 *   x'[t,h,2i]   = y_{2i} cos_t[t,i] - y_{2i+1} sin_t[t,i]
 *   x'[t,h,2i+1] = y_{2i} sin_t[t,i] + y_{2i+1} cos_t[t,i]      (i < 64)
 * in fp32 with one round-to-nearest-even to bf16.  The caller's cos/sin tables
 * ([rows, 64] fp32, device) carry any position scheme (1-D or per-axis angles).
 * Run it on the target rows before bca_step_attend (and on the whole sequence
 * before bca_prefill).  q or k may be NULL (that tensor is left alone; not both).
 * gamma_q / gamma_k: [128] fp32 device (the one for a NULL tensor is unused).
 * Errors: BCA_ERR_UNSUPPORTED for head_dim != 128; BCA_ERR_INVALID_ARG for rows < 0,
 * heads outside [1, 256], eps not finite and > 0, a NULL or non-16-byte-aligned
 * pointer that is needed.  rows == 0 enqueues nothing (pointers unchecked). */
bca_status bca_qk_norm_rope(void* q, void* k, int64_t rows, int32_t heads, int32_t head_dim,
                            const float* gamma_q, const float* gamma_k, const float* cos_t,
                            const float* sin_t, float eps, void* stream);

/* The projection that produces the attention's inputs, with the Q/K norm and the
 * rotary embedding of bca_qk_norm_rope applied in its epilogue (same page and
 * section: the Q/K-norm change sits between the projection and the attention).
 * One linear projection (no bias) of the rows x by w, then, per head:
 *   y          = x w^T                  x [rows, d_model], w [3*heads*128, d_model]
 *                                       (torch Linear layout; output features: Q
 *                                       heads, then K heads, then V heads)
 *   q[t, h, :] = rope(rms_norm(y[t, 128h ..], gamma_q))        (as bca_qk_norm_rope)
 *   k[t, h, :] = rope(rms_norm(y[t, 128(heads+h) ..], gamma_k))
 *   v[t, h, :] = y[t, 128(2 heads+h) ..]
 * Tensor cores with fp32 accumulation; fp32 epilogue; one round-to-nearest-even to
 * bf16.  q, k, v: device bf16 [rows, heads, 128] each (the layout of
 * bca_step_attend / bca_prefill), written in full; no separate normalisation pass
 * reads them again.
 *   x, w          : device bf16, rows d_model elements apart.
 *   gamma_q/k     : [128] fp32 device.  cos_t, sin_t: [rows, 64] fp32 device.
 * Errors: BCA_ERR_UNSUPPORTED for head_dim != 128 or d_model not a positive multiple
 * of 64; BCA_ERR_INVALID_ARG for rows < 0, heads outside [1, 256], eps not finite
 * and > 0, or a NULL / non-16-byte-aligned pointer.  rows == 0 enqueues nothing.
 * dev_status: nullable, receives BCA_ERR_DEVICE_TIMEOUT if a bounded wait expires. */
bca_status bca_qkv_project(const void* x, const void* w, void* q, void* k, void* v, int32_t rows,
                           int32_t d_model, int32_t heads, int32_t head_dim,
                           const float* gamma_q, const float* gamma_k, const float* cos_t,
                           const float* sin_t, float eps, int32_t* dev_status, void* stream);

/* ---- Head-sharded (Ulysses) sequence parallelism -----------------------------
 * "Qwen/Qwen-Image-2.1" (recipes.vllm.ai), "Overview" and "Limitations": the
 * engine's sequence parallelism is Ulysses; "SGLang-Diffusion stöder Qwen-Image-2.1
 * på dag noll", "Hur en driftsättning faktiskt ser ut": Ulysses attention is a
 * verified multi-GPU mode.  N ranks each hold rows_local rows of all H heads; one
 * all-to-all (the caller's, e.g. NCCL) gives each rank all rows of H/N heads, the
 * attention calls run on that head shard (cache slots hold the rank's H/N heads),
 * and a second all-to-all returns O to the row shards.  These two copies lay the
 * buffers out around the exchange (Hn = heads / n_ranks, d = head_dim = 128, bf16):
 *   bca_ulysses_pack   : x[t, g*Hn + j, :] -> send[g, t, j, :]  (block g for rank g)
 *   bca_ulysses_unpack : recv[g, t, j, :] -> x[t, g*Hn + j, :]  (block g from rank g)
 * for t < rows_local.  A received Q/K/V buffer [N][rows_local][Hn][d] is already
 * the [N*rows_local, Hn, d] layout the attention calls take.  x and the buffers
 * must not overlap.  Errors: BCA_ERR_UNSUPPORTED for head_dim != 128;
 * BCA_ERR_INVALID_ARG for rows_local < 0, n_ranks < 1, heads not a positive
 * multiple of n_ranks (at most 256), NULL or non-16-byte-aligned pointers.
 * rows_local == 0 enqueues nothing. */
bca_status bca_ulysses_pack(const void* x, void* send, int64_t rows_local, int32_t heads,
                            int32_t head_dim, int32_t n_ranks, void* stream);
bca_status bca_ulysses_unpack(const void* recv, void* x, int64_t rows_local, int32_t heads,
                              int32_t head_dim, int32_t n_ranks, void* stream);

/* ---- Cached-step graphs ----------------------------------------------------
 * "Qwen-Image-2.1 + vLLM-Omni day-0", "vLLM-Omni's day-0 support" and "Serving
 * architecture: the cross-step prefix KV cache": besides the prefix reuse, the
 * step loop's kernel-launch cost is removed with CUDA graphs.  "Qwen/Qwen-Image-2.1"
 * (recipes.vllm.ai), "CUDA graphs": fixed-shape denoising steps are captured, one
 * entry per image layout (the pages' engine copies prefix K/V into static buffers
 * first and runs quantised caches eagerly; here neither is needed).
 *
 * A step graph is the cached-step attention of n_layers layers for one layout: a
 * fixed request set (cu_target), fixed activation buffers per layer and fixed
 * cache slots per (layer, request).  bca_step_graph_create checks every layer's
 * arguments exactly as bca_step_attend does and records, in layer order, the same
 * kernel launches bca_step_attend would enqueue (each layer after the one before,
 * since the layers share the workspace) into one CUDA graph; bca_step_graph_launch
 * replays them all with one call.  At replay the kernels read the activation
 * buffers and the slots' device memory in place: contents written into the same
 * buffers between replays are used -- nothing is copied into static buffers -- and
 * the outputs are bit-identical to the eager bca_step_attend calls on the same
 * contents.  Pointers, row counts, slot shapes and n_tokens are fixed when the
 * graph is created; another layout needs another graph.  bf16 and e4m3 caches are
 * captured alike; with q8_scratch the e4m3-Q step (its Q quantisation included),
 * with dq_scratch the expand-once step (its expansion kernel included) is recorded.  The graph object lives in host memory (the CUDA driver keeps
 * its own copy of the recorded launches); the library allocates no device memory. */
typedef struct bca_step_graph bca_step_graph; /* opaque */

typedef struct {
  int32_t n_layers;         /* >= 1 */
  const void* const* q_t;   /* [n_layers] device pointers (host array), each as in */
  const void* const* k_t;   /*   bca_step_attend: packed target rows [sum T_r, H, d] */
  const void* const* v_t;
  void* const* o_t;
  const bca_kv_slot* slots; /* [n_layers * n_req] host array, layer-major (read at create) */
  const int32_t* cu_target; /* [n_req + 1] host array, shared by the layers */
  int32_t n_req, heads, head_dim;
  float scale;
  void* workspace;          /* as bca_step_attend (nullable), shared by the layers */
  size_t workspace_bytes;
  int32_t* dev_status;      /* nullable */
  void* q8_scratch;         /* nullable; non-NULL: the layers' bca_step_attend_q8 calls
                               are recorded instead (e4m3 slots), sharing this scratch */
  size_t q8_scratch_bytes;
  void* dq_scratch;         /* nullable; non-NULL: the layers' bca_step_attend_dq calls
                               are recorded instead (e4m3 slots), sharing this scratch
                               (at least the largest layer's bca_step_dq_scratch_bytes);
                               not together with q8_scratch */
  size_t dq_scratch_bytes;
} bca_step_graph_desc;

/* Builds the graph on the current device.  Errors: BCA_ERR_INVALID_ARG for a NULL
 * desc/graph, a bad array, or both q8_scratch and dq_scratch; otherwise the first failing layer's bca_step_attend
 * status (nothing is created then); BCA_ERR_CUDA if capture or instantiation fails. */
bca_status bca_step_graph_create(const bca_step_graph_desc* desc, bca_step_graph** graph);

/* Enqueues one replay (all layers) on `stream` (of the graph's device). */
bca_status bca_step_graph_launch(const bca_step_graph* graph, void* stream);

/* Kernel launches one replay performs (attention + chunk-merge kernels, and the Q
 * quantisation kernel of an e4m3-Q graph or the expansion kernel of a dq graph). */
int32_t bca_step_graph_kernel_nodes(const bca_step_graph* graph);

/* Releases the graph (NULL is ignored).  No replay may be pending on the GPU. */
void bca_step_graph_destroy(bca_step_graph* graph);

/* Human-readable name of a status code (static storage). */
const char* bca_status_string(bca_status status);

/* Upper bound, in nanoseconds, of every device-side wait (default 2e9 = 2 s).
 * Values < 1e6 are raised to 1e6.  Applies to launches enqueued afterwards. */
void bca_set_wait_timeout_ns(uint64_t timeout_ns);

/* Self-check of the bounded-wait path: launches one CTA that waits on a barrier
 * nothing will ever complete, for at most timeout_ns, then stores
 * BCA_ERR_DEVICE_TIMEOUT into *dev_status and returns.  Lets a host test see a
 * device timeout without hanging or faulting the GPU. */
bca_status bca_selftest_wait_timeout(int32_t* dev_status, uint64_t timeout_ns, void* stream);

/* Self-check of the e4m3 encoder's division: for every positive finite bf16 amax
 * and every bf16 x with |x| <= amax, counts (atomically adds to *mismatches, a
 * device uint64 the caller zeroes) the pairs whose e4m3 code from the encoder's
 * reciprocal-and-correction quotient differs from the code of the correctly rounded
 * x / s (s = amax / 448).  Diagnostic only; 0 is expected. */
bca_status bca_selftest_e4m3_division(unsigned long long* mismatches, void* stream);

/* Pipeline tracing (diagnostic; builds compiled with BCA_TRACE only, otherwise
 * BCA_ERR_UNSUPPORTED): attention launches enqueued afterwards record clock64()
 * stamps of CTA `cta`'s producer/MMA/softmax events into dev_buffer
 * ([192 tiles][32 events] uint64, device, caller-owned; cta < 0: none), followed by
 * each CTA's total cycles (one uint64 per CTA, up to 1024 CTAs); NULL turns it off. */
bca_status bca_debug_set_trace(unsigned long long* dev_buffer, int32_t cta);

/* Library version string. */
const char* bca_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BCA_H_ */
