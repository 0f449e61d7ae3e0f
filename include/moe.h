/*
 * moe.h -- C ABI of the routed Mixture-of-Experts FFN layer with low-bit
 * block-quantised experts, for NVIDIA B200 (sm_100a).
 *
 * The layer is the one described by the "Avalon" README and its GGUF model
 * card: 512 routed experts, 10 active per token, 48 layers; expert up/gate
 * tensors in a 3.25-bpw super-block format (one scale per 256 weights, 4-bit
 * sub-scales per 32 weights), down in a 4-bit non-uniform-codebook format,
 * and each expert stored packed as up | gate | down (model card, "Files").
 * The device-side expert-slot lookup follows the "Betelgeuse" post (VRAM
 * slot pool with per-layer capacities, hits resolved on the device, only
 * misses reported); the missed blobs can be pulled from pinned host memory
 * on the stream itself (moe_stage_misses), with no host round trip.
 *
 * Conventions (every entry point):
 *   - Pointers are DEVICE pointers unless the comment says "host".
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy stream).
 *   - The library never allocates memory, never synchronises the stream
 *     (except moe_get_device_status, and moe_stage_table, a once-per-pool
 *     setup call) and never prints.  Memory is owned by
 *     the caller; workspaces are sized with the *_workspace_bytes queries.
 *   - Argument errors are returned synchronously (MOE_ERR_INVALID /
 *     MOE_ERR_SHAPE / MOE_ERR_WORKSPACE) before anything is launched.  A
 *     failed launch returns MOE_ERR_CUDA.  Bad data seen on the device (an
 *     expert id out of range, a missing slot) never traps: the kernel sets
 *     the workspace's device error word and skips the access; read it with
 *     moe_get_device_status.
 *   - Calls on different streams must use different workspaces.
 *   - bf16 and fp16 values are passed as uint16_t bit patterns.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID = 1,     /* null pointer, unknown enum, bad argument   */
  MOE_ERR_SHAPE = 2,       /* a size the format or the kernels reject   */
  MOE_ERR_UNSUPPORTED = 3, /* valid but not implemented                 */
  MOE_ERR_CUDA = 4,        /* a CUDA launch or runtime call failed      */
  MOE_ERR_DEVICE = 5,      /* the device error word was set             */
  MOE_ERR_CAPACITY = 6,    /* slot pool: more misses than free slots    */
  MOE_ERR_TIMEOUT = 7,     /* a bounded device wait gave up             */
  MOE_ERR_WORKSPACE = 8    /* workspace missing or too small            */
} moe_status;

/* Expert weight formats (model card, "Files"; value semantics below).
 *  MOE_Q4_B32 : 32 weights per block, fp16 scale d, 4-bit codes q,
 *               w = d * (q - 8).
 *  MOE_SB3_256: 256-weight super-block, fp16 scale d, eight 4-bit
 *               sub-scales s_j (one per 32 weights), 3-bit codes q,
 *               w = d * (2*s_j + 1) * (2*q - 7) / 8.   (3.1875 bpw)
 *  MOE_NL4_B32: 32 weights per block, fp16 scale d, 4-bit codes q into the
 *               int8 codebook {-127,-104,-83,-65,-49,-35,-22,-10,1,13,25,
 *               38,53,69,89,113}, w = d * cb[q].             (4.5 bpw)
 *  MOE_NL3_256: 256-weight super-block, fp16 scale d, eight 4-bit
 *               sub-scales s_j and eight codebook-shift bits e_j (one per
 *               32 weights), 3-bit codes q into the non-uniform codebook
 *               cb3 = {-15,-10,-6,-2,1,5,9,14}:
 *               w = d * (2*s_j + 1) * (cb3[q] + e_j) / 16.   (3.22 bpw)
 *               This library's own stand-in for the 3-bit non-linear
 *               "K" type the model card lists for up/gate (IQ3_K,
 *               3.44 bpw): the card gives only its name and bit rate, so
 *               neither this layout nor this codebook follows that type.
 *  MOE_SB2_256: 256-weight super-block, fp16 scale d, eight 4-bit
 *               sub-scales s_j (one per 32 weights), 2-bit codes q,
 *               w = d * (2*s_j + 1) * (2*q - 3) / 4.          (2.19 bpw)
 *               This library's own stand-in for the 2-bit type the model
 *               card lists for up/gate (IQ2_S): the card gives only its
 *               name, so the layout and values are this library's.
 * Natural byte layout of a [rows x cols] tensor (rows of blocks along the
 * columns, planar): codes plane, then (SB3, NL3, SB2) sub-scale plane,
 * then the fp16 d plane.  SB3 codes: 96 bytes per super-block, a
 * little-endian bit stream with code i at bit 3i; sub-scale j at bit 4j of
 * a little-endian 32-bit word.  NL3: the SB3 planes (codes, sub-scale
 * words, d), then a plane of one byte per super-block whose bit j is e_j.
 * SB2: codes 64 bytes per super-block, code i at bit 2i, then sub-scale
 * words and d as in SB3.  Q4/NL4 codes: weight i of a row in byte i/2, low
 * nibble for even i.  The *packed* layout (same byte count) is the GPU
 * tile layout that moe_pack_tensor produces and every compute entry point
 * reads. */
typedef enum {
  MOE_Q4_B32 = 1,
  MOE_SB3_256 = 2,
  MOE_NL4_B32 = 3,
  MOE_NL3_256 = 4,
  MOE_SB2_256 = 5
} moe_qfmt;

/* One MoE layer's experts as the FFN sees them.
 * Expert e's blob starts at pool + blob_index[e] * blob_stride and holds the
 * packed tensors up [F x H] | gate [F x H] | down [H x F] back to back (the
 * model card's packed expert layout, "Files": each expert's three tensors
 * adjacent, so that filling a cache slot takes a single copy).  blob_stride must be a multiple
 * of 16 bytes and at least moe_blob_bytes(...). */
typedef struct {
  int H;            /* hidden size                      */
  int F;            /* expert FFN width                 */
  int E;            /* number of routed experts         */
  int fmt_up_gate;  /* moe_qfmt of up and gate          */
  int fmt_down;     /* moe_qfmt of down                 */
  const uint8_t* pool;   /* device, packed expert blobs */
  int64_t blob_stride;   /* bytes between blobs         */
} moe_layer_desc;

/* ---------------------------------------------------------- formats ---- */

/* Bytes of one [rows x cols] tensor in format fmt (natural and packed
 * layouts have the same size); 0 if fmt or the shape is invalid. */
size_t moe_tensor_bytes(int fmt, int rows, int cols);

/* Bytes of one expert blob (up | gate | down, unpadded). */
size_t moe_blob_bytes(int fmt_up_gate, int fmt_down, int H, int F);

/* Natural layout -> packed GPU tile layout (model card, "Files": the expert
 * quant types; the packed layout is this library's own).  `natural` and
 * `packed` are distinct device buffers of moe_tensor_bytes() bytes.
 * Needs rows % 16 == 0, cols % 256 == 0 (SB3, NL3, SB2) or cols % 64 == 0
 * (Q4/NL4). */
moe_status moe_pack_tensor(int fmt, const uint8_t* natural, int rows,
                           int cols, uint8_t* packed, void* stream);

/* Packed tensor -> fp32 [rows x cols] row-major.  The closed forms above
 * are exact in fp32, so the result is bit-exact. */
moe_status moe_dequant(int fmt, const uint8_t* packed, int rows, int cols,
                       float* out, void* stream);

/* Hot-path decoders of moe_dequant_path. */
typedef enum { MOE_DQ_DECODE = 1, MOE_DQ_PREFILL = 2 } moe_dq_path;

/* Packed tensor -> its weights as one of the layer's hot-path decoders
 * produces them (the closed forms of moe_qfmt are the reference; model
 * card, "Files").  A check and debugging export: the FFN kernels never
 * materialise these tensors.
 *   path MOE_DQ_DECODE:  out fp32 [rows x cols] row-major, computed by the
 *        int8 tensor-core tile decoders of the decode kernels (T <= 8),
 *        fed one-hot activations.  Every weight of these formats is exact
 *        in fp32, so the result equals the closed form bit for bit.
 *   path MOE_DQ_PREFILL: out fp16 bits [rows x cols] row-major: the
 *        operand tiles the prefill grouped GEMM's dequantising warps write
 *        to shared memory, un-swizzled.  Each value is the round-to-nearest-
 *        even fp16 of the closed form.  Needs rows % 128 == 0.
 * packed and out 16-byte aligned (else MOE_ERR_INVALID); shape rules of
 * moe_pack_tensor (else MOE_ERR_SHAPE). */
moe_status moe_dequant_path(int fmt, int path, const uint8_t* packed,
                            int rows, int cols, void* out, void* stream);

/* ---------------------------------------------------------- routing ---- */

/* Router and top-k ("Avalon": 512 experts, 10 active; softmax over all E,
 * top-k by probability with ties to the lower index, renormalised).
 *   x        bf16 [T x H] row-major        w_router bf16 [E x H] row-major
 *            (both 16-byte aligned, else MOE_ERR_INVALID)
 *   bias     fp32 [E] added to the logits, or NULL
 *   topk_idx int32 [T x k]: experts by descending weight
 *   topk_w   fp32 [T x k]: renormalised softmax weights (sum to 1)
 *   logits_out fp32 [T x E]: receives the fp32 logits the selection used;
 *            required (NULL returns MOE_ERR_WORKSPACE)
 * Logits: exact bf16 products, fp32 accumulation, one fp32 bias add; for
 * T > 8 and H % 64 == 0 on the 5th-generation tensor cores.
 * Needs 1 <= k <= min(E, 32), E <= 4096, H % 8 == 0. */
moe_status moe_route_topk(const uint16_t* x, int T, int H,
                          const uint16_t* w_router, int E, const float* bias,
                          int k, int32_t* topk_idx, float* topk_w,
                          float* logits_out, void* stream);

/* Workspace of moe_group_tokens. */
size_t moe_group_workspace_bytes(int T, int k, int E);

/* Token-to-expert grouping: the pairs p = t*k + j sorted by expert, stable
 * in p ("MoE GEMM" grouping of the "llama-halo-hybrid" post).
 *   expert_offsets int32 [E+1]: pairs of expert e are
 *                  pair_ids[expert_offsets[e] .. expert_offsets[e+1]-1]
 *   pair_ids       int32 [T*k]
 *   active         int32 [E]: experts with at least one pair, ascending;
 *                  the first *n_active entries are valid
 *   n_active       int32 [1] (device)
 * An expert id outside [0, E) sets the device error word and is dropped. */
moe_status moe_group_tokens(const int32_t* topk_idx, int T, int k, int E,
                            int32_t* expert_offsets, int32_t* pair_ids,
                            int32_t* active, int32_t* n_active, void* ws,
                            size_t ws_bytes, void* stream);

/* A grouping restricted to a list of experts, for computing a layer's
 * experts in waves (prefill through the expert-slot pool: the experts whose
 * blobs are on the device first, the others as their blobs arrive; the
 * prefill prefetch of the "Avalon" README's feature list).  From a grouping made by
 * moe_group_tokens (expert_offsets [E+1], pair_ids [T*k]) and a device list
 * experts[0..n-1] of distinct expert ids, builds the grouping of just those
 * experts' pairs, in the same order: sub_offsets int32 [E+1] (empty ranges
 * for unlisted experts), sub_pairs int32 [T*k] (the first sub_offsets[E]
 * entries are valid), sub_active int32 [E] and sub_n_active int32 [1] as in
 * moe_group_tokens.  An id outside [0, E) sets MOE_ERR_DEVICE in err
 * (device word) and is ignored.  E <= 4096, 0 <= n <= E. */
moe_status moe_group_subset(const int32_t* expert_offsets,
                            const int32_t* pair_ids, int E,
                            const int32_t* experts, int n,
                            int32_t* sub_offsets, int32_t* sub_pairs,
                            int32_t* sub_active, int32_t* sub_n_active,
                            int32_t* err, void* stream);

/* Allocation-free variant of moe_group_tokens (no counterpart in the
 * source pages: it exists for callers of this library that cannot
 * allocate device memory where they call it -- a plugin or custom operator
 * handed only input/output pointers, code where an allocation would
 * synchronise the device or break a capture the caller does not own,
 * real-time loops that forbid allocation).  Same arguments and results as
 * moe_group_tokens, but the scratch lives in a fixed array in the
 * library's own device memory (512.25 KiB, held by every device that loads
 * the library until the process exits) instead of a workspace.
 *   Limits: T*k <= 262144 and E <= 1024, else MOE_ERR_SHAPE.
 *   err  int32 [1] device error word, or NULL to use the array's own word
 *        (cleared at each call; then bad expert ids are not reported).
 *   The first call in each CUDA context (per device) looks up the array's
 *   device address (a runtime symbol lookup); make that first call before
 *   any stream capture.  Do not use the library across a device reset
 *   (cudaDeviceReset): the array lives in the context that loaded it.  Calls that overlap on the GPU (other streams, other host
 *   threads) share the array and race: serialise them.  Nothing is
 *   allocated or freed by this call. */
moe_status moe_group_tokens_static(const int32_t* topk_idx, int T, int k,
                                   int E, int32_t* expert_offsets,
                                   int32_t* pair_ids, int32_t* active,
                                   int32_t* n_active, int32_t* err,
                                   void* stream);

/* ------------------------------------------------------ slot cache ---- */

/* Resolve one layer's chosen experts against its slot partition
 * ("Betelgeuse": VRAM slot pool, per-layer capacities, an in-stream kernel
 * resolves hits and reports only the misses).  One call per (step, layer).
 *   slot_table  int32 [E]      local slot of expert e or -1   (updated)
 *   slot_owner  int32 [n_slots] expert in each slot or -1     (updated)
 *   last_use    uint32 [n_slots] stamp of each slot's last use (updated)
 *   stamp       the stamp written to every slot this call uses or fills
 *   blob_index  int32 [E]: for each chosen expert, slot_base + its slot
 *   miss_expert int32 [T*k]: missed experts, ascending id
 *   miss_slot   int32 [T*k]: the slot each miss was given (its victim)
 *   n_miss      int32 [1] (device)
 *   err         int32 [1] device error word (MOE_ERR_CAPACITY when the
 *               misses outnumber the slots not used by this call; then
 *               nothing is updated)
 * Victim rule: the slot with the smallest last_use among the slots this
 * call has not used or filled, ties to the lowest slot; the evicted
 * expert's table entry becomes -1.  After the call each missed expert's
 * blob goes into pool + blob_index[e] * stride (one copy per expert) before
 * the FFN runs on the same stream: copied by the caller, or pulled from
 * pinned host memory on the stream by moe_stage_misses.  Needs T*k <= 1024,
 * E <= 8192, n_slots <= 8192. */
moe_status moe_slot_resolve(const int32_t* topk_idx, int T, int k, int E,
                            int32_t* slot_table, int32_t* slot_owner,
                            uint32_t* last_use, int n_slots, int slot_base,
                            uint32_t stamp, int32_t* blob_index,
                            int32_t* miss_expert, int32_t* miss_slot,
                            int32_t* n_miss, int32_t* err, void* stream);

/* moe_slot_resolve with the stamp kept on the device, so that a decode
 * step (route -> resolve -> stage -> FFN for every layer) can be captured
 * once as a CUDA graph and replayed step after step with no host argument
 * changing ("Betelgeuse": the whole decode pass as one graph replay).
 *   stamp  uint32 [1] device counter of this partition, 0 before its first
 *          call: the call stamps with *stamp + 1 and stores that value back
 *          (unless it reports an error, when nothing is updated).
 * Resolving each layer once per step with its own counter gives exactly
 * the stamps (and so the victims) of moe_slot_resolve called with
 * stamp = step number, steps counted from 1.  Other arguments, limits and
 * errors as moe_slot_resolve; stamp NULL is MOE_ERR_INVALID. */
moe_status moe_slot_resolve_dev(const int32_t* topk_idx, int T, int k, int E,
                                int32_t* slot_table, int32_t* slot_owner,
                                uint32_t* last_use, int n_slots,
                                int slot_base, uint32_t* stamp,
                                int32_t* blob_index, int32_t* miss_expert,
                                int32_t* miss_slot, int32_t* n_miss,
                                int32_t* err, void* stream);

/* ---------------------------------------- in-stream expert staging ---- */

/* Miss handling without a host round trip per layer ("Betelgeuse": a VRAM
 * slot pool whose misses a pager fills while the decode stream waits).
 * The host copies of the blobs sit in pinned host memory, so the GPU pulls
 * the misses itself; per layer, on one stream (capturable in a graph):
 *   moe_slot_resolve -> moe_stage_misses -> the expert FFN
 * No host thread, flag or second stream is involved. */

/* Build the device table of host blob addresses once: host_blob[i] (host
 * pointers, i = layer * E + e, NULL = not stored) must be 16-byte aligned
 * mapped pinned host memory (cudaHostAlloc, torch pin_memory), else
 * MOE_ERR_INVALID; table is uint64 [n] device memory.  Synchronises
 * `stream`. */
moe_status moe_stage_table(const void* const* host_blob, int n,
                           uint64_t* table, void* stream);

/* Copy this layer's missed blobs (moe_slot_resolve's n_miss / miss_expert /
 * miss_slot, device, P = T*k entries) from their pinned host copies
 * table[layer * E + e] into pool slot slot_base + miss_slot[i], reading
 * host memory over PCIe from one kernel on the stream.  The layer's
 * partition is slots slot_base .. slot_base + n_slots - 1 of a pool of
 * pool_slots slots of blob_stride bytes; blob_bytes are copied per blob.
 * A missing host copy, or a miss_slot outside [0, n_slots), sets
 * MOE_ERR_CAPACITY in err (device word) and skips that blob (so a bad slot
 * never overwrites another layer's expert); a miss count outside [0, P]
 * sets MOE_ERR_DEVICE.  blob_bytes, blob_stride and pool must be multiples
 * of 16 (bytes), 0 <= layer < L and slot_base + n_slots <= pool_slots. */
moe_status moe_stage_misses(const int32_t* n_miss, const int32_t* miss_expert,
                            const int32_t* miss_slot, int P, int layer, int L,
                            int E, const uint64_t* table, uint8_t* pool,
                            int slot_base, int n_slots, int64_t pool_slots,
                            int64_t blob_stride, int64_t blob_bytes,
                            int32_t* err, void* stream);

/* ------------------------------------------------------- expert FFN ---- */

/* Workspace of the FFN entry points (decode and prefill paths). */
size_t moe_ffn_workspace_bytes(int T, int k, int H, int F);

/* Zero a workspace before its first use (the kernels leave their counters
 * at zero when they finish, so this is needed once). */
moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Expert FFN on the grouped pairs: for every pair p of expert e,
 *   h = silu(Wg_e x_t) * (Wu_e x_t),  y_pairs[p] = Wd_e h
 * with the weights dequantised inside the kernel.
 *   x          bf16 [T x H], 16-byte aligned (else MOE_ERR_INVALID);
 *              y_pairs fp32 [T*k x H] (row p = pair p)
 *   expert_offsets/pair_ids/active/n_active: moe_group_tokens' outputs
 *   blob_index int32 [E] or NULL (NULL: expert e's blob is blob e); a
 *              negative entry of a chosen expert sets MOE_ERR_DEVICE
 * Needs H, F multiples of 256 (SB3, NL3, SB2) or 64 (Q4/NL4) and of 16.
 * T <= 8: int8 tensor-core decode kernels.  The weights enter exactly
 *   (int8 codes, integer sub-scale folds, fp32 scales); the activations
 *   are rounded to 15-bit fixed point with one power-of-two scale per
 *   token and 256-column block (split into two int8 halves), h with one
 *   per pair; the integer block sums are exact, the scales apply in fp32.
 *   A bf16 activation keeps every bit when it is at least 2^-6 times the
 *   largest magnitude of its 256-column block.
 * T > 8 with H, F multiples of 128 (the prefill path): grouped GEMMs on the
 *   5th-generation tensor cores in fp16 with fp32 accumulation.  On this
 *   path the grouping may list a subset of the T*k pairs (moe_group_subset):
 *   only the listed pairs' rows of y_pairs are written, and each is
 *   bit-identical to the row the full grouping gives.  Each
 *   weight enters as the round-to-nearest fp16 of its exact value, each
 *   activation row as fp16 after a per-row power-of-two scale that keeps
 *   it below 2^15, and h = silu(g) u is kept as fp16 (silu formed with the
 *   hardware tanh); an |h| beyond the fp16 range sets MOE_ERR_DEVICE.
 * Other shapes: a general SIMT path. */
moe_status moe_expert_ffn_q(const moe_layer_desc* desc, const uint16_t* x,
                            int T, int k, const int32_t* expert_offsets,
                            const int32_t* pair_ids, const int32_t* active,
                            const int32_t* n_active,
                            const int32_t* blob_index, float* y_pairs,
                            void* ws, size_t ws_bytes, void* stream);

/* The two halves of moe_expert_ffn_q, callable on their own (same
 * arguments and workspace; call up, then down, on the same stream).
 *   moe_expert_up_q:   h = silu(Wg x) * (Wu x) for every pair, kept in the
 *                      workspace (decode path: as int8 operands of the down
 *                      projection with one scale per pair and 32 values).
 *   moe_expert_down_q: y_pairs[p] = Wd h_p; y_pairs may be NULL when out is
 *                      given; with out != NULL the weighted combine of
 *                      moe_combine follows (topk_w, residual, out_bf16 as
 *                      there). */
moe_status moe_expert_up_q(const moe_layer_desc* desc, const uint16_t* x,
                           int T, int k, const int32_t* expert_offsets,
                           const int32_t* pair_ids, const int32_t* active,
                           const int32_t* n_active, const int32_t* blob_index,
                           void* ws, size_t ws_bytes, void* stream);
moe_status moe_expert_down_q(const moe_layer_desc* desc, int T, int k,
                             const int32_t* expert_offsets,
                             const int32_t* pair_ids, const int32_t* active,
                             const int32_t* n_active,
                             const int32_t* blob_index, float* y_pairs,
                             const float* topk_w, const float* residual,
                             float* out, uint16_t* out_bf16, void* ws,
                             size_t ws_bytes, void* stream);

/* The prefill path's up/gate GEMM launch alone (T > 8, H and F multiples
 * of 128; else MOE_ERR_UNSUPPORTED): it recomputes h from the grouped fp16
 * activations, row scales and unit plan that a moe_expert_up_q call with
 * the same arguments and workspace staged, reading nothing else of x.  A
 * measurement hook: it times the tensor-core kernel without the activation
 * pass in front of it.  Same result as that moe_expert_up_q call. */
moe_status moe_expert_up_gemm_q(const moe_layer_desc* desc, int T, int k,
                                const int32_t* expert_offsets,
                                const int32_t* pair_ids,
                                const int32_t* active,
                                const int32_t* n_active,
                                const int32_t* blob_index, void* ws,
                                size_t ws_bytes, void* stream);

/* Weighted combine: out[t] = sum_j topk_w[t,j] * y_pairs[t*k+j]
 * (+ residual[t]), summed in j order.  out fp32 [T x H]; out_bf16 bf16
 * [T x H] or NULL; residual fp32 [T x H] or NULL (may alias out). */
moe_status moe_combine(const float* y_pairs, const float* topk_w, int T,
                       int k, int H, const float* residual, float* out,
                       uint16_t* out_bf16, void* stream);

/* Fused expert FFN + combine (the decode fast path): the same result as
 * moe_expert_ffn_q followed by moe_combine, without the caller's y_pairs. */
moe_status moe_expert_ffn_combine_q(const moe_layer_desc* desc,
                                    const uint16_t* x, int T, int k,
                                    const int32_t* expert_offsets,
                                    const int32_t* pair_ids,
                                    const int32_t* active,
                                    const int32_t* n_active,
                                    const int32_t* blob_index,
                                    const float* topk_w,
                                    const float* residual, float* out,
                                    uint16_t* out_bf16, void* ws,
                                    size_t ws_bytes, void* stream);

/* x_out = bf16(r / sqrt(mean(r^2) + 1e-6)) per row: the input of the next
 * layer of a pre-norm residual stack.  r fp32 [T x H]. */
moe_status moe_rmsnorm_bf16(const float* r, int T, int H, uint16_t* x_out,
                            void* stream);

/* Workspace of moe_layer_forward. */
size_t moe_layer_workspace_bytes(int T, int k, int E, int H, int F);

/* One whole MoE layer on one stream: routing, grouping, expert FFN and
 * the weighted combine.  T <= 8 (with T*k at most the SM count and
 * E <= 1024): one cooperative kernel does all of it; it is launched as a
 * programmatic dependent of the work before it on the stream and touches
 * no global memory until that work has completed -- except w_router, whose
 * rows it starts loading at once: w_router must not be written by the work
 * just before the call on the stream (the same holds for the residual
 * variants below).  Otherwise: moe_route_topk, moe_group_tokens, then the expert FFN
 * (the tensor-core prefill path when T > 8 and the shapes allow it) and
 * the combine.  The grouping lives in the workspace.  w_router bf16
 * [E x H]; bias fp32 [E] or NULL; blob_index as in moe_expert_ffn_q;
 * residual/out/out_bf16 as in moe_combine; topk_idx int32 [T x k], topk_w
 * fp32 [T x k] and logits_out fp32 [T x E] (or NULL) receive the routing. */
moe_status moe_layer_forward(const moe_layer_desc* desc, const uint16_t* x,
                             int T, int k, const uint16_t* w_router,
                             const float* bias, const int32_t* blob_index,
                             const float* residual, float* out,
                             uint16_t* out_bf16, int32_t* topk_idx,
                             float* topk_w, float* logits_out, void* ws,
                             size_t ws_bytes, void* stream);

/* ------------------------------------------- pre-norm residual stack ---- */

/* One layer of the 48-layer decode stack ("Avalon": 48 layers of 512
 * experts, top-10) with the residual add between layers:
 *   x = bf16(rmsnorm(r)) per row (eps 1e-6, no learned weight),
 *   r_out = r + MoE(x)            (r_out may alias r: in place)
 * r fp32 [T x H], 16-byte aligned; the other arguments as in
 * moe_layer_forward (w_router, bias, blob_index, topk_idx, topk_w,
 * logits_out or NULL, out_bf16 = bf16 copy of r_out or NULL).  Workspace:
 * moe_layer_workspace_bytes.  T <= 8: one kernel. */
moe_status moe_layer_forward_residual(const moe_layer_desc* desc,
                                      const float* r, int T, int k,
                                      const uint16_t* w_router,
                                      const float* bias,
                                      const int32_t* blob_index, float* r_out,
                                      uint16_t* out_bf16, int32_t* topk_idx,
                                      float* topk_w, float* logits_out,
                                      void* ws, size_t ws_bytes,
                                      void* stream);

/* The same layer in two halves, for callers that act between routing and
 * the expert FFN -- the expert-slot cache ("Betelgeuse": resolve on the
 * device, copy only the misses, then compute; offloaded and resident runs
 * agree bit for bit):
 *   moe_layer_route_residual: x = bf16(rmsnorm(r)), logits, top-k ->
 *     topk_idx [T x k], topk_w [T x k] (and logits_out or NULL).
 *   moe_layer_ffn_residual: r_out = r + sum_j topk_w * FFN_{topk_idx}(x)
 *     with expert e read from pool + blob_index[e] * stride.
 * route then ffn on the same stream and workspace gives bit-for-bit the
 * result of moe_layer_forward_residual with the same blob contents. */
moe_status moe_layer_route_residual(const moe_layer_desc* desc,
                                    const float* r, int T, int k,
                                    const uint16_t* w_router,
                                    const float* bias, int32_t* topk_idx,
                                    float* topk_w, float* logits_out,
                                    void* ws, size_t ws_bytes, void* stream);
moe_status moe_layer_ffn_residual(const moe_layer_desc* desc, const float* r,
                                  int T, int k, const int32_t* topk_idx,
                                  const float* topk_w,
                                  const int32_t* blob_index, float* r_out,
                                  uint16_t* out_bf16, void* ws,
                                  size_t ws_bytes, void* stream);

/* moe_stage_misses then moe_layer_ffn_residual in one launch, with the
 * copies overlapping the compute ("Betelgeuse": the decode pass waits on
 * the pager only for the experts that missed).  The chosen experts that
 * missed (the slot resolve's n_miss / miss_expert / miss_slot, device) are
 * computed after the others; while the hit experts are computed, every
 * block pulls its share of each missed blob from its pinned host copy
 * table[layer * E + e] (moe_stage_table) into pool slot slot_base +
 * miss_slot[i] (the layer's partition: slot_base .. slot_base + n_slots - 1
 * of pool_slots slots of desc->blob_stride bytes at desc->pool), and a
 * missed expert's tiles are read only once all blocks have written theirs
 * (a bounded wait: MOE_ERR_TIMEOUT after 0.5 s).  The result is bit for bit
 * that of the two calls.  Copy errors are reported as in moe_stage_misses,
 * in the workspace's error word.  Needs the one-kernel shapes of
 * moe_layer_forward (T <= 8 ...); other shapes run the two calls in turn. */
moe_status moe_layer_ffn_residual_staged(
    const moe_layer_desc* desc, const float* r, int T, int k,
    const int32_t* topk_idx, const float* topk_w, const int32_t* blob_index,
    float* r_out, uint16_t* out_bf16, const int32_t* n_miss,
    const int32_t* miss_expert, const int32_t* miss_slot, int layer, int L,
    const uint64_t* table, int slot_base, int n_slots, int64_t pool_slots,
    void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream`, read the FFN/grouping workspace's device error word
 * into *host_err (host pointer, may be NULL) and clear it.  Returns
 * MOE_ERR_DEVICE if it was set, MOE_OK otherwise. */
moe_status moe_get_device_status(void* ws, int32_t* host_err, void* stream);

/* Human-readable name of a status code (static string). */
const char* moe_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
