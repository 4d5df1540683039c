/*
 * moe.h -- C ABI of the routed mixture-of-experts FFN layer over MXFP4 expert
 * weights, for NVIDIA B200 (sm_100a).
 *
 * What the layer is (the pages describe it; none prints its formulas):
 *   - DeepSeek-V4-Flash's routed MoE layer: per token only k of E experts run,
 *     and only the activated experts' weights are read from memory
 *     (ainews.cool "antirez ds4 DeepSeek Metal inference", section
 *     技术深度解析: block-sparse matmul over activated experts only).
 *   - routed experts are stored as MXFP4 ("ds4-ssd" README, "Run SSD Sidecar
 *     Mode": native package with bit-exact MXFP4 routed experts).  MXFP4 is the
 *     OCP Microscaling v1.0 format: 32 E2M1 (4-bit) values share one E8M0
 *     power-of-two scale.
 *   - k is a parameter ("ds4-ssd" README, "Experimental Pro Support":
 *     --moe-expert-topk changes the routed expert count); a shared,
 *     always-on expert exists (same section: shared-down prefetch).
 *   - the decode step (T = 1) and the speculative-verify batch of 1 + 4 draft
 *     positions (10100.com ds4-ssd article, "运行模式" / DSpark mode:
 *     --draft-verify 4) are the shapes the layer runs at; prefill runs in
 *     chunks of up to 4K tokens ("ds4-ssd" README, "Validate").
 *
 * Readings where the pages are silent (the same readings as the CPU oracle):
 *   logits = x W_r^T + b (bias used for selection and weights); softmax over
 *   all E, top-k in descending logit order (ties -> lower expert index),
 *   renormalised over the chosen k, no extra scaling; expert
 *   o = W_down (silu(W_gate x) * (W_up x)); y = sum_j w_j o_j (slot order)
 *   + o_shared, rounded to bf16 (RNE).
 *
 * Layouts (all row-major, all device memory unless stated otherwise):
 *   x        [T, H]   bf16 bit patterns (uint16)
 *   W_r      [E, H]   float32 router weights;  bias [E] float32 or NULL
 *   topk_idx [T, k]   int32, descending logit order
 *   topk_w   [T, k]   float32, rows sum to 1
 *   counts   [E]      int32 tokens routed to each expert
 *   offsets  [E + 1]  int32 exclusive scan of counts, offsets[E] = T*k
 *   entries  [T*k]    int32 pair indices p = t*k + j sorted by expert, and by
 *                     ascending token within one expert (stable)
 *   experts  gate_q/up_q [n, I, H/2] u8, gate_s/up_s [n, I, H/32] u8,
 *            down_q [n, H, I/2] u8, down_s [n, H, I/32] u8.  Byte b of a row
 *            holds element 2b in its low nibble and 2b+1 in its high nibble;
 *            scale byte q covers elements 32q..32q+31 of the row.
 *   partial  [T*k + S*T, H] float32: row p = t*k + j is expert idx[t,j]'s
 *            output for token t; rows T*k + t are the shared expert's (S = 1).
 *   y        [T, H]   bf16 bit patterns
 *
 * Constraints (checked on the host before any launch): 1 <= T <= 65536,
 * 32 <= H <= 16384 and H % 32 == 0, 32 <= I <= 16384 and I % 32 == 0,
 * 1 <= E <= 1024, 1 <= k <= min(E, 16); every pointer 16-byte aligned.
 * Violations return MOE_ERR_UNSUPPORTED_SHAPE or MOE_ERR_INVALID_ARG.
 *
 * Ownership and errors: the caller allocates every buffer; the library never
 * allocates or frees device memory.  Calls are asynchronous on `stream`
 * (a cudaStream_t; NULL = legacy default stream) and never synchronise the
 * host.  A launch failure returns MOE_ERR_CUDA.  Faults found on the device
 * (an expert index out of range, ...) are latched in the workspace and read
 * with moe_get_error().  No C++ exception crosses this boundary.
 *
 * Workspace: `ws` is caller-owned device memory of at least
 * moe_workspace_bytes(...) bytes, zeroed once by moe_workspace_init() before
 * its first use.  Its first 16 bytes hold the latched error (status, detail),
 * the wait limit and the debug switches (moe_workspace_set_limits); every call
 * clears the other scratch it relies on itself, so one workspace serves any
 * number of calls of any shapes whose moe_workspace_bytes(...) it covers,
 * including calls replayed from a CUDA graph, as long as calls sharing a
 * workspace are ordered on one stream.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t moe_status_t;
#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1)
#define MOE_ERR_UNSUPPORTED_SHAPE (-2)
#define MOE_ERR_WORKSPACE (-3)
#define MOE_ERR_CUDA (-4)
#define MOE_ERR_TIMEOUT (-5)
#define MOE_ERR_DEVICE_DATA (-6)

/* Debug switches (moe_workspace_set_limits).  MOE_DEBUG_STARVE_FIRST_WAIT:
 * the gate/up kernel leaves its first stage without copies -- on the
 * row-block GEMV the first warp's, on the tensor-core GEMM the first CTA's --
 * so the bounded wait on it runs out and MOE_ERR_TIMEOUT is latched (the
 * error path of a device-side wait, exercised without any fault); the call's
 * output is then undefined.  For tests only. */
#define MOE_DEBUG_STARVE_FIRST_WAIT 1u

typedef struct moe_shape {
  int32_t T; /* tokens in the batch */
  int32_t H; /* hidden size (expert input / output width) */
  int32_t I; /* expert intermediate size */
  int32_t E; /* routed experts */
  int32_t k; /* experts chosen per token */
} moe_shape_t;

/* Device pointers to n_experts MXFP4 experts in the layout above. */
typedef struct moe_mxfp4_experts {
  const uint8_t* gate_q;
  const uint8_t* gate_s;
  const uint8_t* up_q;
  const uint8_t* up_s;
  const uint8_t* down_q;
  const uint8_t* down_s;
  int32_t n_experts;
} moe_mxfp4_experts_t;

/* Expert FFN implementation.  GEMV: CUDA-core streaming kernels (either
 * precision).  GEMM: tcgen05 block-scaled FP4 tensor-core kernels, which
 * require MOE_ACT_MXFP4.  AUTO: GEMM for MOE_ACT_MXFP4 (when the shape allows
 * it: H % 256 == 0, I % 128 == 0), GEMV for MOE_ACT_EXACT. */
#define MOE_PATH_AUTO 0
#define MOE_PATH_GEMV 1
#define MOE_PATH_GEMM 2

/* Activation precision of the expert projections.  EXACT: the bf16 token
 * rows and the fp32 SwiGLU output enter the projections without quantisation
 * (the pages' quality mode, "ds4-ssd" README, "Experimental Pro Support":
 * --quality / --no-int8), with float32 accumulation.  A single token takes
 * the K-split GEMV (float32 products throughout).  On the CUDA-core path for
 * 2 <= T <= 512 (the row-block GEMV, whose products run on f16 tensor-core
 * operands) token row t enters as f16 values of x * 2^-s_t, its largest
 * magnitude scaled into [1, 2) and 2^s_t applied to the sums: every bf16
 * value within 2^-17 of its row's largest magnitude is exact, smaller ones
 * carry an absolute error below 2^-25 of that magnitude.  The SwiGLU output h
 * enters as the pair hi = f16(h 2^-e), lo = f16(h 2^-e - hi) with one power
 * of two 2^e per 32 values (22 significant bits for every value within 2^-18
 * of its block's largest magnitude, an absolute error below 2^-39 of it for
 * the others).  A non-finite value in a token row makes that token's output
 * non-finite.  MXFP4: each projection
 * input row is quantised to MXFP4 in 32-element blocks first (scale
 * 2^(floor(log2 amax) - 2), round-to-nearest-even onto the E2M1 grid,
 * saturating at +-6), as an accelerator path does. */
#define MOE_ACT_EXACT 0
#define MOE_ACT_MXFP4 1

/* Bytes of workspace the calls below need for this shape (any of them).
 * has_shared: 1 if a shared expert is passed.  Returns 0 for an unsupported
 * shape, path or precision (k may exceed E, as for moe_expert_ffn_mxfp4). */
MOE_API size_t moe_workspace_bytes(moe_shape_t shape, int32_t path, int32_t precision,
                           int32_t has_shared);

/* Zero a workspace before its first use (asynchronous memset on stream). */
MOE_API moe_status_t moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Set, for later calls on ws (asynchronous, ordered on stream): the bound of
 * every device-side wait in microseconds (0: the default of 2 s; a wait that
 * runs out latches MOE_ERR_TIMEOUT and its kernel returns) and the debug
 * switches (MOE_DEBUG_*, 0 for none). */
MOE_API moe_status_t moe_workspace_set_limits(void* ws, uint32_t wait_us, uint32_t debug,
                                              void* stream);

/* Router, softmax, top-k and renormalisation.
 * logits[t,e] = sum_h x[t,h] W_r[e,h] + bias[e] in float32 (bias may be NULL);
 * topk_idx/topk_w as described above.  logits_out [T, E] float32 may be NULL.
 * Ties of equal float32 logits go to the lower expert index.  ws must hold the
 * routing part of moe_workspace_bytes(shape, ...); batches above 32 tokens
 * split the router's dot products over up to 16 K ranges when ws also covers
 * the shape's later regions (their sums are added in range order, so every
 * product meets at most 32 + H/32 + 1 float32 roundings). */
MOE_API moe_status_t moe_route_topk(const uint16_t* x, const float* w_router,
                            const float* bias, moe_shape_t shape,
                            float* logits_out, int32_t* topk_idx,
                            float* topk_w, void* ws, size_t ws_bytes,
                            void* stream);

/* Stable counting sort of the T*k (token, slot) pairs by expert: writes
 * counts [E], offsets [E+1] and entries [T*k] (layouts above).  An index
 * outside [0, E) latches MOE_ERR_DEVICE_DATA and the pair is dropped.  Above
 * 2048 pairs, when ws covers the shape's later regions, one CTA per 2048
 * pairs sorts its chunk (same result). */
MOE_API moe_status_t moe_bucket(const int32_t* topk_idx, moe_shape_t shape,
                        int32_t* counts, int32_t* offsets, int32_t* entries,
                        void* ws, size_t ws_bytes, void* stream);

/* Expert SwiGLU FFNs of the routed pairs (and of every token through the
 * shared expert when `shared` is not NULL):
 *   partial[p]      = W_down[e] (silu(W_gate[e] x_t) * (W_up[e] x_t))
 *   for every p = t*k + j listed in entries with e the bucket's expert, and
 *   partial[T*k+t]  = the same through the shared expert.
 * `experts` and `shared` are host pointers to structs of device pointers;
 * experts->n_experts must equal shape.E, shared->n_experts must be 1.
 * Rows of pairs not listed in entries are left untouched.  Here k only sets
 * the pair layout and may exceed shape.E (a rank holding a share of the
 * experts, with offsets pointing at its experts' bucket starts). */
MOE_API moe_status_t moe_expert_ffn_mxfp4(const moe_mxfp4_experts_t* experts,
                                  const moe_mxfp4_experts_t* shared,
                                  const uint16_t* x, const int32_t* offsets,
                                  const int32_t* entries, moe_shape_t shape,
                                  int32_t path, int32_t precision,
                                  float* partial_out, void* ws,
                                  size_t ws_bytes, void* stream);

/* y[t] = bf16_rne( sum_{j<k} topk_w[t,j] * partial[t*k+j]
 *                  + (has_shared ? partial[T*k+t] : 0) ), summed in that
 * order in float32. */
MOE_API moe_status_t moe_combine(const float* partial, const float* topk_w,
                         moe_shape_t shape, int32_t has_shared, uint16_t* y,
                         void* stream);

/* Expert-parallel pieces (a group of ranks each holding a contiguous range of
 * the routed experts; the pages run on one device, this spreads the same
 * layer over several):
 *   y_f32[t] = sum over j < k with e_begin <= topk_idx[t,j] < e_end of
 *              topk_w[t,j] * partial[t*k+j]  (+ partial[T*k+t] if has_shared),
 * summed in slot order in float32 and left in float32 [T, H] so the ranks'
 * results can be added (one all-reduce); rows of pairs outside the range are
 * not read.  0 <= e_begin <= e_end <= shape.E. */
MOE_API moe_status_t moe_combine_range(const float* partial, const float* topk_w,
                                       const int32_t* topk_idx, int32_t e_begin, int32_t e_end,
                                       moe_shape_t shape, int32_t has_shared, float* y_f32,
                                       void* stream);

/* out[i] = bf16_rne(in[i]) for n float32 values (n % 4 == 0). */
MOE_API moe_status_t moe_round_bf16(const float* in, int64_t n, uint16_t* out, void* stream);

/* The whole layer: route -> bucket -> expert FFNs -> combine, on `stream`.
 * topk_idx_out [T,k] and topk_w_out [T,k] may be NULL (kept in ws then). */
MOE_API moe_status_t moe_layer_forward(const uint16_t* x, const float* w_router,
                               const float* bias,
                               const moe_mxfp4_experts_t* experts,
                               const moe_mxfp4_experts_t* shared,
                               moe_shape_t shape, int32_t path,
                               int32_t precision, uint16_t* y,
                               int32_t* topk_idx_out, float* topk_w_out,
                               void* ws, size_t ws_bytes, void* stream);

/* The whole layer like moe_layer_forward (CUDA-core GEMV path) but with no
 * workspace argument and no allocation of any kind.  The pages have no
 * counterpart: this serves callers that may not allocate device memory (a host
 * application that owns every allocation through its own pool, a real-time
 * loop where cudaMalloc/cudaFree could synchronise the device, plug-in code
 * that only receives its input and output tensors).  Scratch is a fixed
 * 16 MiB array inside the library's device image, held on every GPU that loads
 * the library until the process exits; a shape whose moe_workspace_bytes(...,
 * MOE_PATH_GEMV, ...) exceeds it returns MOE_ERR_WORKSPACE.  The first call on
 * a device looks up the array's device address (make it before any stream
 * capture).  Every call reuses the same array, which keeps what the last call
 * left there; each call clears the words it needs at zero itself.  Calls that
 * overlap on the GPU race and must be ordered on one stream.  A device-side
 * error (an expired wait, MOE_ERR_TIMEOUT) is latched in the array and stays
 * there, for this and later calls on the device, until
 * moe_get_error_static() reads it.  Inputs and outputs as for
 * moe_layer_forward; topk_idx_out / topk_w_out may be NULL. */
MOE_API moe_status_t moe_layer_forward_static(const uint16_t* x, const float* w_router,
                                              const float* bias,
                                              const moe_mxfp4_experts_t* experts,
                                              const moe_mxfp4_experts_t* shared,
                                              moe_shape_t shape, int32_t precision,
                                              uint16_t* y, int32_t* topk_idx_out,
                                              float* topk_w_out, void* stream);

/* moe_get_error() for moe_layer_forward_static on the current device:
 * synchronise `stream`, return the first device-side error latched in the
 * static scratch since the last read (MOE_OK if none) and clear it.  Allocates
 * nothing. */
MOE_API moe_status_t moe_get_error_static(void* stream);

/* ---------------------------------------------------------------------------
 * Slot bank: the routed experts in pinned host memory, a bounded set of them
 * resident in device memory.  The ds4-ssd engine streams the experts its
 * router picks into a fixed expert cache ("ds4-ssd" README, "Run SSD Sidecar
 * Mode"); here the backing store is pinned host memory and the bank a
 * caller-owned device region of n_slots experts, filled least recently used
 * first.  A bank is used from one host thread at a time.
 * ------------------------------------------------------------------------- */
typedef struct moe_slot_bank moe_slot_bank_t;

/* Device bytes of a bank of n_slots experts of shape (H, I); 0 if invalid. */
MOE_API size_t moe_slot_bank_bytes(int32_t H, int32_t I, int32_t n_slots);

/* Create a bank over host_experts (HOST pointers to pinned memory, in the
 * canonical layout, n_experts = E) with n_slots slots in slot_mem (device,
 * 16-byte aligned, at least moe_slot_bank_bytes bytes, owned by the caller).
 * The bank object and two small pinned host buffers (the call's expert ids,
 * the expert -> slot map) are host memory the library allocates;
 * moe_slot_bank_destroy frees them.  No device memory is allocated. */
MOE_API moe_status_t moe_slot_bank_create(const moe_mxfp4_experts_t* host_experts, int32_t H,
                                          int32_t I, int32_t n_slots, void* slot_mem,
                                          size_t slot_mem_bytes, moe_slot_bank_t** out);
MOE_API void moe_slot_bank_destroy(moe_slot_bank_t* bank);

/* Make the experts ids[0..n) (host array) resident: experts already in the
 * bank keep their slot, missing ones take the least recently used slots this
 * call does not need, copied host -> device on `stream` (asynchronous);
 * slot_of[i] (host) receives the slot of ids[i].  Calling it ahead of a layer
 * call with the experts expected next prefetches them.  More distinct experts
 * than slots returns MOE_ERR_WORKSPACE. */
MOE_API moe_status_t moe_slot_bank_acquire(moe_slot_bank_t* bank, const int32_t* ids, int32_t n,
                                           int32_t* slot_of, void* stream);

/* The device experts struct of the bank's slots (n_experts = n_slots). */
MOE_API moe_status_t moe_slot_bank_experts(const moe_slot_bank_t* bank,
                                           moe_mxfp4_experts_t* out);

/* Slot hits, misses (host -> device copies) and evictions so far. */
MOE_API moe_status_t moe_slot_bank_stats(const moe_slot_bank_t* bank, int64_t* hits,
                                         int64_t* misses, int64_t* evictions);

/* The layer with its routed experts in a slot bank: route and top-k over all
 * E experts on `stream`, the chosen experts read back to the host (this call
 * synchronises the stream once), made resident, the indices rewritten to
 * slots, then bucket, expert FFNs and combine over the bank.  Same inputs and
 * output as moe_layer_forward; topk_idx_out / topk_w_out are required (expert
 * ids and weights); T * k <= 8192; ws of at least
 * moe_layer_forward_banked_workspace_bytes bytes. */
MOE_API moe_status_t moe_layer_forward_banked(const uint16_t* x, const float* w_router,
                                              const float* bias, moe_slot_bank_t* bank,
                                              const moe_mxfp4_experts_t* shared,
                                              moe_shape_t shape, int32_t path, int32_t precision,
                                              uint16_t* y, int32_t* topk_idx_out,
                                              float* topk_w_out, void* ws, size_t ws_bytes,
                                              void* stream);
MOE_API size_t moe_layer_forward_banked_workspace_bytes(moe_shape_t shape, int32_t n_slots,
                                                        int32_t path, int32_t precision,
                                                        int32_t has_shared);

/* Quantise rows [rows, K] float32 to MXFP4 (codes [rows, K/2], scales
 * [rows, K/32]) with the MOE_ACT_MXFP4 rule above; K % 32 == 0. */
MOE_API moe_status_t moe_act_quant_mxfp4(const float* in, int32_t rows, int32_t K,
                                 uint8_t* q_out, uint8_t* s_out, void* stream);

/* Decode MXFP4 rows (codes [rows, K/2], scales [rows, K/32]) to float32
 * [rows, K] with the conversions the row-block GEMV uses (cvt e2m1x2 -> f16x2
 * for the codes, cvt ue8m0x2 -> bf16x2 for the scales): E2M1 value times
 * 2^(scale-127), scale byte 0 the subnormal 2^-127, byte 255 NaN.  For tests
 * and tools. */
MOE_API moe_status_t moe_decode_mxfp4(const uint8_t* q, const uint8_t* s, int32_t rows,
                              int32_t K, float* out, void* stream);

/* Synchronise `stream`, return the first device-side error latched in ws
 * since the last call (MOE_OK if none) and clear it. */
MOE_API moe_status_t moe_get_error(void* ws, void* stream);

/* Static description of a status code. */
MOE_API const char* moe_status_string(moe_status_t status);

/* Library version, e.g. "0.1.0". */
MOE_API const char* moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
