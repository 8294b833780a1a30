/*
 * mtla.h -- C ABI of the B200 (sm_100a) MTLA attention library, libmtla.so.
 *
 * MTLA (Multi-head Temporal Latent Attention) attends over a KV cache that is
 * compressed twice: every token is reduced to an MLA-style latent c_t (width
 * d_c) plus one decoupled-RoPE key k_t (width d_r), and every s consecutive
 * tokens are merged into one cache slot by a learned gate,
 *   slot_j = sum_{t in block j} w_t [c_t ; RoPE_t(k_t)].
 * Queries attend the slots in the absorbed form (W_UK folded into the query,
 * W_UV applied after the weighted sum) under the stride-aware causal mask:
 * query t sees every finished slot j < floor(t/s) plus its own slot while it
 * is being filled.
 *
 * Sources (page titles and the sections they name):
 *   "Multi-head Temporal Latent Attention" (paper summary page), Method:
 *     (1) merging weights from a hyper-network on the latent times a
 *         positional embedding (Sec. 4.1, Eq. 13), and the in-place update of
 *         the slot being filled at inference;
 *     (2) the stride-aware causal mask for parallel training (Sec. 4.2,
 *         Fig. 2(c));
 *     (3) decoupled-RoPE keys merged along the same axis with the same mask
 *         (Sec. 4.3, Eq. 17); absorption of W^UK and W^UV kept from MLA.
 *   "Multi-Head Latent Attention and Sparse Indexers", "Latent attention
 *     changes the representation": q.(U_K c) = (U_K^T q).c and
 *     sum_j a_j U_V c_j = U_V sum_j a_j c_j.
 *
 * Readings where the pages are silent (fixed by this ABI):
 *   - slots are 0-based: token t lives in slot floor(t/s);
 *   - w_t = sigmoid(G[t mod s] . (c_t * PE_t) + g[t mod s]) with PE_t the
 *     interleaved sinusoid of width d_c and base 10000 (MTLA_GATE_COMPUTED);
 *     the gate may instead be supplied per token (MTLA_GATE_SUPPLIED) or fixed
 *     to 1 (MTLA_GATE_UNIT);
 *   - RoPE rotates interleaved pairs (x_2k, x_2k+1) by t * base^(-2k/d_r);
 *   - the absorbed query is q~ = [W_UK[h]^T qC ; RoPE_t(qR)], the score
 *     scale * <q~, slot>, the output o = W_UV[h] (sum_j a_j slot_j[0:d_c]).
 *
 * Conventions common to every call:
 *   - All tensors are dense, row-major, on the current CUDA device, and the
 *     caller owns them. Every pointer must be 16-byte aligned.
 *   - Storage type: MTLA_BF16 stores activations, weights, cache and output in
 *     bfloat16 (round-to-nearest-even) and computes in fp32; MTLA_FP32 stores
 *     and computes everything in fp32 (no tensor-float rounding anywhere);
 *     MTLA_FP16 stores them in IEEE half precision (round-to-nearest-even) and
 *     computes in fp32 on the CUDA cores (the tensor-core kernels take bf16).
 *     Gate parameters, supplied gates and the open-slot accumulator are
 *     always float32. mtla_linear and the layer calls are bf16 only.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream) and allocate nothing: scratch comes from `workspace`,
 *     whose size mtla_workspace_size() reports.
 *   - Stream order: the first kernel of a bf16 decode step is launched as a
 *     programmatic dependent of the kernel before it, so consecutive steps
 *     overlap. It reads only weights (the absorbed projection W_UK and the
 *     gate's G) before that kernel finishes. That holds for any kernel that does not trigger its
 *     dependents early (ordinary kernels never do). A caller kernel that does
 *     trigger early must write the step's inputs before it triggers. Those
 *     inputs are the positions, latents, queries and gates.
 *   - Argument errors are found on the host before anything is launched and
 *     returned as a status; nothing is written then. Errors found on the
 *     device (a position beyond the cache, a bounded wait that ran out) skip
 *     the affected work and are latched in a device status word that
 *     mtla_get_device_status() reads.
 *   - The library looks up the device addresses of its own device variables
 *     (the status word, the no-allocation scratch array) once per device and
 *     keeps them for the life of the process. A cudaDeviceReset() on a device
 *     invalidates them: calls on that device after such a reset are not
 *     supported.
 */
#ifndef MTLA_H_
#define MTLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MTLA_OK = 0,
    MTLA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or enum      */
    MTLA_ERR_UNSUPPORTED = 2,   /* valid MTLA shape the library has no kernel for */
    MTLA_ERR_CAPACITY = 3,      /* a position does not fit in max_slots slots     */
    MTLA_ERR_CUDA = 4,          /* a CUDA runtime call failed                     */
    MTLA_ERR_TIMEOUT = 5,       /* a bounded device wait ran out (device status)  */
    MTLA_ERR_WORKSPACE = 6      /* workspace smaller than mtla_workspace_size()   */
} mtla_status;

typedef enum { MTLA_BF16 = 0, MTLA_FP32 = 1, MTLA_FP16 = 2 } mtla_dtype;

/* Merging weights (MTLA Sec. 4.1, Eq. 13; the reading of W_t (.) x_t):
 * one scalar per token that scales its whole slot vector x_t = [c_t ; RoPE_t(k_t)]
 * (modes 0-2), or one weight per slot channel (modes 3-4, the reading of W_t as
 * a vector): slot_j = sum_t w_t (.) x_t. The attention is the same for all. */
typedef enum {
    MTLA_GATE_COMPUTED = 0,     /* w_t = sigmoid(G[t mod s] . (c_t*PE_t) + g[t mod s]):
                                   gate_w G [s, d_c] fp32, gate_b g [s] fp32           */
    MTLA_GATE_SUPPLIED = 1,     /* w_t read from gate_in: [B] (decode), [B, T] (prefill) */
    MTLA_GATE_UNIT = 2,         /* w_t = 1                                             */
    MTLA_GATE_CHANNEL_COMPUTED = 3, /* w_t[k] = sigmoid((c_t*PE_t) . G[t mod s][:, k] +
                                   g[t mod s][k]), k < d_c + d_r: gate_w G [s, d_c, d_c+d_r]
                                   fp32 (input channel major), gate_b g [s, d_c+d_r] fp32 */
    MTLA_GATE_CHANNEL_SUPPLIED = 4  /* w_t[k] read from gate_in: [B, d_c+d_r] (decode),
                                   [B, T, d_c+d_r] (prefill)                            */
} mtla_gate_mode;

/* Problem description shared by every call.
 * Supported: 1 <= batch; 1 <= heads <= 128; d_h, d_c, d_r multiples of 16;
 * d_c + d_r <= 576; d_h <= 256; 1 <= stride <= 8; max_slots >= 1; with the
 * per-channel gate modes also d_r <= 128.
 * Anything else: MTLA_ERR_UNSUPPORTED (or INVALID_ARG for non-positive sizes). */
typedef struct {
    int32_t batch;          /* B: sequences                                       */
    int32_t heads;          /* H: query heads (all share the cache, MQA form)     */
    int32_t d_h;            /* per-head width of qC and of the output             */
    int32_t d_c;            /* latent width                                       */
    int32_t d_r;            /* decoupled-RoPE width of keys and query parts       */
    int32_t stride;         /* s: tokens merged into one slot                     */
    int32_t dtype;          /* mtla_dtype                                         */
    int32_t gate_mode;      /* mtla_gate_mode                                     */
    float softmax_scale;    /* 0 => 1/sqrt(d_h + d_r)                             */
    float rope_base;        /* 0 => 10000                                         */
    int32_t max_slots;      /* slots per sequence in the cache buffer             */
} mtla_config;

/* Bytes of scratch that mtla_decode_step (any positions) and mtla_prefill
 * (any T <= max_tokens) need with this config. `bytes` receives the size.
 * Returns INVALID_ARG / UNSUPPORTED for a bad config. Host only. */
mtla_status mtla_workspace_size(const mtla_config* cfg, int32_t max_tokens, size_t* bytes);

/* One incremental decode step: one new token for every sequence
 * (MTLA Method (1): only every s-th step opens a new slot, the steps in
 * between update the slot being filled in place).
 *
 * For each sequence b with t = pos[b]:
 *   w_t per gate_mode; x = [c_new[b] ; RoPE_t(kr_new[b])];
 *   open_slot[b] = (t mod s == 0 ? 0 : open_slot[b]) + w_t x     (fp32)
 *   cache[b, floor(t/s)] = round(open_slot[b])
 *   for every head h: q~ = [W_UK[h]^T q_c[b,h] ; RoPE_t(q_r[b,h])];
 *     out[b,h] = W_UV[h] softmax_j(scale <q~, cache[b,j]>) cache[b,j][0:d_c]
 *     over j = 0 .. floor(t/s).
 *
 *   c_new   [B, d_c]        dtype        kr_new [B, d_r] dtype (before RoPE)
 *   q_c     [B, H, d_h]     dtype        q_r    [B, H, d_r] dtype (before RoPE)
 *   w_uk    [H, d_h, d_c]   dtype        w_uv   [H, d_h, d_c] dtype
 *   gate_w, gate_b     (the COMPUTED modes, shapes under mtla_gate_mode; else may be NULL)
 *   gate_in [B] or [B, d_c+d_r] fp32          (the SUPPLIED modes; else may be NULL)
 *   pos     [B] int32, device: index of this token = tokens already cached.
 *           pos[b] >= max_slots * s skips sequence b and latches CAPACITY.
 *   cache   [B, max_slots, d_c + d_r] dtype, in/out (slot floor(t/s) written)
 *   open_slot [B, d_c + d_r] fp32, in/out (the slot being filled, unrounded)
 *   out     [B, H, d_h]     dtype, out
 *   workspace / workspace_bytes: scratch of at least mtla_workspace_size().
 * Returns OK once the work is enqueued. */
mtla_status mtla_decode_step(const mtla_config* cfg,
                             const void* c_new, const void* kr_new,
                             const void* q_c, const void* q_r,
                             const void* w_uk, const void* w_uv,
                             const float* gate_w, const float* gate_b, const float* gate_in,
                             const int32_t* pos,
                             void* cache, float* open_slot, void* out,
                             void* workspace, size_t workspace_bytes, void* stream);

/* Parallel (training-form) forward over T tokens from position 0
 * (MTLA Method (2)-(3): the stride-aware causal mask lets every position see
 * the finished slots plus its own block's partial slot
 *   P_t = sum_{u = s*floor(t/s)}^{t} w_u [c_u ; RoPE_u(k_u)],
 * so the result equals T incremental decode steps).
 *
 *   c [B,T,d_c], kr [B,T,d_r], q_c [B,T,H,d_h], q_r [B,T,H,d_r]   dtype
 *   w_uk, w_uv, gate_w, gate_b as for decode; gate_in [B,T] or [B,T,d_c+d_r] fp32 (SUPPLIED modes)
 *   out       [B,T,H,d_h] dtype, out
 *   cache_out [B, max_slots, d_c+d_r] dtype, out: slots 0..ceil(T/s)-1 (the
 *             cache a following mtla_decode_step at pos = T continues from);
 *             requires max_slots >= ceil(T/s); must not be NULL.
 *   open_slot_out [B, d_c+d_r] fp32, out, may be NULL: P_{T-1}.
 * T >= 1. Returns OK once the work is enqueued. */
mtla_status mtla_prefill(const mtla_config* cfg, int32_t T,
                         const void* c, const void* kr,
                         const void* q_c, const void* q_r,
                         const void* w_uk, const void* w_uv,
                         const float* gate_w, const float* gate_b, const float* gate_in,
                         void* out, void* cache_out, float* open_slot_out,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Chunked prefill: the parallel forward over T new tokens at positions
 * t0 .. t0+T-1 of every sequence, continuing from the cache state after t0
 * tokens (a long prompt processed in chunks, or a prompt appended to a
 * conversation whose cache exists). MTLA Method (1)-(3): the stride-aware
 * mask lets position i see every finished slot j < floor(i/s) -- those already
 * in the cache and those this chunk completes -- plus its own partial slot; a
 * slot left open at t0 (t0 mod s != 0) continues from the open-slot
 * accumulator, exactly as the in-place update of decoding would continue it.
 * The result equals T calls of mtla_decode_step from the same state, and
 * mtla_prefill over t0+T tokens equals mtla_prefill over t0 followed by this.
 *
 *   t0        tokens already in the cache, the same for every sequence (>= 0)
 *   c, kr, q_c, q_r, gate_in   the new tokens only: [B,T,...] as for mtla_prefill
 *   cache     [B, max_slots, d_c+d_r] dtype, in/out: slots 0 .. ceil(t0/s)-1
 *             hold the state after t0 tokens; slots floor(t0/s) ..
 *             ceil((t0+T)/s)-1 are written (the first may be the open one);
 *             requires ceil((t0+T)/s) <= max_slots (else CAPACITY).
 *   open_slot [B, d_c+d_r] fp32, in/out, not NULL: the accumulator after t0
 *             tokens (read when t0 mod s != 0), then after t0+T tokens.
 *   out, weights, workspace: as for mtla_prefill (mtla_workspace_size with
 *             max_tokens >= T covers it).
 * t0 = 0 is mtla_prefill with cache_out = cache. Returns OK once enqueued. */
mtla_status mtla_prefill_from(const mtla_config* cfg, int32_t t0, int32_t T,
                              const void* c, const void* kr,
                              const void* q_c, const void* q_r,
                              const void* w_uk, const void* w_uv,
                              const float* gate_w, const float* gate_b, const float* gate_in,
                              void* out, void* cache, float* open_slot,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Scratch for mtla_prefill_backward over T tokens. Host only. */
mtla_status mtla_prefill_backward_workspace_size(const mtla_config* cfg, int32_t T, size_t* bytes);

/* Training backward of the parallel forward from position 0 ("Multi-head
 * Temporal Latent Attention", Results: the models are trained from scratch,
 * through the stride-aware mask of Key claims; the gate of Sec. 4.1, Eq. 13,
 * and the block-prefix scan of Sec. 4.2 differentiated as written): given
 * dout, the gradient of a loss L with respect to mtla_prefill's `out`, the
 * gradients of L with respect to every input of that forward.
 *   c, kr, q_c, q_r, w_uk, w_uv, gate_w, gate_b, gate_in: exactly as for
 *       mtla_prefill (storage type cfg->dtype; the gates float32)
 *   dout      [B, T, H, d_h]  storage type
 * Outputs, all float32, contiguous, 16-byte aligned, written whole:
 *   dc [B, T, d_c]   dkr [B, T, d_r]   dq_c [B, T, H, d_h]   dq_r [B, T, H, d_r]
 *   dw_uk, dw_uv [H, d_h, d_c]
 *   dgate_w [s, d_c], dgate_b [s]   (MTLA_GATE_COMPUTED; else may be NULL, untouched)
 *   dgate_in [B, T]                 (MTLA_GATE_SUPPLIED; else may be NULL, untouched)
 * The scalar gate modes only: a per-channel mode gives MTLA_ERR_UNSUPPORTED.
 * cfg->max_slots is not used (any positive value). The forward is recomputed
 * inside (the scan and the absorbed queries) from the inputs. Arithmetic is
 * fp32 on the CUDA cores for both storage types. Returns OK once enqueued;
 * INVALID_ARG for a missing or misaligned pointer or T <= 0, WORKSPACE when
 * workspace_bytes is below mtla_prefill_backward_workspace_size. */
mtla_status mtla_prefill_backward(const mtla_config* cfg, int32_t T,
                                  const void* c, const void* kr,
                                  const void* q_c, const void* q_r,
                                  const void* w_uk, const void* w_uv,
                                  const float* gate_w, const float* gate_b, const float* gate_in,
                                  const void* dout,
                                  float* dc, float* dkr, float* dq_c, float* dq_r,
                                  float* dw_uk, float* dw_uv,
                                  float* dgate_w, float* dgate_b, float* dgate_in,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* The training pair, where the backward runs on the tensor cores (bf16 storage,
 * d_h = 64, d_r = 32, d_c = 128 or 256, scalar gates; UNSUPPORTED otherwise):
 * a forward that keeps what the backward needs (per row the log-sum-exp, O / l
 * and the absorbed query; the partial slots, the slots and the merging
 * weights), and a backward from it that does not recompute the forward.
 * mtla_prefill_train: arguments as for mtla_prefill from position 0 without
 * the cache outputs; `out` receives the same output; `saved` (device memory
 * of at least mtla_prefill_train_saved_size bytes, 16-byte aligned, owned by
 * the caller) receives the kept rows. mtla_prefill_backward_saved: arguments,
 * outputs and errors as for mtla_prefill_backward, plus `saved` from a
 * mtla_prefill_train call on the same config, T and inputs (not checked: a
 * different `saved` gives wrong gradients), and its own (smaller) workspace.
 * Both return OK once enqueued on `stream`. */
mtla_status mtla_prefill_train_saved_size(const mtla_config* cfg, int32_t T, size_t* bytes);
mtla_status mtla_prefill_backward_saved_workspace_size(const mtla_config* cfg, int32_t T, size_t* bytes);
mtla_status mtla_prefill_train(const mtla_config* cfg, int32_t T,
                               const void* c, const void* kr, const void* q_c, const void* q_r,
                               const void* w_uk, const void* w_uv,
                               const float* gate_w, const float* gate_b, const float* gate_in,
                               void* out, void* saved, size_t saved_bytes, void* stream);
mtla_status mtla_prefill_backward_saved(const mtla_config* cfg, int32_t T,
                                        const void* c, const void* kr, const void* q_c, const void* q_r,
                                        const void* w_uk, const void* w_uv,
                                        const float* gate_w, const float* gate_b, const float* gate_in,
                                        const void* saved, const void* dout,
                                        float* dc, float* dkr, float* dq_c, float* dq_r,
                                        float* dw_uk, float* dw_uv,
                                        float* dgate_w, float* dgate_b, float* dgate_in,
                                        void* workspace, size_t workspace_bytes, void* stream);

/* Dense projection on the tensor cores: y[M, N] = x[M, K] . w[N, K]^T with
 * bf16 operands and result and fp32 accumulation. The layer around the path
 * ("Multi-head Temporal Latent Attention", Method: MLA's low-rank compression
 * kept, h_t projected to the shared latent c_t, the decoupled key and the
 * queries; the heads' outputs projected back by W_O) is made of these.
 *   x [M, K], w [N, K], y [M, N]: bf16, row-major, contiguous, 16-byte aligned.
 *   K a multiple of 8 (TMA row pitch); M, N, K >= 1. INVALID_ARG otherwise.
 * Returns OK once enqueued on `stream`. */
mtla_status mtla_linear(const void* x, const void* w, void* y, int32_t M, int32_t N, int32_t K, void* stream);

/* The MTLA layer around the path ("Multi-head Temporal Latent Attention",
 * Method: MLA's low-rank compression kept; "Multi-Head Latent Attention and
 * Sparse Indexers", "Latent attention changes the representation"), bf16 only:
 *   c = h W_DKV^T   k = h W_KR^T   qC = h W_Q^T (heads)   qR = h W_QR^T (heads)
 *   o = the MTLA path on (c, k, qC, qR)       y = o W_O^T
 * Every projection is an mtla_linear GEMM; the absorbed W_UK and W_UV stay in
 * the path's kernels. The weights (all bf16, row-major, 16-byte aligned): */
typedef struct {
    const void* w_dkv;      /* [d_c, d_model]     latent down-projection              */
    const void* w_kr;       /* [d_r, d_model]     decoupled key (RoPE in the path)     */
    const void* w_q;        /* [H * d_h, d_model] per-head queries                      */
    const void* w_qr;       /* [H * d_r, d_model] per-head RoPE query parts             */
    const void* w_uk;       /* [H, d_h, d_c]      as for mtla_decode_step              */
    const void* w_uv;       /* [H, d_h, d_c]                                           */
    const void* w_o;        /* [d_model, H * d_h] output projection                    */
} mtla_layer_weights;

/* Scratch for mtla_layer_forward with T <= max_tokens and for
 * mtla_layer_decode_step (the projections' outputs plus the path's scratch).
 * d_model a positive multiple of 8. Host only. */
mtla_status mtla_layer_workspace_size(const mtla_config* cfg, int32_t d_model, int32_t max_tokens, size_t* bytes);

/* The layer over T tokens of every sequence at positions t0 .. t0+T-1,
 * continuing from the cache state after t0 tokens (t0 = 0: from an empty
 * cache; the path is mtla_prefill_from).
 *   h [B, T, d_model] bf16 in;  y [B, T, d_model] bf16 out
 *   cache, open_slot: as for mtla_prefill_from (in/out; open_slot not NULL)
 *   gate_w, gate_b, gate_in: as for mtla_prefill_from
 * cfg->dtype must be MTLA_BF16 (else UNSUPPORTED). Returns OK once enqueued. */
mtla_status mtla_layer_forward(const mtla_config* cfg, int32_t d_model, int32_t t0, int32_t T, const void* h,
                               const mtla_layer_weights* w, const float* gate_w, const float* gate_b,
                               const float* gate_in, void* y, void* cache, float* open_slot,
                               void* workspace, size_t workspace_bytes, void* stream);

/* One decode step of the layer: h [B, d_model] (the new token of every
 * sequence) -> y [B, d_model]; pos, cache, open_slot and the gates as for
 * mtla_decode_step. cfg->dtype must be MTLA_BF16. */
mtla_status mtla_layer_decode_step(const mtla_config* cfg, int32_t d_model, const void* h,
                                   const mtla_layer_weights* w, const float* gate_w, const float* gate_b,
                                   const float* gate_in, const int32_t* pos, void* cache, float* open_slot,
                                   void* y, void* workspace, size_t workspace_bytes, void* stream);

/* Decode step without a workspace argument, for callers that cannot allocate
 * device memory themselves: code inside a host framework whose pool allocator
 * owns all device memory and forbids raw cudaMalloc, serving loops that cannot
 * afford a cudaMalloc/cudaFree (which may synchronise the device) in the
 * middle of a step, or plug-in hosts that hand over only input and output
 * buffers. The pages describe no such interface: it has no counterpart in the
 * paper.
 *
 * Same arguments, meaning and result as mtla_decode_step, minus `workspace`
 * and `workspace_bytes`: the scratch comes from one array of
 * MTLA_NOALLOC_SCRATCH_BYTES bytes in device memory that libmtla.so declares;
 * every GPU that loads the library holds it until the process exits. The call
 * allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 *   - Limit: a config whose decode scratch (mtla_workspace_size with
 *     max_tokens = 0) exceeds MTLA_NOALLOC_SCRATCH_BYTES is refused on the host
 *     with MTLA_ERR_WORKSPACE before anything is launched.
 *   - Set-up: the first call on a device looks up the array's device address
 *     on that device (cudaGetSymbolAddress, with that device current); make
 *     that first call before any stream capture.
 *   - Sharing: all calls on a device share the one array, which keeps the last
 *     call's contents. Calls whose kernels overlap on the GPU (different
 *     streams with no ordering between them) race on it and give wrong
 *     results; order them, or use mtla_decode_step with separate workspaces. */
#define MTLA_NOALLOC_SCRATCH_BYTES (8u << 20)
mtla_status mtla_decode_step_noalloc(const mtla_config* cfg,
                                     const void* c_new, const void* kr_new,
                                     const void* q_c, const void* q_r,
                                     const void* w_uk, const void* w_uv,
                                     const float* gate_w, const float* gate_b,
                                     const float* gate_in, const int32_t* pos,
                                     void* cache, float* open_slot, void* out, void* stream);

/* Beam-search reorder of the cache, between decode steps. The authors'
 * toolkit decodes with parallel beam search (its project page on
 * sourcepulse.org, "Highlighted Details"); after a step each surviving beam b
 * continues from a parent beam j = src[b], whose cache it must take over:
 *   cache_out[b, 0:n) = cache_in[j, 0:n),  n = ceil(n_tokens[j] / s)
 *   open_out[b]       = open_in[j]
 * The copy is byte exact. Slots n .. max_slots-1 of cache_out[b] are left as
 * they were. Out of place: the caller keeps two caches and swaps them.
 *
 *   src       [B] int32, device: parent of each destination, 0 <= src[b] < B
 *             (duplicates allowed); an index outside skips destination b and
 *             latches INVALID_ARG.
 *   n_tokens  [B] int32, device, indexed by parent: tokens cached in it (its
 *             next decode position); above max_slots * s skips the
 *             destinations that take that parent and latches CAPACITY.
 *   cache_in, cache_out   [B, max_slots, d_c + d_r] dtype; must not overlap.
 *   open_in, open_out     [B, d_c + d_r] fp32; must not overlap.
 * cfg must pass the same checks as for the other calls, but only its batch,
 * d_c, d_r, stride, dtype and max_slots are used. All pointers 16-byte
 * aligned; INVALID_ARG (nothing launched) otherwise or if the buffers
 * overlap. Returns OK once the work is enqueued. */
mtla_status mtla_reorder_cache(const mtla_config* cfg, const int32_t* src, const int32_t* n_tokens,
                               const void* cache_in, const float* open_in,
                               void* cache_out, float* open_out, void* stream);

/* Test hook for the failure path (no counterpart in the pages): launches one
 * CTA that lands a TMA load of 2 KB from `scratch` (device memory, 16-byte
 * aligned, at least 2 KB) and then waits, with the same bounded wait every
 * kernel of the library uses but a limit of `limit_ns` (1 .. 1e9), on an
 * mbarrier nothing arrives on. The wait runs out, MTLA_ERR_TIMEOUT is latched
 * in the device status word, the load is drained and the CTA returns: no
 * hang, no fault, and later calls run normally. INVALID_ARG for a bad
 * argument. Returns OK once enqueued. */
mtla_status mtla_test_wait_timeout(uint64_t limit_ns, void* scratch, void* stream);

/* Synchronises `stream`, then returns and clears the status latched by
 * device-side checks on the current device since the last call (OK if none). */
mtla_status mtla_get_device_status(void* stream);

/* Static English text for a status code. */
const char* mtla_status_string(mtla_status status);

/* Text naming the CUDA call (and its error) behind the last MTLA_ERR_CUDA
 * returned on this host thread; "" if none. Valid until the next call on the
 * same thread. */
const char* mtla_last_error_detail(void);

/* Number of kernels this library has launched in this process (all devices). */
uint64_t mtla_kernel_launches(void);

/* Timing hook for measurement tools (not thread-safe). After this call, the
 * i-th following mtla_decode_step / mtla_prefill call (i = 0, 1, ...) records
 * events[2i] on its stream just before its main attention kernel and
 * events[2i+1] just after it, while i < n_pairs; later calls record nothing.
 * `events` holds cudaEvent_t handles created and owned by the caller and must
 * stay valid while the hook is set. mtla_set_profile_events(NULL, 0) turns
 * the hook off. mtla_profile_events_recorded() returns how many pairs were
 * recorded since the hook was set. Inside stream capture the records become
 * event nodes of the graph (recorded at every replay). */
void mtla_set_profile_events(void* const* events, int32_t n_pairs);
int32_t mtla_profile_events_recorded(void);

#ifdef __cplusplus
}
#endif

#endif /* MTLA_H_ */
