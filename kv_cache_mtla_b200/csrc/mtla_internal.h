// mtla_internal.h -- argument blocks passed from the C ABI to the kernels.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace mtla {

struct Shape {
    int B, H, d_h, d_c, d_r, s, D;
    int gate_mode;          // 0 computed, 1 supplied, 2 unit
    int dtype;              // storage type: kDtypeBF16, kDtypeF32 or kDtypeF16
    int max_slots;
    float scale;            // softmax scale (resolved)
    double log2_rope_base;  // log2 of the RoPE base
    double log2_pe_base;    // log2 of the PE base (10000)
};

struct DecodeArgs {
    Shape sh;
    const void* c_new;
    const void* kr_new;
    const void* q_c;
    const void* q_r;
    const void* w_uk;
    const void* w_uv;
    const float* gate_w;
    const float* gate_b;
    const float* gate_in;
    const int32_t* pos;
    void* cache;
    float* open_slot;
    void* out;
    void* workspace;
    size_t workspace_bytes;
    int* status;            // device status word
};

struct PrefillArgs {
    Shape sh;
    int T;
    int t0;                     // position of the first token (tokens already cached)
    const float* open_slot_in;  // [B, D] the open-slot accumulator after t0 tokens (t0 mod s != 0)
    const void* c;
    const void* kr;
    const void* q_c;
    const void* q_r;
    const void* w_uk;
    const void* w_uv;
    const float* gate_w;
    const float* gate_b;
    const float* gate_in;
    void* out;
    void* cache_out;
    float* open_slot_out;
    void* workspace;
    size_t workspace_bytes;
    int* status;
};

// Chunked prefill (t0 mod s != 0): the open-slot accumulator the chunk starts
// from is copied into `seed_ws` (the last region of the prefill workspace,
// prefill_seed_bytes long) before the scan, which may overwrite the caller's
// open slot; a.open_slot_in then points at the copy. No-op otherwise.
size_t prefill_seed_bytes(const Shape& sh);
cudaError_t prefill_seed(PrefillArgs& a, void* seed_ws, cudaStream_t st);

// Storage types (the values of mtla_dtype).
constexpr int kDtypeBF16 = 0, kDtypeF32 = 1, kDtypeF16 = 2;
inline size_t dtype_bytes(int dtype) { return dtype == kDtypeF32 ? 4 : 2; }

// Scratch layouts (bytes), each region 256-byte aligned.
size_t simt_decode_workspace(const Shape& sh);
size_t simt_prefill_workspace(const Shape& sh, int T);

// Launchers return cudaSuccess or the launch error; they add the number of
// kernels they launched to *launches.
cudaError_t simt_decode(const DecodeArgs& a, int dtype, cudaStream_t st, uint64_t* launches);
cudaError_t simt_prefill(const PrefillArgs& a, int dtype, cudaStream_t st, uint64_t* launches);

// Tensor-core decode (bf16, heads <= 32): shapes it covers, its scratch, launcher.
bool tc_decode_supported(const Shape& sh);
size_t tc_decode_workspace(const Shape& sh);
cudaError_t tc_decode(const DecodeArgs& a, cudaStream_t st, uint64_t* launches);

// Tensor-core decode for many heads (bf16, 32 < heads <= 128, 2-CTA clusters).
bool tc_decode_lh_supported(const Shape& sh);
size_t tc_decode_lh_workspace(const Shape& sh);
cudaError_t tc_decode_lh(const DecodeArgs& a, cudaStream_t st, uint64_t* launches);

// Tensor-core prefill (bf16, d_h = 64, d_c <= 256, slot width <= 320).
bool tc_prefill_supported(const Shape& sh);
size_t tc_prefill_workspace(const Shape& sh, int T);
cudaError_t tc_prefill(const PrefillArgs& a, cudaStream_t st, uint64_t* launches);

// Row pitch (positions) of the per-row statistics [B, H, T] the training
// backward keeps: T rounded up to 4, so that a row is a multiple of 16 bytes
// (a TMA stride).
__host__ __device__ inline int stats_pitch(int T) { return (T + 3) & ~3; }

// The tensor-core prefill from t0 = 0 with what the training backward keeps:
// the merging weights w [B, T] (fp32), per row the log2-domain log-sum-exp
// lse [B, H, stats_pitch(T)] (fp32), O / l obar [B, T, H, d_c] (bf16) and the absorbed
// query qt [B, T, H, D] (bf16) as the score MMAs used it. The partial slots
// stay in the first region of a.workspace (bf16 [B, T, D]).
struct PrefillSave {
    float* w;
    float* lse;
    void* obar;
    void* qt;
};
cudaError_t tc_prefill_save(const PrefillArgs& a, const PrefillSave& sv, cudaStream_t st, uint64_t* launches);

// The masked attention of the training backward on the tensor cores
// (tc_backward.cu; bf16, d_h = 64, d_R = 32, d_c = 128 or 256, scalar gates):
// from the forward's kept rows (qt, lse, obar through delta), dobar and the
// finished slots, the finished-slot parts dqt [B, T, H, D] (fp32, written
// whole) and dF [H, B, n_slots, D] (fp32, per head, written whole).
struct BwdTCInputs {
    const void* qt;        // [B, T, H, D] bf16
    const void* dob;       // [B, T, H, d_c] bf16
    const void* slots;     // [B, n_slots, D] bf16 (the forward's cache rows)
    const void* dout;      // [B, T, H, d_h] bf16
    const void* u;         // [B, n_slots, H d_h] bf16: U_j[h] = W_UV[h] F_j[0:d_c]
    const float* lse;      // [B, H, stats_pitch(T)]
    const float* delta;    // [B, H, stats_pitch(T)]
    float* dqt;
    float* dF;
    int* status;
};
bool tc_backward_supported(const Shape& sh);
// The weight gradients of the training backward on the tensor cores
// (tc_wgrad.cu; bf16 rows, d_h = 64, d_c = 128 or 256), per chunk of token rows:
//   part_k[chunk][h][r][c] = sum_m qc[m, h, r] g[m, h, c]
//   part_v[chunk][h][r][c] = sum_m dout[m, h, r] obar[m, h, c]
// over the chunk's rows m of M = B*T (qc, dout [M, H, d_h]; g, obar [M, H, d_c]);
// adding the n_chunks parts in order gives dW_UK and dW_UV. tc_weight_chunks:
// the chunk count for M rows, at most max_chunks.
int tc_weight_chunks(const Shape& sh, int M, int max_chunks);
cudaError_t tc_weight_parts(const Shape& sh, int M, const void* qc, const void* g, const void* dout,
                            const void* obar, float* part_k, float* part_v, int n_chunks, int* status,
                            cudaStream_t st);
cudaError_t tc_backward_attention(const Shape& sh, int T, const BwdTCInputs& in, cudaStream_t st,
                                  uint64_t* launches);

// y[M, N] = x[M, K] . w[N, K]^T, bf16 in and out, fp32 accumulation (gemm.cu).
// Rows ldx / ldw / ldy elements apart (ldx, ldw multiples of 8).
cudaError_t gemm_bf16(const void* x, int ldx, const void* w, int ldw, void* y, int ldy, int M, int N, int K,
                      int* status, cudaStream_t st, uint64_t* launches);

// Training backward of the parallel forward from position 0 (backward.cu),
// scalar gate modes, fp32 gradients. `a` carries the forward's inputs (t0 0,
// no cache or open slot: the scan writes a scratch copy in the workspace).
struct BackwardGrads {
    const void* dout;      // [B,T,H,d_h] storage type
    float* dc;             // [B,T,d_c]
    float* dkr;            // [B,T,d_R]
    float* dq_c;           // [B,T,H,d_h]
    float* dq_r;           // [B,T,H,d_R]
    float* dw_uk;          // [H,d_h,d_c]
    float* dw_uv;          // [H,d_h,d_c]
    float* dgate_w;        // [s,d_c] (computed gate)
    float* dgate_b;        // [s]
    float* dgate_in;       // [B,T] (supplied gate)
};
size_t prefill_backward_workspace(const Shape& sh, int T, int dtype);
// The training pair (bf16 at the tensor-core widths, scalar gates, t0 = 0):
// the forward keeping what the backward needs in `saved`, and the backward
// from it (no forward recompute).
bool prefill_train_supported(const Shape& sh);
size_t prefill_train_saved_bytes(const Shape& sh, int T);
size_t prefill_backward_saved_workspace(const Shape& sh, int T);
cudaError_t prefill_train(const PrefillArgs& a, void* saved, cudaStream_t st, uint64_t* launches);
cudaError_t prefill_backward_saved(const PrefillArgs& a, const BackwardGrads& g, const void* saved, cudaStream_t st,
                                   uint64_t* launches);
cudaError_t prefill_backward(const PrefillArgs& a, const BackwardGrads& g, int dtype, cudaStream_t st,
                             uint64_t* launches);

// A batch of such products in one launch (gemm.cu): product i reads
// x.p + i * x.batch_stride and w.p + i * w.batch_stride (elements; rows ld
// apart, ld and batch_stride multiples of 8) and writes y + i * y_batch
// (bf16, or float when y_f32).
struct GemmOperand {
    const void* p;
    int ld;
    size_t batch_stride;
};
cudaError_t gemm_batched(const GemmOperand& x, const GemmOperand& w, void* y, int ldy, size_t y_batch, bool y_f32,
                         int M, int N, int K, int batch, int* status, cudaStream_t st, uint64_t* launches);

// Test hook (wait_probe.cu): one CTA whose bounded wait runs out after
// limit_ns; `scratch` is 2 KB of device memory its TMA load reads.
cudaError_t wait_probe(uint64_t limit_ns, void* scratch, int* status, cudaStream_t st, uint64_t* launches);

// Beam-search reorder of the slot cache and open slots (cache_ops.cu).
cudaError_t reorder_cache(const Shape& sh, size_t elem_bytes, const int32_t* src, const int32_t* n_tokens,
                          const void* cache_in, const float* open_in, void* cache_out, float* open_out,
                          int* status, cudaStream_t st, uint64_t* launches);

// Driver entry point cuTensorMapEncodeTiled (NULL if unavailable), looked up once.
void* tensor_map_encoder();
// Streaming multiprocessors of the current device (cached per device).
int sm_count();

// Record which CUDA step failed (read back by mtla_last_error_detail); returns e.
cudaError_t note_error(const char* where, cudaError_t e);

// Profile hook: record the next event pair around the main attention kernel.
void profile_begin(cudaStream_t st);
void profile_end(cudaStream_t st);

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace mtla
