/*
 * mimo_attn.h -- C ABI of the B200 (sm_100a) attention forward for the
 * MiMo-V2 text decoder: the sliding-window layer with a learnable per-head
 * sink and the global causal layer.
 *
 * The operation (miles PR #3648 "add MiMo-V2.6-Flash-RL support", Motivation
 * and Design Notes; miles docs "MiMo-V2.6-Flash", section 1 Model Introduction
 * and section 5.4 Notable quirks; Megatron-LM issue #2976, Architecture
 * Analysis; Megatron-Bridge API doc "mimo_v2_flash_bridge", module summary):
 *
 *   For every packed sequence b (tokens cu_seqlens[b] .. cu_seqlens[b+1]-1),
 *   local position p and query head h, with KV head g = h / (Hq / Hkv):
 *     q~ = rope(q[t, h], p), k~_j = rope(k[s_b + j, g], j)   (first rope_dims
 *          dims, rotate-half pairs (i, i + rope_dims/2), theta_i =
 *          rope_base^(-2i/rope_dims), positions restart at 0 per sequence)
 *     keys j with 0 <= j <= p and (global layer, or p - j <= window)
 *     s_j = q~ . k~_j / sqrt(head_dim_qk)
 *     lse = ln( sum_j exp(s_j) + exp(sink[h]) )   (sink term only if sink != NULL)
 *     out[t, h] = sum_j exp(s_j - lse) * v_scale * v[s_b + j, g]
 *   window = 128 gives the query plus 128 previous keys, 129 in total (miles
 *   docs section 5.4); window = 127 gives the 128-key HF variant.
 *
 * Conventions for every entry point:
 *   - Device pointers are caller-owned CUDA global memory on the current
 *     device; host pointers are caller-owned host memory.  The library keeps
 *     no caller pointer after a call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Kernels run asynchronously on it; only the entry points that
 *     say so synchronise.
 *   - Return values are mimo_status codes.  Argument checks happen before any
 *     CUDA call, so a rejected call has no side effect.
 *   - All tensors are dense, row-major and contiguous in THD layout
 *     (tokens, heads, dims).  Every device pointer must be 16-byte aligned,
 *     and the attention output `out` of the forward and KV-cache entry
 *     points 32-byte aligned (its rows are written with 32-byte stores);
 *     otherwise MIMO_ERR_INVALID_ARG.
 */
#ifndef MIMO_ATTN_H_
#define MIMO_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MIMO_API __attribute__((visibility("default")))
#else
#define MIMO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MIMO_LAYER_SWA = 0,    /* sliding window (`window` previous keys) with optional sink */
  MIMO_LAYER_GLOBAL = 1  /* causal over the whole sequence, no sink */
} mimo_layer_kind;

typedef enum {
  MIMO_OK = 0,
  MIMO_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer, inconsistent dims */
  MIMO_ERR_UNSUPPORTED = 2, /* valid for the method but not built: head dims other than 192/128, rope_dims != 64 */
  MIMO_ERR_CUDA = 3,        /* a CUDA runtime/driver call or kernel launch failed */
  MIMO_ERR_TIMEOUT = 4,     /* a kernel's bounded wait ran out (reported by mimo_attn_check) */
  MIMO_ERR_RANGE = 5,       /* a rotated Q/K value exceeded the FP16 range (|x| > 65504) */
  MIMO_ERR_BAD_SEQLENS = 6, /* the kernel found cu_seqlens inconsistent with dims (reported by mimo_attn_check) */
  MIMO_ERR_SCRATCH_LIMIT = 7 /* mimo_attn_fwd_noalloc: T * Hkv * 128 bytes exceed its fixed scratch */
} mimo_status;

/* Shapes.  Supported: head_dim_qk = 192, head_dim_v = 128,
 * num_q_heads % num_kv_heads == 0, num_seqs >= 1, total_tokens >= 0,
 * max_seqlen >= every sequence length (it sizes the launch grid). */
typedef struct {
  int32_t num_seqs;
  int32_t total_tokens;
  int32_t max_seqlen;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim_qk;
  int32_t head_dim_v;
} mimo_attn_dims;

/*
 * Attention forward on device buffers.
 *   q          bf16 [T, Hq, 192]          (device)
 *   k          bf16 [T, Hkv, 192]         (device)
 *   v          bf16 [T, Hkv, 128]         (device)
 *   sink       fp32 [Hq] or NULL          (device) per-query-head sink logit in
 *              score units (not multiplied by the softmax scale); it joins the
 *              softmax denominator and carries no value.  SWA only: a non-NULL
 *              sink with MIMO_LAYER_GLOBAL is MIMO_ERR_INVALID_ARG.
 *   cu_seqlens int32 [num_seqs + 1]       (device) cu[0] = 0, non-decreasing,
 *              cu[num_seqs] = T, lengths <= max_seqlen.  The host cannot read it
 *              without a sync, so a violation is detected by the kernel, which
 *              skips that sequence and records MIMO_ERR_BAD_SEQLENS for
 *              mimo_attn_check.  Empty sequences are allowed.
 *   layer_kind MIMO_LAYER_SWA or MIMO_LAYER_GLOBAL
 *   window     SWA: keys j with p - window <= j <= p (window >= 0); ignored for GLOBAL
 *   rope_base  RoPE base (1e4 for SWA, 1e7 for global in MiMo-V2.6), > 0
 *   rope_dims  must be 64 (the first 64 of the 192 Q/K dims are rotated)
 *   v_scale    factor applied to V before P.V (0.707 in the model)
 *   out        bf16 [T, Hq, 128]          (device) every row of every head is written
 *   lse        fp32 [Hq, T]               (device) natural-log normaliser, including
 *              the sink term
 * Range: rotated Q/K rope dims enter the tensor cores as FP16 (the pass-through
 * dims stay BF16).  A rotated value is x_i cos(a) - x_{i+32} sin(a) (or its
 * partner), at most sqrt(2) max(|x_i|, |x_{i+32}|) in magnitude, so inputs
 * whose first 64 dims stay within 65504 / sqrt(2) = 46318 in magnitude never
 * overflow.  Larger inputs may, depending on the position; a rotated value
 * above 65504 in magnitude (the largest finite FP16) is recorded as
 * MIMO_ERR_RANGE for mimo_attn_check and that call's output is not valid.
 * Scratch: when a two-head kernel that reads K's rope dims pre-rotated runs
 * (the pipelined kernel, and the window kernel where it is chosen, see
 * mimo_attn_set_kernel), the call rotates them once into T * Hkv * 128 bytes
 * of transient device scratch from a library-owned stream-ordered pool
 * (cudaMallocFromPoolAsync on `stream`, cudaFreeAsync on the same stream).
 * The pool's release threshold is 0: later calls on the stream reuse the
 * memory without synchronizing, and the next synchronization returns it to
 * the device, so nothing persists between synchronized calls.  Does not
 * synchronise.
 */
MIMO_API int mimo_attn_fwd(const void* q, const void* k, const void* v, const float* sink,
                  const int32_t* cu_seqlens, const mimo_attn_dims* dims, int layer_kind,
                  int window, double rope_base, int rope_dims, float v_scale, void* out,
                  float* lse, void* stream);

/*
 * Bytes of device workspace mimo_attn_fwd_host needs for these dims
 * (q, k, v, sink, cu_seqlens, out and lse, each 256-byte aligned).
 * Returns 0 for invalid dims.
 */
MIMO_API size_t mimo_attn_host_workspace_size(const mimo_attn_dims* dims, int has_sink);

/*
 * End-to-end forward from HOST buffers (same layouts and meaning as
 * mimo_attn_fwd; q/k/v/out are bf16 bit patterns in host memory, pinned for
 * asynchronous copies).  The caller passes a device workspace of at least
 * mimo_attn_host_workspace_size bytes, 256-byte aligned.  The call copies the
 * inputs host->device on `stream`, runs the forward, copies out and lse
 * device->host and synchronises the stream before returning, so the host
 * buffers hold the result on return.  Takes the same transient scratch as
 * mimo_attn_fwd.
 */
MIMO_API int mimo_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                       const float* sink_host, const int32_t* cu_seqlens_host,
                       const mimo_attn_dims* dims, int layer_kind, int window, double rope_base,
                       int rope_dims, float v_scale, void* out_host, float* lse_host,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronises `stream`, then reads and clears the library's device error
 * word for the current device: MIMO_ERR_TIMEOUT, MIMO_ERR_RANGE or
 * MIMO_ERR_BAD_SEQLENS if a kernel recorded one since the last check (the
 * lowest-numbered one is returned), MIMO_ERR_CUDA if the sync failed, else
 * MIMO_OK.
 */
MIMO_API int mimo_attn_check(void* stream);

/*
 * Failure-detection self test: launches one CTA that waits on a shared-memory
 * barrier nothing ever arrives on, with a wait limit of `limit_ns`
 * nanoseconds (1e3 .. 1e10).  The wait gives up, records MIMO_ERR_TIMEOUT
 * and the kernel returns; this call synchronises `stream` and returns what
 * mimo_attn_check returns (MIMO_ERR_TIMEOUT when the bounded wait works).
 */
MIMO_API int mimo_attn_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/* Static description of a status code (never NULL). */
MIMO_API const char* mimo_attn_status_string(int status);

/*
 * Same operation, arguments and results as mimo_attn_fwd, for callers that
 * cannot allocate device memory during the call -- for example a framework
 * that has already reserved the device for its own caching allocator, or a
 * serving loop that forbids allocation on its hot path.  (This entry point
 * has no counterpart in the pages that describe the layer; it only changes
 * where the scratch lives.)
 *   - The rotated-K scratch (T * Hkv * 128 bytes) lives in a fixed device
 *     array inside the library, mimo_attn_noalloc_scratch_bytes() bytes
 *     (32 MiB), that every GPU which loads the library holds until the
 *     process exits.  Larger problems are rejected with
 *     MIMO_ERR_SCRATCH_LIMIT before anything is launched.
 *   - The call makes no cudaMalloc/cudaFree or pool allocation.
 *   - The first call on a device, with that device current, looks up the
 *     array's device address and sets kernel attributes; make that first
 *     call before any stream capture.
 *   - Every call uses the same array, so calls that overlap on the GPU (on
 *     different streams, or on one stream without ordering) race; calls on
 *     one stream are ordered and safe.  Each call rewrites every scratch row
 *     it reads, so nothing needs clearing between calls.
 */
MIMO_API int mimo_attn_fwd_noalloc(const void* q, const void* k, const void* v, const float* sink,
                                   const int32_t* cu_seqlens, const mimo_attn_dims* dims, int layer_kind,
                                   int window, double rope_base, int rope_dims, float v_scale, void* out,
                                   float* lse, void* stream);

/* Size in bytes of the fixed scratch array mimo_attn_fwd_noalloc uses. */
MIMO_API size_t mimo_attn_noalloc_scratch_bytes(void);

/* Kernel selection for mimo_attn_fwd and mimo_attn_fwd_noalloc (process-wide;
 * default AUTO).
 *   MIMO_KERNEL_AUTO       for a sliding-window call with 0 <= window <= 128:
 *                          WINDOW_PACKED when Hq/Hkv is 4 or 8, else WINDOW when
 *                          Hq/Hkv is even; PIPELINED when Hq/Hkv is even otherwise
 *                          (the global layer, longer windows); else SIMPLE
 *   MIMO_KERNEL_SIMPLE     one CTA per (128-query tile, head), every step serialised;
 *                          any Hq/Hkv ratio (the cross-check path)
 *   MIMO_KERNEL_PIPELINED  warp-specialised persistent kernel, two heads per CTA,
 *                          online softmax over any number of key tiles;
 *                          Hq/Hkv must be even
 *   MIMO_KERNEL_WINDOW     the same roles, specialised for sliding windows of at
 *                          most 128 keys: both key tiles of a query tile are
 *                          scored first and softmaxed in one pass; Hq/Hkv must be
 *                          even and the call a sliding-window one with
 *                          window <= 128
 *   MIMO_KERNEL_WINDOW_PACKED  sliding windows of at most 128 keys with the
 *                          Hq/Hkv query heads of a KV group packed into each
 *                          128-row tile (128/G tokens x G heads): a tile spans
 *                          128/G + 128 keys instead of 256, K/V stream through
 *                          a ring of 16-key blocks, and RoPE of both Q and K is
 *                          applied in shared memory (no pre-pass, no scratch);
 *                          Hq/Hkv must be 4 or 8 and the call a sliding-window
 *                          one with window <= 128
 * A forced choice whose condition fails makes the call return
 * MIMO_ERR_UNSUPPORTED.  Returns MIMO_ERR_INVALID_ARG for any other value.
 * All kernels compute the same operation; they differ only in the order of
 * floating-point rounding (where the softmax maximum is taken and when it is
 * applied), well inside the stated tolerances. */
typedef enum {
  MIMO_KERNEL_AUTO = 0,
  MIMO_KERNEL_SIMPLE = 1,
  MIMO_KERNEL_PIPELINED = 2,
  MIMO_KERNEL_WINDOW = 3,
  MIMO_KERNEL_WINDOW_PACKED = 4
} mimo_kernel_choice;
MIMO_API int mimo_attn_set_kernel(int choice);

/*
 * Kernel timing for measurement tools.  After mimo_attn_profile_start, every
 * forward that runs a persistent kernel (window, packed window or pipelined)
 * records a CUDA event pair (events owned by the library) around that kernel
 * on the call's stream.
 * mimo_attn_profile_stop ends recording, waits for the recorded events, and
 * returns how many attention-kernel launches were recorded and their summed
 * duration in milliseconds (the K RoPE pre-pass is excluded).  Process-wide.
 */
MIMO_API int mimo_attn_profile_start(void);
MIMO_API int mimo_attn_profile_stop(int* launches, double* total_ms);
/*
 * Records the event pair around every stride-th attention-kernel launch only
 * (stride >= 1; 1, the default, records every launch), so that the events can
 * sit inside a timed region with little effect on it.  The count restarts at
 * mimo_attn_profile_start.  MIMO_ERR_INVALID_ARG for stride < 1.
 */
MIMO_API int mimo_attn_profile_set_stride(int stride);

/*
 * Attention of new query tokens against a KV cache with page size 1: decode,
 * speculative-draft verification and chunked prefill for the same two layer
 * kinds (miles docs "MiMo-V2.6-Flash" section 3.2 SGLang: page size 1,
 * chunked prefill of up to 49152 tokens, 8 speculative draft tokens).
 *
 *   q           bf16 [total_q, Hq, 192]   (device) the new tokens of every
 *               sequence, THD-packed by cu_q
 *   k_cache     bf16 [cache_rows, Hkv, 192] (device) K as mimo_attn_fwd takes it
 *               (not rotated); v_cache bf16 [cache_rows, Hkv, 128]
 *   kv_indices  int32 [total_kv]          (device) cache row of every key:
 *               sequence b's keys, in position order, are entries
 *               kv_indptr[b] .. kv_indptr[b+1]-1; the new tokens' K and V
 *               are already in the cache (the last q_len_b entries)
 *   kv_indptr   int32 [num_seqs + 1]      (device) kv_indptr[0] = 0, nondecreasing
 *   cu_q        int32 [num_seqs + 1]      (device) cu_q[0] = 0, cu_q[B] = total_q
 *   sink, layer_kind, window, rope_base, rope_dims, v_scale: as mimo_attn_fwd
 *   out         bf16 [total_q, Hq, 128]   (device); lse fp32 [Hq, total_q] (device)
 * Query i of sequence b (1 <= q_len_b <= kv_len_b) sits at position
 * kv_len_b - q_len_b + i and attends the keys mimo_attn_fwd would give it, so
 * out and lse equal the forward's rows for those positions.  Chunked
 * prefill: the max_q_len * Hq/Hkv query rows of a KV head may exceed 128, up
 * to 2^20 (else MIMO_ERR_UNSUPPORTED); both kernels run them in 128-row
 * tiles; every q_len_b,
 * kv_len_b must be at most max_q_len, max_kv_len.  Inconsistent cu_q /
 * kv_indptr, q_len_b > kv_len_b and cache rows outside [0, cache_rows) are
 * recorded as MIMO_ERR_BAD_SEQLENS for mimo_attn_check (such rows are left
 * unwritten; an index outside the cache is never dereferenced).  Scratch: a
 * partial result per key split, total_q * Hq * splits * 520 bytes (plus 512
 * bytes) from the library's stream-ordered pool; with one split (the keys a
 * row sees fit one split: always on sliding-window layers) the tensor-core
 * kernel writes out and lse directly and the partials go unused.  Does not
 * synchronise.  (The pages give no
 * interface; this one mirrors mimo_attn_fwd.)
 */
typedef struct {
  int32_t num_seqs, total_q, total_kv, cache_rows, max_q_len, max_kv_len;
  int32_t num_q_heads, num_kv_heads, head_dim_qk, head_dim_v;
} mimo_decode_dims;
MIMO_API int mimo_attn_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* kv_indices,
                              const int32_t* kv_indptr, const int32_t* cu_q, const float* sink,
                              const mimo_decode_dims* dims, int layer_kind, int window, double rope_base,
                              int rope_dims, float v_scale, void* out, float* lse, void* stream);

/*
 * Selects the kernel mimo_attn_decode launches (process-wide; default AUTO):
 *   MIMO_DECODE_AUTO        the tensor-core kernel
 *   MIMO_DECODE_CUDA_CORES  FP32 on the CUDA cores, 32 keys per step (the
 *                           cross-check path)
 *   MIMO_DECODE_TENSOR      tcgen05: a 128-row tile of the query rows of one
 *                           KV head as the M = 128 operand, K/V gathered by
 *                           index into shared memory 64 keys per step, S and
 *                           O in TMEM
 * Both cut the query rows of a KV head into 128-row tiles (chunked prefill).
 * Both compute the same operation; they differ in rounding order (the
 * tensor-core kernel rounds P to BF16 and the rotated dims of Q and K to FP16,
 * as the forward does).  Returns MIMO_ERR_INVALID_ARG for any other value.
 */
typedef enum { MIMO_DECODE_AUTO = 0, MIMO_DECODE_CUDA_CORES = 1, MIMO_DECODE_TENSOR = 2 } mimo_decode_choice;
MIMO_API int mimo_attn_set_decode_kernel(int choice);

/* Kernel of mimo_attn_bwd: 0 automatic (tensor cores), 1 FP32 CUDA cores (the cross-check: FP32
 * throughout, about 4x slower on the sliding layer at 4096 tokens), 2 tensor cores (tcgen05, BF16
 * operands: the rotated Q / K dims, P and dS each rounded once to BF16).  Process-wide. */
MIMO_API int mimo_attn_set_bwd_kernel(int choice);

/*
 * Backward of mimo_attn_fwd (miles PR #3648 trains this layer; the LSE with the
 * sink included is the convention it needs).  Inputs as mimo_attn_fwd, plus the
 * forward's out (bf16 [T, Hq, 128]) and lse (fp32 [Hq, T]), dout = dL/dout
 * (bf16 [T, Hq, 128]) and dlse = dL/dlse (fp32 [Hq, T], NULL = 0), all device.
 * Outputs (device, fp32, overwritten): dq [T, Hq, 192], dk [T, Hkv, 192],
 * dv [T, Hkv, 128] and dsink [Hq] (required iff sink is given).  dL/ds_j =
 * P_j (dout . v_scale v_j - D + dlse) with D = dout . out; the rotation of the
 * first 64 dims is taken back by its transpose.  By default on the tensor
 * cores, or in FP32 on the CUDA cores (mimo_attn_set_bwd_kernel); both
 * accumulate with atomics, so the result is not bit-reproducible run to run.
 * Scratch: Hq * T * 4 bytes from the library's pool.  Does not synchronise.
 */
MIMO_API int mimo_attn_bwd(const void* q, const void* k, const void* v, const float* sink,
                           const int32_t* cu_seqlens, const mimo_attn_dims* dims, int layer_kind,
                           int window, double rope_base, int rope_dims, float v_scale, const void* out,
                           const float* lse, const void* dout, const float* dlse, float* dq, float* dk,
                           float* dv, float* dsink, void* stream);

/*
 * FP8 blockwise dequant of a weight matrix (Megatron-Bridge API doc
 * "mimo_v2_flash_bridge", _dequant_fp8_blockwise: out = fp8 value times
 * scale_inv; miles docs section 3.1: each kv-head shard of the fused qkv_proj
 * has its own block scales).  codes: E4M3 bytes [rows, cols] (device, 16-byte
 * aligned, cols a multiple of 16); scale_inv: fp32 [ceil(rows / block_rows),
 * ceil(cols / block_cols)] (device); out: bf16 [rows, cols] (device), each the
 * round-to-nearest-even of the exact product.  The pages do not give the block
 * size (128 x 128 is the usual one).  cols not a multiple of 16 or above
 * 2^31 - 1: MIMO_ERR_UNSUPPORTED; negative sizes, block sizes below 1, null
 * or misaligned pointers: MIMO_ERR_INVALID_ARG; no rows or no columns: nothing
 * to do.  Does not synchronise.
 */
MIMO_API int mimo_fp8_dequant_blockwise(const void* codes, const float* scale_inv, int64_t rows, int64_t cols,
                                        int block_rows, int block_cols, void* out, void* stream);

/*
 * Split of the kv-head-interleaved fused QKV output (miles docs section 1 and
 * 3.1) into the q, k, v this library's attention takes: fused bf16
 * [T, Hkv * (Hq/Hkv * 192 + 192 + 128)], where KV group g holds its query heads,
 * then its K head, then its V head; q bf16 [T, Hq, 192], k [T, Hkv, 192],
 * v [T, Hkv, 128].  All device, 16-byte aligned.  Does not synchronise.
 */
MIMO_API int mimo_qkv_split(const void* fused, int64_t tokens, int num_q_heads, int num_kv_heads, void* q,
                            void* k, void* v, void* stream);

/*
 * Output projection linear_proj of the attention (miles PR #3648, commit
 * message on MiMoV2SelfAttention: the projection is built for the 128-dim V
 * heads): y = x . w^T with x bf16 [tokens, in_features] (the attention output
 * [T, Hq, 128] viewed as [T, Hq * 128]), w bf16 [out_features, in_features]
 * (a Linear weight, no bias), y bf16 [tokens, out_features]; FP32
 * accumulation, one rounding of each output to BF16.  A plain GEMM: it runs
 * on cuBLAS, loaded at the first call (MIMO_ERR_CUDA if it cannot be loaded).
 * Features must be multiples of 8 and at most 2^31 - 1 (else
 * MIMO_ERR_UNSUPPORTED).  Device pointers, 16-byte aligned.  Does not
 * synchronise.
 */
MIMO_API int mimo_linear_proj(const void* x, const void* w, int64_t tokens, int64_t in_features,
                              int64_t out_features, void* y, void* stream);

/*
 * MoE routing (miles docs section 1: 256 routed experts, top-8 sigmoid routing
 * with a fixed score-correction bias; router logits in FP32 per the SGLang
 * cookbook section 2).  logits fp32 [T, E], bias fp32 [E] (E a multiple of 32,
 * at most 256); ids int32 [T, top_k] in descending score + bias (ties to the
 * lower expert), weights fp32 [T, top_k]: the chosen experts' sigmoid scores,
 * normalised to sum to one when normalize != 0.  The choice is taken on FP32
 * keys fp32(sigmoid) + bias.  The pages do not say where the bias enters or
 * whether the weights are normalised: this is the plain reading.  Device
 * pointers.  Does not synchronise.
 */
MIMO_API int mimo_moe_route(const float* logits, const float* bias, int64_t tokens, int num_experts, int top_k,
                            int normalize, int32_t* ids, float* weights, void* stream);

/* ABI version: (major << 16) | minor. */
MIMO_API int mimo_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MIMO_ATTN_H_ */
