/*
 * mea.h — C ABI of libmea, exact memory-efficient attention for B200 (sm_100a).
 *
 * What the library computes (all entry points):
 *
 *     out = softmax(Q K^T * scale + bias) V,   lse = log(sum(exp(Q K^T * scale + bias)))
 *
 * row by row, over a packed batch of variable-length segments that never attend to one
 * another (the block-diagonal mask of "Cómo construir transformadores con memoria eficiente
 * con xFormers…", section 4 "packed variable-length batch", and technique 1 "Packed Sequences &
 * BlockDiagonalMask" of "How to Build Memory-Efficient Transformers with xFormers…"), optionally
 * under an implicit lower-triangular causal mask (technique 5 of the latter), with grouped-query
 * attention (the G key/value heads of "group query attention gqa", each shared by R = Hq/Hkv
 * query heads; R = Hq is MQA) and an optional per-head ALiBi additive bias (technique 3).
 * The score matrix is computed tile by tile with an online softmax and never reaches global
 * memory (the blockwise engine of "大模型推理加速终极指南", section 1).
 *
 * Notation and layouts (row-major, contiguous, 16-byte aligned base pointers):
 *   T_q, T_k   total packed query / key tokens;   Hq, Hkv   query / key-value heads; D head_dim
 *   q   [T_q, Hq,  D]  fp16 or bf16          out [T_q, Hq, D] same dtype as q
 *   k,v [T_k, Hkv, D]  same dtype            lse [Hq, T_q] fp32 (natural log), may be NULL
 *   cu_seqlens_q / cu_seqlens_k: int32 [n_seqs+1] prefix sums of segment lengths, in DEVICE
 *   memory; segment s owns query rows [cu_q[s], cu_q[s+1]) and key rows [cu_k[s], cu_k[s+1]).
 *   Query head h reads key/value head h / R (the repeat_interleave grouping).
 *   D: a multiple of 8 from 8 to 256 (mea_forward and the decode entry points), from 8 to 128
 *   (mea_backward); a multiple of 16 from 16 to 128 with e4m3 inputs (mea_forward_fp8).
 *
 * Per segment s with L_q = cu_q[s+1]-cu_q[s], L_k = cu_k[s+1]-cu_k[s], query row i sits at key
 * position p_i = i + L_k - L_q (bottom-right alignment: the last query sees the last key).
 *   MEA_MASK_NONE:   row i attends to keys j in [0, L_k)
 *   MEA_MASK_CAUSAL: row i attends to keys j in [0, min(p_i, L_k-1)]
 *   ALiBi (alibi_slopes != NULL): bias(i, j) = -slope[h] * |p_i - j|, added after scaling.
 * A row with no admissible key (L_k = 0, or causal with p_i < 0) gets out = 0, lse = -inf.
 *
 * Ownership: the caller owns and allocates every buffer; the library never allocates device
 * memory in these calls. Errors: arguments are validated before anything is launched and a
 * negative mea_status is returned with nothing launched; MEA_ERR_CUDA reports a failed launch.
 * Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream) and never
 * synchronise the host.
 */
#ifndef MEA_H_
#define MEA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MEA_OK = 0,
  MEA_ERR_NULL = -1,          /* a required pointer is NULL                                   */
  MEA_ERR_SHAPE = -2,         /* negative/zero sizes, total or max_seqlen out of range        */
  MEA_ERR_HEADS = -3,         /* n_heads_q % n_heads_kv != 0, or a head count < 1             */
  MEA_ERR_HEAD_DIM = -4,      /* head_dim outside the entry point's set (see Notation)        */
  MEA_ERR_DTYPE = -5,         /* dtype not MEA_F16 / MEA_BF16                                 */
  MEA_ERR_ALIGN = -6,         /* a tensor base pointer is not 16-byte aligned (TMA needs it)  */
  MEA_ERR_MASK = -7,          /* mask_kind not a mea_mask value                               */
  MEA_ERR_WORKSPACE = -8,     /* workspace NULL or smaller than the size function says        */
  MEA_ERR_CUDA = -9,          /* a CUDA runtime/driver call or a launch failed                */
  MEA_ERR_DEVICE_TIMEOUT = -10, /* a kernel gave up on a bounded wait (see mea_device_error)  */
  MEA_ERR_DEVICE = -11,       /* the current device is not an sm_100 part                     */
  MEA_ERR_SCALE = -12,        /* scale is not finite                                           */
  MEA_ERR_SCRATCH_LIMIT = -13 /* the problem needs more scratch than the fixed static array    */
} mea_status;

typedef enum { MEA_F16 = 0, MEA_BF16 = 1 } mea_dtype;

typedef enum {
  MEA_MASK_NONE = 0,   /* block-diagonal only                                   */
  MEA_MASK_CAUSAL = 1  /* block-diagonal plus bottom-right lower-triangular    */
} mea_mask;

/*
 * mea_forward — packed variable-length attention forward (prefill / training forward).
 *
 * Computes out and lse as defined above for every (segment, query row, query head).
 *   n_seqs        number of segments (>= 1); cu_seqlens_* hold n_seqs+1 entries each.
 *   total_q/k     T_q = cu_seqlens_q[n_seqs], T_k = cu_seqlens_k[n_seqs] (given by the caller
 *                 so that the host never reads device memory; they size the TMA views).
 *   max_seqlen_q  the largest L_q, or an upper bound on it. It only sizes the grid: every CTA
 *                 reads the true lengths from cu_seqlens_q, so a smaller value still produces
 *                 every row (more slowly, on fewer CTAs); 0 is treated as 1.
 *   scale         multiplies Q K^T before the bias (1/sqrt(D) is the usual choice).
 *   alibi_slopes  NULL, or DEVICE fp32 [n_heads_q] slopes (2^(-8(h+1)/Hq) is the usual choice).
 *   dtype         mea_dtype of q, k, v and out.
 * Returns MEA_OK or a negative mea_status. Segments with L_q = 0 produce nothing.
 * MEA_ERR_HEADS also covers head counts so large that the kernel's integer head-block-to-group
 * mapping could round wrongly ((H/P - 1) * (R/P - 1) >= 2^32, with R = n_heads_q / n_heads_kv
 * and P its largest power-of-two divisor up to 128); no realistic head count reaches it.
 * Performance: the work items (a pair of query tiles of one segment and one block of query heads)
 * are balanced over the GPU's SMs heaviest first; with up to 256 segments every CTA ranks them
 * by length on chip, longer lists are walked in segment order (still complete, less balanced).
 */
int mea_forward(const void* q, const void* k, const void* v, void* out, float* lse,
                const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int n_seqs,
                int total_q, int total_k, int max_seqlen_q, int n_heads_q, int n_heads_kv,
                int head_dim, float scale, int mask_kind, const float* alibi_slopes,
                int dtype, void* stream);

/*
 * mea_decode_workspace_size — bytes of device workspace mea_decode_splitkv needs.
 *   split_keys is the number of keys per split-KV chunk (0 = the library's choice for these
 *   sizes; pass the same value to mea_decode_splitkv). Returns 0 for invalid arguments.
 *   The workspace holds, for every chunk, one partial output row and one partial lse per query
 *   head of the chunk's group, in fp32.
 */
size_t mea_decode_workspace_size(int n_seqs, int total_k, int n_heads_q, int n_heads_kv,
                                 int head_dim, int split_keys);

/*
 * mea_decode_splitkv — one query token per request against a packed KV cache, split along the
 * keys (the split-K attention of "大模型推理加速终极指南", section 1) and merged by
 * log-sum-exp.
 *   q    [n_seqs, n_heads_q, D]   one token per request      out [n_seqs, n_heads_q, D]
 *   k,v  [total_k, n_heads_kv, D] packed, request b owns rows [cu_k[b], cu_k[b+1])
 *   lse  [n_heads_q, n_seqs] fp32 or NULL
 * The single query is the newest token of its request (p = L_k - 1), so it attends to all L_k
 * keys; mask_kind is accepted for symmetry and CAUSAL equals NONE here.
 *   workspace/workspace_bytes: caller-owned device scratch of at least
 *   mea_decode_workspace_size(...) bytes, 256-byte aligned; its contents need no initialisation.
 *   split_keys: keys per chunk, a multiple of 64 (0 = library's choice: the largest power of
 *   two from 128 to 2048 that leaves about half a (chunk, head block) work item per SM or more).
 * Two kernels are launched on `stream`: the split kernel and the log-sum-exp merge kernel.
 */
int mea_decode_splitkv(const void* q, const void* k, const void* v, void* out, float* lse,
                       const int32_t* cu_seqlens_k, int n_seqs, int total_k, int max_seqlen_k,
                       int n_heads_q, int n_heads_kv, int head_dim, float scale, int mask_kind,
                       const float* alibi_slopes, int dtype, void* workspace,
                       size_t workspace_bytes, int split_keys, void* stream);

/*
 * mea_decode_splitkv_noalloc — mea_decode_splitkv without a caller-provided workspace.
 *
 * The pages have no counterpart to this entry point: it exists for callers of the library, not
 * for the method. Some callers cannot call cudaMalloc at all. For example, a plugin running
 * inside a host runtime that has already reserved the device memory it will ever use and hands
 * its plugins only their input and output tensors; or a latency-bound serving loop that must not
 * pay for an allocation (and the device synchronisation an allocation can imply) on every decode
 * step. This variant takes the same arguments as mea_decode_splitkv minus the workspace, and
 * keeps the split-KV partials in a fixed array of MEA_DECODE_NOALLOC_SCRATCH_BYTES bytes that is
 * part of the library itself (a file-scope __device__ array). Each GPU that loads the library
 * holds that array until the process exits.
 *
 *   - It allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *   - The caller still provides q, k, v, out and (optionally) lse, as for mea_decode_splitkv.
 *   - split_keys = 0 starts from the library's chunk size and doubles it until the partials fit
 *     in the array; an explicit split_keys is used as given. If the partials
 *     ((ceil(total_k / chunk) + n_seqs) * n_heads_q * (head_dim + 1) floats, each region rounded
 *     up to 256 bytes) cannot fit, the call returns MEA_ERR_SCRATCH_LIMIT and launches nothing.
 *   - The first call on a device looks up the array's device address on that device (one
 *     cudaGetSymbolAddress, with that device current); make that first call before any stream
 *     capture on that device. The address belongs to the CUDA context that is current during
 *     the call: it is remembered per device together with that context, and looked up again
 *     (the same way) when a later call runs under another context of the device, for example
 *     after cudaDeviceReset.
 *   - All calls share the one array and it keeps whatever the last call wrote. Nothing in it needs
 *     to start at zero (every partial is written before it is read). Two calls whose kernels
 *     overlap on the GPU (different streams, or different host threads, without ordering between
 *     them) race on the array and give wrong results: order them on one stream or with events.
 * Returns MEA_OK or a negative mea_status, like mea_decode_splitkv.
 */
#define MEA_DECODE_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int mea_decode_splitkv_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                               const int32_t* cu_seqlens_k, int n_seqs, int total_k,
                               int max_seqlen_k, int n_heads_q, int n_heads_kv, int head_dim,
                               float scale, int mask_kind, const float* alibi_slopes, int dtype,
                               int split_keys, void* stream);

/*
 * mea_forward_fp8 — mea_forward with 8-bit e4m3 q, k, v (FP8 forward on the tensor cores).
 *
 * The inputs are e4m3 values (1 sign, 4 exponent, 3 mantissa bits, bias 7, largest finite 448,
 * no infinities) with per-tensor descales: the attention is that of q_descale*q,
 * k_descale*k, v_descale*v (exact products of the decoded values), with the same segments,
 * masks, GQA grouping, ALiBi and scale as mea_forward. Q K^T accumulates in fp32; P is rounded
 * to e4m3 for the P V product (its row sum and lse use the fp32 values); out is written in
 * out_dtype (MEA_BF16 or MEA_F16), lse in fp32 natural log.
 *   q, k, v   DEVICE e4m3 [total_q, n_heads_q, D] / [total_k, n_heads_kv, D].
 *   head_dim  a multiple of 16 from 16 to 128 (MEA_ERR_HEAD_DIM otherwise).
 * Other arguments, errors and ownership as mea_forward.
 */
int mea_forward_fp8(const void* q, const void* k, const void* v, void* out, float* lse,
                    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int n_seqs,
                    int total_q, int total_k, int max_seqlen_q, int n_heads_q, int n_heads_kv,
                    int head_dim, float scale, int mask_kind, const float* alibi_slopes,
                    float q_descale, float k_descale, float v_descale, int out_dtype,
                    void* stream);

/*
 * mea_backward_workspace_size — bytes of workspace mea_backward needs: two fp32 per (query
 * head, query token) and per each of 128 pad rows a head (delta = rowsum(dout * out) and the
 * row's exponent term, computed by the first kernel), 4096 bytes for the segments' launch
 * order, plus 256 bytes of alignment slack.
 */
size_t mea_backward_workspace_size(int total_q, int n_heads_q);

/*
 * mea_backward — gradients of the packed attention of mea_forward (training backward).
 *
 * For L = sum(out * dout), computes dq = dL/dq, dk = dL/dk, dv = dL/dv of the definition above
 * (the same segments, masks, GQA grouping, ALiBi slopes and scale as the forward call), as the
 * derivative of the forward definition: with P the row softmax of the scaled, biased, masked
 * scores, dS = P * (dout V^T - rowsum(dout * out)), dq = scale * dS K, dk = scale * dS^T Q
 * (summed over the heads of a KV group), dv = P^T dout (likewise summed).
 *   q, k, v, out  DEVICE, the forward's inputs and output (same layout and dtype as mea_forward).
 *   lse           DEVICE fp32 [n_heads_q, total_q], the forward's lse (required).
 *   dout          DEVICE gradient of out, layout and dtype of out.
 *   dq, dk, dv    DEVICE outputs, layouts of q, k, v; every element is written (keys no query
 *                 sees and rows that see no key get 0).
 *   n_seqs        1 .. 65535 segments.
 *   max_seqlen_q/k upper bounds on every L_q / L_k (they size the grids; MEA_ERR_SHAPE when
 *                 ceil(max_seqlen_q / 128) * n_heads_q / 4 would pass 2^31 - 1).
 *   workspace     DEVICE, at least mea_backward_workspace_size(total_q, n_heads_q) bytes, owned
 *                 by the caller; 16-byte aligned.
 * No atomics: the result is deterministic. Asynchronous on `stream`. Returns MEA_OK or a
 * negative mea_status (MEA_ERR_WORKSPACE when the workspace is missing or too small).
 */
int mea_backward(const void* q, const void* k, const void* v, const void* out, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv, const int32_t* cu_seqlens_q,
                 const int32_t* cu_seqlens_k, int n_seqs, int total_q, int total_k,
                 int max_seqlen_q, int max_seqlen_k, int n_heads_q, int n_heads_kv, int head_dim,
                 float scale, int mask_kind, const float* alibi_slopes, int dtype, void* workspace,
                 size_t workspace_bytes, void* stream);

/*
 * mea_decode_paged — mea_decode_splitkv over a paged K/V cache (serving layout): request b's key
 * t (0 <= t < L_b) lives in cache block block_table[b * max_blocks + t / block_size], slot
 * t % block_size. Same arithmetic, masks, output and workspace as mea_decode_splitkv.
 *   k_cache, v_cache  DEVICE [num_blocks, block_size, n_heads_kv, head_dim], dtype of q.
 *   block_table       DEVICE int32 [n_seqs, max_blocks]; entries past ceil(L_b / block_size)
 *                     are not read. An id outside [0, num_blocks) reads as zeros (never faults).
 *   cu_seqlens_k      DEVICE int32 [n_seqs + 1], prefix sums of the requests' key counts L_b.
 *   block_size        16, 32, or a multiple of 64.
 *   total_k           an upper bound on cu_seqlens_k[n_seqs] (for example num_blocks *
 *                     block_size); it sizes the workspace exactly as in mea_decode_splitkv:
 *                     mea_decode_workspace_size(n_seqs, total_k, ...).
 *   max_seqlen_k      an upper bound on every L_b, at most max_blocks * block_size.
 * Slots of a block past the end of its sequence may hold any bits (they are never used).
 */
int mea_decode_paged(const void* q, const void* k_cache, const void* v_cache,
                     const int32_t* block_table, const int32_t* cu_seqlens_k, void* out,
                     float* lse, int n_seqs, int num_blocks, int block_size, int max_blocks,
                     int total_k, int max_seqlen_k, int n_heads_q, int n_heads_kv, int head_dim,
                     float scale, int mask_kind, const float* alibi_slopes, int dtype,
                     void* workspace, size_t workspace_bytes, int split_keys, void* stream);

/* mea_status_string — a static English description of a mea_status value. */
const char* mea_status_string(int status);

/*
 * mea_device_error — reads (and, if `clear` != 0, resets) the device-side error word of the
 * current device. Kernels bound every wait; one that gives up records a non-zero code here
 * (bits 0..7: which wait, bits 8..15: which kernel) and returns early. Synchronises the device.
 * Returns MEA_OK and stores the word in *code, or MEA_ERR_CUDA.
 */
int mea_device_error(int* code, int clear);

/*
 * mea_set_wait_timeout_ns — the bound, in nanoseconds, on every wait inside the kernels
 * (default 2e9). Applies to launches made after the call, from any thread.
 */
void mea_set_wait_timeout_ns(unsigned long long ns);

/*
 * mea_wait_selftest — exercises the bounded wait that every kernel uses, with nothing else in
 * flight: one warp initialises a shared-memory mbarrier (arrival count 1) and waits on its
 * first phase with the given bound (`timeout_ns`, 0 means the current mea_set_wait_timeout_ns
 * value). With `arrive` != 0 the warp first arrives itself, so the wait completes at once and
 * the error word stays 0; with `arrive` == 0 nothing ever arrives, the wait gives up after the
 * bound, records MEA_SELFTEST_WAIT_CODE in the device error word (if it was 0) and the kernel
 * returns normally. This is how a caller (or a test) checks that a timed-out wait leaves the
 * context usable and reports through mea_device_error. Asynchronous on `stream`; returns
 * MEA_OK, or MEA_ERR_CUDA if the launch fails.
 */
#define MEA_SELFTEST_WAIT_CODE 0x7f01
int mea_wait_selftest(unsigned long long timeout_ns, int arrive, void* stream);

/* mea_version — library version string. */
const char* mea_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MEA_H_ */
