/*
 * exact_attention_ring_b200 — C ABI of the B200 (sm_100a) exact-attention library.
 *
 * Exact scaled-dot-product attention O = softmax(scale * Q K^T) V, computed tile
 * by tile with an online softmax so that the N x N score matrix never reaches
 * device memory ("1-Flash-Attention.md", sections "Tiling（分块）技术" and
 * "递归计算softmax"; FlashAttention V2 page: Q tiles in the outer loop, K/V in the
 * inner loop, normalisation once at the end). Single-query decode splits the
 * key range across thread blocks and merges the partial results by their
 * log-sum-exp (FlashAttention V2 page, Flash-Decoding paragraph; FlashAttention-3
 * page, the split-K combine step). Ring attention (context parallelism) shards a
 * long sequence across devices and merges each device's per-shard results the
 * same way (attn_fwd_f32, attn_merge; FlashAttention-3 page, RingAttention).
 * The backward pass (attn_bwd) recomputes P from the saved log-sum-exp; the
 * FP8 forward (attn_quant_fp8, attn_quant_fp8_rotate, attn_fwd_fp8) runs on
 * block-quantised E4M3 inputs, optionally after incoherent processing
 * (FlashAttention-3 page).
 *
 * Conventions shared by every call:
 *  - All tensors are dense, contiguous, row-major device buffers owned by the
 *    caller. The library allocates nothing, never synchronises, and only
 *    enqueues work on `stream` (0 = the legacy default stream). Every call is
 *    asynchronous like a kernel launch.
 *  - bf16 buffers hold IEEE bfloat16 bit patterns; float buffers hold IEEE fp32.
 *  - Every pointer must be 16-byte aligned and must not alias another argument.
 *  - Arguments are checked before anything is launched; a failed check returns a
 *    status and enqueues nothing. A launch failure returns ATTN_ERR_CUDA.
 *  - Sequence lengths (N, L) are at most 2^31 - 256, so that the block and tile
 *    counts rounded up from them fit an int; a longer one is
 *    ATTN_ERR_INVALID_ARG (attn_decode_default_splits returns 0).
 *  - Every wait inside a kernel is bounded. A kernel whose wait runs out records
 *    ATTN_ERR_TIMEOUT in a device-side status word and returns early (its outputs
 *    are then undefined); attn_device_status() reads and clears that word.
 *  - LSE is the natural-log log-sum-exp of the scaled, masked scores of a row:
 *    lse_i = ln sum_{j visible} exp(scale * q_i . k_j).
 *  - Kernels are launched with programmatic stream serialization: a kernel's
 *    blocks may be scheduled while the previous kernel in the stream finishes,
 *    but each waits for that kernel's completion before its first access to
 *    device memory, so the stream's order of memory effects is unchanged.
 *  - Calls may be captured in CUDA graphs. A non-causal attn_fwd (and
 *    attn_fwd_f16, attn_fwd_f32) hands out its work items through one of 64
 *    device counters, taken by successive launches in turn and back at zero when
 *    the launch's kernel ends; a call whose last round of query blocks would
 *    leave most SMs idle makes two launches (the second, in 128-row halves,
 *    right behind the first) and takes two counters: at most 32 such calls may
 *    be in flight at once, and a captured call keeps its counters at every
 *    replay, so replays of one graph must not run concurrently with each other.
 */
#ifndef EXACT_ATTENTION_RING_B200_ATTN_H
#define EXACT_ATTENTION_RING_B200_ATTN_H

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as the CUDA runtime's cudaStream_t (an opaque driver stream). */
typedef struct CUstream_st* attn_stream_t;

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, Hq % Hkv != 0, bad scale */
    ATTN_ERR_UNSUPPORTED = 2, /* a head dimension other than 64 or 128 */
    ATTN_ERR_CUDA = 3,        /* a CUDA runtime call or a launch failed */
    ATTN_ERR_TIMEOUT = 4      /* a bounded in-kernel wait ran out (see attn_device_status) */
} attn_status_t;

/*
 * attn_fwd — prefill forward pass.
 * Defined by: "1-Flash-Attention.md", "问题分析" (S = Q K^T, A = softmax(S/sqrt(d)),
 * O = A V on (batch, heads, seq_len, head_dim) tensors) and "使用注意事项"
 * (causal flag; head_dim 64 or 128; fp16/bf16 inputs), computed by the tiled
 * online-softmax recurrence of "递归计算softmax"; softmax_scale as in "框架集成".
 *
 *  q    [B, Hq,  N, d] bf16 (device, read)
 *  k, v [B, Hkv, N, d] bf16 (device, read)
 *  o    [B, Hq,  N, d] bf16 (device, written): O rounded to nearest-even bf16
 *  lse  [B, Hq,  N]    fp32 (device, written): natural-log LSE per row
 *  B, Hq, Hkv, N >= 1; Hq % Hkv == 0; query head h reads key/value head
 *      h / (Hq / Hkv) (grouped-query / multi-query attention).
 *  d     64 or 128 (else ATTN_ERR_UNSUPPORTED).
 *  causal  0: every row sees all N keys; 1: row i sees keys j <= i.
 *  scale   finite and > 0 (typically 1/sqrt(d)).
 * Any N >= 1 is accepted (no power-of-two requirement); ragged tiles are masked.
 */
attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                       int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                       attn_stream_t stream);

/*
 * attn_fwd_f32 — attn_fwd with O written in fp32 (O_acc / l, not rounded to
 * bf16): the form a partial result takes when it is merged further, e.g. one
 * key/value block of ring attention folded in with attn_merge. Same method,
 * arguments, layouts, checks and errors as attn_fwd except
 *  o  [B, Hq, N, d] fp32 (device, written).
 * bf16(o of attn_fwd_f32) with round-to-nearest-even equals o of attn_fwd.
 */
attn_status_t attn_fwd_f32(const void* q, const void* k, const void* v, float* o, float* lse,
                           int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                           attn_stream_t stream);

/*
 * attn_decode_splitkv — split-KV (Flash-Decoding) partials for one query token.
 * Defined by: FlashAttention V2 page, Flash-Decoding paragraph (the key/value
 * sequence is split across thread blocks for single-query decode); each split is
 * the attention of "1-Flash-Attention.md", "问题分析", restricted to its keys.
 *
 *  q        [B, Hq, d]      bf16 (device, read): the one query of each sequence
 *  k, v     [B, Hkv, L, d]  bf16 (device, read): the key/value cache
 *  o_part   [B, Hq, S, d]   fp32 (device, written): normalised partial outputs
 *  lse_part [B, Hq, S]      fp32 (device, written): natural-log LSE per split
 *  S = num_splits, 1 <= S <= L. Split s covers keys [s*C, min(L, (s+1)*C)) with
 *  C = 128 * ceil(ceil(L / S) / 128). A split with no keys gets lse = -inf, o = 0.
 *  d 64 or 128; Hq % Hkv == 0; scale finite and > 0.
 *  If a bounded wait inside the kernel runs out (attn_device_status then reports
 *  ATTN_ERR_TIMEOUT), the splits it abandoned are written as empty (lse = -inf,
 *  o = 0): the results of that call are not attention and must be discarded.
 */
attn_status_t attn_decode_splitkv(const void* q, const void* k, const void* v,
                                  float* o_part, float* lse_part,
                                  int B, int Hq, int Hkv, int L, int d, int num_splits,
                                  float scale, attn_stream_t stream);

/*
 * attn_combine — log-sum-exp weighted merge of split partials.
 * Defined by: FlashAttention-3 page (the split-K combine step,
 * combine_attn_seqk_parallel): with M = max_s lse_s and w_s = exp(lse_s - M),
 * O = sum_s w_s O_s / sum_s w_s and LSE = M + ln sum_s w_s; a split with
 * lse_s = -inf has weight 0.
 *
 *  o_part   [B, Hq, S, d] fp32 (device, read)
 *  lse_part [B, Hq, S]    fp32 (device, read)
 *  o        [B, Hq, d]    bf16 (device, written)
 *  lse      [B, Hq]       fp32 (device, written)
 *  d 64 or 128; 1 <= S <= 12000 (one weight per split is kept in shared
 *  memory; larger S returns ATTN_ERR_INVALID_ARG); at least one split of
 *  every (b, h) must be non-empty.
 */
attn_status_t attn_combine(const float* o_part, const float* lse_part, void* o, float* lse,
                           int B, int Hq, int num_splits, int d, attn_stream_t stream);

/*
 * attn_merge — folds the attention of one key/value block into a running result:
 * the merge step of ring attention (context parallelism), where the key/value
 * shards of a long sequence travel around a ring of devices and each device
 * attends its query shard to every shard in turn, one attn_fwd per shard.
 * Defined by: FlashAttention-3 page (attention over a key range split into parts
 * is the log-sum-exp weighted merge of the parts: its split-K combine and the
 * RingAttention derivation it refers to). Blocks come in fp32 so that a ring
 * rounds its result to bf16 once, at the last merge. Per row, with
 * M = max(lse_acc, lse_blk),
 * wa = exp(lse_acc - M), wb = exp(lse_blk - M):
 *   o_acc <- (wa o_acc + wb o_blk) / (wa + wb),   lse_acc <- M + ln(wa + wb);
 * a side whose lse is -inf has weight 0; a row with both -inf is left as it was.
 *
 *  o_acc   [rows, d] fp32 (device): read unless init; written unless out is given
 *  lse_acc [rows]    fp32 (device): read unless init; always written
 *  o_blk   [rows, d] fp32 (device, read): e.g. the o of attn_fwd_f32, rows = B*Hq*N
 *  lse_blk [rows]    fp32 (device, read): the matching lse
 *  out     [rows, d] bf16 (device, written) or NULL: when given, the merged O is
 *          written here (bf16, round to nearest even) instead of into o_acc —
 *          the last merge of a ring
 *  init    nonzero: o_acc and lse_acc are not read; the result is the block itself
 *  rows >= 1; d 64 or 128. o_acc, out and o_blk must not overlap.
 */
attn_status_t attn_merge(float* o_acc, float* lse_acc, const float* o_blk, const float* lse_blk,
                         void* out, long long rows, int d, int init, attn_stream_t stream);

/*
 * attn_bwd — gradients of exact attention with respect to q, k and v, given the
 * output gradient dout and the forward pass's o and lse (attn_fwd, same inputs).
 * P is recomputed from q, k and lse instead of being stored (FlashAttention V2
 * page, opening paragraph: tiling and recomputation; Flash Attention notes,
 * "使用注意事项": the backward pass keeps the softmax terms in fp32). For the
 * visible keys j of row i, with P_ij = exp(scale q_i . k_j - lse_i):
 *   dP_ij = dout_i . v_j,  Delta_i = dout_i . o_i,  dS_ij = P_ij (dP_ij - Delta_i),
 *   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,  dv_j = sum_i P_ij dout_i,
 * dk and dv summed over the G = Hq / Hkv query heads that read a key/value head.
 * P and dS enter the tensor-core products rounded to bf16; sums are fp32.
 *
 *  q, o, dout [B, Hq, N, d]  bf16 (device, read)
 *  k, v       [B, Hkv, N, d] bf16 (device, read)
 *  lse        [B, Hq, N]     fp32 (device, read): the lse attn_fwd returned
 *  delta      [B, Hq, N]     fp32 (device): workspace, overwritten with Delta
 *  dq         [B, Hq, N, d]  bf16 (device, written)
 *  dk, dv     [B, Hkv, N, d] bf16 (device, written)
 *  B*Hq <= 65535; 1 <= N <= 65535 * 128; d 64 or 128 (else
 *  ATTN_ERR_UNSUPPORTED); causal 0/1 (query i sees keys j <= i); scale finite
 *  and > 0. Outputs must not overlap the inputs. Three launches on `stream`:
 *  Delta, then dk/dv (one block per 128-key tile and key/value head), then dq
 *  (one block per 128-row query tile and query head); under the causal mask the
 *  blocks with the most work start first.
 */
attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                       const void* dout, float* delta, void* dq, void* dk, void* dv,
                       int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                       attn_stream_t stream);

/*
 * attn_quant_fp8, attn_quant_fp8_rotate, attn_fwd_fp8 — the forward pass on
 * FP8 (E4M3) inputs. FlashAttention-3 page: FP8 computation with block
 * quantisation and incoherent processing. Reading of "block
 * quantisation": one fp32 scale per block of 128 consecutive rows of a
 * (batch, head) plane — or one per plane — s = amax / 448 with amax the
 * largest |x| of the block (s = 1 for an all-zero block), code = E4M3(x / s),
 * round to nearest even, IEEE fp32 division; the code stands for
 * E4M3(code) * s.
 *
 * attn_quant_fp8 quantises x [planes, N, d] bf16 (device, read):
 *  codes   transpose == 0: [planes, N, d] uint8; transpose == 1: [planes, d, Np]
 *          uint8 with Np = 128 * ceil(N / 128), codes of keys >= N zero
 *  scales  [planes, ceil(N / 128)] fp32 (written); with per_plane != 0 every
 *          block of a plane gets the plane's scale
 *  d 64 or 128 (else ATTN_ERR_UNSUPPORTED); planes <= 65535. One launch for
 *  per-block row-major codes (per_plane 0, transpose 0), three otherwise.
 *
 * attn_quant_fp8_rotate quantises like attn_quant_fp8 (per_plane 0,
 * transpose 0) after incoherent processing of every row. Reading of the page's
 * "incoherent processing" (it gives no detail): each row x of Q and of K is
 * replaced by y = H (signs o x) / sqrt(d), H the d x d Sylvester Hadamard
 * matrix and signs a vector of random +1 / -1 shared by Q and K. H H^T = d I,
 * so the rotation is orthogonal and Q K^T is unchanged, while an outlier in one
 * coordinate is spread over all d before quantisation. y is computed in fp32
 * as the fast Walsh-Hadamard transform (butterflies (a, b) -> (a + b, a - b) of
 * span 1, 2, ..., d/2 in that order) and one multiplication by the fp32 value
 * nearest 1 / sqrt(d); the codes and scales are those of the block quantisation
 * of y. Rotate Q and K with the same signs and leave V as it is: attn_fwd_fp8 on
 * the results computes the attention of the original inputs.
 *  x       [planes, N, d] bf16 (device, read)
 *  signs   [d] fp32, each +1 or -1 (device, read; the caller draws them)
 *  codes   [planes, N, d] uint8 (written), scales [planes, ceil(N / 128)] (written)
 *  d 64 or 128 (else ATTN_ERR_UNSUPPORTED); planes <= 65535. One launch.
 *
 * attn_fwd_fp8 computes O and LSE (as attn_fwd) from quantised inputs:
 *  q8  [B, Hq, N, 128]  codes from attn_quant_fp8(q, ..., per_plane 0, transpose 0)
 *  k8  [B, Hkv, N, 128] codes from attn_quant_fp8(k, ..., per_plane 0, transpose 0)
 *  vt8 [B, Hkv, 128, Np] codes from attn_quant_fp8(v, ..., per_plane 1, transpose 1)
 *  sq, sk, sv           the matching scales
 *  o   [B, Hq, N, 128] bf16, lse [B, Hq, N] fp32 (written)
 * S = Q8 K8^T runs on the tensor cores in E4M3 with fp32 accumulation and the
 * block scales applied to the fp32 scores; P is rounded to E4M3 for the P V
 * product (kept at most 2^8 by rescaling O whenever a row's maximum grows by
 * more than 8 in log2 units); l sums the fp32 P. d must be 128 (else
 * ATTN_ERR_UNSUPPORTED); B*Hq <= 65535; other checks as attn_fwd.
 */
attn_status_t attn_quant_fp8(const void* x, void* codes, float* scales, int planes, int N, int d,
                             int per_plane, int transpose, attn_stream_t stream);
attn_status_t attn_quant_fp8_rotate(const void* x, const float* signs, void* codes, float* scales,
                                    int planes, int N, int d, attn_stream_t stream);
attn_status_t attn_fwd_fp8(const void* q8, const void* k8, const void* vt8, const float* sq,
                           const float* sk, const float* sv, void* o, float* lse,
                           int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                           attn_stream_t stream);

/*
 * attn_fwd_f16, attn_decode_splitkv_f16, attn_combine_f16 — the same three calls
 * for IEEE fp16 inputs (the pages list FP16 beside BF16 among the supported
 * dtypes: "1-Flash-Attention.md", "使用注意事项"). Arguments, layouts, checks and
 * errors as for the bf16 calls; every 16-bit buffer (q, k, v, o) holds fp16
 * bit patterns, P is rounded to fp16 for the P V product, and o is written as
 * fp16 (round to nearest even). lse and the split partials stay fp32.
 */
attn_status_t attn_fwd_f16(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                           attn_stream_t stream);
attn_status_t attn_decode_splitkv_f16(const void* q, const void* k, const void* v,
                                      float* o_part, float* lse_part,
                                      int B, int Hq, int Hkv, int L, int d, int num_splits,
                                      float scale, attn_stream_t stream);
attn_status_t attn_combine_f16(const float* o_part, const float* lse_part, void* o, float* lse,
                               int B, int Hq, int num_splits, int d, attn_stream_t stream);

/*
 * attn_decode_default_splits — the split count attn_decode_splitkv is tuned for
 * on a 148-SM B200: it maximises the busy fraction of the waves of (batch,
 * kv-head, split) blocks times the fraction of each block's time spent
 * streaming (a block's start-up is worth about 260 keys). Pure host
 * arithmetic; returns 1 <= S <= ceil(L / 128), or 0 on bad arguments.
 */
int attn_decode_default_splits(int B, int Hq, int Hkv, int L);

/* Human-readable name of a status code (static storage). */
const char* attn_status_string(attn_status_t status);

/*
 * attn_device_status — synchronises `stream`, then reads and clears the
 * device-side status word that kernels set when a bounded wait runs out.
 * Returns ATTN_OK, ATTN_ERR_TIMEOUT, or ATTN_ERR_CUDA if synchronisation failed.
 * Uses the current CUDA device.
 */
attn_status_t attn_device_status(attn_stream_t stream);

/*
 * attn_selftest_bounded_wait — launches one thread that waits on a barrier that
 * nothing completes, with a wait limit of `limit_us` microseconds (1..10^6), so
 * that the timeout path can be exercised without faulting or hanging the GPU.
 * The wait runs out, the kernel records ATTN_ERR_TIMEOUT and returns. Enqueued
 * on `stream`; read the result with attn_device_status().
 */
attn_status_t attn_selftest_bounded_wait(int limit_us, attn_stream_t stream);

/*
 * attn_decode_noalloc — split-KV decode plus combine that allocates nothing.
 * The pages have no counterpart: this is a service for callers that cannot
 * allocate device memory for the split partials (an engine whose device memory
 * is owned by its own pool, a plug-in that must not allocate, a latency-critical
 * loop that cannot afford cudaMalloc). It computes what attn_decode_splitkv
 * followed by attn_combine computes, with the same arguments except that the
 * partials live in a fixed 4 MiB array built into the library (1,048,576 floats;
 * every GPU that loads the library holds it until the process exits).
 *
 *  q [B, Hq, d], k/v [B, Hkv, L, d] bf16 (device, read)
 *  o [B, Hq, d] bf16, lse [B, Hq] fp32 (device, written)
 *  num_splits, d, scale: as for attn_decode_splitkv.
 * Limit: B * Hq * num_splits * (d + 1) <= 1,048,576 and num_splits <= 12000
 * (the combine's bound); larger problems, and any argument attn_decode_splitkv
 * or attn_combine would reject, return ATTN_ERR_INVALID_ARG before anything is
 * enqueued (use fewer splits, or the attn_decode_splitkv + attn_combine pair
 * with caller-owned partials).
 * The first call on a device looks up the array's device address (with that
 * device current) and the library keeps it for the life of the process; make
 * that first call before any stream capture. After cudaDeviceReset (or anything
 * else that tears down and recreates the device's primary context) the kept
 * address is stale: such a process must not call attn_decode_noalloc again.
 * The call never calls cudaMalloc, cudaFree or any allocating routine. All calls
 * on a device share the one array and it keeps the last call's contents;
 * nothing in it needs clearing, because every partial is written before it is
 * read (a split abandoned after a bounded wait ran out is written as empty, and
 * attn_device_status reports ATTN_ERR_TIMEOUT: discard that call's o and lse).
 * Calls that can overlap on the GPU (different streams without ordering
 * between them) race on the array and must not be issued.
 */
attn_status_t attn_decode_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                                  int B, int Hq, int Hkv, int L, int d, int num_splits, float scale,
                                  attn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_ATTENTION_RING_B200_ATTN_H */
