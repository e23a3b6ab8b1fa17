/*
 * unipin.h - C ABI of the B200 (sm_100a) library for UniPinRec's cross-stage
 * KV reuse: the M-FALCON masked prefill attention, the write of the past K/V
 * into a preallocated cache pool, and the rank decode that scores candidate
 * tokens against a slot of that pool.
 *
 * Sources (the method is described in prose only):
 *   [notes]  UniPinRec reproduction notes (slinene.github.io, ai-papers-daily,
 *            "unipinrec-unified-retrieval-ranking-masked-action-kv-share"),
 *            sub-module details §3 "attention mask", §6 "serving:
 *            cross-process KV sharing".
 *   [review] UniPinRec paper review (liuzhao09.github.io,
 *            "pinterest-unipinrec"), §2.2 joint objective, §2.4 co-serving,
 *            Faiss and the cross-stage KV cache.
 *
 * Conventions shared by every call:
 *   - Tensors are bfloat16, row-major, in device memory owned by the caller.
 *     Packed token tensors are [T, H, D]: token t, head h, element d at
 *     ((t * H + h) * D + d).  Every tensor pointer must be 16-byte aligned.
 *   - Ragged batches use int32 offset arrays in device memory: cu_seqlens of
 *     length B+1 (segment b = tokens cu_seqlens[b] .. cu_seqlens[b+1]-1).
 *   - Supported head dims: D in {32, 64, 128}.
 *   - Heads: queries have H heads, keys and values H_kv heads with H a multiple
 *     of H_kv; query head h reads key/value head h / (H / H_kv) (grouped-query
 *     attention; H_kv = H is plain multi-head attention).  [notes] §6 names the
 *     pool's H "KV heads": the pool has H_kv heads.
 *   - Every call is asynchronous on `stream` (a cudaStream_t, NULL = the
 *     legacy default stream), does no host synchronisation, allocates
 *     nothing and keeps no pointer after it returns.  The first call of each
 *     entry point on a device sets kernel attributes and resolves a driver
 *     entry point, so make one call before capturing a CUDA graph.
 *   - Host-checkable errors come back as the return value and launch nothing.
 *     Errors the kernels find in device arrays (a length or slot id out of
 *     range) and bounded waits that ran out of time are stored into
 *     *dev_status (device int, may be NULL; 0 = no error, the first error
 *     wins); a kernel never traps.  The rows of a segment or request found
 *     out of range are written as zeros when the segment's own rows lie
 *     inside the tensors (rows of a segment whose cu_seqlens range is
 *     itself out of bounds are not written).  After a timeout the output is
 *     undefined.  The caller clears *dev_status and reads it back when it
 *     likes.
 */
#ifndef UNIPIN_H
#define UNIPIN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    UNIPIN_OK = 0,
    UNIPIN_ERR_INVALID_ARG = -1,    /* null pointer, negative size, inconsistent shapes */
    UNIPIN_ERR_UNSUPPORTED = -2,    /* D not in {32, 64, 128}; device is not sm_100 */
    UNIPIN_ERR_MISALIGNED = -3,     /* a tensor pointer is not 16-byte aligned */
    UNIPIN_ERR_OUT_OF_RANGE = -4,   /* slot >= S, n > n_cap, layer >= L, a length > the stated max */
    UNIPIN_ERR_CUDA = -5,           /* a CUDA runtime / driver call failed */
    UNIPIN_ERR_DEVICE_TIMEOUT = -6  /* a bounded device wait expired (reported via dev_status) */
} unipin_status;

/* Element type of a pool's K and V. */
typedef enum {
    UNIPIN_POOL_BF16 = 0,   /* bfloat16 */
    UNIPIN_POOL_E4M3 = 1    /* FP8 E4M3 codes with one scale for K and one for V */
} unipin_pool_dtype;

/*
 * The KV cache pool ([review] §2.4, [notes] §6): one preallocated tensor of
 * shape [L, S, H, n_cap, D] for K and one for V (layer, slot, KV head,
 * history position, head dim), row-major, caller-owned device memory.  Row
 * (l, s, h, j) starts at element (((l * S + s) * H + h) * n_cap + j) * D.
 * A slot holds one user's past K/V; rows j >= that user's n are never read.
 *
 * dtype UNIPIN_POOL_BF16: elements are bfloat16; k_scale and v_scale are ignored.
 * dtype UNIPIN_POOL_E4M3: elements are FP8 E4M3 codes (1 byte; the format's
 *   fn form: bias 7, no infinity, largest finite 448).  The pages apply E4M3 to
 *   their linear layers ([notes]/[review] FP8 sections); storing the pool in it
 *   is this library's extension, halving its size.  Writing x stores
 *   E4M3(x * (1 / k_scale)) (the reciprocal and the product in float32, nearest
 *   value with ties to even, magnitudes saturated at 448); attention reads code c
 *   as bfloat16(value(c) * k_scale) (float32 product, nearest even), and alike
 *   for V.  Scales must be finite and positive; with powers of two the read is
 *   exact.
 */
typedef struct {
    void* k;
    void* v;
    int L, S, H, n_cap, D;
    int dtype;            /* unipin_pool_dtype */
    float k_scale;        /* UNIPIN_POOL_E4M3 only */
    float v_scale;
} unipin_kvpool;

/*
 * Masked prefill attention over B packed segments [n_b past || k_b candidates]
 * ([notes] §3, [review] §2.2):
 *   past row i < n_b      attends to keys j <= i (causal, diagonal included);
 *   candidate row i >= n_b attends to every past key j < n_b and to itself,
 *                          never to another candidate.
 *   O_i = softmax_j(scale * q_i . k_j) v_j over the allowed keys, computed with
 *   fp32 scores, fp32 online softmax and fp32 accumulation (P rounded to bf16
 *   for the P.V product).
 *
 *   q              [T, H, D] bf16, T = total_tokens = cu_seqlens[B]
 *   k, v           [T, H_kv, D] bf16
 *   out            [T, H, D], fp32 if out_fp32 != 0 else bf16 (round to nearest even)
 *   lse            optional fp32 [T, H] (NULL: not written): per row and head the
 *                  log-sum-exp of its scores in base-2 units,
 *                  lse_i = log2(sum_j 2^(scale * log2(e) * q_i . k_j)) over the allowed
 *                  keys j, so the weight of key j is 2^(scale*log2(e)*q_i.k_j - lse_i).
 *                  The backward pass (unipin_masked_prefill_bwd) takes it.
 *   cu_seqlens     device int32 [B+1]; past_lens device int32 [B], 0 <= n_b <= len_b
 *   max_seqlen     host int >= every len_b (sizes the grid; a longer segment is a device error)
 *   scale          softmax scale, normally 1/sqrt(D)
 *   pool, slot_ids optional (pool == NULL: no pool write).  When given (pool->H ==
 *                  H_kv), the past K/V of segment b is also written to pool rows
 *                  [layer, slot_ids[b], h, 0:n_b) exactly as unipin_kvpool_write does:
 *                  into a bfloat16 pool by the same kernel from the K/V tiles it loads
 *                  anyway, into an E4M3 pool by a second kernel of the same call.
 *   workspace      optional device scratch, 16-byte aligned (NULL allowed).  With at
 *                  least unipin_masked_prefill_workspace_size() bytes, the persistent
 *                  thread blocks take (segment, head, query-tile pair) work items from
 *                  a shared counter; without it each block takes a fixed stride of
 *                  items.  Same result either way.  Two calls that overlap in time
 *                  must not share a workspace.
 * Returns UNIPIN_OK or a negative unipin_status.
 */
int unipin_masked_prefill_attn(const void* q, const void* k, const void* v, void* out, int out_fp32, float* lse,
                               const int* cu_seqlens, const int* past_lens, int B, int H, int H_kv, int D,
                               int max_seqlen, int total_tokens, float scale, const unipin_kvpool* pool,
                               const int* slot_ids, int layer, void* workspace, size_t workspace_bytes,
                               int* dev_status, void* stream);

/* Bytes of scratch that let unipin_masked_prefill_attn hand out work
 * dynamically (a work counter the call zeroes on `stream` before its kernel). */
size_t unipin_masked_prefill_workspace_size(void);

/*
 * Gradients of the masked prefill ([review] §2.2: the joint objective trains
 * [past || candidates] in one forward pass under this mask, so the backward
 * pass runs over the same allowed pairs).  With P_ij the forward's weights
 * (rebuilt from lse) and dO the gradient of the loss with respect to out:
 *   dV_j = sum_i P_ij dO_i
 *   dS_ij = P_ij (dO_i . v_j - dO_i . O_i)
 *   dQ_i = scale * sum_j dS_ij k_j,   dK_j = scale * sum_i dS_ij q_i
 * over allowed (i, j) only: a past key collects gradient from the later past
 * rows and from every candidate row of its segment, a candidate's own key and
 * value only from its own row.  Scores, probabilities and accumulation are
 * fp32; P and dS are rounded to bf16 as tensor-core operands.
 *   q              [T, H, D] bf16; k, v [T, H_kv, D] bf16: the forward's inputs
 *   out            [T, H, D] bf16, the forward's output (bf16 mode)
 *   dout           [T, H, D] bf16, the gradient with respect to out
 *   lse            fp32 [T, H] as written by unipin_masked_prefill_attn
 *   dq             fp32 [T, H, D], dk and dv fp32 [T, H_kv, D] (a key/value head
 *                  sums its query heads' gradients); written in full (dq is accumulated
 *                  across key tiles with atomic adds, so its low bits depend on
 *                  their order)
 *   D              32, 64 or 128 (UNIPIN_ERR_UNSUPPORTED otherwise)
 *   workspace      device scratch of at least
 *                  unipin_masked_prefill_bwd_workspace_size(total_tokens, H) bytes
 *                  (the per-row dO . O), 16-byte aligned; not shared by overlapping calls
 * Other arguments and errors as unipin_masked_prefill_attn.  Rows of a segment
 * found out of range on the device get zero gradients.
 */
int unipin_masked_prefill_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
                              const float* lse, float* dq, float* dk, float* dv, const int* cu_seqlens,
                              const int* past_lens, int B, int H, int H_kv, int D, int max_seqlen,
                              int total_tokens, float scale, void* workspace, size_t workspace_bytes,
                              int* dev_status, void* stream);

/* Bytes of workspace unipin_masked_prefill_bwd needs: 4 * total_tokens * H, rounded up to 16. */
size_t unipin_masked_prefill_bwd_workspace_size(int total_tokens, int H);

/*
 * Pool write ([review] §2.4: retrieval writes the past K/V of every layer
 * into the shared pool; [notes] §6: pool [L, S, H, n, D], slot reuse):
 *   pool.k[layer, slot_ids[b], h, j, :] = k[cu_seqlens[b] + j, h, :]   for j < past_lens[b]
 * and the same for v.  Into a bfloat16 pool a byte copy (bit-exact); into an
 * E4M3 pool each element quantized as the pool's description says.  Nothing
 * else in the pool is touched.  Slot ids within one call must be distinct (a repeated id leaves
 * that slot holding one of the writers' rows, unspecified which).
 *   k, v           [T, H, D] bf16 with T = cu_seqlens[B]
 *   max_past       host int >= every past_lens[b] (sizes the grid)
 *   total_tokens   T, the number of rows of k and v (rows read are checked against it)
 */
int unipin_kvpool_write(const unipin_kvpool* pool, int layer, const void* k, const void* v,
                        const int* cu_seqlens, const int* past_lens, const int* slot_ids, int B, int max_past,
                        int total_tokens, int* dev_status, void* stream);

/*
 * Rank decode ([review] §2.4: the ranking node forwards only the candidate
 * tokens and lets them attend to the cached history K/V; [notes] §6: read
 * the request's slot, cost O(nk)).  Request r has k_r candidates (rows
 * cu_seqlens_c[r] .. cu_seqlens_c[r+1]-1 of q_c/k_c/v_c) and n_r = past_lens[r]
 * cached rows in slot slot_ids[r] of `pool` at `layer`.  Candidate c attends
 * to pool rows 0..n_r-1 of that slot and to itself (its own k_c, v_c) - the
 * same mask as the candidate rows of the prefill, so it returns what the
 * prefill returns for those rows.
 *   q_c            [T_c, H, D] bf16, T_c = total_cand = cu_seqlens_c[R]
 *   k_c, v_c       [T_c, pool->H, D] bf16 (the candidates' own keys and values;
 *                  H must be a multiple of the pool's key/value heads)
 *   out            [T_c, H, D], fp32 if out_fp32 else bf16
 *   max_k          host int >= every k_r (sizes the grid and picks the kernel: with
 *                  max_k * G <= 64 (G = H / pool->H) and D in {64, 128} the pool keys
 *                  are the tensor-core M dimension, the G query heads of a key/value
 *                  head share one sweep of its history, and a request's key range is
 *                  swept by several thread blocks, the bandwidth-bound case;
 *                  otherwise 128-candidate query tiles run through the prefill engine)
 *   workspace      optional device scratch, 16-byte aligned (NULL allowed).  With at
 *                  least 256 bytes the blocks take work items from a shared counter
 *                  (zeroed by the call on `stream`); with at least
 *                  unipin_rank_decode_workspace_size(...) bytes the pool sweep of
 *                  each request is also split over several thread blocks (split-n)
 *                  when that helps, and the splits are merged (in the kernel for
 *                  max_k * G <= 64, by a second kernel otherwise; the per-request
 *                  arrival counters the in-kernel merge uses are zeroed by the call
 *                  on `stream`).  The result is the same either way up to fp32
 *                  rounding.  Two calls that overlap in time must not share a
 *                  workspace.
 */
int unipin_rank_decode_attn(const void* q_c, const void* k_c, const void* v_c, void* out, int out_fp32,
                            const int* cu_seqlens_c, const int* slot_ids, const int* past_lens, int R, int H,
                            int D, int max_k, int total_cand, float scale, const unipin_kvpool* pool, int layer,
                            void* workspace, size_t workspace_bytes, int* dev_status, void* stream);

/* Bytes of workspace unipin_rank_decode_attn uses at most for these sizes
 * (n_cap = the pool's rows per slot) over a bfloat16 pool: 256 for the work
 * counter, plus the split-n partial results (and, for max_k <= 64 candidate
 * columns, one arrival counter per request and head) when it would split.  The
 * split grows with the device's SM count; the size returned covers the
 * current device and a 148-SM B200. */
size_t unipin_rank_decode_workspace_size(int R, int H, int H_kv, int D, int max_k, int total_cand, int n_cap);

/* The same for a given pool of either dtype.  Over an UNIPIN_POOL_E4M3 pool:
 *   - with max_k * G <= 64 and D = 128, or max_k * G <= 32 and D = 64, and with
 *     k_scale and v_scale both bfloat16 values in [2^-117, 2^118], the
 *     small-candidate kernel reads the codes itself (each key tile lands in
 *     shared memory as codes and is expanded there to the bfloat16 values the
 *     tensor cores take), so the workspace is as for a bfloat16 pool: optional,
 *     only for split-n;
 *   - otherwise the call first dequantizes rows 0..n_r-1 of each request's slot
 *     (layer `layer`) into bfloat16 in the workspace and then decodes from
 *     there, so it needs a workspace: this size, which includes
 *     R * pool->H * pool->n_cap * pool->D * 4 bytes for those rows; with less it
 *     returns UNIPIN_ERR_INVALID_ARG.
 * Either way code c stands for bfloat16(value(c) * scale). */
size_t unipin_rank_decode_pool_workspace_size(const unipin_kvpool* pool, int R, int H, int max_k, int total_cand);

/*
 * Rank decode that allocates nothing and takes no workspace.  There is no
 * counterpart to this on the pages; it exists for callers that cannot call
 * cudaMalloc at decode time: a serving process whose device memory is already
 * handed to another framework's pool, or a loop that must not allocate after
 * start-up.  Arguments and results are those of unipin_rank_decode_attn,
 * and so are its errors, with one more: the scratch it needs (a work counter
 * and, when the pool sweep is split, the split-n partial results and arrival
 * counters) lives in a device array of unipin_rank_decode_noalloc_scratch_bytes()
 * bytes (32 MiB) that the library reserves on every device it is loaded on
 * and keeps until the process exits.
 *   - If unipin_rank_decode_workspace_size(R, H, pool->H, D, max_k,
 *     total_cand, pool->n_cap) exceeds that size, the pool sweep is not split
 *     (as unipin_rank_decode_attn does with a small workspace): the same
 *     result, computed more slowly.
 *   - An UNIPIN_POOL_E4M3 pool is taken only where the small-candidate kernel
 *     reads its codes (see unipin_rank_decode_pool_workspace_size); otherwise
 *     the call returns UNIPIN_ERR_UNSUPPORTED: the dequantized rows it would
 *     decode from do not fit a fixed array.
 *   - The first call on a device looks up the array's device address; make
 *     that first call before any stream capture.
 *   - Every call shares the one array and it keeps the last call's contents
 *     (the call zeroes the work counter it needs on `stream` itself), so two
 *     calls that overlap on the GPU - on different streams, or from different
 *     host threads - race and may give wrong results.  Serialise them.
 */
int unipin_rank_decode_attn_noalloc(const void* q_c, const void* k_c, const void* v_c, void* out, int out_fp32,
                                    const int* cu_seqlens_c, const int* slot_ids, const int* past_lens, int R,
                                    int H, int D, int max_k, int total_cand, float scale,
                                    const unipin_kvpool* pool, int layer, int* dev_status, void* stream);

/* Size of the array behind unipin_rank_decode_attn_noalloc (32 MiB). */
size_t unipin_rank_decode_noalloc_scratch_bytes(void);

/*
 * Cross-process sharing of a pool ([notes] §6 "serving: cross-process KV
 * sharing": retrieval and ranking are separate OS processes with separate
 * CUDA contexts; each retrieval replica preallocates its [L, S, H, n, D] pool
 * and exports CUDA IPC handles for it, and the ranking process maps the same
 * device memory and reads the KV without a trip through the host).
 *
 * unipin_kvpool_share is plain bytes and may be written to a file or a
 * socket as it is: the IPC handles of the device allocations that hold
 * pool.k and pool.v, the byte offsets of the pool inside them, and the shape.
 */
typedef struct {
    unsigned char k_handle[64];       /* cudaIpcMemHandle_t of the allocation holding pool.k */
    unsigned char v_handle[64];       /* same for pool.v */
    unsigned long long k_offset;      /* byte offset of pool.k inside its allocation */
    unsigned long long v_offset;
    int L, S, H, n_cap, D;
    int dtype;                        /* pool.dtype, pool.k_scale, pool.v_scale */
    float k_scale, v_scale;
} unipin_kvpool_share;

/* Exporter side: fill *out for `pool`.  The pool's tensors must lie in memory
 * from cudaMalloc (not from virtual-memory mapping or cudaMallocAsync pools),
 * and must stay allocated while any importer has it open.
 * Returns UNIPIN_ERR_INVALID_ARG for a null or malformed pool or a pointer
 * that is not device memory, UNIPIN_ERR_OUT_OF_RANGE if the pool extends past
 * its allocation, UNIPIN_ERR_CUDA if the handle cannot be created. */
int unipin_kvpool_share_export(const unipin_kvpool* pool, unipin_kvpool_share* out);

/* Importer side (another process, on a device that can reach the exporter's):
 * map the shared pool into this process; *out is then a pool usable by every
 * call of this library.  A process cannot open a handle it exported itself
 * (UNIPIN_ERR_CUDA). */
int unipin_kvpool_share_open(const unipin_kvpool_share* in, unipin_kvpool* out);

/* Importer side: unmap a pool opened from `in`; clears opened->k and ->v. */
int unipin_kvpool_share_close(const unipin_kvpool_share* in, unipin_kvpool* opened);

/*
 * Slot assignment for the pool ([notes] §6: slots are reused in rotation;
 * [review] §2.4: the retrieval stage hands the ranking node the slot id of
 * each request).  Host-side and thread-safe.  acquire hands out n distinct
 * free slots, scanning in round-robin order from the slot after the last one
 * it handed out, so consecutive requests rotate through the pool; release
 * returns slots once the ranking side is done with them.
 */
typedef struct unipin_slot_ring unipin_slot_ring;

/* A ring over slots 0..S-1, all free.  UNIPIN_ERR_INVALID_ARG if S < 1. */
int unipin_slot_ring_create(int S, unipin_slot_ring** out);

/* Writes n free slot ids into the host array slot_ids and marks them in use.
 * If fewer than n are free, takes none and returns UNIPIN_ERR_OUT_OF_RANGE. */
int unipin_slot_ring_acquire(unipin_slot_ring* ring, int n, int* slot_ids);

/* Marks the n slots free again.  All or nothing: an id out of range, not in
 * use, or repeated in the list gives UNIPIN_ERR_INVALID_ARG and frees none. */
int unipin_slot_ring_release(unipin_slot_ring* ring, int n, const int* slot_ids);

/* Number of free slots (or UNIPIN_ERR_INVALID_ARG for a null ring). */
int unipin_slot_ring_free_count(unipin_slot_ring* ring);

void unipin_slot_ring_destroy(unipin_slot_ring* ring);

/* Human-readable name of a unipin_status value. */
const char* unipin_status_string(int status);

/*
 * Self-test of the bounded device wait used by every kernel: launches one
 * warp that waits on a barrier nothing ever completes, with a limit of
 * limit_us microseconds.  The wait gives up, stores UNIPIN_ERR_DEVICE_TIMEOUT
 * into *dev_status and the kernel returns normally.  Exists so tests can
 * check the timeout path without any kernel hanging.
 */
int unipin_selftest_bounded_wait(int* dev_status, unsigned int limit_us, void* stream);

/*
 * Self-test of the exp2 the softmax evaluates on the FMA pipe for one score
 * pair in four (a degree-3 polynomial after rounding the argument to an
 * integer, see csrc/sm100_ptx.cuh): y[i] = 2^x[i] for n device floats, so
 * tests can compare it with CUDA's exp2f.  Arguments below -127 give 0.
 */
int unipin_selftest_exp2(const float* x, float* y, int n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* UNIPIN_H */
