/*
 * yocopp.h - C ABI of the B200 (sm_100a) YOCO / YOCO++ cross-layer KV cache
 * hot path: the fused residual composition + cache append, and the
 * split-K GQA decode attention that every cross-decoder layer runs over the
 * single shared cache.
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers of the current CUDA device,
 *    owned by the caller.  The library never allocates or frees them and
 *    keeps no reference after the call returns.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL is the legacy default stream).  A YOCOPP_OK return means the work
 *    was enqueued; it does not wait for it.
 *  - Host-side argument checks return a negative yocopp_status and enqueue
 *    nothing.  Nothing is thrown across the ABI.
 *  - Values the host cannot see without synchronising (positions, lengths,
 *    block-table entries) are checked in the kernels; a violation skips the
 *    offending access and records a code that yocopp_get_device_status()
 *    returns.  Kernels never trap.
 *  - Element types: YOCOPP_BF16 (storage bf16, fp32 arithmetic) or
 *    YOCOPP_F32.  q, K, V, the cache and the output share one type.
 */
#ifndef YOCOPP_H
#define YOCOPP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum yocopp_status {
    YOCOPP_OK = 0,
    YOCOPP_EINVAL = -1,        /* null pointer, bad size, unsupported shape */
    YOCOPP_EDTYPE = -2,        /* unknown or unsupported element type */
    YOCOPP_ECAPACITY = -3,     /* a position / length beyond the cache (device check) */
    YOCOPP_EWORKSPACE = -4,    /* workspace missing, misaligned or too small */
    YOCOPP_ECUDA = -5,         /* a CUDA runtime/driver call failed */
    YOCOPP_EDEVICE_CHECK = -6, /* a kernel met an invalid block-table entry */
    YOCOPP_ETIMEOUT = -7       /* a bounded wait inside a kernel ran out */
} yocopp_status;

typedef enum yocopp_dtype {
    YOCOPP_BF16 = 0,
    YOCOPP_F32 = 1
} yocopp_dtype;

/*
 * One layer's KV cache (caller-owned device memory).
 *
 * Contiguous (block_table == NULL):
 *   k, v : [batch][num_kv_heads][capacity][head_dim]
 * Paged (block_table != NULL):
 *   k, v : [num_blocks][num_kv_heads][block_size][head_dim]
 *   block_table : int32 [batch][max_blocks_per_seq]; position p of sequence b
 *   lives in block block_table[b][p / block_size], slot p % block_size;
 *   capacity must equal block_size * max_blocks_per_seq.
 * In both layouts each (token, head) row is head_dim contiguous elements and
 * each (sequence or block, head) plane is contiguous, which is what lets the
 * decode kernel stage K/V tiles with TMA.
 *
 * Supported: head_dim in {64, 128}; block_size in {16, 32, 64, 128, 256};
 * k and v 16-byte aligned.  In YOCO++ (section 2, "cache strategy") a
 * self-decoder layer's cache holds the composed K'_i, V'_i; the cross-decoder
 * layers all read layer L/2's cache, the shared cache.
 */
typedef struct yocopp_cache {
    void* k;
    void* v;
    const int32_t* block_table;
    int32_t dtype;               /* yocopp_dtype */
    int32_t batch;
    int32_t num_kv_heads;
    int32_t head_dim;
    int32_t capacity;            /* positions per sequence */
    int32_t block_size;          /* paged only (ignored when contiguous) */
    int32_t max_blocks_per_seq;  /* paged only */
    int32_t num_blocks;          /* paged only: blocks in the pool */
} yocopp_cache;

/*
 * yocopp_compose_append - YOCO++ residual KV composition fused with the
 * cache write (YOCO++: Enhancing YOCO with KV Residual Connections,
 * section 2 "method", composition equations; section 2 key innovation 1,
 * cache strategy: the composed values are what is stored).
 *
 * For every new token t of sequence b, KV head h and channel c:
 *   K'[t,h,c] = lambda * (alpha[0] * K1[t,h,c] + alpha[1] * Ki[t,h,c])
 *   V'[t,h,c] = lambda * (alpha[2] * V1[t,h,c] + alpha[3] * Vi[t,h,c])
 * computed in fp32 with error-free products and sums for the inner weighted
 * sum (so near-cancelling terms keep their low bits), then multiplied by
 * lambda, rounded once to the cache type, and written to cache positions
 * pos[b] .. pos[b] + n_b - 1.  A stored bf16 value is the exact composition
 * rounded once to nearest-even bf16 (not a rounding of an fp32 intermediate);
 * only a value within about 2^-48 (relative) of a bf16 rounding midpoint can
 * land on the other neighbour, so it is always within one bf16 ulp.
 *
 *   K1, V1, Ki, Vi : device, [total_new][num_kv_heads][head_dim], cache dtype,
 *                    16-byte aligned.  Rows are token-major and packed over
 *                    the batch: sequence b's new tokens are rows
 *                    [cu_new[b], cu_new[b+1]) or, when cu_new == NULL,
 *                    [b * n_uniform, (b + 1) * n_uniform).  K1/V1 are the
 *                    current tokens' layer-1 values (they may alias Ki/Vi).
 *   alpha          : HOST, 4 floats {aK1, aK2, aV1, aV2}.
 *   lambda         : the scale factor (35 in YOCO++, section 2, key innovation 2).
 *   cache          : HOST descriptor of the destination cache.
 *   pos            : device int32 [cache->batch], first position written.
 *   cu_new         : device int32 [cache->batch + 1] prefix offsets, or NULL.
 *   n_uniform      : tokens per sequence when cu_new == NULL (>= 0).
 *   total_new      : number of input rows (= cu_new[batch] or batch*n_uniform).
 *
 * Layer 1 (raw K_1, V_1 stored) is alpha = {0, 1/lambda, 0, 1/lambda}, which
 * reproduces the inputs bit for bit in bf16 (section 2, initialization).
 * A row whose position is outside [0, capacity), or whose block-table entry
 * is outside [0, num_blocks), is not written and the device status records
 * YOCOPP_ECAPACITY / YOCOPP_EDEVICE_CHECK.  No other cache slot is touched.
 */
int32_t yocopp_compose_append(const void* K1, const void* V1, const void* Ki, const void* Vi,
                              const float alpha[4], float lambda, const yocopp_cache* cache,
                              const int32_t* pos, const int32_t* cu_new, int32_t n_uniform,
                              int64_t total_new, void* stream);

/*
 * yocopp_decode_attn_workspace_size - bytes of device workspace that
 * yocopp_decode_attn needs for this cache shape and query-head count on the
 * current device (it depends on the device's SM count).  Returns a negative
 * yocopp_status on invalid arguments.  The workspace holds a call generation
 * that the kernel itself advances (so calls captured in a CUDA graph replay
 * correctly), the per-split partial softmax state (max, sum of exponentials,
 * weighted value sum) from the start of the buffer upwards, and one arrival
 * counter per (sequence, kv-head) plane at the END of the buffer
 * (workspace_bytes as passed, rounded down to 256).
 *
 * Zero-fill the workspace once before its first use.  After that it never
 * needs clearing, also not after a failed call, as long as every call on it
 * passes the same workspace_bytes, the same query-group size (num_q_heads /
 * num_kv_heads) and the same head_dim; batch and lengths may change freely
 * between calls (the partials' extent only grows with the plane count, so it
 * never reaches the counters of a call with more planes).  Zero-fill it again
 * before using it with another group size, head_dim or workspace_bytes.  A
 * workspace that was not zero-filled can make a call report
 * YOCOPP_EWORKSPACE through yocopp_get_device_status and leave output rows
 * unwritten.
 */
int64_t yocopp_decode_attn_workspace_size(const yocopp_cache* cache, int32_t num_q_heads);

/*
 * yocopp_decode_attn - one decode step of a cross-decoder layer over the
 * shared cache (You Only Cache Once, abstract: the cross-decoder reuses the
 * cached KVs through cross-attention; YOCO++ section 2: every upper-half
 * layer reads (K'_{L/2}, V'_{L/2}); section 3: decoding reads one KV set).
 *
 * For sequence b and query head h with KV head g = h / (num_q_heads /
 * num_kv_heads) (contiguous GQA grouping):
 *   s_t = scale * <q[b,h,:], K'[b,t,g,:]>   for t in [0, seq_lens[b])
 *   out[b,h,:] = sum_t softmax(s)_t * V'[b,t,g,:]
 * fp32 arithmetic, online softmax over key tiles split across the GPU, then
 * an exact log-sum-exp merge of the splits by the last CTA to finish each
 * (sequence, kv-head) plane: one kernel launch.  seq_lens[b] == 0 gives zeros.
 * The kernel is launched as a programmatic dependent of the previous work in
 * the stream (it waits for that work before reading any input).
 *
 *   q         : device [batch][num_q_heads][head_dim], cache dtype, 16-byte aligned.
 *   cache     : HOST descriptor of the shared cache.
 *   seq_lens  : device int32 [batch]; positions attended (the token being
 *               decoded is already appended).  A length above capacity is
 *               clamped and YOCOPP_ECAPACITY recorded on the device.
 *   out       : device [batch][num_q_heads][head_dim], cache dtype.
 *   num_q_heads : multiple of num_kv_heads, group size in {1, 2, 4}.
 *   scale     : softmax scale; 0 selects 1/sqrt(head_dim).
 *   workspace : device, >= yocopp_decode_attn_workspace_size() bytes, 256-byte
 *               aligned, not shared with a concurrently running call.
 */
int32_t yocopp_decode_attn(const void* q, const yocopp_cache* cache, const int32_t* seq_lens,
                           void* out, int32_t num_q_heads, float scale, void* workspace,
                           int64_t workspace_bytes, void* stream);

/*
 * yocopp_decode_attn_fused - the read-time alternative the composition is
 * designed to avoid (YOCO++, section 1 on FusedKV and section 3: combining
 * several layers' KVs while decoding costs extra I/O; composing before the
 * cache write keeps decoding at one KV set per layer).  Same attention as
 * yocopp_decode_attn over K' = lambda (alpha[0] K_1 + alpha[1] K_i) and
 * V' = lambda (alpha[2] V_1 + alpha[3] V_i), but K', V' are formed in fp32
 * at read time (never rounded to the cache type) from two RAW caches, so
 * every decode step reads twice the bytes.  The exact FusedKV combination is
 * not given by the pages; this is the YOCO++ formula evaluated at read time.
 *   cache_i : raw K_i, V_i of layer L/2;  cache_1 : raw K_1, V_1 of layer 1;
 *             identical shape, dtype, layout and block table.
 * Other arguments as yocopp_decode_attn (its workspace size applies).
 */
int32_t yocopp_decode_attn_fused(const void* q, const yocopp_cache* cache_i, const yocopp_cache* cache_1,
                                 const float alpha[4], float lambda, const int32_t* seq_lens, void* out,
                                 int32_t num_q_heads, float scale, void* workspace, int64_t workspace_bytes,
                                 void* stream);

/*
 * yocopp_decode_attn_partial - yocopp_decode_attn over this caller's cached
 * positions only, kept unnormalised so that it can be merged with results
 * over other positions of the same sequences (for example other GPUs' shards
 * of one long context; You Only Cache Once, abstract: the cache scales to
 * 1M tokens, more than one GPU holds).  Arguments as yocopp_decode_attn,
 * with `partial` in place of `out`:
 *   partial : device fp32 [batch][num_q_heads][head_dim + 2]; per row the
 *             weighted sum o[c] = sum_t 2^(s'_t - m) V'_t[c] for c < head_dim,
 *             then m = max_t s'_t and l = sum_t 2^(s'_t - m), where
 *             s'_t = scale * log2(e) * <q, K'_t> (base-2 logits).  A sequence
 *             with no positions gives o = 0, m = -inf, l = 0.
 */
int32_t yocopp_decode_attn_partial(const void* q, const yocopp_cache* cache, const int32_t* seq_lens,
                                   float* partial, int32_t num_q_heads, float scale, void* workspace,
                                   int64_t workspace_bytes, void* stream);

/*
 * yocopp_decode_combine - exact log-sum-exp merge of num_parts partial results
 * (each laid out as yocopp_decode_attn_partial writes them) into the output:
 *   partials : device fp32 [num_parts][rows][head_dim + 2], rows = batch * num_q_heads
 *   out      : device [rows][head_dim] of `dtype`
 * out = sum_r 2^(m_r - M) o_r / sum_r 2^(m_r - M) l_r with M = max_r m_r;
 * rows with no positions in any part give 0.
 */
int32_t yocopp_decode_combine(const float* partials, int32_t num_parts, int64_t rows, int32_t head_dim,
                              int32_t dtype, void* out, void* stream);

/*
 * yocopp_decode_attn_static - yocopp_decode_attn without a caller workspace.
 * The pages describe no such call: this entry point exists for callers that
 * cannot allocate device memory on this path, such as a host framework that
 * owns all device memory through its own pool and gives plug-in libraries no
 * allocator, or a serving loop in which cudaMalloc's implicit device-wide
 * synchronisation is not acceptable.
 *
 * Same arguments and results as yocopp_decode_attn, minus the workspace: the
 * split partials and arrival counters live in a fixed 4 MiB array inside the
 * library (every device that loads the library holds it until the process
 * exits).  Nothing is allocated or freed by this call.
 *   - The array's last 64 KiB hold the arrival counters of up to 8192
 *     (sequence, kv-head) planes at a fixed place; the split partials use the
 *     rest.  A shape with batch * num_kv_heads > 8192, or whose partials do
 *     not fit, returns YOCOPP_EWORKSPACE and enqueues nothing.  On a 148-SM
 *     device at head_dim 128 that is batch * num_kv_heads <= 1688 with 4
 *     query heads per KV head, 3673 with 2 and 7642 with 1 (partials:
 *     (2 * 148 + batch * num_kv_heads) * G * (head_dim + 2) * 4 bytes, each of
 *     the three arrays rounded up to 256, within 4 MiB - 64 KiB - 256).
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress with that device current); make that first call
 *     before any stream capture.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents.  It starts zero-filled when the library is loaded; since the
 *     counters never move and the partials never reach them, every call (also
 *     a failed one, and whatever the previous call's shape) leaves it usable
 *     by the next, so nothing ever needs clearing.  Calls whose execution
 *     overlaps on the GPU (different streams, or different host threads) race
 *     on it and give wrong results: serialise them.
 */
int32_t yocopp_decode_attn_static(const void* q, const yocopp_cache* cache, const int32_t* seq_lens,
                                  void* out, int32_t num_q_heads, float scale, void* stream);

/*
 * yocopp_prefill_attn - causal attention of a self-decoder layer's prefill
 * tokens over that layer's own cache, on the tensor cores (YOCO++: Enhancing
 * YOCO with KV Residual Connections, section 2 "cache strategy": a lower-half
 * layer caches its composed K'_i, V'_i and attends over them; section 3:
 * prefill is compute-bound, the composition adding only a little I/O).
 * Call it after yocopp_compose_append has written the tokens' composed rows
 * (the composition and this attention are two kernels in one stream).
 *
 * Query row j of sequence b sits at cache position p_b + j (p_b = pos[b], or
 * 0 when pos == NULL) and, for query head h and KV head g = h / (num_q_heads /
 * num_kv_heads):
 *   s_u = scale * <q[b,j,h,:], K'[b,g,u,:]>   for u in [0, p_b + j]
 *   out[b,j,h,:] = sum_u softmax(s)_u * V'[b,g,u,:]
 * with fp32 scores and accumulation, P rounded to bf16 for the value product.
 *
 *   q       : device bf16 [total_q][num_q_heads][128], 16-byte aligned; rows
 *             token-major and packed over the batch like yocopp_compose_append's
 *             inputs: sequence b's rows are [cu_q[b], cu_q[b+1]) or, when
 *             cu_q == NULL, [b * n_uniform, (b + 1) * n_uniform).
 *   cache   : HOST descriptor; bf16, head_dim 128, contiguous or paged (any
 *             block size yocopp_cache allows).  Positions [0, p_b + n_b) of
 *             sequence b must hold the composed rows; a block-table entry
 *             outside [0, num_blocks) for such a position records
 *             YOCOPP_EDEVICE_CHECK (that block is not read).
 *   pos     : device int32 [batch] or NULL (all 0; a whole-prompt prefill).
 *   cu_q    : device int32 [batch + 1] prefix offsets, or NULL.
 *   n_uniform : rows per sequence when cu_q == NULL.
 *   total_q : rows of q and out (= cu_q[batch] or batch * n_uniform).
 *   max_q   : with cu_q, an upper bound of every n_b (sizes the grid);
 *             ignored when cu_q == NULL.
 *   out     : device bf16 [total_q][num_q_heads][128], 16-byte aligned.
 *   num_q_heads : multiple of num_kv_heads.
 *   scale   : softmax scale; 0 selects 1/sqrt(128).
 * A sequence with p_b < 0, p_b + n_b > capacity or n_b > max_q is skipped and
 * YOCOPP_ECAPACITY recorded on the device; a decreasing cu_q records
 * YOCOPP_EDEVICE_CHECK.  Output rows of skipped sequences are not written.
 * Returns YOCOPP_EDTYPE for fp32 caches and YOCOPP_EINVAL for other shapes.
 */
int32_t yocopp_prefill_attn(const void* q, const yocopp_cache* cache, const int32_t* pos, const int32_t* cu_q,
                            int32_t n_uniform, int64_t total_q, int32_t max_q, void* out, int32_t num_q_heads,
                            float scale, void* stream);

/*
 * yocopp_prefill_compose_attn - yocopp_compose_append followed by
 * yocopp_prefill_attn in ONE launch: the composition of the prefill rows
 * fused with the causal attention over them (YOCO++: Enhancing YOCO with KV
 * Residual Connections, section 2, composition equations and cache strategy;
 * section 3: prefill is compute-bound and the composition adds only a little
 * I/O, which here overlaps the attention's tensor-core work).  The launch
 * holds, per sequence, one composition CTA for each 128-row query tile (all
 * KV heads) besides the attention CTAs; the composition CTAs of sequence b+1
 * run ahead of the attention CTAs of sequence b, and an attention CTA waits
 * (bounded, on a flag in the workspace) until the rows of a key tile are
 * composed before loading it.  Results equal the two calls': the cache gets
 * the same bits as yocopp_compose_append writes and the outputs those of
 * yocopp_prefill_attn.
 *
 *   K1, V1, Ki, Vi : raw rows as for yocopp_compose_append, packed like q
 *                    ([total_q][num_kv_heads][128] bf16, rows of sequence b
 *                    at [cu_q[b], cu_q[b+1]) or b * n_uniform ..); they are
 *                    composed into cache positions pos[b] + j.
 *   alpha, lambda  : as for yocopp_compose_append (HOST alpha[4]).
 *   q ... scale    : as for yocopp_prefill_attn.
 *   workspace      : device, >= yocopp_prefill_compose_attn_workspace_size()
 *                    bytes, 256-byte aligned, zero-filled once before its first
 *                    use; it never needs clearing after that (a call generation
 *                    advanced by the kernel tags the flags), for any later
 *                    shape.  Not shared with a concurrently running call.
 * Positions before pos[b] must already hold composed rows, as for
 * yocopp_prefill_attn.  A wait that runs out records YOCOPP_ETIMEOUT.
 */
int64_t yocopp_prefill_compose_attn_workspace_size(const yocopp_cache* cache, int32_t max_q);
int32_t yocopp_prefill_compose_attn(const void* K1, const void* V1, const void* Ki, const void* Vi,
                                    const float alpha[4], float lambda, const void* q, const yocopp_cache* cache,
                                    const int32_t* pos, const int32_t* cu_q, int32_t n_uniform, int64_t total_q,
                                    int32_t max_q, void* out, int32_t num_q_heads, float scale, void* workspace,
                                    int64_t workspace_bytes, void* stream);

/*
 * yocopp_get_device_status - the first error code recorded by a kernel on
 * the current device since the last reset (YOCOPP_OK if none).  Synchronous:
 * it waits for the device.  reset != 0 clears the record.
 */
int32_t yocopp_get_device_status(int32_t reset);

/* Human-readable name of a yocopp_status value (static string). */
const char* yocopp_status_string(int32_t status);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int32_t yocopp_version(void);

/*
 * yocopp_set_decode_kernel - which score product later yocopp_decode_attn /
 * _partial / _static launches use (process-wide, host-side):
 *   0  the default, which is 2;
 *   1  CUDA-core packed fp32 FMA for q.k (every dtype and head_dim);
 *   2  tcgen05 tensor cores for the query-group x key-tile product where
 *      supported (bf16, head_dim 128, batch up to about 2400; otherwise the
 *      CUDA-core kernel runs).
 * Both give the same results within rounding; the value sum and the softmax
 * run on the CUDA cores in both.  Returns YOCOPP_EINVAL for other values.
 */
int32_t yocopp_set_decode_kernel(int32_t which);

/*
 * yocopp_testing_set_decode_fault - failure-injection hook for tests.
 * Host-side, process-wide; affects later yocopp_decode_attn and
 * yocopp_prefill_attn launches.
 *   drop_tile     : decode: index (in the split plan's flattened tile order) of
 *                   one tile whose load is never issued, so the consumers' wait
 *                   on it can only run out; prefill: index of the key tile
 *                   whose K load the first CTA never issues; -1 disables the
 *                   injection.
 *   wait_limit_ns : limit of every bounded wait inside the decode and prefill
 *                   kernels (default 2 s); must be > 0.
 * With a dropped tile the kernel records YOCOPP_ETIMEOUT, waits (bounded) for
 * its own copies still in flight, and returns; the context stays usable.
 * Returns YOCOPP_EINVAL for wait_limit_ns <= 0.
 */
int32_t yocopp_testing_set_decode_fault(int32_t drop_tile, int64_t wait_limit_ns);

/*
 * yocopp_testing_set_decode_prefetch - switch for the early L2 prefetch of the
 * tensor-core decode kernel (on by default).  Host-side, process-wide; affects
 * later decode launches.  Launched while the previous kernel in the stream
 * still runs, that kernel guesses, before its programmatic wait, each CTA's
 * first tiles from the lengths and block tables as they stand and prefetches
 * them into L2; everything it computes reads the inputs again after the wait.
 *   enabled : 1 = prefetch (default), 0 = no prefetch.
 * The results are the same bits either way.  Returns YOCOPP_EINVAL for other
 * values.
 */
int32_t yocopp_testing_set_decode_prefetch(int32_t enabled);

#ifdef __cplusplus
}
#endif

#endif /* YOCOPP_H */
