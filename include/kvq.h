/*
 * kvq.h -- C ABI of the B200 (sm_100a) KVarN-style quantized paged KV cache.
 *
 * What the library computes.  The KVarN pages describe a vLLM attention
 * backend whose cache blocks go through a Hadamard rotation, a variance
 * normalisation and asymmetric low-bit quantisation (4-bit keys, 2-bit values
 * by default, preset flag kvarn_k4v2_g128), with the group scales folded into
 * attention at read time:
 *   - "Трюк Huawei с KV-кэшем" (beyondheadline.xyz), lede and section
 *     "Заявка, которая ломает привычный компромисс";
 *   - "KVarN vs TurboQuant" (dothoosh.com), the four-stage pipeline list and
 *     the kv_cache_dtype flag paragraph.
 * The pages give no formula or layout; the library fixes them as follows.
 *
 * Write path, per 128-element K or V head vector x of one token:
 *   r = R x, R = H/sqrt(128), H the natural-order Sylvester Hadamard matrix;
 *   mu, sigma = mean and population standard deviation of r (sigma = 0 -> 1);
 *   u = (r - mu)/sigma, lo = min u, hi = max u;
 *   S = fp16(sigma (hi - lo)/(2^b - 1)), Z = fp16(mu + sigma lo)   [g128]
 *   c_i = clamp(rne((r_i - Z)/S), 0, 2^b - 1) (all 0 when S == 0), b = k_bits
 *   for keys and v_bits for values (4 and 2 by default).  Dequantized
 *   vector: x^ = R (S c + Z).
 *
 * Read path (decode), for query head j of sequence b, kv head h = j / G,
 * G = Hq/Hkv, tau = softmax_scale (<= 0 means 1/sqrt(128)):
 *   o = sum_t softmax_t(tau <q, k^_t>) v^_t over the seq_lens[b] cached
 *   tokens.  The kernel computes it with the scales folded in: q~ = R q once,
 *   s_t = tau (S_K,t <q~, c_K,t> + Z_K,t sum(q~)), o~ = sum_t p_t (S_V,t c_V,t
 *   + Z_V,t), o = R o~ once.
 *
 * Pool layout (the ABI; the pages leave it open).  A pool is num_blocks
 * physical blocks of block_size (16) token slots for each of num_kv_heads
 * heads.  Segment (p, h) starts at byte (p*num_kv_heads + h) * SEG and holds,
 * for the default k4v2_g128 (SEG = 1664):
 *   [0,1024)    K codes, 16 rows of 64 B; element i at byte i/2, low nibble
 *               for even i
 *   [1024,1536) V codes, 16 rows of 32 B; element i at byte i/4, bits 2(i%4)
 *   [1536,1568) S_K[16]  [1568,1600) Z_K[16]
 *   [1600,1632) S_V[16]  [1632,1664) Z_V[16]          (fp16, little endian)
 * Slot s of the pool is block s/16, row s%16 (vLLM slot mapping).  That is
 * 104 bytes per token per kv head against 512 for an fp16 cache (4.92x).
 * The other presets (k4v4, k2v2, k8v4, all g128) keep the same order: 16 K
 * rows of 16*k_bits B, 16 V rows of 16*v_bits B, then S_K, Z_K, S_V, Z_V;
 * a b-bit element i sits at bits [b*i, b*i+b) of its row, little endian.
 * SEG = 16*128*(k_bits+v_bits)/8 + 128: 2176, 1152 and 3200 bytes.
 *
 * Conventions.
 *   - The caller owns every buffer.  Device pointers are CUDA device memory
 *     of the current device; host pointers are ordinary host memory.  The
 *     library allocates nothing and keeps no state except cached device
 *     attributes and one device status word per device (see
 *     kvq_last_device_status).
 *   - Calls that take a stream are asynchronous on that stream (a
 *     cudaStream_t passed as void*, NULL = legacy default stream) and return
 *     after validating arguments and enqueueing work.
 *   - Every entry point returns 0 (KVQ_OK) or a negative kvq_status.  No
 *     exception, abort or device trap ever leaves the library: argument
 *     errors are caught on the host; out-of-range block ids and slots met on
 *     the device are skipped and recorded in the device status word.
 *   - Supported geometry: head_dim 128, group 128, block_size 16, and one of
 *     four presets (k_bits, v_bits) = (4, 2) (the pages' default,
 *     kvarn_k4v2_g128), (4, 4), (2, 2) or (8, 4); num_q_heads a multiple of
 *     num_kv_heads with G = Hq/Hkv in {1, 2, 4, 8}.  Anything else returns
 *     KVQ_ERR_UNSUPPORTED.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID = -1,        /* null pointer, negative size, bad enum value */
  KVQ_ERR_UNSUPPORTED = -2,    /* geometry or preset the kernels do not cover */
  KVQ_ERR_CUDA = -3,           /* a CUDA runtime call failed (launch, query)  */
  KVQ_ERR_POOL_EXHAUSTED = -4, /* kvq_block_table: not enough physical blocks */
  KVQ_ERR_OUT_OF_RANGE = -5,   /* block id or slot outside the pool           */
  KVQ_ERR_DEVICE_TIMEOUT = -6, /* a bounded device-side wait gave up          */
  KVQ_ERR_WORKSPACE = -7       /* workspace missing, misaligned or too small  */
} kvq_status;

typedef enum { KVQ_F16 = 0, KVQ_BF16 = 1, KVQ_F32 = 2 } kvq_dtype;

/* One cache pool.  pool is device memory of kvq_cache_bytes(desc) bytes,
 * 16-byte aligned, owned by the caller; its initial contents do not matter. */
typedef struct {
  int32_t num_blocks;   /* physical blocks in the pool (>= 0)             */
  int32_t block_size;   /* token slots per block: 16                      */
  int32_t num_kv_heads; /* Hkv >= 1                                       */
  int32_t head_dim;     /* 128                                            */
  int32_t k_bits;       /* 4 (or 2, 8: see kvq_parse_dtype)               */
  int32_t v_bits;       /* 2 (or 4)                                       */
  int32_t group;        /* elements per scale/zero group: 128 (= head_dim) */
  void* pool;           /* device pointer                                 */
} kvq_cache_desc;

/* Parse a cache dtype string of the form "kvarn_k<kb>v<vb>_g<g>", the vLLM
 * flag named on the KVarN pages ("KVarN vs TurboQuant", flag paragraph).
 * Host only.  Writes the three numbers and returns KVQ_OK for a well-formed
 * string (KVQ_ERR_UNSUPPORTED if it is well formed but not one of the
 * presets the kernels cover: k4v2_g128, k4v4_g128, k2v2_g128, k8v4_g128),
 * KVQ_ERR_INVALID otherwise.  Output pointers may not be NULL. */
int kvq_parse_dtype(const char* s, int32_t* k_bits, int32_t* v_bits, int32_t* group);

/* Bytes of the pool described by desc (num_blocks * num_kv_heads * SEG, SEG
 * = 1664 for k4v2_g128, 2176 for k4v4, 1152 for k2v2, 3200 for k8v4), or 0
 * if desc is NULL or unsupported.  Host only.  The pool is the paged cache
 * the KVarN backend writes into ("блоки кэша": the cache blocks of "Трюк
 * Huawei с KV-кэшем", section "Заявка, которая ломает привычный
 * компромисс", whose 3-5x capacity over FP16 is this byte count's ratio to
 * 512 bytes per token-head); per-token cache bytes are the quantity the
 * HBM-math section of "Kompresja pamięci podręcznej KV to decyzja
 * infrastrukturalna..." (encorp.ai) reasons with. */
size_t kvq_cache_bytes(const kvq_cache_desc* desc);

/* Assign physical blocks to sequences, host only (no device work): the job
 * of vLLM's paged block manager, which the KVarN backend plugs into ("Трюк
 * Huawei с KV-кэшем": lede, a ready vLLM backend; section "Заявка, которая
 * ломает привычный компромисс": the cache blocks; "KVarN vs TurboQuant"
 * (dothoosh.com), next-step list: fixed-size pages today, variable page
 * sizes announced).  Here it builds the tables the tests and benchmarks use.
 * Sequence b needs ceil(seq_lens[b]/block_size) blocks, which are taken in
 * order from a permutation of 0..num_blocks-1: the identity when
 * shuffle_seed == 0, otherwise a seeded shuffle (SplitMix64-driven
 * Fisher-Yates), as a fragmented vLLM block manager would hand them out.
 * block_table_out is [batch * max_blocks_per_seq] host int32, row-major,
 * unused entries set to -1; *blocks_used_out (may be NULL) gets the total.
 * Returns KVQ_ERR_POOL_EXHAUSTED if the pool is too small and
 * KVQ_ERR_INVALID if a sequence needs more than max_blocks_per_seq blocks. */
int kvq_block_table(int32_t num_blocks, int32_t block_size, const int32_t* seq_lens, int32_t batch,
                    int32_t max_blocks_per_seq, uint64_t shuffle_seed, int32_t* block_table_out,
                    int32_t* blocks_used_out);

/* slots_out[i] = block_table[seq_ids[i]][positions[i]/block_size] *
 * block_size + positions[i] % block_size, host only: vLLM's slot rule for
 * where a token's entry goes in the paged cache (the vLLM backend and its
 * cache blocks of "Трюк Huawei с KV-кэшем", section "Заявка, которая ломает
 * привычный компромисс"); kvq_quantize_append takes these slots.  An entry whose block
 * is -1 gives -1 (the write path then skips that token).  All pointers are
 * host memory; returns KVQ_ERR_INVALID for a negative position or a position
 * beyond the table row. */
int kvq_slot_mapping(const int32_t* block_table, int32_t max_blocks_per_seq,
                     const int32_t* positions, const int32_t* seq_ids, int32_t n_tokens,
                     int32_t block_size, int32_t* slots_out);

/* Cache write (the write path above, one kernel launch).
 * k, v: device, n_tokens rows; row t starts at element t*token_stride and
 * holds [num_kv_heads, 128] contiguous elements of in_dtype (F16 or BF16);
 * token_stride >= num_kv_heads*128 and a multiple of 8; k and v 16-byte
 * aligned.  slot_mapping: device int32 [n_tokens]; a negative slot skips the
 * token; a slot at or beyond num_blocks*16 is skipped and recorded as
 * KVQ_ERR_OUT_OF_RANGE in the device status word.  n_tokens == 0 is a no-op.
 * Tokens with distinct slots may share a block. */
int kvq_quantize_append(const kvq_cache_desc* desc, const void* k, const void* v,
                        kvq_dtype in_dtype, int32_t n_tokens, int64_t token_stride,
                        const int32_t* slot_mapping, void* stream);

/* Workspace bytes kvq_decode_attention needs for this problem on the current
 * device (split-K partials plus one int32 ticket per (sequence, kv head)),
 * or 0 for an unsupported geometry.  Host only (reads cached device
 * attributes).  The read path (scale folding at read time, "KVarN vs
 * TurboQuant" (dothoosh.com), pipeline list, fourth stage) is split across
 * the context because a long-context decode is bound by dragging the cache
 * through HBM (HBM-math section of "Kompresja pamięci podręcznej KV to
 * decyzja infrastrukturalna..." (encorp.ai)); these are the partial results
 * of the splits. */
size_t kvq_decode_workspace_bytes(const kvq_cache_desc* desc, int32_t batch, int32_t num_q_heads,
                                  int32_t max_seq_len);

/* Decode attention over the packed cache (the read path above, one kernel
 * launch: query rotation, paged split-K scan with scale folding, in-kernel
 * split combine by atomic ticket, output rotation).
 * q: device [batch, num_q_heads, 128] of q_dtype (F16, BF16 or F32).
 * block_table: device int32 [batch, max_blocks_per_seq]; seq_lens: device
 * int32 [batch], each in [0, max_seq_len]; max_seq_len sizes the split
 * grid and must be >= every seq_lens[b] (a longer sequence is truncated and
 * recorded as KVQ_ERR_OUT_OF_RANGE).  out: device [batch, num_q_heads, 128]
 * of out_dtype (F32, BF16 or F16); a sequence of length 0 gives zeros.
 * workspace: device, 16-byte aligned, at least kvq_decode_workspace_bytes
 * bytes, zero-filled by the caller once before its first use; every call
 * leaves it ready for the next call (tickets reset themselves).  Calls that
 * share a workspace must be ordered on one stream.  A block id outside the
 * pool is read as nothing (the token is skipped) and recorded as
 * KVQ_ERR_OUT_OF_RANGE in the device status word. */
int kvq_decode_attention(const kvq_cache_desc* desc, const void* q, kvq_dtype q_dtype,
                         int32_t batch, int32_t num_q_heads, const int32_t* block_table,
                         int32_t max_blocks_per_seq, const int32_t* seq_lens,
                         int32_t max_seq_len, float softmax_scale, void* out,
                         kvq_dtype out_dtype, void* workspace, size_t ws_bytes, void* stream);

/* As kvq_decode_attention / kvq_decode_workspace_bytes, with the split-K
 * granularity chosen by the caller: blocks_per_split physical blocks (of 16
 * tokens) per CTA; 0 picks the default.  A value that would cut a sequence
 * into more than 64 splits is raised to ceil(blocks / 64); a value above
 * 2048 blocks (32768 tokens) is lowered to 2048, or to that 64-split minimum
 * if it is larger, since a longer split loses accuracy in the kernel's
 * fixed-point probabilities (the default plan obeys the same bound).  The
 * workspace size depends on it. */
size_t kvq_decode_workspace_bytes_ex(const kvq_cache_desc* desc, int32_t batch,
                                     int32_t num_q_heads, int32_t max_seq_len,
                                     int32_t blocks_per_split);
int kvq_decode_attention_ex(const kvq_cache_desc* desc, const void* q, kvq_dtype q_dtype,
                            int32_t batch, int32_t num_q_heads, const int32_t* block_table,
                            int32_t max_blocks_per_seq, const int32_t* seq_lens,
                            int32_t max_seq_len, float softmax_scale, void* out,
                            kvq_dtype out_dtype, void* workspace, size_t ws_bytes,
                            int32_t blocks_per_split, void* stream);

/* One decode step of a cache that grows by one token per sequence: for each
 * sequence b with L = seq_lens[b] > 0, the new token's K and V rows (k_new,
 * v_new: device, row b at element b*token_stride, [num_kv_heads, 128] of
 * in_dtype F16 or BF16, 16-byte aligned, token_stride a multiple of 8 and
 * >= num_kv_heads*128; the rows of all batch sequences must be readable,
 * an empty sequence's row is read and ignored) are quantized into position
 * L-1, i.e. slot
 * block_table[b][(L-1)/16]*16 + (L-1)%16 -- the bytes kvq_quantize_append
 * writes for that slot -- and then the decode attention of
 * kvq_decode_attention runs over positions 0 .. L-1, the new token included.
 * One kernel launch: the CTA whose split holds position L-1 writes the new
 * row before it reads that block.  The same arguments, workspace and status
 * rules as kvq_decode_attention; the new token's block must not be read by
 * another sequence of the same call.  A seq_lens[b] outside [0,
 * max_seq_len] or beyond the table row appends nothing for that sequence
 * (the pool is left as it was), truncates its read as kvq_decode_attention
 * does and records KVQ_ERR_OUT_OF_RANGE.  Follows the KVarN write path (Hadamard
 * rotation, variance normalisation, asymmetric RTN) and read path (scale
 * folding at read time) of "KVarN vs TurboQuant" (dothoosh.com). */
int kvq_append_decode_attention(const kvq_cache_desc* desc, const void* k_new, const void* v_new,
                                kvq_dtype in_dtype, int64_t token_stride, const void* q,
                                kvq_dtype q_dtype, int32_t batch, int32_t num_q_heads,
                                const int32_t* block_table, int32_t max_blocks_per_seq,
                                const int32_t* seq_lens, int32_t max_seq_len, float softmax_scale,
                                void* out, kvq_dtype out_dtype, void* workspace, size_t ws_bytes,
                                void* stream);

/* kvq_decode_attention without a caller-provided workspace, for callers that
 * cannot allocate device memory at call time: code that runs inside a memory
 * pool or allocator that forbids runtime allocations, embedded or plugin
 * callers that receive only input and output buffers, and hosts whose
 * allocation calls would synchronise the device in the middle of a step.
 * (The pages have no counterpart; this is a packaging convenience.)
 * Arguments are those of kvq_decode_attention minus the workspace; the
 * default split plan is used.  The split-K scratch is a fixed 32 MiB array
 * inside the library's device image, so every GPU that loads the library
 * holds it until the process exits; a problem whose scratch would exceed
 * 32 MiB returns KVQ_ERR_WORKSPACE and launches nothing.  No allocation is
 * made by this call: it clears the scratch's ticket area with an
 * asynchronous memset and launches the decode kernel on the stream.  The
 * first call on each device looks up the scratch's device address (a one-time
 * set-up), so make that first call before any stream capture.  All calls on
 * a device share the one scratch array: calls that may overlap on the GPU
 * (different streams without ordering between them) race and give wrong
 * results; order them on one stream. */
int kvq_decode_attention_noalloc(const kvq_cache_desc* desc, const void* q, kvq_dtype q_dtype,
                                 int32_t batch, int32_t num_q_heads, const int32_t* block_table,
                                 int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                 int32_t max_seq_len, float softmax_scale, void* out,
                                 kvq_dtype out_dtype, void* stream);

/* ---- bf16 window of sink and recent tokens ------------------------------
 * "Kompresja pamięci podręcznej KV to decyzja infrastrukturalna..."
 * (encorp.ai), OSCAR section: the first ("sink") tokens and the most recent
 * tokens of a sequence stay in BF16 while the history is compressed.  Here
 * the history is the KVarN pool above, which keeps every position; the
 * window holds the raw rows of the positions read unquantized: for a
 * sequence of length L, positions t < sink and t >= L - recent.
 *
 * Window buffer (device memory the caller owns, 16-byte aligned): bf16
 * [num_seqs][num_kv_heads][sink + recent][2 (K, V)][128]; row t holds sink
 * position t (t < sink), row sink + t % recent holds recent position t.
 * Limits: sink in [0, 64], recent in [0, 1024]. */
typedef struct {
  void* data;
  int32_t num_seqs;
  int32_t num_kv_heads;
  int32_t sink;
  int32_t recent;
} kvq_window_desc;

/* Bytes of the window buffer: num_seqs * num_kv_heads * (sink + recent) *
 * 2 * 128 * 2; 0 for an invalid descriptor. */
size_t kvq_window_bytes(const kvq_window_desc* w);

/* Copy the raw K and V rows of n_tokens new tokens into the window: token n
 * (bf16, element (n, h, i) of k and v at n*token_stride + h*128 + i, as in
 * kvq_quantize_append: k and v 16-byte aligned, token_stride >=
 * num_kv_heads*128 and a multiple of 8) of sequence seq_ids[n] at position positions[n] goes
 * to its sink row when positions[n] < sink and to its ring row when
 * recent > 0; a negative sequence id skips the token.  seq_ids and
 * positions are device int32 arrays.  Call it for every appended token, as
 * well as kvq_quantize_append (the pool keeps every position, so a token
 * that leaves the recent window is read from the pool).  A sequence id >=
 * num_seqs or a negative position is skipped and recorded as
 * KVQ_ERR_OUT_OF_RANGE.  The tokens of one call must go to distinct rows
 * (at most one position per ring row of a sequence; the order of writes to
 * one row within a call is not defined).  Asynchronous on the stream. */
int kvq_window_append(const kvq_window_desc* w, const void* k, const void* v, int64_t token_stride,
                      const int32_t* seq_ids, const int32_t* positions, int32_t n_tokens, void* stream);

/* Workspace bytes of kvq_decode_attention_window (its split plan has one
 * record more per head than kvq_decode_attention's: the window's). */
size_t kvq_decode_window_workspace_bytes(const kvq_cache_desc* desc, int32_t batch, int32_t num_q_heads,
                                         int32_t max_seq_len);

/* kvq_decode_attention with the window's raw rows standing in at the window
 * positions of every sequence (sequence b of the batch is window sequence
 * b; w->num_kv_heads must equal the pool's): attention over positions
 * 0 .. L-1 where t < sink and t >= L - recent read the window and every
 * other position reads the pool, as kvq_decode_attention does.  One launch:
 * the split CTAs skip the window positions of the pool, and one more CTA per
 * (sequence, kv head) attends over the window rows (in fp32) and hands its
 * partial (o, m, l), rotated into the cache's domain, to the same split-K
 * merge.  Same arguments, workspace rules (sized by
 * kvq_decode_window_workspace_bytes) and status rules as
 * kvq_decode_attention; batch must not exceed w->num_seqs. */
int kvq_decode_attention_window(const kvq_cache_desc* desc, const kvq_window_desc* w, const void* q,
                                kvq_dtype q_dtype, int32_t batch, int32_t num_q_heads,
                                const int32_t* block_table, int32_t max_blocks_per_seq,
                                const int32_t* seq_lens, int32_t max_seq_len, float softmax_scale, void* out,
                                kvq_dtype out_dtype, void* workspace, size_t ws_bytes, void* stream);

/* Synchronise the stream, then read and clear the current device's status
 * word: KVQ_OK, or the first error that a kernel recorded since the last
 * read (KVQ_ERR_OUT_OF_RANGE, KVQ_ERR_DEVICE_TIMEOUT).  Returns
 * KVQ_ERR_CUDA if the synchronisation itself fails.  (The pages have no
 * counterpart: this is how the kernels, which never trap, report bad block
 * ids, slots and lengths and bounded waits that ran out.) */
int kvq_last_device_status(void* stream);

/* Failure-detection self-test (the pages have no counterpart).  Every
 * device-side wait of the kernels is bounded in time: after one second
 * (1000000 us, the largest value limit_us takes) it gives up and the kernel
 * records KVQ_ERR_DEVICE_TIMEOUT in the device status word, without a trap,
 * and returns with nothing of its own left in flight.  This call launches
 * one warp that makes such a wait, with the same code, on a barrier that
 * nothing ever arrives at, giving up after limit_us microseconds (1 ..
 * 1000000), so that a test can watch the path run: kvq_last_device_status
 * then returns KVQ_ERR_DEVICE_TIMEOUT and the context stays usable.
 * elapsed_ns (device memory, may be NULL) receives the time the wait took.
 * Asynchronous on the stream; KVQ_ERR_INVALID for limit_us out of range. */
int kvq_selftest_wait_timeout(uint32_t limit_us, uint64_t* elapsed_ns, void* stream);

/* Static description of a status code; never NULL.  (The pages have no
 * counterpart: error reporting of this library.) */
const char* kvq_error_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* KVQ_H */
