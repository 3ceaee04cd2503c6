/*
 * kvq_oracle.h -- CPU oracle for the KVarN k4v2_g128 quantized paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow, obviously-correct
 * restatement of what the cache write path and the decode read path compute.
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * load it.  It shares no code, header, table or helper with the CUDA library
 * under bit_kv_cache_18_b200/; neither side includes or links the other.
 *
 * Arithmetic is IEEE double throughout, except for the two places where the
 * format itself stores fp16 (the per-group scale S and zero point Z), which
 * are rounded to binary16 with round-to-nearest-even exactly as stored.
 *
 * Sources (the method is described on five web pages, none of which prints a
 * formula, a bit layout or code):
 *   - "Трюк Huawei с KV-кэшем" (beyondheadline.xyz), section "Заявка, которая
 *     ломает привычный компромисс": the cache blocks are run through a Hadamard
 *     rotation, variance normalisation and asymmetric low-bit quantisation,
 *     4-bit keys and 2-bit values by default, flag kvarn_k4v2_g128.
 *   - "KVarN vs TurboQuant" (dothoosh.com), the four-stage pipeline list:
 *     Hadamard rotation; variance normalisation; asymmetric round-to-nearest
 *     quantisation; scale folding at read time.
 *   - "Kompresja pamięci podręcznej KV..." (encorp.ai), section on HBM math:
 *     Llama-3.1-70B BF16 needs about 0.31 MB of KV cache per token, about
 *     40 GB at 128K tokens.
 *
 * Readings taken where the pages are silent:
 *   - R = H/sqrt(d) with H the natural-order Sylvester Hadamard matrix,
 *     H[i][j] = (-1)^popcount(i & j); no random signs ("no calibration").
 *   - Variance normalisation = per-vector standardisation u = (r - mu)/sigma
 *     with population sigma; sigma = 0 is replaced by 1.
 *   - One group of 128 elements along head_dim per (token, kv head, K|V).
 *   - Asymmetric min/max RTN: S = fp16(sigma*(hi-lo)/(2^b-1)),
 *     Z = fp16(mu + sigma*lo), c = clamp(rne((r - Z)/S), 0, 2^b-1) using the
 *     stored S and Z; S == 0 gives all-zero codes.  Dequant: r^ = S*c + Z.
 *   - Segment layout per (physical block p, kv head h), index p*Hkv + h:
 *     [K codes: block_size rows of d*kb/8 bytes][V codes: rows of d*vb/8]
 *     [S_K x block_size][Z_K x block_size][S_V x block_size][Z_V x block_size]
 *     (fp16, little endian).  Element i of a code row sits at byte i*b/8,
 *     bit offset (i*b) mod 8 (low nibble first for 4-bit).
 *   - Decode: s_t = tau * <q, k^_t> in the original domain, softmax, o = sum
 *     p_t v^_t; tau = 1/sqrt(d) unless given; query head j reads kv head
 *     j / (Hq/Hkv).  Sequence length 0 gives a zero output.
 */
#ifndef KVQ_ORACLE_H
#define KVQ_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Input element types understood by the oracle. */
enum { KVQO_F16 = 0, KVQO_BF16 = 1, KVQO_F32 = 2 };

/* Geometry of one cache pool.  d must be a power of two; bits in {2,4,8}. */
typedef struct {
  int32_t num_blocks;
  int32_t block_size;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t k_bits;
  int32_t v_bits;
} kvqo_geom;

/* ---- binary16 / bfloat16 ------------------------------------------------ */
uint16_t kvqo_f64_to_f16(double x);  /* IEEE 754 binary16, RNE, overflow->inf */
double kvqo_f16_to_f64(uint16_t h);
double kvqo_bf16_to_f64(uint16_t b);

/* ---- rotation ----------------------------------------------------------- */
/* H[i*d + j] = (-1)^popcount(i&j).  Returns 0, or -1 if d is not a power of 2. */
int kvqo_hadamard(int32_t d, int8_t* H);
/* r = (H x)/sqrt(d) by the explicit matrix product.  x and r may not alias. */
int kvqo_rotate(int32_t d, const double* x, double* r);

/* ---- one group ---------------------------------------------------------- */
/* Full write-path definition for one vector x (length d, group = d).
 * normalize = 0 replaces mu by 0 and sigma by 1 (used by the invariant test).
 * Outputs: codes[d] in 0..2^bits-1, stored fp16 bits of S and Z, and the
 * rotated vector r[d] (may be NULL).  Returns 0 on success. */
int kvqo_quantize_vector(int32_t d, const double* x, int32_t bits, int32_t normalize,
                         uint8_t* codes, uint16_t* S, uint16_t* Z, double* r);
/* Step 5 alone: codes of an already rotated vector r under given fp16 S, Z. */
int kvqo_codes_given_meta(int32_t d, const double* r, int32_t bits, uint16_t S, uint16_t Z,
                          uint8_t* codes);
/* The unrounded quotient (r_i - Z)/S for every element, for tie accounting. */
int kvqo_quotients(int32_t d, const double* r, uint16_t S, uint16_t Z, double* quot);
/* The two unrounded metadata values sigma*(hi-lo)/(2^b-1) and mu + sigma*lo. */
int kvqo_meta_exact(int32_t d, const double* x, int32_t bits, int32_t normalize,
                    double* s_exact, double* z_exact);
/* x^ = R (S*c + Z); rhat (may be NULL) receives S*c + Z. */
int kvqo_dequantize_vector(int32_t d, const uint8_t* codes, uint16_t S, uint16_t Z,
                           double* xhat, double* rhat);

/* ---- paged pool --------------------------------------------------------- */
size_t kvqo_segment_bytes(const kvqo_geom* g);
size_t kvqo_pool_bytes(const kvqo_geom* g);
/* Write one token's packed K/V group into (block p, row o) of kv head h. */
int kvqo_pack_token(const kvqo_geom* g, uint8_t* pool, int32_t p, int32_t o, int32_t h,
                    const uint8_t* kcodes, uint16_t Sk, uint16_t Zk,
                    const uint8_t* vcodes, uint16_t Sv, uint16_t Zv);
/* Read them back. */
int kvqo_unpack_token(const kvqo_geom* g, const uint8_t* pool, int32_t p, int32_t o, int32_t h,
                      uint8_t* kcodes, uint16_t* Sk, uint16_t* Zk,
                      uint8_t* vcodes, uint16_t* Sv, uint16_t* Zv);

/* Cache write: K and V are [n_tokens] rows of [Hkv, d] elements of in_dtype,
 * row t starting at element t*token_stride.  slots[t] < 0 skips token t;
 * otherwise block = slots[t] / block_size, row = slots[t] % block_size.
 * Returns 0, -1 for bad arguments, -5 for a slot outside the pool. */
int kvqo_quantize_append(const kvqo_geom* g, uint8_t* pool, const void* k, const void* v,
                         int32_t in_dtype, int32_t n_tokens, int64_t token_stride,
                         const int32_t* slots, int32_t normalize);

/* Decode attention for one (sequence b, query head j).  q_row is the d
 * elements of that head (q_dtype).  form 0 = plain definition (dequantize to
 * the original domain, explicit softmax); form 1 = rotated-domain folding of
 * S and Z into q.k and p.v with one rotation of q and of the output.  out[d]
 * in double.  Returns 0, -1 bad args, -5 block id outside the pool. */
int kvqo_decode_one(const kvqo_geom* g, const uint8_t* pool, const void* q_row, int32_t q_dtype,
                    int32_t num_q_heads, int32_t j, const int32_t* block_table_row,
                    int32_t seq_len, double softmax_scale, int32_t form, double* out);

/* All (b, j) pairs: q [batch, Hq, d], out [batch, Hq, d] double.
 * nthreads <= 1 runs on the calling thread; otherwise std::thread workers
 * split the (b, j) pairs (used only to time the oracle on many cores). */
int kvqo_decode_attention(const kvqo_geom* g, const uint8_t* pool, const void* q, int32_t q_dtype,
                          int32_t batch, int32_t num_q_heads, const int32_t* block_table,
                          int32_t max_blocks_per_seq, const int32_t* seq_lens,
                          double softmax_scale, int32_t form, int32_t nthreads, double* out);

/* Unquantized attention in double for one query head j over seq_len raw K/V
 * rows laid out as in the write path (row t at element t*token_stride, each
 * row [Hkv, d]); used only to report the error that quantisation adds. */
int kvqo_attention_dense(int32_t d, int32_t num_kv_heads, const void* k, const void* v,
                         int32_t kv_dtype, int64_t token_stride, int32_t seq_len,
                         const void* q_row, int32_t q_dtype, int32_t num_q_heads, int32_t j,
                         double softmax_scale, double* out);

/* ---- bf16 window of sink and recent tokens ------------------------------
 * ("Kompresja pamięci podręcznej KV..." (encorp.ai), OSCAR section: the first
 * "sink" tokens and the most recent tokens stay in BF16 while the history is
 * compressed.)  Reading: for a sequence of length L, position t is kept raw
 * when t < sink or t >= L - recent; every other position reads its quantized
 * token from the pool, which holds every position.  The raw rows live in a
 * window buffer of bf16 [num_seqs][num_kv_heads][sink + recent][2 (K, V)][d]:
 * row t holds sink position t (t < sink), row sink + t % recent holds a
 * recent position t.
 *
 * Window append: token n (its K and V rows laid out as in the write path,
 * element (n, h, i) at n*token_stride + h*d + i, bf16 bits) of sequence
 * seq_ids[n] at position positions[n] is copied to its sink row when
 * positions[n] < sink and to its ring row when recent > 0; tokens with a
 * negative sequence id are skipped.  Returns 0, or -1 for bad arguments. */
int kvqo_window_append(int32_t d, int32_t num_kv_heads, int32_t sink, int32_t recent, int32_t num_seqs,
                       uint16_t* win, const uint16_t* k, const uint16_t* v, int64_t token_stride,
                       const int32_t* seq_ids, const int32_t* positions, int32_t n_tokens);

/* Decode attention over the quantized pool with the window's raw rows
 * standing in at the window positions (sequence b uses window sequence b).
 * Plain original-domain definition, as kvqo_decode_attention form 0. */
int kvqo_decode_attention_window(const kvqo_geom* g, const uint8_t* pool, const uint16_t* win,
                                 int32_t sink, int32_t recent, const void* q, int32_t q_dtype,
                                 int32_t batch, int32_t num_q_heads, const int32_t* block_table,
                                 int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                 double softmax_scale, int32_t nthreads, double* out);

/* ---- byte accounting ---------------------------------------------------- */
/* Packed bytes per token per kv head: d*(kb+vb)/8 codes + 4 fp16 metadata. */
double kvqo_packed_bytes_per_token_head(int32_t d, int32_t k_bits, int32_t v_bits);
/* Unquantized bytes per token of a model: layers * Hkv * d * 2 (K,V) * elem. */
double kvqo_dense_bytes_per_token(int32_t layers, int32_t num_kv_heads, int32_t d,
                                  int32_t bytes_per_elem);

#ifdef __cplusplus
}
#endif
#endif
