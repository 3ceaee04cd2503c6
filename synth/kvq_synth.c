/*
 * kvq_synth.c -- seeded, counter-based synthetic inputs for the KV-cache
 * tests and benchmark.
 *
 * This module holds no arithmetic of the quantisation method.  Its only job is
 * to produce the same input bits for the CPU oracle and for the CUDA library.
 * Every value is a pure function of (seed, tensor id, element index), so any
 * slice of a huge input can be regenerated on its own.
 *
 * Generator: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014; constants as published by Vigna) applied to
 * a counter; 53-bit uniforms in (0,1); normals by the Box-Muller transform
 * (cosine branch only, one normal per pair of uniforms).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static uint64_t sm64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static uint64_t stream_key(uint64_t seed, uint64_t tensor_id) {
  return sm64(sm64(seed) ^ sm64(tensor_id + 0x632BE59BD9B4E019ull));
}

/* Uniform in (0,1) from counter c of a stream. */
static double unif(uint64_t key, uint64_t c) {
  const uint64_t x = sm64(key ^ sm64(c));
  return ((double)(x >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

static double normal(uint64_t key, uint64_t e) {
  const double u1 = unif(key, 2 * e);
  const double u2 = unif(key, 2 * e + 1);
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

/* float -> bfloat16 bits, round to nearest even (finite inputs). */
static uint16_t to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  const uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

static uint16_t to_f16(float f) {
  _Float16 h = (_Float16)f;
  uint16_t u;
  memcpy(&u, &h, 2);
  return u;
}

/* dtype: 0 = fp16 bits, 1 = bf16 bits, 2 = float32, 3 = float64 */
static void store(void* out, int dtype, int64_t i, double v) {
  if (dtype == 0)
    ((uint16_t*)out)[i] = to_f16((float)v);
  else if (dtype == 1)
    ((uint16_t*)out)[i] = to_bf16((float)v);
  else if (dtype == 2)
    ((float*)out)[i] = (float)v;
  else
    ((double*)out)[i] = v;
}

/* n standard normals for elements [offset, offset + n) of a stream. */
void synth_normal(uint64_t seed, uint64_t tensor_id, int64_t offset, int64_t n, int dtype,
                  void* out) {
  const uint64_t key = stream_key(seed, tensor_id);
  for (int64_t i = 0; i < n; ++i) store(out, dtype, i, normal(key, (uint64_t)(offset + i)));
}

/* Per (kv head) outlier channels: n_out distinct channels of d, each with a
 * factor uniform in [fmin, fmax]; channels[h*n_out + k], factors likewise. */
void synth_outliers(uint64_t seed, uint64_t tensor_id, int32_t num_heads, int32_t d,
                    int32_t n_out, double fmin, double fmax, int32_t* channels,
                    double* factors) {
  const uint64_t key = stream_key(seed, tensor_id ^ 0x5A5A5A5Aull);
  for (int32_t h = 0; h < num_heads; ++h) {
    uint64_t c = (uint64_t)h << 32;
    for (int32_t k = 0; k < n_out; ++k) {
      int32_t ch;
      int dup;
      do {
        ch = (int32_t)(unif(key, c++) * d);
        if (ch >= d) ch = d - 1;
        dup = 0;
        for (int32_t m = 0; m < k; ++m) dup |= channels[h * n_out + m] == ch;
      } while (dup);
      channels[h * n_out + k] = ch;
      factors[h * n_out + k] = fmin + (fmax - fmin) * unif(key, c++);
    }
  }
}

/* K or V rows for tokens [t0, t0 + n_tokens) of a [T, Hkv, d] tensor:
 * N(0,1) per element times the head's outlier factor on its outlier channels,
 * rounded to dtype.  out is dense [n_tokens, Hkv, d]. */
void synth_kv(uint64_t seed, uint64_t tensor_id, int64_t t0, int64_t n_tokens,
              int32_t num_heads, int32_t d, int32_t n_out, double fmin, double fmax,
              int dtype, void* out) {
  const uint64_t key = stream_key(seed, tensor_id);
  int32_t ch[64 * 16];
  double fa[64 * 16];
  double scale[4096];
  if (num_heads > 64 || n_out > 16 || (int64_t)num_heads * d > 4096) return;
  synth_outliers(seed, tensor_id, num_heads, d, n_out, fmin, fmax, ch, fa);
  for (int32_t h = 0; h < num_heads; ++h) {
    for (int32_t i = 0; i < d; ++i) scale[h * d + i] = 1.0;
    for (int32_t k = 0; k < n_out; ++k) scale[h * d + ch[h * n_out + k]] = fa[h * n_out + k];
  }
  const int64_t row = (int64_t)num_heads * d;
  for (int64_t t = 0; t < n_tokens; ++t)
    for (int64_t e = 0; e < row; ++e)
      store(out, dtype, t * row + e, normal(key, (uint64_t)((t0 + t) * row + e)) * scale[e]);
}

/* n integers uniform in [lo, hi]. */
void synth_uniform_int(uint64_t seed, uint64_t tensor_id, int64_t n, int32_t lo, int32_t hi,
                       int32_t* out) {
  const uint64_t key = stream_key(seed, tensor_id);
  const double span = (double)hi - (double)lo + 1.0;
  for (int64_t i = 0; i < n; ++i) {
    int64_t v = lo + (int64_t)(unif(key, (uint64_t)i) * span);
    if (v > hi) v = hi;
    out[i] = (int32_t)v;
  }
}

/* A seeded permutation of 0..n-1 (Fisher-Yates driven by the stream). */
void synth_permutation(uint64_t seed, uint64_t tensor_id, int64_t n, int32_t* out) {
  const uint64_t key = stream_key(seed, tensor_id);
  for (int64_t i = 0; i < n; ++i) out[i] = (int32_t)i;
  for (int64_t i = n - 1; i > 0; --i) {
    int64_t j = (int64_t)(unif(key, (uint64_t)i) * (double)(i + 1));
    if (j > i) j = i;
    const int32_t tmp = out[i];
    out[i] = out[j];
    out[j] = tmp;
  }
}
