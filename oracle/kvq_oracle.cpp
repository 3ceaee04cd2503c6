// kvq_oracle.cpp -- CPU oracle for the KVarN k4v2_g128 quantized paged KV cache.
//
// TEST INFRASTRUCTURE ONLY (see kvq_oracle.h).  Plain double-precision
// restatement of the write path (rotate, normalise, asymmetric RTN, pack) and
// of decode attention over the packed paged cache.  Nothing here is blocked,
// fused or reordered beyond what the definitions say; speed is irrelevant.
#include "kvq_oracle.h"

#include <cmath>
#include <cstring>
#include <thread>
#include <vector>

namespace {

bool is_pow2(int32_t d) { return d > 0 && (d & (d - 1)) == 0; }

int popcount32(uint32_t x) {
  int n = 0;
  while (x) {
    n += x & 1u;
    x >>= 1;
  }
  return n;
}

bool bits_ok(int32_t b) { return b == 2 || b == 4 || b == 8; }

// Value of element i of an input row, widened to double.
double load_elem(const void* base, int32_t dtype, int64_t i) {
  if (dtype == KVQO_F16) return kvqo_f16_to_f64(static_cast<const uint16_t*>(base)[i]);
  if (dtype == KVQO_BF16) return kvqo_bf16_to_f64(static_cast<const uint16_t*>(base)[i]);
  return static_cast<double>(static_cast<const float*>(base)[i]);
}

// Bytes occupied by one code row of d elements at b bits.
size_t row_bytes(int32_t d, int32_t b) { return static_cast<size_t>(d) * b / 8; }

struct SegmentOffsets {
  size_t k_codes, v_codes, s_k, z_k, s_v, z_v, total;
};

SegmentOffsets segment_offsets(const kvqo_geom* g) {
  SegmentOffsets o;
  const size_t bs = static_cast<size_t>(g->block_size);
  o.k_codes = 0;
  o.v_codes = o.k_codes + bs * row_bytes(g->head_dim, g->k_bits);
  o.s_k = o.v_codes + bs * row_bytes(g->head_dim, g->v_bits);
  o.z_k = o.s_k + 2 * bs;
  o.s_v = o.z_k + 2 * bs;
  o.z_v = o.s_v + 2 * bs;
  o.total = o.z_v + 2 * bs;
  return o;
}

bool geom_ok(const kvqo_geom* g) {
  return g && g->num_blocks >= 0 && g->block_size > 0 && g->num_kv_heads > 0 &&
         is_pow2(g->head_dim) && bits_ok(g->k_bits) && bits_ok(g->v_bits) &&
         (g->head_dim * g->k_bits) % 8 == 0 && (g->head_dim * g->v_bits) % 8 == 0;
}

void put_u16(uint8_t* p, uint16_t v) {
  p[0] = static_cast<uint8_t>(v & 0xFF);
  p[1] = static_cast<uint8_t>(v >> 8);
}
uint16_t get_u16(const uint8_t* p) { return static_cast<uint16_t>(p[0] | (p[1] << 8)); }

// Element i of a code row at b bits: byte i*b/8, bit offset (i*b) mod 8.
void put_code(uint8_t* row, int32_t i, int32_t b, uint8_t c) {
  const int64_t bit = static_cast<int64_t>(i) * b;
  const int64_t byte = bit / 8;
  const int shift = static_cast<int>(bit % 8);
  const uint8_t mask = static_cast<uint8_t>(((1u << b) - 1u) << shift);
  row[byte] = static_cast<uint8_t>((row[byte] & ~mask) | ((c << shift) & mask));
}
uint8_t get_code(const uint8_t* row, int32_t i, int32_t b) {
  const int64_t bit = static_cast<int64_t>(i) * b;
  return static_cast<uint8_t>((row[bit / 8] >> (bit % 8)) & ((1u << b) - 1u));
}

}  // namespace

extern "C" {

// ---------------------------------------------------------------------------
// binary16 from double, written from the IEEE 754 definition: 1 sign bit,
// 5 exponent bits (bias 15), 10 fraction bits; subnormals are k * 2^-24.
// Round to nearest, ties to even (std::nearbyint in the default mode).
uint16_t kvqo_f64_to_f16(double x) {
  if (std::isnan(x)) return 0x7E00;
  const uint16_t sign = std::signbit(x) ? 0x8000 : 0;
  const double a = std::fabs(x);
  if (a == 0.0) return sign;
  if (std::isinf(a)) return static_cast<uint16_t>(sign | 0x7C00);
  int e;
  std::frexp(a, &e);  // a = m * 2^e, m in [0.5, 1): unbiased exponent is e-1
  const int E = e - 1;
  if (E < -14) {
    // subnormal range: value = k * 2^-24, k in [0, 1024]; k == 1024 is the
    // smallest normal, whose bit pattern is also 1024.
    const double k = std::nearbyint(std::ldexp(a, 24));
    return static_cast<uint16_t>(sign | static_cast<uint16_t>(k));
  }
  double k = std::nearbyint(std::ldexp(a, 10 - E));  // in [1024, 2048]
  int Eb = E;
  if (k >= 2048.0) {
    k = 1024.0;
    Eb += 1;
  }
  if (Eb > 15) return static_cast<uint16_t>(sign | 0x7C00);
  return static_cast<uint16_t>(sign | ((Eb + 15) << 10) | (static_cast<int>(k) - 1024));
}

double kvqo_f16_to_f64(uint16_t h) {
  const int s = (h >> 15) & 1;
  const int e = (h >> 10) & 0x1F;
  const int f = h & 0x3FF;
  double v;
  if (e == 0)
    v = std::ldexp(static_cast<double>(f), -24);
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = std::ldexp(static_cast<double>(1024 + f), e - 25);
  return s ? -v : v;
}

double kvqo_bf16_to_f64(uint16_t b) {
  const uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return static_cast<double>(f);
}

// ---------------------------------------------------------------------------
int kvqo_hadamard(int32_t d, int8_t* H) {
  if (!is_pow2(d) || !H) return -1;
  for (int32_t i = 0; i < d; ++i)
    for (int32_t j = 0; j < d; ++j)
      H[static_cast<size_t>(i) * d + j] = (popcount32(static_cast<uint32_t>(i & j)) & 1) ? -1 : 1;
  return 0;
}

int kvqo_rotate(int32_t d, const double* x, double* r) {
  if (!is_pow2(d) || !x || !r || x == r) return -1;
  std::vector<int8_t> H(static_cast<size_t>(d) * d);
  kvqo_hadamard(d, H.data());
  const double inv = 1.0 / std::sqrt(static_cast<double>(d));
  for (int32_t i = 0; i < d; ++i) {
    double acc = 0.0;
    for (int32_t j = 0; j < d; ++j) acc += H[static_cast<size_t>(i) * d + j] * x[j];
    r[i] = acc * inv;
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Steps 1-4 of the write path for one group: returns r, mu, sigma, lo, hi.
static void stats_of(int32_t d, const double* x, int32_t normalize, std::vector<double>& r,
                     double& mu, double& sigma, double& lo, double& hi) {
  r.assign(static_cast<size_t>(d), 0.0);
  kvqo_rotate(d, x, r.data());  // step 1: r = R x
  mu = 0.0;
  sigma = 1.0;
  if (normalize) {  // step 2: per-vector mean and population standard deviation
    double s = 0.0;
    for (int32_t i = 0; i < d; ++i) s += r[i];
    mu = s / d;
    double v = 0.0;
    for (int32_t i = 0; i < d; ++i) v += (r[i] - mu) * (r[i] - mu);
    sigma = std::sqrt(v / d);
    if (sigma == 0.0) sigma = 1.0;
  }
  // step 3: range of the normalised values u = (r - mu)/sigma
  lo = (r[0] - mu) / sigma;
  hi = lo;
  for (int32_t i = 1; i < d; ++i) {
    const double u = (r[i] - mu) / sigma;
    if (u < lo) lo = u;
    if (u > hi) hi = u;
  }
}

int kvqo_meta_exact(int32_t d, const double* x, int32_t bits, int32_t normalize, double* s_exact,
                    double* z_exact) {
  if (!is_pow2(d) || !x || !bits_ok(bits) || !s_exact || !z_exact) return -1;
  std::vector<double> r;
  double mu, sigma, lo, hi;
  stats_of(d, x, normalize, r, mu, sigma, lo, hi);
  const double levels = static_cast<double>((1 << bits) - 1);
  *s_exact = sigma * (hi - lo) / levels;
  *z_exact = mu + sigma * lo;
  return 0;
}

int kvqo_codes_given_meta(int32_t d, const double* r, int32_t bits, uint16_t S, uint16_t Z,
                          uint8_t* codes) {
  if (!is_pow2(d) || !r || !bits_ok(bits) || !codes) return -1;
  const double s = kvqo_f16_to_f64(S);
  const double z = kvqo_f16_to_f64(Z);
  const double top = static_cast<double>((1 << bits) - 1);
  for (int32_t i = 0; i < d; ++i) {
    if (s == 0.0) {  // a zero scale stores every element as code 0
      codes[i] = 0;
      continue;
    }
    double c = std::nearbyint((r[i] - z) / s);  // round half to even
    if (c < 0.0) c = 0.0;
    if (c > top) c = top;
    codes[i] = static_cast<uint8_t>(c);
  }
  return 0;
}

int kvqo_quotients(int32_t d, const double* r, uint16_t S, uint16_t Z, double* quot) {
  if (!is_pow2(d) || !r || !quot) return -1;
  const double s = kvqo_f16_to_f64(S);
  const double z = kvqo_f16_to_f64(Z);
  for (int32_t i = 0; i < d; ++i) quot[i] = (s == 0.0) ? 0.0 : (r[i] - z) / s;
  return 0;
}

int kvqo_quantize_vector(int32_t d, const double* x, int32_t bits, int32_t normalize,
                         uint8_t* codes, uint16_t* S, uint16_t* Z, double* r_out) {
  if (!is_pow2(d) || !x || !bits_ok(bits) || !codes || !S || !Z) return -1;
  std::vector<double> r;
  double mu, sigma, lo, hi;
  stats_of(d, x, normalize, r, mu, sigma, lo, hi);
  const double levels = static_cast<double>((1 << bits) - 1);
  *S = kvqo_f64_to_f16(sigma * (hi - lo) / levels);  // step 4
  *Z = kvqo_f64_to_f16(mu + sigma * lo);
  kvqo_codes_given_meta(d, r.data(), bits, *S, *Z, codes);  // step 5
  if (r_out) std::memcpy(r_out, r.data(), sizeof(double) * d);
  return 0;
}

int kvqo_dequantize_vector(int32_t d, const uint8_t* codes, uint16_t S, uint16_t Z, double* xhat,
                           double* rhat) {
  if (!is_pow2(d) || !codes || !xhat) return -1;
  const double s = kvqo_f16_to_f64(S);
  const double z = kvqo_f16_to_f64(Z);
  std::vector<double> rh(static_cast<size_t>(d));
  for (int32_t i = 0; i < d; ++i) rh[i] = s * codes[i] + z;  // step 6: r^ = S c + Z
  kvqo_rotate(d, rh.data(), xhat);                           // x^ = R r^ (R = R^T = R^-1)
  if (rhat) std::memcpy(rhat, rh.data(), sizeof(double) * d);
  return 0;
}

// ---------------------------------------------------------------------------
size_t kvqo_segment_bytes(const kvqo_geom* g) {
  if (!geom_ok(g)) return 0;
  return segment_offsets(g).total;
}

size_t kvqo_pool_bytes(const kvqo_geom* g) {
  if (!geom_ok(g)) return 0;
  return segment_offsets(g).total * static_cast<size_t>(g->num_blocks) * g->num_kv_heads;
}

static uint8_t* segment_ptr(const kvqo_geom* g, uint8_t* pool, int32_t p, int32_t h) {
  return pool + (static_cast<size_t>(p) * g->num_kv_heads + h) * segment_offsets(g).total;
}

int kvqo_pack_token(const kvqo_geom* g, uint8_t* pool, int32_t p, int32_t o, int32_t h,
                    const uint8_t* kcodes, uint16_t Sk, uint16_t Zk, const uint8_t* vcodes,
                    uint16_t Sv, uint16_t Zv) {
  if (!geom_ok(g) || !pool || !kcodes || !vcodes) return -1;
  if (p < 0 || p >= g->num_blocks || o < 0 || o >= g->block_size || h < 0 ||
      h >= g->num_kv_heads)
    return -5;
  const SegmentOffsets so = segment_offsets(g);
  uint8_t* seg = segment_ptr(g, pool, p, h);
  uint8_t* krow = seg + so.k_codes + static_cast<size_t>(o) * row_bytes(g->head_dim, g->k_bits);
  uint8_t* vrow = seg + so.v_codes + static_cast<size_t>(o) * row_bytes(g->head_dim, g->v_bits);
  for (int32_t i = 0; i < g->head_dim; ++i) put_code(krow, i, g->k_bits, kcodes[i]);
  for (int32_t i = 0; i < g->head_dim; ++i) put_code(vrow, i, g->v_bits, vcodes[i]);
  put_u16(seg + so.s_k + 2 * o, Sk);
  put_u16(seg + so.z_k + 2 * o, Zk);
  put_u16(seg + so.s_v + 2 * o, Sv);
  put_u16(seg + so.z_v + 2 * o, Zv);
  return 0;
}

int kvqo_unpack_token(const kvqo_geom* g, const uint8_t* pool, int32_t p, int32_t o, int32_t h,
                      uint8_t* kcodes, uint16_t* Sk, uint16_t* Zk, uint8_t* vcodes,
                      uint16_t* Sv, uint16_t* Zv) {
  if (!geom_ok(g) || !pool || !kcodes || !vcodes || !Sk || !Zk || !Sv || !Zv) return -1;
  if (p < 0 || p >= g->num_blocks || o < 0 || o >= g->block_size || h < 0 ||
      h >= g->num_kv_heads)
    return -5;
  const SegmentOffsets so = segment_offsets(g);
  const uint8_t* seg = segment_ptr(g, const_cast<uint8_t*>(pool), p, h);
  const uint8_t* krow =
      seg + so.k_codes + static_cast<size_t>(o) * row_bytes(g->head_dim, g->k_bits);
  const uint8_t* vrow =
      seg + so.v_codes + static_cast<size_t>(o) * row_bytes(g->head_dim, g->v_bits);
  for (int32_t i = 0; i < g->head_dim; ++i) kcodes[i] = get_code(krow, i, g->k_bits);
  for (int32_t i = 0; i < g->head_dim; ++i) vcodes[i] = get_code(vrow, i, g->v_bits);
  *Sk = get_u16(seg + so.s_k + 2 * o);
  *Zk = get_u16(seg + so.z_k + 2 * o);
  *Sv = get_u16(seg + so.s_v + 2 * o);
  *Zv = get_u16(seg + so.z_v + 2 * o);
  return 0;
}

int kvqo_quantize_append(const kvqo_geom* g, uint8_t* pool, const void* k, const void* v,
                         int32_t in_dtype, int32_t n_tokens, int64_t token_stride,
                         const int32_t* slots, int32_t normalize) {
  if (!geom_ok(g) || !pool || n_tokens < 0 || (n_tokens > 0 && (!k || !v || !slots))) return -1;
  if (in_dtype != KVQO_F16 && in_dtype != KVQO_BF16 && in_dtype != KVQO_F32) return -1;
  const int32_t d = g->head_dim;
  const int32_t H = g->num_kv_heads;
  if (token_stride < static_cast<int64_t>(H) * d) return -1;
  for (int32_t t = 0; t < n_tokens; ++t) {
    if (slots[t] < 0) continue;
    if (slots[t] / g->block_size >= g->num_blocks) return -5;
  }
  std::vector<double> xk(d), xv(d);
  std::vector<uint8_t> ck(d), cv(d);
  for (int32_t t = 0; t < n_tokens; ++t) {
    const int32_t slot = slots[t];
    if (slot < 0) continue;  // padding token: nothing is written
    const int32_t p = slot / g->block_size;
    const int32_t o = slot % g->block_size;
    for (int32_t h = 0; h < H; ++h) {
      const int64_t base = static_cast<int64_t>(t) * token_stride + static_cast<int64_t>(h) * d;
      for (int32_t i = 0; i < d; ++i) {
        xk[i] = load_elem(k, in_dtype, base + i);
        xv[i] = load_elem(v, in_dtype, base + i);
      }
      uint16_t Sk, Zk, Sv, Zv;
      kvqo_quantize_vector(d, xk.data(), g->k_bits, normalize, ck.data(), &Sk, &Zk, nullptr);
      kvqo_quantize_vector(d, xv.data(), g->v_bits, normalize, cv.data(), &Sv, &Zv, nullptr);
      kvqo_pack_token(g, pool, p, o, h, ck.data(), Sk, Zk, cv.data(), Sv, Zv);
    }
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Every cached token of one (sequence, kv head): dequantized K and V rows in
// the original domain (form 0), or the raw codes plus widened metadata S_K,
// Z_K, S_V, Z_V (form 1).  Returns -5 for a block id outside the pool.
struct Gathered {
  std::vector<double> khat, vhat;   // [L, d] original domain
  std::vector<uint8_t> kc, vc;      // [L, d] codes
  std::vector<double> meta;         // [L, 4]
};

static int gather_tokens(const kvqo_geom* g, const uint8_t* pool, int32_t h,
                         const int32_t* bt_row, int32_t seq_len, int32_t form, Gathered& out) {
  const int32_t d = g->head_dim;
  const size_t n = static_cast<size_t>(seq_len) * d;
  if (form == 0) {
    out.khat.assign(n, 0.0);
    out.vhat.assign(n, 0.0);
  } else {
    out.kc.assign(n, 0);
    out.vc.assign(n, 0);
    out.meta.assign(static_cast<size_t>(seq_len) * 4, 0.0);
  }
  std::vector<uint8_t> ck(d), cv(d);
  for (int32_t t = 0; t < seq_len; ++t) {
    const int32_t p = bt_row[t / g->block_size];  // paged gather
    const int32_t o = t % g->block_size;
    if (p < 0 || p >= g->num_blocks) return -5;
    uint16_t Sk, Zk, Sv, Zv;
    kvqo_unpack_token(g, pool, p, o, h, ck.data(), &Sk, &Zk, cv.data(), &Sv, &Zv);
    const size_t row = static_cast<size_t>(t) * d;
    if (form == 0) {
      kvqo_dequantize_vector(d, ck.data(), Sk, Zk, &out.khat[row], nullptr);
      kvqo_dequantize_vector(d, cv.data(), Sv, Zv, &out.vhat[row], nullptr);
    } else {
      std::memcpy(&out.kc[row], ck.data(), d);
      std::memcpy(&out.vc[row], cv.data(), d);
      out.meta[4 * static_cast<size_t>(t) + 0] = kvqo_f16_to_f64(Sk);
      out.meta[4 * static_cast<size_t>(t) + 1] = kvqo_f16_to_f64(Zk);
      out.meta[4 * static_cast<size_t>(t) + 2] = kvqo_f16_to_f64(Sv);
      out.meta[4 * static_cast<size_t>(t) + 3] = kvqo_f16_to_f64(Zv);
    }
  }
  return 0;
}

// Softmax weights of scores s (max subtracted), their sum in *l.
static std::vector<double> softmax_weights(const std::vector<double>& s, double* l) {
  double m = s[0];
  for (size_t t = 1; t < s.size(); ++t) m = s[t] > m ? s[t] : m;
  std::vector<double> p(s.size());
  *l = 0.0;
  for (size_t t = 0; t < s.size(); ++t) {
    p[t] = std::exp(s[t] - m);
    *l += p[t];
  }
  return p;
}

// softmax(s) then o = sum_t p_t * rows_t, all in double.
static void softmax_combine(int32_t d, const std::vector<double>& s,
                            const std::vector<double>& rows, double* out) {
  double l;
  const std::vector<double> p = softmax_weights(s, &l);
  for (int32_t i = 0; i < d; ++i) out[i] = 0.0;
  for (size_t t = 0; t < s.size(); ++t)
    for (int32_t i = 0; i < d; ++i) out[i] += p[t] * rows[t * d + i];
  for (int32_t i = 0; i < d; ++i) out[i] /= l;
}

// One query head against the gathered tokens of its kv head.
static void attend(int32_t d, int32_t seq_len, const double* q, double tau, int32_t form,
                   const Gathered& gt, double* out) {
  if (seq_len == 0) {
    for (int32_t i = 0; i < d; ++i) out[i] = 0.0;
    return;
  }
  std::vector<double> s(static_cast<size_t>(seq_len));
  if (form == 0) {
    // plain definition: s_t = tau <q, k^_t>, o = softmax(s) . v^
    for (int32_t t = 0; t < seq_len; ++t) {
      double dot = 0.0;
      for (int32_t i = 0; i < d; ++i) dot += q[i] * gt.khat[static_cast<size_t>(t) * d + i];
      s[t] = tau * dot;
    }
    softmax_combine(d, s, gt.vhat, out);
    return;
  }
  // form 1, scale folding at read time in the rotated domain:
  //   q~ = R q,  s_t = tau (S_K,t * sum_i q~_i c_K,t,i + Z_K,t * sum_i q~_i)
  //   o~ = (sum_t p_t S_V,t c_V,t + (sum_t p_t Z_V,t) 1) / sum_t p_t,  o = R o~
  std::vector<double> qr(d), orot(d, 0.0);
  kvqo_rotate(d, q, qr.data());
  double qsum = 0.0;
  for (int32_t i = 0; i < d; ++i) qsum += qr[i];
  for (int32_t t = 0; t < seq_len; ++t) {
    double dot = 0.0;
    for (int32_t i = 0; i < d; ++i) dot += qr[i] * gt.kc[static_cast<size_t>(t) * d + i];
    s[t] = tau * (gt.meta[4 * static_cast<size_t>(t)] * dot +
                  gt.meta[4 * static_cast<size_t>(t) + 1] * qsum);
  }
  double l;
  const std::vector<double> p = softmax_weights(s, &l);
  double zeta = 0.0;
  for (int32_t t = 0; t < seq_len; ++t) {
    const double ps = p[t] * gt.meta[4 * static_cast<size_t>(t) + 2];
    for (int32_t i = 0; i < d; ++i) orot[i] += ps * gt.vc[static_cast<size_t>(t) * d + i];
    zeta += p[t] * gt.meta[4 * static_cast<size_t>(t) + 3];
  }
  for (int32_t i = 0; i < d; ++i) orot[i] = (orot[i] + zeta) / l;
  kvqo_rotate(d, orot.data(), out);
}

int kvqo_decode_one(const kvqo_geom* g, const uint8_t* pool, const void* q_row, int32_t q_dtype,
                    int32_t num_q_heads, int32_t j, const int32_t* block_table_row,
                    int32_t seq_len, double softmax_scale, int32_t form, double* out) {
  if (!geom_ok(g) || !pool || !q_row || !out || num_q_heads <= 0 ||
      num_q_heads % g->num_kv_heads != 0 || j < 0 || j >= num_q_heads || seq_len < 0 ||
      (seq_len > 0 && !block_table_row) || (form != 0 && form != 1))
    return -1;
  const int32_t d = g->head_dim;
  const int32_t G = num_q_heads / g->num_kv_heads;
  const int32_t h = j / G;
  const double tau = softmax_scale > 0.0 ? softmax_scale : 1.0 / std::sqrt(static_cast<double>(d));
  std::vector<double> q(d);
  for (int32_t i = 0; i < d; ++i) q[i] = load_elem(q_row, q_dtype, i);
  Gathered gt;
  const int rc = gather_tokens(g, pool, h, block_table_row, seq_len, form, gt);
  if (rc) return rc;
  attend(d, seq_len, q.data(), tau, form, gt, out);
  return 0;
}

namespace {
struct DecodeJob {
  const kvqo_geom* g;
  const uint8_t* pool;
  const void* q;
  int32_t q_dtype, batch, hq, mbps;
  const int32_t* bt;
  const int32_t* lens;
  double tau;
  int32_t form;
  double* out;
  const uint16_t* win;  // bf16 window of sink and recent tokens (form 0 only), or null
  int32_t sink, recent;
};

// Element (b, h, row, kv, i) of a window buffer.
size_t win_index(int32_t H, int32_t rows, int32_t d, int32_t b, int32_t h, int32_t row, int32_t kv,
                 int32_t i) {
  return ((((static_cast<size_t>(b) * H + h) * rows + row) * 2 + kv) * d) + i;
}

// All query heads of one (sequence b, kv head h): the tokens are dequantized
// once and every query head of the group attends to them.
int run_pair(const DecodeJob& J, int32_t b, int32_t h) {
  const int32_t d = J.g->head_dim;
  const int32_t G = J.hq / J.g->num_kv_heads;
  const int32_t L = J.lens[b];
  if (L < 0 || (L + J.g->block_size - 1) / J.g->block_size > J.mbps) return -1;
  Gathered gt;
  const int rc = gather_tokens(J.g, J.pool, h, J.bt + static_cast<size_t>(b) * J.mbps, L,
                               J.form, gt);
  if (rc) return rc;
  if (J.win) {  // window positions take the raw rows
    const int32_t rows = J.sink + J.recent;
    for (int32_t t = 0; t < L; ++t) {
      int32_t row = -1;
      if (t < J.sink)
        row = t;
      else if (J.recent > 0 && t >= L - J.recent)
        row = J.sink + t % J.recent;
      if (row < 0) continue;
      for (int32_t i = 0; i < d; ++i) {
        gt.khat[static_cast<size_t>(t) * d + i] =
            kvqo_bf16_to_f64(J.win[win_index(J.g->num_kv_heads, rows, d, b, h, row, 0, i)]);
        gt.vhat[static_cast<size_t>(t) * d + i] =
            kvqo_bf16_to_f64(J.win[win_index(J.g->num_kv_heads, rows, d, b, h, row, 1, i)]);
      }
    }
  }
  std::vector<double> q(d);
  for (int32_t jj = 0; jj < G; ++jj) {
    const int32_t j = h * G + jj;
    const int64_t qbase = (static_cast<int64_t>(b) * J.hq + j) * d;
    for (int32_t i = 0; i < d; ++i) q[i] = load_elem(J.q, J.q_dtype, qbase + i);
    attend(d, L, q.data(), J.tau, J.form, gt, J.out + qbase);
  }
  return 0;
}

// Every (sequence, kv head) pair of a decode job, on up to nthreads threads.
int run_all(const DecodeJob& J, int32_t nthreads) {
  const int32_t H = J.g->num_kv_heads;
  const int64_t pairs = static_cast<int64_t>(J.batch) * H;
  if (nthreads <= 1 || pairs <= 1) {
    for (int64_t w = 0; w < pairs; ++w) {
      const int rc = run_pair(J, static_cast<int32_t>(w / H), static_cast<int32_t>(w % H));
      if (rc) return rc;
    }
    return 0;
  }
  const int32_t nt = static_cast<int32_t>(nthreads < pairs ? nthreads : pairs);
  std::vector<int> rcs(static_cast<size_t>(nt), 0);
  std::vector<std::thread> pool_threads;
  for (int32_t w = 0; w < nt; ++w) {
    pool_threads.emplace_back([&, w]() {
      for (int64_t x = w; x < pairs; x += nt) {
        const int rc = run_pair(J, static_cast<int32_t>(x / H), static_cast<int32_t>(x % H));
        if (rc) {
          rcs[w] = rc;
          return;
        }
      }
    });
  }
  for (auto& th : pool_threads) th.join();
  for (int rc : rcs)
    if (rc) return rc;
  return 0;
}
}  // namespace

int kvqo_decode_attention(const kvqo_geom* g, const uint8_t* pool, const void* q, int32_t q_dtype,
                          int32_t batch, int32_t num_q_heads, const int32_t* block_table,
                          int32_t max_blocks_per_seq, const int32_t* seq_lens,
                          double softmax_scale, int32_t form, int32_t nthreads, double* out) {
  if (!geom_ok(g) || !pool || !q || !out || !seq_lens || !block_table || batch < 0 ||
      num_q_heads <= 0 || num_q_heads % g->num_kv_heads != 0 || max_blocks_per_seq < 0 ||
      (form != 0 && form != 1))
    return -1;
  DecodeJob J{g,
              pool,
              q,
              q_dtype,
              batch,
              num_q_heads,
              max_blocks_per_seq,
              block_table,
              seq_lens,
              softmax_scale > 0.0 ? softmax_scale
                                  : 1.0 / std::sqrt(static_cast<double>(g->head_dim)),
              form,
              out,
              nullptr,
              0,
              0};
  return run_all(J, nthreads);
}

int kvqo_window_append(int32_t d, int32_t num_kv_heads, int32_t sink, int32_t recent, int32_t num_seqs,
                       uint16_t* win, const uint16_t* k, const uint16_t* v, int64_t token_stride,
                       const int32_t* seq_ids, const int32_t* positions, int32_t n_tokens) {
  if (!is_pow2(d) || num_kv_heads <= 0 || sink < 0 || recent < 0 || num_seqs < 0 || n_tokens < 0 ||
      (n_tokens > 0 && (!win || !k || !v || !seq_ids || !positions)))
    return -1;
  const int32_t rows = sink + recent;
  for (int32_t n = 0; n < n_tokens; ++n) {
    const int32_t b = seq_ids[n], t = positions[n];
    if (b < 0) continue;
    if (b >= num_seqs || t < 0) return -1;
    for (int32_t h = 0; h < num_kv_heads; ++h) {
      const int64_t src = static_cast<int64_t>(n) * token_stride + static_cast<int64_t>(h) * d;
      for (int32_t kv = 0; kv < 2; ++kv) {
        const uint16_t* x = kv == 0 ? k : v;
        if (t < sink)
          for (int32_t i = 0; i < d; ++i) win[win_index(num_kv_heads, rows, d, b, h, t, kv, i)] = x[src + i];
        if (recent > 0)
          for (int32_t i = 0; i < d; ++i)
            win[win_index(num_kv_heads, rows, d, b, h, sink + t % recent, kv, i)] = x[src + i];
      }
    }
  }
  return 0;
}

int kvqo_decode_attention_window(const kvqo_geom* g, const uint8_t* pool, const uint16_t* win,
                                 int32_t sink, int32_t recent, const void* q, int32_t q_dtype,
                                 int32_t batch, int32_t num_q_heads, const int32_t* block_table,
                                 int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                 double softmax_scale, int32_t nthreads, double* out) {
  if (!geom_ok(g) || !pool || !q || !out || !seq_lens || !block_table || batch < 0 ||
      num_q_heads <= 0 || num_q_heads % g->num_kv_heads != 0 || max_blocks_per_seq < 0 || sink < 0 ||
      recent < 0 || (sink + recent > 0 && !win))
    return -1;
  DecodeJob J{g,
              pool,
              q,
              q_dtype,
              batch,
              num_q_heads,
              max_blocks_per_seq,
              block_table,
              seq_lens,
              softmax_scale > 0.0 ? softmax_scale : 1.0 / std::sqrt(static_cast<double>(g->head_dim)),
              0,
              out,
              sink + recent > 0 ? win : nullptr,
              sink,
              recent};
  return run_all(J, nthreads);
}

int kvqo_attention_dense(int32_t d, int32_t num_kv_heads, const void* k, const void* v,
                         int32_t kv_dtype, int64_t token_stride, int32_t seq_len,
                         const void* q_row, int32_t q_dtype, int32_t num_q_heads, int32_t j,
                         double softmax_scale, double* out) {
  if (!is_pow2(d) || num_kv_heads <= 0 || !q_row || !out || seq_len < 0 ||
      (seq_len > 0 && (!k || !v)) || num_q_heads % num_kv_heads != 0 || j < 0 ||
      j >= num_q_heads)
    return -1;
  const int32_t h = j / (num_q_heads / num_kv_heads);
  const double tau = softmax_scale > 0.0 ? softmax_scale : 1.0 / std::sqrt(static_cast<double>(d));
  if (seq_len == 0) {
    for (int32_t i = 0; i < d; ++i) out[i] = 0.0;
    return 0;
  }
  std::vector<double> s(static_cast<size_t>(seq_len)), rows(static_cast<size_t>(seq_len) * d);
  for (int32_t t = 0; t < seq_len; ++t) {
    const int64_t base = static_cast<int64_t>(t) * token_stride + static_cast<int64_t>(h) * d;
    double dot = 0.0;
    for (int32_t i = 0; i < d; ++i) {
      dot += load_elem(q_row, q_dtype, i) * load_elem(k, kv_dtype, base + i);
      rows[static_cast<size_t>(t) * d + i] = load_elem(v, kv_dtype, base + i);
    }
    s[t] = tau * dot;
  }
  softmax_combine(d, s, rows, out);
  return 0;
}

// ---------------------------------------------------------------------------
double kvqo_packed_bytes_per_token_head(int32_t d, int32_t k_bits, int32_t v_bits) {
  return static_cast<double>(d) * (k_bits + v_bits) / 8.0 + 4.0 * 2.0;
}

double kvqo_dense_bytes_per_token(int32_t layers, int32_t num_kv_heads, int32_t d,
                                  int32_t bytes_per_elem) {
  return static_cast<double>(layers) * num_kv_heads * d * 2.0 * bytes_per_elem;
}

}  // extern "C"
