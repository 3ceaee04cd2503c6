// kvq_host.cu -- the extern "C" entry points declared in include/kvq.h:
// argument validation, the split-K plan, host-only block-table helpers, the
// device status word, and the kernel launches.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "kvq_internal.cuh"

namespace kvq {

namespace {

__device__ int g_kvq_status = 0;

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {0};
int* g_status_ptr[kMaxDevices] = {nullptr};
std::mutex g_attr_mutex;

bool supported_desc(const kvq_cache_desc* d) {
  return d->head_dim == kHeadDim && d->group == kHeadDim && d->block_size == kBlockSize &&
         preset_supported(d->k_bits, d->v_bits);
}

int check_desc(const kvq_cache_desc* d) {
  if (!d) return KVQ_ERR_INVALID;
  if (d->num_blocks < 0 || d->num_kv_heads <= 0 || d->block_size <= 0 || d->head_dim <= 0 ||
      d->k_bits <= 0 || d->v_bits <= 0 || d->group <= 0)
    return KVQ_ERR_INVALID;
  if (!supported_desc(d)) return KVQ_ERR_UNSUPPORTED;
  return KVQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

}  // namespace

// Fixed split-K scratch for kvq_decode_attention_noalloc.  It lives in the
// module image, so every GPU that loads this library holds the full 32 MiB
// until the process exits.  Host code must never pass the symbol itself to
// a kernel (on the host it is only a stand-in): the device address comes
// from cudaGetSymbolAddress, once per device, with that device current.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;
static __device__ __align__(256) uint8_t g_kvq_scratch[kStaticScratchBytes];
void* g_scratch_ptr[kMaxDevices] = {nullptr};

void* device_scratch_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_attr_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_kvq_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

int* device_status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  if (g_status_ptr[dev]) return g_status_ptr[dev];
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_kvq_status) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lk(g_attr_mutex);
  g_status_ptr[dev] = static_cast<int*>(p);
  return g_status_ptr[dev];
}

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < kMaxDevices && g_sm_count[dev] > 0) return g_sm_count[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  if (dev < kMaxDevices) {
    std::lock_guard<std::mutex> lk(g_attr_mutex);
    g_sm_count[dev] = n;
  }
  return n;
}

// Split-K plan.  The context of every sequence is cut into nsplit splits of
// blocks_per_split blocks; one CTA owns one (sequence, kv head, split) and
// walks it in chunks of decode_chunk_blocks() blocks.  The default picks
// nsplit (at most decode_max_splits()) by a small cost model: CTAs run in
// waves of (SMs x resident CTAs per SM), a CTA costs its chunks plus a fixed
// start-up worth about two chunks (the first loads, the query rotation, the
// partial record), and every extra split adds a tenth of a chunk of merge
// work.  Default splits are whole chunks.  A requested blocks_per_split is
// raised if it would need more splits than the cap, and lowered to
// decode_max_split_blocks(), the block ids a CTA stages in shared memory;
// a sequence longer than cap x that many blocks is not supported.

int plan_decode(int32_t batch, int32_t num_kv_heads, int32_t num_q_heads, int32_t max_seq_len,
                int32_t bps_request, DecodePlan* plan, int32_t extra_records) {
  if (batch < 0 || num_kv_heads <= 0 || num_q_heads <= 0 || max_seq_len < 0 || bps_request < 0)
    return KVQ_ERR_INVALID;
  const int64_t nb = (static_cast<int64_t>(max_seq_len) + kBlockSize - 1) / kBlockSize;
  const int64_t cap = decode_max_splits();
  const int64_t cb = decode_chunk_blocks();
  const int64_t bmax = decode_max_split_blocks();
  if (nb > bmax * cap) return KVQ_ERR_UNSUPPORTED;
  int64_t bps = bps_request;
  if (nb == 0) {
    bps = 1;
  } else if (bps == 0) {
    const int64_t units = static_cast<int64_t>(batch) * num_kv_heads;
    const int64_t slots = static_cast<int64_t>(device_sm_count()) * decode_ctas_per_sm();
    const int64_t bmax_c = (bmax + cb - 1) / cb * cb;  // in whole chunks
    double best = 1e300;
    bps = std::min((nb + cb - 1) / cb * cb, bmax_c);
    int64_t last = -1;
    for (int64_t n = 1; n <= cap && n <= nb; ++n) {
      const int64_t b = ((nb + n - 1) / n + cb - 1) / cb * cb;  // whole chunks
      const int64_t ns = (nb + b - 1) / b;
      if (ns > cap || b == last || b > bmax_c) continue;
      last = b;
      const int64_t waves = (units * ns + slots - 1) / slots;
      const double cost = static_cast<double>(waves) * (static_cast<double>(b) / cb + 2.0) + 0.1 * ns;
      if (cost < best) {
        best = cost;
        bps = b;
      }
    }
  } else {
    if ((nb + bps - 1) / bps > cap) bps = (nb + cap - 1) / cap;
    if (bps > bmax) bps = bmax;  // (cap x bmax blocks cover the sequence)
  }
  const int64_t nsplit = nb > 0 ? (nb + bps - 1) / bps : 1;
  plan->blocks_per_split = static_cast<int32_t>(bps);
  plan->nsplit = static_cast<int32_t>(nsplit);
  plan->nrec = static_cast<int32_t>(nsplit + extra_records);
  plan->ticket_bytes = ((static_cast<size_t>(batch) * num_kv_heads * sizeof(int32_t)) + 255) / 256 * 256;
  plan->partial_bytes = static_cast<size_t>(batch) * num_q_heads * plan->nrec * kPartialFloats * sizeof(float);
  plan->total_bytes = plan->ticket_bytes + plan->partial_bytes;
  return KVQ_OK;
}

}  // namespace kvq

using namespace kvq;

extern "C" {

const char* kvq_error_string(int status) {
  switch (status) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported geometry or preset";
    case KVQ_ERR_CUDA: return "CUDA runtime error";
    case KVQ_ERR_POOL_EXHAUSTED: return "block pool exhausted";
    case KVQ_ERR_OUT_OF_RANGE: return "block id or slot outside the pool";
    case KVQ_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case KVQ_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    default: return "unknown status";
  }
}

int kvq_parse_dtype(const char* s, int32_t* k_bits, int32_t* v_bits, int32_t* group) {
  if (!s || !k_bits || !v_bits || !group) return KVQ_ERR_INVALID;
  const char* prefix = "kvarn_k";
  if (std::strncmp(s, prefix, std::strlen(prefix)) != 0) return KVQ_ERR_INVALID;
  const char* p = s + std::strlen(prefix);
  auto read_int = [&](int32_t* out) -> bool {
    if (*p < '0' || *p > '9') return false;
    int64_t v = 0;
    while (*p >= '0' && *p <= '9') {
      v = v * 10 + (*p - '0');
      if (v > 1 << 20) return false;
      ++p;
    }
    *out = static_cast<int32_t>(v);
    return true;
  };
  int32_t kb, vb, g;
  if (!read_int(&kb) || *p++ != 'v' || !read_int(&vb) || *p++ != '_' || *p++ != 'g' ||
      !read_int(&g) || *p != '\0')
    return KVQ_ERR_INVALID;
  *k_bits = kb;
  *v_bits = vb;
  *group = g;
  return (preset_supported(kb, vb) && g == kHeadDim) ? KVQ_OK : KVQ_ERR_UNSUPPORTED;
}

size_t kvq_cache_bytes(const kvq_cache_desc* desc) {
  if (check_desc(desc) != KVQ_OK) return 0;
  return static_cast<size_t>(desc->num_blocks) * desc->num_kv_heads * seg_bytes(desc->k_bits, desc->v_bits);
}

int kvq_block_table(int32_t num_blocks, int32_t block_size, const int32_t* seq_lens, int32_t batch,
                    int32_t max_blocks_per_seq, uint64_t shuffle_seed, int32_t* block_table_out,
                    int32_t* blocks_used_out) {
  if (num_blocks < 0 || block_size <= 0 || batch < 0 || max_blocks_per_seq < 0 ||
      (batch > 0 && (!seq_lens || !block_table_out)))
    return KVQ_ERR_INVALID;
  int64_t need = 0;
  for (int32_t b = 0; b < batch; ++b) {
    if (seq_lens[b] < 0) return KVQ_ERR_INVALID;
    const int64_t nb = (static_cast<int64_t>(seq_lens[b]) + block_size - 1) / block_size;
    if (nb > max_blocks_per_seq) return KVQ_ERR_INVALID;
    need += nb;
  }
  if (need > num_blocks) return KVQ_ERR_POOL_EXHAUSTED;
  int32_t* order = static_cast<int32_t*>(std::malloc(sizeof(int32_t) * (num_blocks > 0 ? num_blocks : 1)));
  if (!order) return KVQ_ERR_INVALID;
  for (int32_t i = 0; i < num_blocks; ++i) order[i] = i;
  if (shuffle_seed != 0) {
    const uint64_t key = splitmix64(shuffle_seed);
    for (int32_t i = num_blocks - 1; i > 0; --i) {
      const uint64_t r = splitmix64(key ^ splitmix64(static_cast<uint64_t>(i)));
      const int32_t j = static_cast<int32_t>(r % static_cast<uint64_t>(i + 1));
      const int32_t t = order[i];
      order[i] = order[j];
      order[j] = t;
    }
  }
  int64_t pos = 0;
  for (int32_t b = 0; b < batch; ++b) {
    const int64_t nb = (static_cast<int64_t>(seq_lens[b]) + block_size - 1) / block_size;
    int32_t* row = block_table_out + static_cast<int64_t>(b) * max_blocks_per_seq;
    for (int64_t i = 0; i < max_blocks_per_seq; ++i) row[i] = i < nb ? order[pos + i] : -1;
    pos += nb;
  }
  std::free(order);
  if (blocks_used_out) *blocks_used_out = static_cast<int32_t>(need);
  return KVQ_OK;
}

int kvq_slot_mapping(const int32_t* block_table, int32_t max_blocks_per_seq,
                     const int32_t* positions, const int32_t* seq_ids, int32_t n_tokens,
                     int32_t block_size, int32_t* slots_out) {
  if (n_tokens < 0 || block_size <= 0 || max_blocks_per_seq < 0 ||
      (n_tokens > 0 && (!block_table || !positions || !seq_ids || !slots_out)))
    return KVQ_ERR_INVALID;
  for (int32_t i = 0; i < n_tokens; ++i) {
    if (positions[i] < 0 || seq_ids[i] < 0) return KVQ_ERR_INVALID;
    const int32_t blk = positions[i] / block_size;
    if (blk >= max_blocks_per_seq) return KVQ_ERR_INVALID;
    const int32_t p = block_table[static_cast<int64_t>(seq_ids[i]) * max_blocks_per_seq + blk];
    slots_out[i] = p < 0 ? -1 : p * block_size + positions[i] % block_size;
  }
  return KVQ_OK;
}

int kvq_quantize_append(const kvq_cache_desc* desc, const void* k, const void* v,
                        kvq_dtype in_dtype, int32_t n_tokens, int64_t token_stride,
                        const int32_t* slot_mapping, void* stream) {
  int rc = check_desc(desc);
  if (rc != KVQ_OK) return rc;
  if (n_tokens < 0) return KVQ_ERR_INVALID;
  if (in_dtype != KVQ_F16 && in_dtype != KVQ_BF16) return in_dtype == KVQ_F32 ? KVQ_ERR_UNSUPPORTED : KVQ_ERR_INVALID;
  if (n_tokens == 0) return KVQ_OK;
  if (!desc->pool || !k || !v || !slot_mapping) return KVQ_ERR_INVALID;
  if (!aligned16(desc->pool) || !aligned16(k) || !aligned16(v)) return KVQ_ERR_INVALID;
  if (token_stride < static_cast<int64_t>(desc->num_kv_heads) * kHeadDim || token_stride % 8 != 0)
    return KVQ_ERR_INVALID;
  QuantizeArgs a;
  a.pool = static_cast<uint8_t*>(desc->pool);
  a.num_blocks = desc->num_blocks;
  a.num_kv_heads = desc->num_kv_heads;
  a.k = k;
  a.v = v;
  a.in_dtype = in_dtype;
  a.n_tokens = n_tokens;
  a.token_stride = token_stride;
  a.slots = slot_mapping;
  a.k_bits = desc->k_bits;
  a.v_bits = desc->v_bits;
  a.status = device_status_ptr();
  if (!a.status) return KVQ_ERR_CUDA;
  return launch_quantize(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

size_t kvq_decode_workspace_bytes_ex(const kvq_cache_desc* desc, int32_t batch, int32_t num_q_heads,
                                     int32_t max_seq_len, int32_t blocks_per_split) {
  if (check_desc(desc) != KVQ_OK || num_q_heads <= 0 || num_q_heads % desc->num_kv_heads != 0)
    return 0;
  DecodePlan plan;
  if (plan_decode(batch, desc->num_kv_heads, num_q_heads, max_seq_len, blocks_per_split, &plan) != KVQ_OK)
    return 0;
  return plan.total_bytes;
}

size_t kvq_decode_workspace_bytes(const kvq_cache_desc* desc, int32_t batch, int32_t num_q_heads,
                                  int32_t max_seq_len) {
  return kvq_decode_workspace_bytes_ex(desc, batch, num_q_heads, max_seq_len, 0);
}

namespace {
// The new-token rows of a fused append + decode call.
struct AppendRows {
  const void* k;
  const void* v;
  kvq_dtype dtype;
  int64_t token_stride;
};

int decode_impl(const kvq_cache_desc* desc, const void* q, kvq_dtype q_dtype, int32_t batch, int32_t num_q_heads,
                const int32_t* block_table, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                int32_t max_seq_len, float softmax_scale, void* out, kvq_dtype out_dtype, void* workspace,
                size_t ws_bytes, int32_t blocks_per_split, void* stream, const AppendRows* app,
                const kvq_window_desc* win = nullptr) {
  int rc = check_desc(desc);
  if (rc != KVQ_OK) return rc;
  if (batch < 0 || num_q_heads <= 0 || max_blocks_per_seq < 0 || max_seq_len < 0 ||
      blocks_per_split < 0)
    return KVQ_ERR_INVALID;
  if (q_dtype < KVQ_F16 || q_dtype > KVQ_F32 || out_dtype < KVQ_F16 || out_dtype > KVQ_F32)
    return KVQ_ERR_INVALID;
  if (num_q_heads % desc->num_kv_heads != 0) return KVQ_ERR_UNSUPPORTED;
  const int32_t G = num_q_heads / desc->num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return KVQ_ERR_UNSUPPORTED;
  if (batch == 0) return KVQ_OK;
  if (!desc->pool || !q || !block_table || !seq_lens || !out) return KVQ_ERR_INVALID;
  if (!aligned16(desc->pool)) return KVQ_ERR_INVALID;
  const bool use_win = win != nullptr && win->sink + win->recent > 0;
  if (use_win && batch > win->num_seqs) return KVQ_ERR_INVALID;
  DecodePlan plan;
  rc = plan_decode(batch, desc->num_kv_heads, num_q_heads, max_seq_len, blocks_per_split, &plan, use_win ? 1 : 0);
  if (rc != KVQ_OK) return rc;
  if (!workspace || !aligned16(workspace) || ws_bytes < plan.total_bytes) return KVQ_ERR_WORKSPACE;
  if (!std::isfinite(softmax_scale)) return KVQ_ERR_INVALID;
  const float tau = softmax_scale > 0.0f ? softmax_scale : 0.088388347648318440550f;
  DecodeArgs a;
  a.pool = static_cast<const uint8_t*>(desc->pool);
  a.num_blocks = desc->num_blocks;
  a.num_kv_heads = desc->num_kv_heads;
  a.q = q;
  a.q_dtype = q_dtype;
  a.batch = batch;
  a.num_q_heads = num_q_heads;
  a.block_table = block_table;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.seq_lens = seq_lens;
  a.max_seq_len = max_seq_len;
  a.scale_log2 = tau * 1.4426950408889634074f;
  a.out = out;
  a.out_dtype = out_dtype;
  a.tickets = static_cast<int32_t*>(workspace);
  a.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + plan.ticket_bytes);
  a.blocks_per_split = plan.blocks_per_split;
  a.nsplit = plan.nsplit;
  a.k_bits = desc->k_bits;
  a.v_bits = desc->v_bits;
  a.status = device_status_ptr();
  a.k_new = app ? static_cast<const uint8_t*>(app->k) : nullptr;
  a.v_new = app ? static_cast<const uint8_t*>(app->v) : nullptr;
  a.new_bf16 = app && app->dtype == KVQ_BF16 ? 1 : 0;
  a.new_stride_bytes = app ? app->token_stride * 2 : 0;
  a.win = use_win ? static_cast<const uint16_t*>(win->data) : nullptr;
  a.win_sink = use_win ? win->sink : 0;
  a.win_recent = use_win ? win->recent : 0;
  a.nrec = plan.nrec;
  if (!a.status) return KVQ_ERR_CUDA;
  return launch_decode(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}
}  // namespace

int kvq_decode_attention_ex(const kvq_cache_desc* desc, const void* q, kvq_dtype q_dtype,
                            int32_t batch, int32_t num_q_heads, const int32_t* block_table,
                            int32_t max_blocks_per_seq, const int32_t* seq_lens,
                            int32_t max_seq_len, float softmax_scale, void* out,
                            kvq_dtype out_dtype, void* workspace, size_t ws_bytes,
                            int32_t blocks_per_split, void* stream) {
  return decode_impl(desc, q, q_dtype, batch, num_q_heads, block_table, max_blocks_per_seq, seq_lens, max_seq_len,
                     softmax_scale, out, out_dtype, workspace, ws_bytes, blocks_per_split, stream, nullptr);
}

int kvq_append_decode_attention(const kvq_cache_desc* desc, const void* k_new, const void* v_new,
                                kvq_dtype in_dtype, int64_t token_stride, const void* q,
                                kvq_dtype q_dtype, int32_t batch, int32_t num_q_heads,
                                const int32_t* block_table, int32_t max_blocks_per_seq,
                                const int32_t* seq_lens, int32_t max_seq_len, float softmax_scale,
                                void* out, kvq_dtype out_dtype, void* workspace, size_t ws_bytes,
                                void* stream) {
  const int rc = check_desc(desc);
  if (rc != KVQ_OK) return rc;
  if (in_dtype != KVQ_F16 && in_dtype != KVQ_BF16) return KVQ_ERR_INVALID;
  if (batch > 0 && (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new))) return KVQ_ERR_INVALID;
  if (token_stride < static_cast<int64_t>(desc->num_kv_heads) * kHeadDim || token_stride % 8 != 0)
    return KVQ_ERR_INVALID;
  const AppendRows app{k_new, v_new, in_dtype, token_stride};
  return decode_impl(desc, q, q_dtype, batch, num_q_heads, block_table, max_blocks_per_seq, seq_lens, max_seq_len,
                     softmax_scale, out, out_dtype, workspace, ws_bytes, 0, stream, &app);
}

namespace {
// The geometry of a window descriptor; with need_data, also its buffer.
int check_window(const kvq_window_desc* w, bool need_data = true) {
  if (!w || w->num_seqs < 0 || w->num_kv_heads <= 0 || w->sink < 0 || w->sink > kMaxWindowSink ||
      w->recent < 0 || w->recent > kMaxWindowRecent)
    return KVQ_ERR_INVALID;
  if (need_data && w->num_seqs > 0 && w->sink + w->recent > 0 && (!w->data || !aligned16(w->data)))
    return KVQ_ERR_INVALID;
  return KVQ_OK;
}
}  // namespace

size_t kvq_window_bytes(const kvq_window_desc* w) {
  if (check_window(w, false) != KVQ_OK) return 0;
  return static_cast<size_t>(w->num_seqs) * w->num_kv_heads * (w->sink + w->recent) * 2 * kHeadDim * 2;
}

int kvq_window_append(const kvq_window_desc* w, const void* k, const void* v, int64_t token_stride,
                      const int32_t* seq_ids, const int32_t* positions, int32_t n_tokens, void* stream) {
  int rc = check_window(w);
  if (rc != KVQ_OK) return rc;
  if (n_tokens < 0) return KVQ_ERR_INVALID;
  if (n_tokens == 0 || w->sink + w->recent == 0 || w->num_seqs == 0) return KVQ_OK;
  if (!k || !v || !seq_ids || !positions || !aligned16(k) || !aligned16(v)) return KVQ_ERR_INVALID;
  if (token_stride < static_cast<int64_t>(w->num_kv_heads) * kHeadDim || token_stride % 8 != 0)
    return KVQ_ERR_INVALID;
  WindowAppendArgs a;
  a.win = static_cast<uint16_t*>(w->data);
  a.num_seqs = w->num_seqs;
  a.num_kv_heads = w->num_kv_heads;
  a.sink = w->sink;
  a.recent = w->recent;
  a.k = static_cast<const uint16_t*>(k);
  a.v = static_cast<const uint16_t*>(v);
  a.token_stride = token_stride;
  a.seq_ids = seq_ids;
  a.positions = positions;
  a.n_tokens = n_tokens;
  a.status = device_status_ptr();
  if (!a.status) return KVQ_ERR_CUDA;
  return launch_window_append(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

size_t kvq_decode_window_workspace_bytes(const kvq_cache_desc* desc, int32_t batch, int32_t num_q_heads,
                                         int32_t max_seq_len) {
  if (check_desc(desc) != KVQ_OK || num_q_heads <= 0 || num_q_heads % desc->num_kv_heads != 0) return 0;
  DecodePlan plan;
  if (plan_decode(batch, desc->num_kv_heads, num_q_heads, max_seq_len, 0, &plan, 1) != KVQ_OK) return 0;
  return plan.total_bytes;
}

int kvq_decode_attention_window(const kvq_cache_desc* desc, const kvq_window_desc* w, const void* q,
                                kvq_dtype q_dtype, int32_t batch, int32_t num_q_heads,
                                const int32_t* block_table, int32_t max_blocks_per_seq,
                                const int32_t* seq_lens, int32_t max_seq_len, float softmax_scale, void* out,
                                kvq_dtype out_dtype, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_desc(desc);
  if (rc != KVQ_OK) return rc;
  rc = check_window(w);
  if (rc != KVQ_OK) return rc;
  if (w->num_kv_heads != desc->num_kv_heads) return KVQ_ERR_INVALID;
  return decode_impl(desc, q, q_dtype, batch, num_q_heads, block_table, max_blocks_per_seq, seq_lens, max_seq_len,
                     softmax_scale, out, out_dtype, workspace, ws_bytes, 0, stream, nullptr, w);
}

int kvq_decode_attention(const kvq_cache_desc* desc, const void* q, kvq_dtype q_dtype, int32_t batch,
                         int32_t num_q_heads, const int32_t* block_table, int32_t max_blocks_per_seq,
                         const int32_t* seq_lens, int32_t max_seq_len, float softmax_scale, void* out,
                         kvq_dtype out_dtype, void* workspace, size_t ws_bytes, void* stream) {
  return kvq_decode_attention_ex(desc, q, q_dtype, batch, num_q_heads, block_table, max_blocks_per_seq,
                                 seq_lens, max_seq_len, softmax_scale, out, out_dtype, workspace, ws_bytes,
                                 0, stream);
}

int kvq_decode_attention_noalloc(const kvq_cache_desc* desc, const void* q, kvq_dtype q_dtype,
                                 int32_t batch, int32_t num_q_heads, const int32_t* block_table,
                                 int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                 int32_t max_seq_len, float softmax_scale, void* out,
                                 kvq_dtype out_dtype, void* stream) {
  int rc = check_desc(desc);
  if (rc != KVQ_OK) return rc;
  // the argument rules of kvq_decode_attention, checked before the scratch
  // is sized (decode_impl repeats them)
  if (batch < 0 || num_q_heads <= 0) return KVQ_ERR_INVALID;
  if (num_q_heads % desc->num_kv_heads != 0) return KVQ_ERR_UNSUPPORTED;
  if (batch == 0) return KVQ_OK;
  DecodePlan plan;
  rc = plan_decode(batch, desc->num_kv_heads, num_q_heads, max_seq_len, 0, &plan);
  if (rc != KVQ_OK) return rc;
  if (plan.total_bytes > kStaticScratchBytes) return KVQ_ERR_WORKSPACE;  // beyond the fixed scratch
  void* scratch = device_scratch_ptr();
  if (!scratch) return KVQ_ERR_CUDA;
  // The scratch keeps whatever the previous call left; the tickets must start
  // at zero (the partials are always written before they are read).
  if (cudaMemsetAsync(scratch, 0, plan.ticket_bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KVQ_ERR_CUDA;
  return kvq_decode_attention_ex(desc, q, q_dtype, batch, num_q_heads, block_table, max_blocks_per_seq,
                                 seq_lens, max_seq_len, softmax_scale, out, out_dtype, scratch,
                                 kStaticScratchBytes, 0, stream);
}

int kvq_selftest_wait_timeout(uint32_t limit_us, uint64_t* elapsed_ns, void* stream) {
  if (limit_us == 0 || static_cast<uint64_t>(limit_us) * 1000u > wait_limit_ns()) return KVQ_ERR_INVALID;
  int* status = device_status_ptr();
  if (!status) return KVQ_ERR_CUDA;
  return launch_wait_probe(status, static_cast<uint64_t>(limit_us) * 1000u, elapsed_ns,
                           static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KVQ_OK
             : KVQ_ERR_CUDA;
}

int kvq_last_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return KVQ_ERR_CUDA;
  int host = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&host, g_kvq_status, sizeof(int)) != cudaSuccess) return KVQ_ERR_CUDA;
  if (host != 0 && cudaMemcpyToSymbol(g_kvq_status, &zero, sizeof(int)) != cudaSuccess)
    return KVQ_ERR_CUDA;
  return host;
}

}  // extern "C"
