// kvq_window.cu -- the bf16 window of sink and recent tokens: row copies.
//
// "Kompresja pamięci podręcznej KV..." (encorp.ai), OSCAR section: the first
// ("sink") tokens and the most recent tokens of a sequence stay in BF16 while
// the history is compressed.  The pool keeps every position; the window
// keeps the raw rows of the positions read unquantized.  Layout (include/
// kvq.h): bf16 [num_seqs][num_kv_heads][sink + recent][2 (K, V)][128], row t
// for sink position t, row sink + t % recent for recent position t.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

// One warp per (token, kv head): lanes 0-15 move the K row, lanes 16-31 the
// V row, 16 bytes each, into the sink row and/or the ring row.
__global__ void __launch_bounds__(256) window_append_kernel(WindowAppendArgs a) {
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  if (wid >= static_cast<int64_t>(a.n_tokens) * a.num_kv_heads) return;
  const int n = static_cast<int>(wid / a.num_kv_heads), h = static_cast<int>(wid % a.num_kv_heads);
  const int sq = a.seq_ids[n], t = a.positions[n];
  if (sq < 0) return;
  if (sq >= a.num_seqs || t < 0) {
    if (lane == 0 && h == 0) record_status(a.status, KVQ_ERR_OUT_OF_RANGE);
    return;
  }
  const int kv = lane >> 4, piece = lane & 15;
  const uint16_t* src = (kv == 0 ? a.k : a.v) + static_cast<int64_t>(n) * a.token_stride + h * kHeadDim;
  const uint4 x = __ldg(reinterpret_cast<const uint4*>(src) + piece);
  const int rows = a.sink + a.recent;
  uint16_t* base = a.win + (static_cast<int64_t>(sq) * a.num_kv_heads + h) * rows * (2 * kHeadDim) + kv * kHeadDim;
  if (t < a.sink) reinterpret_cast<uint4*>(base + static_cast<int64_t>(t) * (2 * kHeadDim))[piece] = x;
  if (a.recent > 0)
    reinterpret_cast<uint4*>(base + static_cast<int64_t>(a.sink + t % a.recent) * (2 * kHeadDim))[piece] = x;
}

}  // namespace

cudaError_t launch_window_append(const WindowAppendArgs& a, cudaStream_t stream) {
  const int64_t warps = static_cast<int64_t>(a.n_tokens) * a.num_kv_heads;
  if (warps == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((warps + 7) / 8));
  return launch_pdl(window_append_kernel, grid, dim3(256), 0, stream, a);
}

}  // namespace kvq
