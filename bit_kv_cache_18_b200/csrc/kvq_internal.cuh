// kvq_internal.cuh -- shared pieces of the sm_100a KV-cache kernels.
//
// Format constants of the k4v2_g128 pool (see include/kvq.h for the layout and
// the pages it follows), the device status word, small PTX wrappers and the
// launcher entry points that kvq_host.cu calls.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

// ---- pool formats (presets k<KB>v<VB>_g128, 16-token blocks) ----------------
// A segment (block, kv head): 16 rows of K codes, 16 rows of V codes (element
// i of a b-bit row at bit b*i of the row, little-endian), then S_K, Z_K,
// S_V, Z_V as 16 fp16 each.
constexpr int kHeadDim = 128;
constexpr int kBlockSize = 16;
template <int KB, int VB>
struct Fmt {
  static constexpr int kKBits = KB;
  static constexpr int kVBits = VB;
  static constexpr int kKRowBytes = kHeadDim * KB / 8;
  static constexpr int kVRowBytes = kHeadDim * VB / 8;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kBlockSize * kKRowBytes;
  static constexpr int kOffSK = kOffV + kBlockSize * kVRowBytes;
  static constexpr int kOffZK = kOffSK + 2 * kBlockSize;
  static constexpr int kOffSV = kOffZK + 2 * kBlockSize;
  static constexpr int kOffZV = kOffSV + 2 * kBlockSize;
  static constexpr int kSegBytes = kOffZV + 2 * kBlockSize;
  static_assert(kSegBytes % 128 == 0, "segments stay 128-byte aligned");
};
static_assert(Fmt<4, 2>::kSegBytes == 1664, "the default preset's segment");
// The presets built: k4v2 (the pages' default), k4v4, k2v2, k8v4.
constexpr bool preset_supported(int kb, int vb) {
  return (kb == 4 && (vb == 2 || vb == 4)) || (kb == 2 && vb == 2) || (kb == 8 && vb == 4);
}
constexpr int seg_bytes(int kb, int vb) { return kBlockSize * kHeadDim * (kb + vb) / 8 + 8 * kBlockSize; }

// Split-K partial record in the decode workspace: o~[128], m (log2 domain), l.
constexpr int kPartialFloats = kHeadDim + 4;

// ---- device status word ----------------------------------------------------
// One int per device (a module-scope __device__ variable in kvq_host.cu whose
// address the host looks up once per device and passes to every kernel).
// Kernels record the first error with a compare-and-swap from 0;
// kvq_last_device_status reads and clears it.
__device__ __forceinline__ void record_status(int* status, int code) { atomicCAS(status, 0, code); }
int* device_status_ptr();  // nullptr if the lookup failed

// ---- small helpers -----------------------------------------------------------
__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float load_as_f32(const void* p, int dtype, int64_t i) {
  if (dtype == KVQ_F32) return static_cast<const float*>(p)[i];
  const uint16_t u = static_cast<const uint16_t*>(p)[i];
  if (dtype == KVQ_BF16) return __uint_as_float(static_cast<uint32_t>(u) << 16);
  return __half2float(__ushort_as_half(u));
}

__device__ __forceinline__ void store_from_f32(void* p, int dtype, int64_t i, float v) {
  if (dtype == KVQ_F32)
    static_cast<float*>(p)[i] = v;
  else if (dtype == KVQ_BF16)
    static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else
    static_cast<__half*>(p)[i] = __float2half_rn(v);
}

// ---- write path, one warp per head vector ------------------------------------
// Rotate, normalise, quantise and pack one 128-element K (is_v false: KB
// bits) or V (VB bits) head vector (bf16 or fp16, 16-byte aligned at src)
// into row row_in_block of segment seg, lane l holding elements 4l .. 4l+3:
// the two lowest butterfly stages in registers, the five others by shuffles,
// the statistics as warp reductions.  The arithmetic is that of the bulk
// write path (moments of y = sqrt(128) r, fp16 S and Z, codes from the stored
// S and Z); only the summation order differs.  Each lane then owns whole
// bytes of the packed row: the 4 b bits of its four codes.
// Method: "KVarN vs TurboQuant" (dothoosh.com), pipeline list: Hadamard
// rotation, variance normalisation, asymmetric round-to-nearest.
// quantize_vector_warp_raw takes the lane's 8 source bytes already loaded.
// Lane's four codes (c[j] = element 4 lane + j) into a packed B-bit row.
template <int B>
__device__ __forceinline__ void store_lane_codes(uint8_t* row, const uint32_t (&c)[4], int lane) {
  if (B == 2)
    row[lane] = static_cast<uint8_t>(c[0] | c[1] << 2 | c[2] << 4 | c[3] << 6);
  else if (B == 4)
    reinterpret_cast<uint16_t*>(row)[lane] = static_cast<uint16_t>(c[0] | c[1] << 4 | c[2] << 8 | c[3] << 12);
  else
    reinterpret_cast<uint32_t*>(row)[lane] = c[0] | c[1] << 8 | c[2] << 16 | c[3] << 24;
}
template <bool kBF16, int KB, int VB>
__device__ __forceinline__ void quantize_vector_warp_raw(uint2 raw, uint8_t* seg, int row_in_block, bool is_v,
                                                         int lane) {
  using F = Fmt<KB, VB>;
  constexpr float kMagicRne = 12582912.0f;  // 1.5 * 2^23: low mantissa bits hold rne of the addend
  float y[4];
  if (kBF16) {
    y[0] = bf16lo_to_f32(raw.x);
    y[1] = bf16hi_to_f32(raw.x);
    y[2] = bf16lo_to_f32(raw.y);
    y[3] = bf16hi_to_f32(raw.y);
  } else {
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
    y[0] = a.x;
    y[1] = a.y;
    y[2] = b.x;
    y[3] = b.y;
  }
  // Walsh-Hadamard butterflies (unnormalised): strides 1, 2 in registers,
  // strides 4 .. 64 across lanes (the lower index keeps u + v)
  {
    const float a0 = y[0] + y[1], a1 = y[0] - y[1], a2 = y[2] + y[3], a3 = y[2] - y[3];
    y[0] = a0 + a2;
    y[1] = a1 + a3;
    y[2] = a0 - a2;
    y[3] = a1 - a3;
  }
#pragma unroll
  for (int st = 1; st < 32; st <<= 1) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float o = __shfl_xor_sync(0xffffffffu, y[j], st);
      y[j] = (lane & st) ? o - y[j] : y[j] + o;
    }
  }
  float sum = (y[0] + y[1]) + (y[2] + y[3]);
  float sq = fmaf(y[0], y[0], fmaf(y[1], y[1], fmaf(y[2], y[2], y[3] * y[3])));
  float ymin = fminf(fminf(y[0], y[1]), fminf(y[2], y[3]));
  float ymax = fmaxf(fmaxf(y[0], y[1]), fmaxf(y[2], y[3]));
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    sq += __shfl_xor_sync(0xffffffffu, sq, o);
    ymin = fminf(ymin, __shfl_xor_sync(0xffffffffu, ymin, o));
    ymax = fmaxf(ymax, __shfl_xor_sync(0xffffffffu, ymax, o));
  }
  const float levels = is_v ? static_cast<float>((1 << VB) - 1) : static_cast<float>((1 << KB) - 1);
  constexpr float kInvSqrtD = 0.088388347648318440550f;
  const float mean = sum * (1.0f / kHeadDim);
  const float var = fmaxf(sq * (1.0f / kHeadDim) - mean * mean, 0.0f);
  float sigma = sqrtf(var);
  if (sigma == 0.0f) sigma = 1.0f;
  const float lo = (ymin - mean) / sigma;
  const float hi = (ymax - mean) / sigma;
  const __half Sh = __float2half_rn(kInvSqrtD * (sigma * (hi - lo)) / levels);
  const __half Zh = __float2half_rn(kInvSqrtD * (mean + sigma * lo));
  const float Sf = __half2float(Sh);
  const float Zf = __half2float(Zh);
  uint32_t c[4] = {0u, 0u, 0u, 0u};
  if (Sf != 0.0f) {
    const float a = kInvSqrtD / Sf;
    const float b = -Zf / Sf;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float t = fminf(fmaxf(fmaf(y[j], a, b), 0.0f), levels);
      c[j] = __float_as_uint(t + kMagicRne) & 0xFFu;
    }
  }
  if (is_v) {
    store_lane_codes<VB>(seg + F::kOffV + row_in_block * F::kVRowBytes, c, lane);
    if (lane == 0) {
      reinterpret_cast<__half*>(seg + F::kOffSV)[row_in_block] = Sh;
      reinterpret_cast<__half*>(seg + F::kOffZV)[row_in_block] = Zh;
    }
  } else {
    store_lane_codes<KB>(seg + F::kOffK + row_in_block * F::kKRowBytes, c, lane);
    if (lane == 0) {
      reinterpret_cast<__half*>(seg + F::kOffSK)[row_in_block] = Sh;
      reinterpret_cast<__half*>(seg + F::kOffZK)[row_in_block] = Zh;
    }
  }
}

// elements 4 lane .. 4 lane + 3 (8 bytes) of the vector at src
template <bool kBF16, int KB, int VB>
__device__ __forceinline__ void quantize_vector_warp(const uint8_t* src, uint8_t* seg, int row_in_block, bool is_v,
                                                     int lane) {
  quantize_vector_warp_raw<kBF16, KB, VB>(*reinterpret_cast<const uint2*>(src + 8 * lane), seg, row_in_block, is_v,
                                          lane);
}

// ---- programmatic dependent launch ------------------------------------------
// Every kernel here is launched with programmatic stream serialization: it
// may become resident while the kernel before it in the stream is still
// finishing.  It executes pdl_wait() before it reads or writes any memory
// that an earlier kernel may touch (inputs, pool, workspace, outputs), and
// pdl_trigger(), which lets the next kernel's CTAs become resident and set
// up, at a point chosen by the tensor-memory rule below.
//
// Tensor-memory rule.  The decode and bulk-quantize kernels allocate tensor
// memory (256 of an SM's 512 columns) before their pdl_wait(), and an
// allocation blocks until the columns are free.  A CTA that waits in
// pdl_wait() for grid A must therefore never hold columns that a CTA of A
// still has to allocate.  Each kernel triggers only after its own CTA
// holds all the tensor memory it will ever take (the bulk quantize: right
// after its allocation; decode: after its deallocation), so by the time a
// dependent CTA allocates, every CTA of the grid before it has either
// allocated already or finished.  Shared memory backs this up: no SM can
// hold three CTAs of these kernels at once (each asks for more than a third
// of the SM's 228 KB), so at most two 256-column allocations meet on an SM.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---- launchers (return cudaError_t of the launch) ---------------------------
struct QuantizeArgs {
  uint8_t* pool;
  int32_t num_blocks;
  int32_t num_kv_heads;
  const void* k;
  const void* v;
  int32_t in_dtype;
  int32_t n_tokens;
  int64_t token_stride;
  const int32_t* slots;
  int* status;
  int32_t k_bits, v_bits;  // preset
};
cudaError_t launch_quantize(const QuantizeArgs& a, cudaStream_t stream);

struct DecodeArgs {
  const uint8_t* pool;
  int32_t num_blocks;
  int32_t num_kv_heads;
  const void* q;
  int32_t q_dtype;
  int32_t batch;
  int32_t num_q_heads;
  const int32_t* block_table;
  int32_t max_blocks_per_seq;
  const int32_t* seq_lens;
  int32_t max_seq_len;
  float scale_log2;  // softmax scale times log2(e)
  void* out;
  int32_t out_dtype;
  int32_t* tickets;   // [batch * num_kv_heads]
  float* partials;    // [batch, num_q_heads, nsplit, kPartialFloats]
  int32_t blocks_per_split;
  int32_t nsplit;
  int* status;
  // optional one-token append at position seq_lens[b] - 1 before the scan
  const uint8_t* k_new;  // nullptr: no append
  const uint8_t* v_new;
  int32_t new_bf16;
  int64_t new_stride_bytes;
  int32_t k_bits, v_bits;  // preset
  // optional bf16 window of sink and recent tokens: CTA x = nsplit of each
  // (b, h) attends over it and hands in record nsplit (nrec = nsplit + 1)
  const uint16_t* win;  // nullptr: no window (nrec = nsplit)
  int32_t win_sink, win_recent;
  int32_t nrec;  // records per (b, query head) in partials
};
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);

// Window append (kvq_window_append).
struct WindowAppendArgs {
  uint16_t* win;
  int32_t num_seqs, num_kv_heads, sink, recent;
  const uint16_t* k;
  const uint16_t* v;
  int64_t token_stride;  // elements
  const int32_t* seq_ids;
  const int32_t* positions;
  int32_t n_tokens;
  int* status;
};
cudaError_t launch_window_append(const WindowAppendArgs& a, cudaStream_t stream);
constexpr int kMaxWindowSink = 64;
constexpr int kMaxWindowRecent = 1024;

// Failure-detection self-test (kvq_selftest_wait_timeout) and the time after
// which a kernel's bounded wait gives up.
cudaError_t launch_wait_probe(int* status, uint64_t limit_ns, uint64_t* elapsed_ns, cudaStream_t stream);
uint64_t wait_limit_ns();

// Split-K plan of a decode call on the current device.
struct DecodePlan {
  int32_t blocks_per_split;
  int32_t nsplit;
  int32_t nrec;          // records per (b, query head): nsplit + extra_records
  size_t ticket_bytes;   // rounded up to 256
  size_t partial_bytes;
  size_t total_bytes;
};
int plan_decode(int32_t batch, int32_t num_kv_heads, int32_t num_q_heads, int32_t max_seq_len,
                int32_t blocks_per_split_request, DecodePlan* plan,
                int32_t extra_records = 0);

int device_sm_count();
int decode_ctas_per_sm();  // resident decode CTAs per SM on the current device
int decode_max_splits();   // upper bound the split plan respects
int decode_max_split_blocks();  // longest split (blocks) a decode CTA takes
int decode_chunk_blocks();  // blocks the decode kernel takes per step (splits are multiples of it)

// Raise a kernel's dynamic shared-memory limit once per device (a host call
// that is not a stream operation, so it is also safe while a stream is being
// captured into a graph).
template <auto kKernel>
cudaError_t ensure_smem_limit(int bytes) {
  static bool done[64] = {};  // one flag array per kernel (template argument)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(kKernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
  return e;
}

}  // namespace kvq
