// kvq_quantize.cu -- cache write path: rotate, normalise, quantise, pack.
//
// One thread owns one 128-element K or V head vector end to end, so the
// Walsh-Hadamard transform, the mean/variance/min/max reductions and the
// packing all stay in that thread's registers and need no shuffles.  The
// butterflies use Blackwell's packed f32x2 add/sub: the thread keeps the
// vector as 64 pairs (x[k], x[k+64]); the stride-64 stage is done first as
// scalars and the six remaining stages run on whole pairs.
//
// Rows reach shared memory through 16-byte cp.async copies that are coalesced
// across the warp (two 256-byte rows per instruction) into a 272-byte pitch,
// which makes the per-thread row reads bank-conflict free; each warp double
// buffers its 32-row tiles.  Codes leave as 16-byte stores into the paged
// segment (64 B of K codes or 32 B of V codes per row) plus two fp16 stores.
//
// Method ("Трюк Huawei с KV-кэшем", section "Заявка, которая ломает
// привычный компромисс"; "KVarN vs TurboQuant", pipeline list): Hadamard
// rotation, variance normalisation, asymmetric round-to-nearest; the exact
// definition and pool layout are stated in include/kvq.h.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kWarps = 4;
constexpr int kRows = 32;                  // vectors per warp tile, one per lane
constexpr int kPitch = kHeadDim * 2 + 16;  // 272-byte smem pitch of a 256-byte row
constexpr int kTileBytes = kRows * kPitch;

typedef unsigned long long u64;

__device__ __forceinline__ u64 pk(float a, float b) {
  u64 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk(u64 v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ void upk_u(u64 v, uint32_t& a, uint32_t& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=r"(a), "=r"(b) : "l"(v));
}
__device__ __forceinline__ u64 add2(u64 a, u64 b) {
  u64 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ u64 sub2(u64 a, u64 b) {
  u64 d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ u64 fma2(u64 a, u64 b, u64 c) {
  u64 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float min3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N));
}

// Stage the 32 rows of tile `tile` (vectors tile*32 .. tile*32+31 of one of
// the two tensors) into smem.  Row r of the tile is vector n = tile*32 + r,
// i.e. token n / Hkv, head n % Hkv.  Lane l copies chunk (16 B) l of rows
// 2j and 2j+1 in iteration j; the row addresses are computed once per lane
// (its own vector) and handed around with shuffles.
__device__ __forceinline__ void stage_tile(uint32_t sbuf, const uint8_t* src, int64_t n_vec,
                                           int hkv, int64_t stride_bytes, int64_t tile, int lane) {
  const int64_t n = tile * kRows + lane;
  const bool mine_valid = n < n_vec;
  const int64_t tok = mine_valid ? n / hkv : 0;
  const int hh = mine_valid ? static_cast<int>(n - tok * hkv) : 0;
  const uint8_t* my_row = src + tok * stride_bytes + static_cast<int64_t>(hh) * (kHeadDim * 2);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int row = 2 * j + (lane >> 4);
    const int col = lane & 15;
    const uint8_t* row_ptr = reinterpret_cast<const uint8_t*>(
        __shfl_sync(0xffffffffu, static_cast<unsigned long long>(reinterpret_cast<uintptr_t>(my_row)), row));
    const bool valid = tile * kRows + row < n_vec;
    cp_async16(sbuf + row * kPitch + col * 16, valid ? row_ptr + col * 16 : src, valid);
  }
}

// 128 elements of the thread's row in smem -> pairs P[k] = (x[k], x[k+64])
// after the stride-64 butterfly (x[k] + x[k+64], x[k] - x[k+64]).
template <bool kBF16>
__device__ __forceinline__ void load_row(const uint8_t* row, u64 (&P)[64]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint4 lo = *reinterpret_cast<const uint4*>(row + j * 16);       // x[8j .. 8j+7]
    const uint4 hi = *reinterpret_cast<const uint4*>(row + j * 16 + 128);  // x[64+8j ..]
    const uint32_t wl[4] = {lo.x, lo.y, lo.z, lo.w};
    const uint32_t wh[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float a0, a1, b0, b1;
      if (kBF16) {
        a0 = bf16lo_to_f32(wl[e]);
        a1 = bf16hi_to_f32(wl[e]);
        b0 = bf16lo_to_f32(wh[e]);
        b1 = bf16hi_to_f32(wh[e]);
      } else {
        const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&wl[e]));
        const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&wh[e]));
        a0 = fa.x;
        a1 = fa.y;
        b0 = fb.x;
        b1 = fb.y;
      }
      P[8 * j + 2 * e] = pk(a0 + b0, a0 - b0);
      P[8 * j + 2 * e + 1] = pk(a1 + b1, a1 - b1);
    }
  }
}

// The remaining six butterfly stages (strides 1..32) on whole pairs.
__device__ __forceinline__ void fwht_pairs(u64 (&P)[64]) {
#pragma unroll
  for (int s = 1; s < 64; s <<= 1) {
#pragma unroll
    for (int k = 0; k < 64; ++k) {
      if ((k & s) == 0) {
        const u64 a = P[k], b = P[k + s];
        P[k] = add2(a, b);
        P[k + s] = sub2(a, b);
      }
    }
  }
}

// Code of pair element with the integer in the low mantissa bits: the value
// t = q + 1.5*2^23 has ulp 1, so its low bits hold rne(q) (ties to even).
constexpr float kMagic = 12582912.0f;

template <int kBits>
__device__ __forceinline__ void quantize_store(u64 (&P)[64], uint8_t* seg, int row_in_block) {
  constexpr float kLevels = static_cast<float>((1 << kBits) - 1);
  constexpr float kInvSqrtD = 0.088388347648318440550f;  // 1/sqrt(128)

  // variance normalisation statistics of r = y / sqrt(128), computed on y
  u64 s2 = 0ull, q2 = 0ull;
  {
    u64 acc_s[8], acc_q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      acc_s[i] = P[i];
      acc_q[i] = fma2(P[i], P[i], 0ull);
    }
#pragma unroll
    for (int k = 8; k < 64; ++k) {
      acc_s[k & 7] = add2(acc_s[k & 7], P[k]);
      acc_q[k & 7] = fma2(P[k], P[k], acc_q[k & 7]);
    }
#pragma unroll
    for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
      for (int i = 0; i < w; ++i) {
        acc_s[i] = add2(acc_s[i], acc_s[i + w]);
        acc_q[i] = add2(acc_q[i], acc_q[i + w]);
      }
    s2 = acc_s[0];
    q2 = acc_q[0];
  }
  float sa, sb, qa, qb;
  upk(s2, sa, sb);
  upk(q2, qa, qb);
  const float mean = (sa + sb) * (1.0f / kHeadDim);
  const float var = fmaxf((qa + qb) * (1.0f / kHeadDim) - mean * mean, 0.0f);
  float sigma = sqrtf(var);
  if (sigma == 0.0f) sigma = 1.0f;

  // range of y (min/max of u = (y - mean)/sigma sit at the same elements)
  float ymin, ymax;
  {
    float mn[8], mx[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float a, b;
      upk(P[i], a, b);
      mn[i] = fminf(a, b);
      mx[i] = fmaxf(a, b);
    }
#pragma unroll
    for (int k = 8; k < 64; ++k) {
      float a, b;
      upk(P[k], a, b);
      mn[k & 7] = min3(mn[k & 7], a, b);
      mx[k & 7] = max3(mx[k & 7], a, b);
    }
    ymin = min3(min3(mn[0], mn[1], mn[2]), min3(mn[3], mn[4], mn[5]), fminf(mn[6], mn[7]));
    ymax = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
  }
  const float lo = (ymin - mean) / sigma;
  const float hi = (ymax - mean) / sigma;
  const __half Sh = __float2half_rn(kInvSqrtD * (sigma * (hi - lo)) / kLevels);
  const __half Zh = __float2half_rn(kInvSqrtD * (mean + sigma * lo));
  const float Sf = __half2float(Sh);
  const float Zf = __half2float(Zh);

  // codes: q = (r - Z)/S = y * (c/S) - Z/S, rounded to nearest even, clamped
  uint32_t words[16];
  if (Sf == 0.0f) {
#pragma unroll
    for (int m = 0; m < 16; ++m) words[m] = 0u;
  } else {
    const float a = kInvSqrtD / Sf;
    const float b = -Zf / Sf;
    const u64 a2 = pk(a, a), b2 = pk(b, b), m2 = pk(kMagic, kMagic);
    // q is monotone in y, so clamping is needed only if an extreme leaves range
    const float cmin = fmaf(ymin, a, b) + kMagic;
    const float cmax = fmaf(ymax, a, b) + kMagic;
    const bool clamp = (cmin < kMagic) || (cmax > kMagic + kLevels);
#pragma unroll
    for (int k = 0; k < 64; ++k) {
      u64 t = fma2(P[k], a2, b2);
      if (clamp) {
        float ta, tb;
        upk(t, ta, tb);
        t = pk(fminf(fmaxf(ta, 0.0f), kLevels), fminf(fmaxf(tb, 0.0f), kLevels));
      }
      P[k] = add2(t, m2);
    }
    // pack: element i < 64 is P[i].x, element i >= 64 is P[i-64].y
    if (kBits == 4) {
#pragma unroll
      for (int m = 0; m < 16; ++m) {  // word m = elements 8m .. 8m+7
        uint32_t c[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int i = 8 * m + e;
          uint32_t lo_bits, hi_bits;
          upk_u(P[i & 63], lo_bits, hi_bits);
          c[e] = (i < 64) ? lo_bits : hi_bits;
        }
        const uint32_t b0 = c[0] + 16u * c[1], b1 = c[2] + 16u * c[3];
        const uint32_t b2 = c[4] + 16u * c[5], b3 = c[6] + 16u * c[7];
        words[m] = prmt(prmt(b0, b1, 0x0040u), prmt(b2, b3, 0x0040u), 0x5410u);
      }
    } else {
#pragma unroll
      for (int m = 0; m < 8; ++m) {  // word m = elements 16m .. 16m+15
        uint32_t c[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int i = 16 * m + e;
          uint32_t lo_bits, hi_bits;
          upk_u(P[i & 63], lo_bits, hi_bits);
          c[e] = (i < 64) ? lo_bits : hi_bits;
        }
        uint32_t by[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          by[q] = c[4 * q] + 4u * c[4 * q + 1] + 16u * c[4 * q + 2] + 64u * c[4 * q + 3];
        words[m] = prmt(prmt(by[0], by[1], 0x0040u), prmt(by[2], by[3], 0x0040u), 0x5410u);
      }
    }
  }

  if (kBits == 4) {
    uint4* dst = reinterpret_cast<uint4*>(seg + kOffK + row_in_block * kKRowBytes);
#pragma unroll
    for (int m = 0; m < 4; ++m)
      dst[m] = make_uint4(words[4 * m], words[4 * m + 1], words[4 * m + 2], words[4 * m + 3]);
    reinterpret_cast<__half*>(seg + kOffSK)[row_in_block] = Sh;
    reinterpret_cast<__half*>(seg + kOffZK)[row_in_block] = Zh;
  } else {
    uint4* dst = reinterpret_cast<uint4*>(seg + kOffV + row_in_block * kVRowBytes);
#pragma unroll
    for (int m = 0; m < 2; ++m)
      dst[m] = make_uint4(words[4 * m], words[4 * m + 1], words[4 * m + 2], words[4 * m + 3]);
    reinterpret_cast<__half*>(seg + kOffSV)[row_in_block] = Sh;
    reinterpret_cast<__half*>(seg + kOffZV)[row_in_block] = Zh;
  }
}

template <bool kBF16>
__global__ void __launch_bounds__(kWarps * 32)
    quantize_kernel(uint8_t* __restrict__ pool, int32_t num_blocks, int32_t hkv,
                    const uint8_t* __restrict__ k, const uint8_t* __restrict__ v,
                    int32_t n_tokens, int64_t stride_bytes, const int32_t* __restrict__ slots, int* status) {
  extern __shared__ __align__(16) uint8_t smem[];
  pdl_trigger();  // (the grid is persistent: every CTA is resident at once)
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const uint32_t buf0 = smem_u32(smem + warp * 2 * kTileBytes);
  const uint8_t* my_buf0 = smem + warp * 2 * kTileBytes;

  const int64_t n_vec = static_cast<int64_t>(n_tokens) * hkv;
  const int64_t tiles_per_tensor = (n_vec + kRows - 1) / kRows;
  const int64_t total_tiles = 2 * tiles_per_tensor;  // K tiles, then V tiles
  const int64_t warp_id = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;

  int64_t tile = warp_id;
  if (tile >= total_tiles) return;
  int stage = 0;
  {
    const bool isv = tile >= tiles_per_tensor;
    stage_tile(buf0, isv ? v : k, n_vec, hkv, stride_bytes, isv ? tile - tiles_per_tensor : tile,
               lane);
    cp_async_commit();
  }
  for (; tile < total_tiles; tile += nwarps) {
    const int64_t next = tile + nwarps;
    if (next < total_tiles) {
      const bool nv = next >= tiles_per_tensor;
      stage_tile(buf0 + (stage ^ 1) * kTileBytes, nv ? v : k, n_vec, hkv, stride_bytes,
                 nv ? next - tiles_per_tensor : next, lane);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();

    const bool is_v = tile >= tiles_per_tensor;
    const int64_t n = (is_v ? tile - tiles_per_tensor : tile) * kRows + lane;
    if (n < n_vec) {
      const int64_t tok = n / hkv;
      const int h = static_cast<int>(n - tok * hkv);
      const int32_t slot = slots[tok];
      if (slot >= 0) {
        const int32_t p = slot / kBlockSize;
        if (p >= num_blocks) {
          record_status(status, KVQ_ERR_OUT_OF_RANGE);
        } else {
          uint8_t* seg = pool + (static_cast<int64_t>(p) * hkv + h) * kSegBytes;
          u64 P[64];
          load_row<kBF16>(my_buf0 + stage * kTileBytes + lane * kPitch, P);
          fwht_pairs(P);
          if (is_v)
            quantize_store<kVBits>(P, seg, slot % kBlockSize);
          else
            quantize_store<kKBits>(P, seg, slot % kBlockSize);
        }
      }
    }
    __syncwarp();
    stage ^= 1;
  }
}


// ---- small appends (a few tokens per call, as in decode) --------------------
// One warp per head vector (quantize_vector_warp in kvq_internal.cuh).
constexpr int kSmallWarps = 4;
constexpr int64_t kSmallMaxVecs = 1024;  // at most this many head vectors per tensor

template <bool kBF16>
__global__ void __launch_bounds__(kSmallWarps * 32)
    quantize_small_kernel(uint8_t* __restrict__ pool, int32_t num_blocks, int32_t hkv,
                          const uint8_t* __restrict__ k, const uint8_t* __restrict__ v, int32_t n_tokens,
                          int64_t stride_bytes, const int32_t* __restrict__ slots, int* status) {
  pdl_trigger();  // (the whole grid is resident at once)
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t n_vec = static_cast<int64_t>(n_tokens) * hkv;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * kSmallWarps + (threadIdx.x >> 5);
  if (w >= 2 * n_vec) return;
  const bool is_v = w >= n_vec;
  const int64_t n = is_v ? w - n_vec : w;
  const int64_t tok = n / hkv;
  const int h = static_cast<int>(n - tok * hkv);
  const int32_t slot = slots[tok];
  if (slot < 0) return;
  const int32_t p = slot / kBlockSize;
  if (p >= num_blocks) {
    if (lane == 0) record_status(status, KVQ_ERR_OUT_OF_RANGE);
    return;
  }
  const int row_in_block = slot % kBlockSize;
  uint8_t* seg = pool + (static_cast<int64_t>(p) * hkv + h) * kSegBytes;

  quantize_vector_warp<kBF16>((is_v ? v : k) + tok * stride_bytes + static_cast<int64_t>(h) * (kHeadDim * 2), seg,
                              row_in_block, is_v, lane);
}

}  // namespace

cudaError_t launch_quantize(const QuantizeArgs& a, cudaStream_t stream) {
  if (a.n_tokens == 0) return cudaSuccess;
  const int64_t n_vec = static_cast<int64_t>(a.n_tokens) * a.num_kv_heads;
  const int64_t stride_bytes = a.token_stride * 2;
  if (n_vec <= kSmallMaxVecs) {
    const unsigned grid = static_cast<unsigned>((2 * n_vec + kSmallWarps - 1) / kSmallWarps);
    if (a.in_dtype == KVQ_BF16)
      return launch_pdl(quantize_small_kernel<true>, dim3(grid), dim3(kSmallWarps * 32), 0, stream, a.pool,
                        a.num_blocks, a.num_kv_heads, static_cast<const uint8_t*>(a.k),
                        static_cast<const uint8_t*>(a.v), a.n_tokens, stride_bytes, a.slots, a.status);
    else
      return launch_pdl(quantize_small_kernel<false>, dim3(grid), dim3(kSmallWarps * 32), 0, stream, a.pool,
                        a.num_blocks, a.num_kv_heads, static_cast<const uint8_t*>(a.k),
                        static_cast<const uint8_t*>(a.v), a.n_tokens, stride_bytes, a.slots, a.status);
    return cudaGetLastError();
  }
  const int64_t tiles = 2 * ((n_vec + kRows - 1) / kRows);
  const int smem = kWarps * 2 * kTileBytes;
  const int sms = device_sm_count();
  int64_t grid = (tiles + kWarps - 1) / kWarps;
  const int64_t cap = static_cast<int64_t>(sms) * 3;
  if (grid > cap) grid = cap;
  if (a.in_dtype == KVQ_BF16) {
    const cudaError_t e = ensure_smem_limit<quantize_kernel<true>>(smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(quantize_kernel<true>, dim3(static_cast<unsigned>(grid)), dim3(kWarps * 32), smem, stream,
                      a.pool, a.num_blocks, a.num_kv_heads, static_cast<const uint8_t*>(a.k),
                      static_cast<const uint8_t*>(a.v), a.n_tokens, stride_bytes, a.slots, a.status);
  } else {
    const cudaError_t e = ensure_smem_limit<quantize_kernel<false>>(smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(quantize_kernel<false>, dim3(static_cast<unsigned>(grid)), dim3(kWarps * 32), smem, stream,
                      a.pool, a.num_blocks, a.num_kv_heads, static_cast<const uint8_t*>(a.k),
                      static_cast<const uint8_t*>(a.v), a.n_tokens, stride_bytes, a.slots, a.status);
  }
  return cudaGetLastError();
}

}  // namespace kvq
