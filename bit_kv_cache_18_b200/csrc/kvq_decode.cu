// kvq_decode.cu -- decode attention over the packed paged cache.
//
// One CTA owns one (sequence b, kv head h, split of the context).  It
//   1. rotates the G query heads of kv head h once, q~ = R q, and sums them
//      (the zero points enter every score as Z_K,t * sum(q~));
//   2. walks its blocks through the block table, scoring each token with the
//      key scale folded in, s_t = tau*log2(e)*(S_K,t <q~, c_K,t> + Z_K,t sum q~),
//      keeping a running max and sum per head (online softmax, base 2);
//   3. accumulates o~ += p_t S_V,t c_V,t and zeta += p_t Z_V,t in the rotated
//      domain and writes (o~ + zeta, m, l) as its split's partial;
//   4. takes a ticket; the last CTA of (b, h) merges the splits and rotates
//      the merged output back once, o = R o~ / l.
// Scale folding at read time and the single rotations of the query and the
// output follow the KVarN pipeline list ("KVarN vs TurboQuant", dothoosh.com,
// fourth stage) and the definitions in include/kvq.h.  No CTA ever waits for
// another: the last one to finish does the merge.
#include <math_constants.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kThreads = 128;

// In-place Walsh-Hadamard transform of G rows of 128 floats in shared memory,
// followed by the 1/sqrt(128) factor; all kThreads threads take part.
template <int G>
__device__ __forceinline__ void fwht_rows_smem(float (*rows)[kHeadDim]) {
#pragma unroll 1
  for (int s = 1; s < kHeadDim; s <<= 1) {
    for (int w = threadIdx.x; w < G * (kHeadDim / 2); w += kThreads) {
      const int g = w / (kHeadDim / 2);
      const int k = w % (kHeadDim / 2);
      const int i = (k / s) * 2 * s + (k % s);
      const float a = rows[g][i], b = rows[g][i + s];
      rows[g][i] = a + b;
      rows[g][i + s] = a - b;
    }
    __syncthreads();
  }
  for (int w = threadIdx.x; w < G * kHeadDim; w += kThreads)
    rows[w / kHeadDim][w % kHeadDim] *= 0.088388347648318440550f;
  __syncthreads();
}

template <int G>
__global__ void __launch_bounds__(kThreads) decode_kernel(DecodeArgs a) {
  const int split = blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int tid = threadIdx.x;

  __shared__ float qr[G][kHeadDim];
  __shared__ float qsum[G];
  __shared__ __align__(16) uint8_t seg[kSegBytes];
  __shared__ float sc[kBlockSize][G];
  __shared__ float pw[kBlockSize][G];
  __shared__ float alpha_s[G];
  __shared__ float st_m[G], st_l[G], st_z[G];
  __shared__ int is_last;

  // effective length of this sequence
  int L = a.seq_lens[b];
  if (L < 0 || L > a.max_seq_len || L > a.max_blocks_per_seq * kBlockSize) {
    if (tid == 0) record_status(a.status, KVQ_ERR_OUT_OF_RANGE);
    L = L < 0 ? 0 : L;
    L = L > a.max_seq_len ? a.max_seq_len : L;
    L = L > a.max_blocks_per_seq * kBlockSize ? a.max_blocks_per_seq * kBlockSize : L;
  }
  const int nb = (L + kBlockSize - 1) / kBlockSize;
  const int blk0 = split * a.blocks_per_split;
  const int blk1 = min(nb, blk0 + a.blocks_per_split);

  // 1. query rotation and its sum
  for (int i = tid; i < G * kHeadDim; i += kThreads) {
    const int g = i / kHeadDim;
    const int64_t qi = (static_cast<int64_t>(b) * a.num_q_heads + h * G + g) * kHeadDim + i % kHeadDim;
    qr[g][i % kHeadDim] = load_as_f32(a.q, a.q_dtype, qi);
  }
  __syncthreads();
  fwht_rows_smem<G>(qr);
  {
    const int warp = tid >> 5, lane = tid & 31;
    for (int g = warp; g < G; g += kThreads / 32) {
      float s = qr[g][lane] + qr[g][lane + 32] + qr[g][lane + 64] + qr[g][lane + 96];
#pragma unroll
      for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) qsum[g] = s;
    }
  }
  if (tid < G) {
    st_m[tid] = -CUDART_INF_F;
    st_l[tid] = 0.0f;
    st_z[tid] = 0.0f;
  }
  __syncthreads();

  float acc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) acc[g] = 0.0f;

  // 2./3. paged scan of this split
  for (int blk = blk0; blk < blk1; ++blk) {
    const int32_t p = a.block_table[static_cast<int64_t>(b) * a.max_blocks_per_seq + blk];
    if (p < 0 || p >= a.num_blocks) {  // uniform across the CTA
      if (tid == 0) record_status(a.status, KVQ_ERR_OUT_OF_RANGE);
      continue;
    }
    const int ntok = min(kBlockSize, L - blk * kBlockSize);
    const uint4* src = reinterpret_cast<const uint4*>(
        a.pool + (static_cast<int64_t>(p) * a.num_kv_heads + h) * kSegBytes);
    for (int i = tid; i < kSegBytes / 16; i += kThreads) reinterpret_cast<uint4*>(seg)[i] = src[i];
    __syncthreads();

    // scores: token o = tid/8, dims 16*part .. 16*part+15
    {
      const int o = tid >> 3, part = tid & 7;
      const uint2 w = *reinterpret_cast<const uint2*>(seg + kOffK + o * kKRowBytes + part * 8);
      float dot[G];
#pragma unroll
      for (int g = 0; g < G; ++g) dot[g] = 0.0f;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const uint32_t word = e < 8 ? w.x : w.y;
        const float c = static_cast<float>((word >> (4 * (e & 7))) & 15u);
#pragma unroll
        for (int g = 0; g < G; ++g) dot[g] = fmaf(qr[g][16 * part + e], c, dot[g]);
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int off = 4; off; off >>= 1) dot[g] += __shfl_xor_sync(0xffffffffu, dot[g], off);
      }
      if (part == 0) {
        const float Sk = __half2float(reinterpret_cast<const __half*>(seg + kOffSK)[o]);
        const float Zk = __half2float(reinterpret_cast<const __half*>(seg + kOffZK)[o]);
#pragma unroll
        for (int g = 0; g < G; ++g)
          sc[o][g] = o < ntok ? a.scale_log2 * fmaf(Sk, dot[g], Zk * qsum[g]) : -CUDART_INF_F;
      }
    }
    __syncthreads();

    // online softmax update, one thread per head
    if (tid < G) {
      const int g = tid;
      float mnew = st_m[g];
      for (int o = 0; o < kBlockSize; ++o) mnew = fmaxf(mnew, sc[o][g]);
      const float alpha = st_m[g] == -CUDART_INF_F ? 0.0f : exp2f(st_m[g] - mnew);
      float lsum = 0.0f, zsum = 0.0f;
      for (int o = 0; o < kBlockSize; ++o) {
        const float pp = o < ntok ? exp2f(sc[o][g] - mnew) : 0.0f;
        pw[o][g] = pp * __half2float(reinterpret_cast<const __half*>(seg + kOffSV)[o]);
        lsum += pp;
        zsum = fmaf(pp, __half2float(reinterpret_cast<const __half*>(seg + kOffZV)[o]), zsum);
      }
      st_l[g] = fmaf(st_l[g], alpha, lsum);
      st_z[g] = fmaf(st_z[g], alpha, zsum);
      st_m[g] = mnew;
      alpha_s[g] = alpha;
    }
    __syncthreads();

    // p.v with the value scale folded into p: thread = dimension
    {
      const int d = tid;
#pragma unroll
      for (int g = 0; g < G; ++g) acc[g] *= alpha_s[g];
      for (int o = 0; o < kBlockSize; ++o) {
        const uint8_t byte = seg[kOffV + o * kVRowBytes + d / 4];
        const float c = static_cast<float>((byte >> (2 * (d & 3))) & 3u);
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g] = fmaf(pw[o][g], c, acc[g]);
      }
    }
    __syncthreads();
  }

  // split partial: o~ (unnormalised, zero points included), m, l
  {
    const int d = tid;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float* rec = a.partials +
                   ((static_cast<int64_t>(b) * a.num_q_heads + h * G + g) * a.nsplit + split) * kPartialFloats;
      rec[d] = acc[g] + st_z[g];
      if (d == 0) {
        rec[kHeadDim] = st_m[g];
        rec[kHeadDim + 1] = st_l[g];
      }
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int t = atomicAdd(&a.tickets[b * a.num_kv_heads + h], 1);
    is_last = (t == a.nsplit - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  // 4. merge the splits (thread = dimension) and rotate back
  {
    const int d = tid;
#pragma unroll 1
    for (int g = 0; g < G; ++g) {
      const float* recs = a.partials + ((static_cast<int64_t>(b) * a.num_q_heads + h * G + g) * a.nsplit) * kPartialFloats;
      float M = -CUDART_INF_F;
      for (int s = 0; s < a.nsplit; ++s) {
        const float l = __ldcg(recs + s * kPartialFloats + kHeadDim + 1);
        if (l > 0.0f) M = fmaxf(M, __ldcg(recs + s * kPartialFloats + kHeadDim));
      }
      float lsum = 0.0f, o = 0.0f;
      for (int s = 0; s < a.nsplit; ++s) {
        const float l = __ldcg(recs + s * kPartialFloats + kHeadDim + 1);
        if (l > 0.0f) {
          const float w = exp2f(__ldcg(recs + s * kPartialFloats + kHeadDim) - M);
          lsum = fmaf(l, w, lsum);
          o = fmaf(__ldcg(recs + s * kPartialFloats + d), w, o);
        }
      }
      qr[g][d] = lsum > 0.0f ? o / lsum : 0.0f;
    }
  }
  __syncthreads();
  fwht_rows_smem<G>(qr);
  for (int i = tid; i < G * kHeadDim; i += kThreads) {
    const int g = i / kHeadDim;
    const int64_t oi = (static_cast<int64_t>(b) * a.num_q_heads + h * G + g) * kHeadDim + i % kHeadDim;
    store_from_f32(a.out, a.out_dtype, oi, qr[g][i % kHeadDim]);
  }
  if (tid == 0) a.tickets[b * a.num_kv_heads + h] = 0;  // ready for the next call
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  const dim3 grid(a.nsplit, a.num_kv_heads, a.batch);
  const int G = a.num_q_heads / a.num_kv_heads;
  switch (G) {
    case 1: decode_kernel<1><<<grid, kThreads, 0, stream>>>(a); break;
    case 2: decode_kernel<2><<<grid, kThreads, 0, stream>>>(a); break;
    case 4: decode_kernel<4><<<grid, kThreads, 0, stream>>>(a); break;
    case 8: decode_kernel<8><<<grid, kThreads, 0, stream>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace kvq
