// kvq_decode.cu -- decode attention over the packed paged cache.
//
// One CTA owns one (sequence b, kv head h, split of the context); its eight
// warps take the split's blocks round robin.  The CTA
//   1. rotates the G query heads of kv head h once, q~ = R q (in-smem FWHT),
//      and sums them: zero points enter every score as Z_K,t * sum(q~);
//   2. per warp, streams its 16-token segments (1664 B each) into a private
//      ring of shared-memory stages with 16-byte cp.async copies, eight
//      segments in flight, reading block-table entries 32 at a time one
//      window ahead;
//   3. per segment, computes q~.c_K for all G heads and 16 tokens on the
//      tensor cores, folds the key scale and zero point into the score,
//      updates a base-2 online softmax, folds the value scale into the
//      probabilities, p' = p S_V, and accumulates p'.c_V on the tensor cores
//      plus zeta += p Z_V;
//   4. merges its warps, writes the split's partial (o~, m, l); the last CTA
//      of (b, h) to take a ticket merges the splits and rotates the result
//      back once, o = R o~ / l.
// Scale folding at read time and the single rotations of the query and the
// output follow the KVarN pipeline list ("KVarN vs TurboQuant", dothoosh.com,
// fourth stage) and the definitions in include/kvq.h.  No CTA ever waits for
// another.
//
// Tensor-core mapping (mma.sync m16n8k16, fp16 in, fp32 accumulate).  Rows
// m = 0..7 hold the G <= 8 query heads, rows 8..15 the same heads again as the
// low half of a two-term fp16 split (x = hi + lo, hi = fp16(x), lo =
// fp16(x - hi)), so the split that keeps 22 bits of the rotated query and of
// p S_V costs no extra instruction: it fills rows a single head group would
// leave empty.  QK: A = q~ (16 x 16 dims), B = codes (16 dims x 8 tokens).
// PV: A = p' (16 x 16 tokens), B = codes (16 tokens x 8 dims).  The QK
// accumulator layout is exactly the PV A-operand layout, so probabilities
// never leave registers.
//
// Code unpacking.  A 4-bit or 2-bit code masked in place into the mantissa of
// fp16 1024.0 (0x6400) and the bias then subtracted (one packed fp16 sub per
// two codes) gives the code, times a power of two fixed by its bit position,
// as an exact normal fp16 number.  The power of two of each operand slot is
// known statically and folded into the query fragment (keys) or into the
// final output scaling (values).  Leaving the codes as fp16 subnormals would
// save the subtraction, but measured on B200 that loses accuracy in the
// tensor-core sums (decode error about 2e-3 instead of 3e-5).
#include <math_constants.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kStages = 8;          // segments in flight per warp
constexpr int kMaxSplits = 64;      // the plan never cuts a sequence finer

template <int W>
struct __align__(128) DecodeSmem {
  uint8_t stage[W][kStages][kSegBytes];  // per-warp segment rings (then merge scratch)
  float q[8][kHeadDim];                  // rotated query rows (then the merged output)
  float qsum[8];
  float wm[W][8];
  float wl[W][8];
  int is_last;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N));
}

// 1664-byte segment, 104 chunks of 16 B: lane l copies chunks l, l+32, l+64
// and, for l < 8, l+96.
__device__ __forceinline__ void copy_segment(uint8_t* dst, const uint8_t* src, int lane) {
  const uint32_t d = smem_u32(dst);
#pragma unroll
  for (int k = 0; k < 3; ++k) cp_async16(d + (lane + 32 * k) * 16, src + (lane + 32 * k) * 16);
  if (lane < 8) cp_async16(d + (lane + 96) * 16, src + (lane + 96) * 16);
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Two-term fp16 split of a pair: hi = fp16(x), lo = fp16(x - hi).
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 f = __half22float2(h);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = pack_half2(x0 - f.x, x1 - f.y);
}

// (1024 + c) - 1024 = c exactly, for both halves.
constexpr uint32_t kBias = 0x64006400u;
__device__ __forceinline__ uint32_t unbias(uint32_t x) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(x), "r"(kBias));
  return d;
}

__device__ __forceinline__ float2 half2_at(const uint8_t* p) {
  return __half22float2(*reinterpret_cast<const __half2*>(p));
}

// In-place FWHT of 8 rows of 128 floats in smem and the 1/sqrt(128) factor.
template <int kThreads>
__device__ __forceinline__ void fwht8_smem(float (*rows)[kHeadDim]) {
#pragma unroll 1
  for (int s = 1; s < kHeadDim; s <<= 1) {
    for (int w = threadIdx.x; w < 8 * (kHeadDim / 2); w += kThreads) {
      const int g = w / (kHeadDim / 2);
      const int k = w % (kHeadDim / 2);
      const int i = (k / s) * 2 * s + (k % s);
      const float x = rows[g][i], y = rows[g][i + s];
      rows[g][i] = x + y;
      rows[g][i + s] = x - y;
    }
    __syncthreads();
  }
  for (int w = threadIdx.x; w < 8 * kHeadDim; w += kThreads)
    rows[w / kHeadDim][w % kHeadDim] *= 0.088388347648318440550f;
  __syncthreads();
}

template <int G, int W>
__global__ void __launch_bounds__(W * 32, 1) decode_kernel(DecodeArgs a) {
  constexpr int kThreads = W * 32;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecodeSmem<W>& sm = *reinterpret_cast<DecodeSmem<W>*>(smem_raw);
  const int split = blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int g = lane >> 2;  // fragment row group: query head g (hi), g+8 (lo)
  const int c = lane & 3;   // fragment column pair

  // effective length of this sequence
  int L = a.seq_lens[b];
  if (L < 0 || L > a.max_seq_len || L > a.max_blocks_per_seq * kBlockSize) {
    if (tid == 0) record_status(a.status, KVQ_ERR_OUT_OF_RANGE);
    L = max(L, 0);
    L = min(L, a.max_seq_len);
    L = min(L, a.max_blocks_per_seq * kBlockSize);
  }
  const int nb = (L + kBlockSize - 1) / kBlockSize;
  const int blk0 = split * a.blocks_per_split;
  const int blk1 = min(nb, blk0 + a.blocks_per_split);
  // this warp's blocks: blk0 + warp + W*j, j = 0 .. nmine-1
  const int nmine = blk1 > blk0 + warp ? (blk1 - blk0 - warp + W - 1) / W : 0;
  const int32_t* bt_row = a.block_table + static_cast<int64_t>(b) * a.max_blocks_per_seq + blk0 + warp;
  const uint8_t* pool_h = a.pool + static_cast<int64_t>(h) * kSegBytes;
  const int64_t pstride = static_cast<int64_t>(a.num_kv_heads) * kSegBytes;

  // ---- 1. block-table windows (lane l holds the entry of local block 32k+l)
  //      and the first kStages segments in flight
  int32_t win0 = lane < nmine ? bt_row[W * lane] : -1;
  int32_t win1 = 32 + lane < nmine ? bt_row[W * (32 + lane)] : -1;
  int wbase = 0;
  uint32_t valid_bits = 0;  // bit s: the segment staged in slot s is real
#pragma unroll
  for (int i = 0; i < kStages; ++i) {
    const int32_t p = __shfl_sync(0xffffffffu, win0, i);
    if (i < nmine) {
      if (p >= 0 && p < a.num_blocks) {
        copy_segment(sm.stage[warp][i], pool_h + p * pstride, lane);
        valid_bits |= 1u << i;
      } else if (lane == 0) {
        record_status(a.status, KVQ_ERR_OUT_OF_RANGE);
      }
    }
    cp_async_commit();
  }

  // ---- 2. rotate the query (overlaps the copies in flight)
  for (int i = tid; i < 8 * kHeadDim; i += kThreads) {
    const int gg = i / kHeadDim;
    float v = 0.0f;
    if (gg < G) {
      const int64_t qi = (static_cast<int64_t>(b) * a.num_q_heads + h * G + gg) * kHeadDim + i % kHeadDim;
      v = load_as_f32(a.q, a.q_dtype, qi);
    }
    sm.q[gg][i % kHeadDim] = v;
  }
  __syncthreads();
  fwht8_smem<kThreads>(sm.q);
  if (warp < 8) {
    const int gg = warp;
    float s = sm.q[gg][lane] + sm.q[gg][lane + 32] + sm.q[gg][lane + 64] + sm.q[gg][lane + 96];
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) sm.qsum[gg] = s;
  }
  __syncthreads();

  // QK A fragments.  k-step kk reads word w = 4c + kk/2 of a key row (dims
  // 8w..8w+7).  Slots (2c, 2c+1) take dims (8w+e, 8w+e+4) and slots
  // (2c+8, 2c+9) take (8w+e+1, 8w+e+5), e = 0 for even kk and 2 for odd kk;
  // the second pair's codes sit 4 bits higher (x16), so its q is /16.
  uint32_t qa[8][4];
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const int w = 4 * c + (kk >> 1);
    const int e = (kk & 1) ? 2 : 0;
    const float* qr = sm.q[g];
    split_pair(qr[8 * w + e], qr[8 * w + e + 4], qa[kk][0], qa[kk][1]);
    split_pair(qr[8 * w + e + 1] * 0.0625f, qr[8 * w + e + 5] * 0.0625f, qa[kk][2], qa[kk][3]);
  }
  const float zq = a.scale_log2 * sm.qsum[g];
  const float kscale = a.scale_log2;

  // PV B operand: n-tile nt covers dims 8nt..8nt+7, column g is dim 8nt+g:
  // byte 2(nt&1) + g/4 of word nt/2 of a value row, crumb g%4 (kept in place,
  // so column g's codes carry a factor 4^(g%4)).
  const uint32_t vsel0 = static_cast<uint32_t>((g >> 2) | ((4 + (g >> 2)) << 8));
  const uint32_t vsel1 = static_cast<uint32_t>((2 + (g >> 2)) | ((6 + (g >> 2)) << 8));
  const uint32_t vmask = 0x00030003u << (2 * (g & 3));

  float o[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.0f;
  float m_ref = -CUDART_INF_F;
  float l_part = 0.0f, z_part = 0.0f;

  // ---- 3. the paged scan
#pragma unroll 1
  for (int i = 0; i < nmine; ++i) {
    const int slot = i % kStages;
    cp_async_wait<kStages - 1>();
    __syncwarp();
    if (valid_bits & (1u << slot)) {
      const uint8_t* sg = sm.stage[warp][slot];
      const int ntok = min(kBlockSize, L - (blk0 + warp + W * i) * kBlockSize);

      // scores: n-tile j holds tokens 8j..8j+7, column g is token 8j+g; two
      // accumulator chains per n-tile (even / odd k-steps) halve the latency
      float sacc[2][2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) sacc[j][ch][0] = sacc[j][ch][1] = sacc[j][ch][2] = sacc[j][ch][3] = 0.0f;
      }
      const uint4 kw0 = *reinterpret_cast<const uint4*>(sg + kOffK + g * kKRowBytes + 16 * c);
      const uint4 kw1 = *reinterpret_cast<const uint4*>(sg + kOffK + (8 + g) * kKRowBytes + 16 * c);
      const uint32_t words[2][4] = {{kw0.x, kw0.y, kw0.z, kw0.w}, {kw1.x, kw1.y, kw1.z, kw1.w}};
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint32_t w = (kk & 1) ? (words[j][kk >> 1] >> 8) : words[j][kk >> 1];
          mma16816(sacc[j][kk & 1], qa[kk], unbias((w & 0x000F000Fu) | kBias), unbias((w & 0x00F000F0u) | kBias));
        }
      }
      // fold S_K, Z_K: s = tau log2e (S_K 2^24 (hi + lo) + Z_K sum q~)
      float sc[4];
      float mx = -CUDART_INF_F;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float2 sk = half2_at(sg + kOffSK + 4 * (4 * j + c));
        const float2 zk = half2_at(sg + kOffZK + 4 * (4 * j + c));
        const int t0 = 8 * j + 2 * c;
        const float d0 = (sacc[j][0][0] + sacc[j][1][0]) + (sacc[j][0][2] + sacc[j][1][2]);
        const float d1 = (sacc[j][0][1] + sacc[j][1][1]) + (sacc[j][0][3] + sacc[j][1][3]);
        sc[2 * j] = t0 < ntok ? fmaf(kscale * sk.x, d0, zk.x * zq) : -CUDART_INF_F;
        sc[2 * j + 1] = t0 + 1 < ntok ? fmaf(kscale * sk.y, d1, zk.y * zq) : -CUDART_INF_F;
        mx = fmaxf(mx, fmaxf(sc[2 * j], sc[2 * j + 1]));
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      if (mx > m_ref) {  // new running max for head g: rescale this thread's state
        const float alpha = m_ref == -CUDART_INF_F ? 0.0f : exp2f(m_ref - mx);
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
          o[nt][0] *= alpha;
          o[nt][1] *= alpha;
          o[nt][2] *= alpha;
          o[nt][3] *= alpha;
        }
        l_part *= alpha;
        z_part *= alpha;
        m_ref = mx;
      }
      // probabilities with the value scale folded in: p' = p S_V
      float pv[4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float2 sv = half2_at(sg + kOffSV + 4 * (4 * j + c));
        const float2 zv = half2_at(sg + kOffZV + 4 * (4 * j + c));
        const int t0 = 8 * j + 2 * c;
        const float p0 = t0 < ntok ? exp2f(sc[2 * j] - m_ref) : 0.0f;
        const float p1 = t0 + 1 < ntok ? exp2f(sc[2 * j + 1] - m_ref) : 0.0f;
        l_part += p0 + p1;
        pv[2 * j] = t0 < ntok ? p0 * sv.x : 0.0f;
        pv[2 * j + 1] = t0 + 1 < ntok ? p1 * sv.y : 0.0f;
        if (t0 < ntok) z_part = fmaf(p0, zv.x, z_part);
        if (t0 + 1 < ntok) z_part = fmaf(p1, zv.y, z_part);
      }
      uint32_t pa[4];
      split_pair(pv[0], pv[1], pa[0], pa[1]);
      split_pair(pv[2], pv[3], pa[2], pa[3]);

      // p'.c_V: value rows of tokens 2c, 2c+1, 8+2c, 9+2c
      const uint4* vr = reinterpret_cast<const uint4*>(sg + kOffV);
      const uint4 va0 = vr[(2 * c) * 2], va1 = vr[(2 * c) * 2 + 1];
      const uint4 vb0 = vr[(2 * c + 1) * 2], vb1 = vr[(2 * c + 1) * 2 + 1];
      const uint4 vc0 = vr[(8 + 2 * c) * 2], vc1 = vr[(8 + 2 * c) * 2 + 1];
      const uint4 vd0 = vr[(9 + 2 * c) * 2], vd1 = vr[(9 + 2 * c) * 2 + 1];
      const uint32_t tA[8] = {va0.x, va0.y, va0.z, va0.w, va1.x, va1.y, va1.z, va1.w};
      const uint32_t tB[8] = {vb0.x, vb0.y, vb0.z, vb0.w, vb1.x, vb1.y, vb1.z, vb1.w};
      const uint32_t tC[8] = {vc0.x, vc0.y, vc0.z, vc0.w, vc1.x, vc1.y, vc1.z, vc1.w};
      const uint32_t tD[8] = {vd0.x, vd0.y, vd0.z, vd0.w, vd1.x, vd1.y, vd1.z, vd1.w};
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const uint32_t sel = (nt & 1) ? vsel1 : vsel0;
        const uint32_t b0 = unbias((__byte_perm(tA[nt >> 1], tB[nt >> 1], sel) & vmask) | kBias);
        const uint32_t b1 = unbias((__byte_perm(tC[nt >> 1], tD[nt >> 1], sel) & vmask) | kBias);
        mma16816(o[nt], pa, b0, b1);
      }
    } else if (lane == 0 && i >= kStages) {
      record_status(a.status, KVQ_ERR_OUT_OF_RANGE);
    }
    __syncwarp();
    // refill this slot with the warp's block j = i + kStages
    const int j = i + kStages;
    if (j < nmine) {
      if (j >= wbase + 32) {  // slide the block-table window by 32 entries
        win0 = win1;
        wbase += 32;
        win1 = wbase + 32 + lane < nmine ? bt_row[W * (wbase + 32 + lane)] : -1;
      }
      const int32_t p = __shfl_sync(0xffffffffu, win0, j - wbase);
      if (p >= 0 && p < a.num_blocks) {
        copy_segment(sm.stage[warp][slot], pool_h + p * pstride, lane);
        valid_bits |= 1u << slot;
      } else {
        valid_bits &= ~(1u << slot);
      }
    }
    cp_async_commit();
  }
  cp_async_wait<0>();

  // ---- 4. merge: lanes of a head, then warps, then splits
  l_part += __shfl_xor_sync(0xffffffffu, l_part, 1);
  l_part += __shfl_xor_sync(0xffffffffu, l_part, 2);
  z_part += __shfl_xor_sync(0xffffffffu, z_part, 1);
  z_part += __shfl_xor_sync(0xffffffffu, z_part, 2);
  __syncthreads();  // every warp is done with its stages: reuse them
  float(*wo)[8][kHeadDim] = reinterpret_cast<float(*)[8][kHeadDim]>(&sm.stage[0][0][0]);
  {
    // column n of n-tile nt is dim 8nt + n with code factor 4^(n%4) 2^-24
    const float f0 = 1.0f / static_cast<float>(1 << (2 * ((2 * c) & 3)));
    const float f1 = 1.0f / static_cast<float>(1 << (2 * ((2 * c + 1) & 3)));
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      wo[warp][g][8 * nt + 2 * c] = fmaf(o[nt][0] + o[nt][2], f0, z_part);
      wo[warp][g][8 * nt + 2 * c + 1] = fmaf(o[nt][1] + o[nt][3], f1, z_part);
    }
    if (c == 0) {
      sm.wm[warp][g] = m_ref;
      sm.wl[warp][g] = l_part;
    }
  }
  __syncthreads();
  for (int t = tid; t < G * kHeadDim; t += kThreads) {
    const int gg = t / kHeadDim, d = t % kHeadDim;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < W; ++w)
      if (sm.wl[w][gg] > 0.0f) M = fmaxf(M, sm.wm[w][gg]);
    float lsum = 0.0f, acc = 0.0f;
#pragma unroll
    for (int w = 0; w < W; ++w) {
      if (sm.wl[w][gg] > 0.0f) {
        const float f = exp2f(sm.wm[w][gg] - M);
        lsum = fmaf(sm.wl[w][gg], f, lsum);
        acc = fmaf(wo[w][gg][d], f, acc);
      }
    }
    float* rec =
        a.partials + ((static_cast<int64_t>(b) * a.num_q_heads + h * G + gg) * a.nsplit + split) * kPartialFloats;
    if (a.nsplit == 1) {
      sm.q[gg][d] = lsum > 0.0f ? acc / lsum : 0.0f;  // nothing to merge: finish here
    } else {
      rec[d] = acc;
      if (d == 0) {
        rec[kHeadDim] = M;
        rec[kHeadDim + 1] = lsum;
      }
    }
  }
  if (a.nsplit > 1) {
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      const int t = atomicAdd(&a.tickets[b * a.num_kv_heads + h], 1);
      sm.is_last = (t == a.nsplit - 1);
    }
    __syncthreads();
    if (!sm.is_last) return;
    __threadfence();

    // the last CTA of (b, h) merges the splits: (m, l) of every split into
    // smem, merge weights per head, then every output element as a weighted
    // sum of its nsplit partials (float4 loads, eight in flight per thread)
    float* mls = reinterpret_cast<float*>(&sm.stage[0][0][0]);  // [G][nsplit] m, then l, then w
    const int ns = a.nsplit;
    const float* base = a.partials + (static_cast<int64_t>(b) * a.num_q_heads + h * G) * ns * kPartialFloats;
    for (int t = tid; t < G * ns; t += kThreads) {
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(base + static_cast<int64_t>(t) * kPartialFloats + kHeadDim));
      mls[t] = ml.x;
      mls[G * ns + t] = ml.y;
    }
    __syncthreads();
    if (warp < G) {
      const int gg = warp;
      float M = -CUDART_INF_F;
      for (int s = lane; s < ns; s += 32)
        if (mls[G * ns + gg * ns + s] > 0.0f) M = fmaxf(M, mls[gg * ns + s]);
#pragma unroll
      for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
      float lsum = 0.0f;
      for (int s = lane; s < ns; s += 32) {
        const float l = mls[G * ns + gg * ns + s];
        if (l > 0.0f) lsum = fmaf(l, exp2f(mls[gg * ns + s] - M), lsum);
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
      const float inv = lsum > 0.0f ? 1.0f / lsum : 0.0f;
      for (int s = lane; s < ns; s += 32) {
        const float l = mls[G * ns + gg * ns + s];
        mls[2 * G * ns + gg * ns + s] = l > 0.0f ? exp2f(mls[gg * ns + s] - M) * inv : 0.0f;
      }
    }
    __syncthreads();
    for (int t = tid; t < G * (kHeadDim / 4); t += kThreads) {
      const int gg = t / (kHeadDim / 4), q4 = t % (kHeadDim / 4);
      const float* w = mls + 2 * G * ns + gg * ns;
      const float4* src = reinterpret_cast<const float4*>(base + static_cast<int64_t>(gg) * ns * kPartialFloats) + q4;
      constexpr int kStride = kPartialFloats / 4;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      int s = 0;
      for (; s + 8 <= ns; s += 8) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = __ldcg(src + (s + u) * kStride);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float wu = w[s + u];
          acc.x = fmaf(v[u].x, wu, acc.x);
          acc.y = fmaf(v[u].y, wu, acc.y);
          acc.z = fmaf(v[u].z, wu, acc.z);
          acc.w = fmaf(v[u].w, wu, acc.w);
        }
      }
      for (; s < ns; ++s) {
        const float4 v = __ldcg(src + s * kStride);
        const float wu = w[s];
        acc.x = fmaf(v.x, wu, acc.x);
        acc.y = fmaf(v.y, wu, acc.y);
        acc.z = fmaf(v.z, wu, acc.z);
        acc.w = fmaf(v.w, wu, acc.w);
      }
      sm.q[gg][4 * q4] = acc.x;
      sm.q[gg][4 * q4 + 1] = acc.y;
      sm.q[gg][4 * q4 + 2] = acc.z;
      sm.q[gg][4 * q4 + 3] = acc.w;
    }
    if (tid == 0) a.tickets[b * a.num_kv_heads + h] = 0;  // ready for the next call
  }
  for (int t = G * kHeadDim + tid; t < 8 * kHeadDim; t += kThreads) sm.q[t / kHeadDim][t % kHeadDim] = 0.0f;
  __syncthreads();

  // rotate back once and store
  fwht8_smem<kThreads>(sm.q);
  for (int i = tid; i < G * kHeadDim; i += kThreads) {
    const int gg = i / kHeadDim;
    const int64_t oi = (static_cast<int64_t>(b) * a.num_q_heads + h * G + gg) * kHeadDim + i % kHeadDim;
    store_from_f32(a.out, a.out_dtype, oi, sm.q[gg][i % kHeadDim]);
  }
}

constexpr int kDecodeWarps = 8;

template <int G>
cudaError_t launch_g(const DecodeArgs& a, cudaStream_t stream) {
  constexpr int W = kDecodeWarps;
  const int smem = static_cast<int>(sizeof(DecodeSmem<W>));
  const cudaError_t e = ensure_smem_limit<decode_kernel<G, W>>(smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(a.nsplit, a.num_kv_heads, a.batch);
  decode_kernel<G, W><<<grid, W * 32, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

int decode_ctas_per_sm() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
  if (cached[dev] > 0) return cached[dev];
  constexpr int W = kDecodeWarps;
  const int smem = static_cast<int>(sizeof(DecodeSmem<W>));
  int n = 0;
  if (ensure_smem_limit<decode_kernel<8, W>>(smem) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_kernel<8, W>, W * 32, smem) != cudaSuccess || n < 1)
    n = 1;
  cached[dev] = n;
  return n;
}

int decode_max_splits() { return kMaxSplits; }

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.num_q_heads / a.num_kv_heads) {
    case 1: return launch_g<1>(a, stream);
    case 2: return launch_g<2>(a, stream);
    case 4: return launch_g<4>(a, stream);
    case 8: return launch_g<8>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace kvq
