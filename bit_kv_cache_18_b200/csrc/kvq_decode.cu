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

#ifndef KVQ_DECODE_WARPS
#define KVQ_DECODE_WARPS 8
#endif
constexpr int kDecodeWarps = KVQ_DECODE_WARPS;          // warps per CTA
constexpr int kStages = kDecodeWarps == 8 ? 6 : 8;      // segments in flight per warp
constexpr int kMinCtasPerSm = kDecodeWarps == 8 ? 2 : 3;
constexpr float kRescaleLog2 = 8.0f;  // lazy running-max threshold (log2 units)
constexpr int kMaxSplits = 64;      // the plan never cuts a sequence finer

template <int W>
struct __align__(128) DecodeSmem {
  uint8_t stage[W][kStages][kSegBytes];  // per-warp segment rings (then merge scratch)
  uint64_t bar[W][kStages];              // one mbarrier per stage
  uint4 qfrag[8][32];                    // QK A fragments, [k-step][lane]
  float q[8][kHeadDim];                  // rotated query rows (then the merged output)
  float qsum[8];
  float wm[W][8];
  float wl[W][8];
  float wf[8][W];  // per head: weight of each warp in the CTA merge
  float hm[8];
  float hl[8];
  int is_last;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// ---- TMA bulk copies completed on mbarriers ---------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
// One 1664-byte segment, global -> shared, by the TMA engine, issued by the
// lanes whose predicate is set (one per warp) without a branch: an
// async-proxy fence (orders earlier reads of the slot), the barrier's
// expected byte count, and the bulk copy that completes it.
__device__ __forceinline__ void bulk_load_segment_if(bool pred, uint8_t* dst, const uint8_t* src, uint64_t* bar) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
      "@p fence.proxy.async.shared::cta;\n"
      "@p mbarrier.arrive.expect_tx.shared::cta.b64 _, [%2], %3;\n"
      "@p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %3, [%2]; }" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(smem_u32(bar)), "r"(kSegBytes), "r"(static_cast<uint32_t>(pred))
      : "memory");
}
// One 1664-byte segment, global -> shared, by the TMA engine; the barrier
// expects the bytes and completes its phase when they have landed.
__device__ __forceinline__ void bulk_load_segment(uint8_t* dst, const uint8_t* src, uint64_t* bar) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(kSegBytes)
               : "memory");
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(kSegBytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}
// Bounded, warp-uniform wait for a barrier phase (every lane polls; the warp
// leaves together): false if the copy never arrived, in which case the caller
// records KVQ_ERR_DEVICE_TIMEOUT instead of hanging.
constexpr uint32_t kWaitLimit = 1u << 22;
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  for (uint32_t it = 0; it < kWaitLimit; ++it)
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  return false;
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
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

constexpr uint32_t kBias = 0x64006400u;
// (x & mask) | bias in one LOP3 (mask an immediate, bias a register), then
// the bias subtracted: the masked codes as exact fp16 numbers.
template <uint32_t kMask>
__device__ __forceinline__ uint32_t codes_f16(uint32_t x, uint32_t bias) {
  uint32_t t, d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(t) : "r"(x), "n"(kMask), "r"(bias));
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(t), "r"(bias));
  return d;
}


__device__ __forceinline__ float2 half2_at(const uint8_t* p) {
  return __half22float2(*reinterpret_cast<const __half2*>(p));
}

// Walsh-Hadamard transform of one 128-vector held by a warp, element
// lane + 32k in x[k]: the stride-32 and stride-64 butterflies in registers,
// strides 1..16 by shuffles (the lower index of a pair keeps u + v, the upper
// one u - v), then the 1/sqrt(128) factor times `scale`.
__device__ __forceinline__ void fwht_warp(float (&x)[4], int lane, float scale) {
  const float y0 = x[0] + x[1], y1 = x[0] - x[1], y2 = x[2] + x[3], y3 = x[2] - x[3];
  x[0] = y0 + y2;
  x[2] = y0 - y2;
  x[1] = y1 + y3;
  x[3] = y1 - y3;
#pragma unroll
  for (int st = 1; st < 32; st <<= 1) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float o = __shfl_xor_sync(0xffffffffu, x[k], st);
      x[k] = (lane & st) ? o - x[k] : x[k] + o;
    }
  }
  const float f = 0.088388347648318440550f * scale;
#pragma unroll
  for (int k = 0; k < 4; ++k) x[k] *= f;
}

__device__ __forceinline__ float ex2(float x) {  // 2^x (MUFU.EX2); ex2(-inf) = 0
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int G, int W>
__global__ void __launch_bounds__(W * 32, kMinCtasPerSm) decode_kernel(DecodeArgs a) {
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
  //      and the first kStages segments in flight (lane 0 drives the TMA)
  int32_t win0 = lane < nmine ? bt_row[W * lane] : -1;
  int32_t win1 = 32 + lane < nmine ? bt_row[W * (32 + lane)] : -1;
  int wbase = 0;
  if (lane == 0) {
#pragma unroll
    for (int s2 = 0; s2 < kStages; ++s2) mbar_init(&sm.bar[warp][s2], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  uint32_t valid_bits = 0;  // bit s: a copy into slot s is in flight / landed
  uint32_t phase_bits = 0;  // bit s: parity of slot s's next completion
#pragma unroll
  for (int i = 0; i < kStages; ++i) {
    const int32_t p = __shfl_sync(0xffffffffu, win0, i);
    if (i < nmine) {
      if (p >= 0 && p < a.num_blocks) {
        if (lane == 0) bulk_load_segment(sm.stage[warp][i], pool_h + p * pstride, &sm.bar[warp][i]);
        valid_bits |= 1u << i;
      } else if (lane == 0) {
        record_status(a.status, KVQ_ERR_OUT_OF_RANGE);
      }
    }
  }

  // ---- 2. rotate the query (overlaps the copies in flight): warp w < 8
  //      owns query head w of this kv head.  tau*log2(e) is folded into q~,
  //      so scores come out of the MMA already in base-2 logits.
  for (int gg = warp; gg < 8; gg += W) {
    float x[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (gg < G) {
      const int64_t q0 = (static_cast<int64_t>(b) * a.num_q_heads + h * G + gg) * kHeadDim;
#pragma unroll
      for (int k = 0; k < 4; ++k) x[k] = load_as_f32(a.q, a.q_dtype, q0 + lane + 32 * k);
    }
    fwht_warp(x, lane, a.scale_log2);
    float s4 = (x[0] + x[1]) + (x[2] + x[3]);
#pragma unroll
    for (int o = 16; o; o >>= 1) s4 += __shfl_xor_sync(0xffffffffu, s4, o);
#pragma unroll
    for (int k = 0; k < 4; ++k) sm.q[gg][lane + 32 * k] = x[k];
    if (lane == 0) sm.qsum[gg] = s4;
  }
  __syncthreads();

  // QK A fragments in smem, [k-step][lane], built by warp kk for its k-step
  // and read back with one 16-byte load per k-step.  k-step kk reads word
  // w = 4c + kk/2 of a key row (dims 8w..8w+7).  Slots (2c, 2c+1) take dims
  // (8w+e, 8w+e+4) and slots (2c+8, 2c+9) take (8w+e+1, 8w+e+5), e = 0 for
  // even kk and 2 for odd kk; the second pair's codes sit 4 bits higher (x16),
  // so its q is /16.
  for (int kk = warp; kk < 8; kk += W) {
    const int w = 4 * c + (kk >> 1);
    const int e = (kk & 1) ? 2 : 0;
    const float* qr = sm.q[g];
    uint4 f;
    split_pair(qr[8 * w + e], qr[8 * w + e + 4], f.x, f.y);
    split_pair(qr[8 * w + e + 1] * 0.0625f, qr[8 * w + e + 5] * 0.0625f, f.z, f.w);
    sm.qfrag[kk][lane] = f;
  }
  const float zq = sm.qsum[g];
  __syncthreads();

  // PV B operand through ldmatrix.trans: 8x8 tiles of 16-bit elements of the
  // value rows (tokens x 8 crumbs).  Tile i covers tokens 8(i/2)..8(i/2)+7 and
  // dims 64(i%2)..64(i%2)+63; after the transpose lane (g, c) holds, for
  // tokens (2c, 2c+1) of the tile, the 16 bits of dims 64h+8g .. 64h+8g+7.
  // n-tile (h, k) takes crumb k of those 16 bits, i.e. column g is dim
  // 64h + 8g + k.  Crumbs 0..4 are masked in place (code times 4^k), crumbs
  // 5..7 after a 10-bit shift (code times 4^(k-5)).
  const int ld_tok = ((lane >> 4) << 3) + (lane & 7);
  const int ld_half = (lane >> 3) & 1;

  uint32_t bias;
  asm volatile("mov.b32 %0, %1;" : "=r"(bias) : "n"(kBias));

  float o[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.0f;
  float m_ref = -CUDART_INF_F;
  float l_part = 0.0f, z_part = 0.0f;

  // ---- 3. the paged scan
  bool timed_out = false;
  int slot = 0;
#pragma unroll 1
  for (int i = 0; i < nmine; ++i, slot = (slot + 1 == kStages) ? 0 : slot + 1) {
    if (valid_bits & (1u << slot)) {
      if (!mbar_wait(&sm.bar[warp][slot], (phase_bits >> slot) & 1u)) {
        timed_out = true;
        break;
      }
      phase_bits ^= 1u << slot;
    }
    if (valid_bits & (1u << slot)) {
      const uint8_t* sg = sm.stage[warp][slot];
      const int ntok = min(kBlockSize, L - (blk0 + warp + W * i) * kBlockSize);

      // scores: n-tile j holds tokens 8j..8j+7, column g is token 8j+g
      float sacc[2][2][4];  // [n-tile][chain: even / odd k-steps]
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) sacc[j][ch][0] = sacc[j][ch][1] = sacc[j][ch][2] = sacc[j][ch][3] = 0.0f;
      const uint4 kw0 = *reinterpret_cast<const uint4*>(sg + kOffK + g * kKRowBytes + 16 * c);
      const uint4 kw1 = *reinterpret_cast<const uint4*>(sg + kOffK + (8 + g) * kKRowBytes + 16 * c);
      const uint32_t words[2][4] = {{kw0.x, kw0.y, kw0.z, kw0.w}, {kw1.x, kw1.y, kw1.z, kw1.w}};
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint4 f = sm.qfrag[kk][lane];
        const uint32_t qa[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint32_t w = (kk & 1) ? (words[j][kk >> 1] >> 8) : words[j][kk >> 1];
          mma16816(sacc[j][kk & 1], qa, codes_f16<0x000F000Fu>(w, bias), codes_f16<0x00F000F0u>(w, bias));
        }
      }
      // fold S_K, Z_K: s = tau log2e (S_K (hi + lo) + Z_K sum q~)
      float sc[4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float2 sk = half2_at(sg + kOffSK + 4 * (4 * j + c));
        const float2 zk = half2_at(sg + kOffZK + 4 * (4 * j + c));
        const float d0 = (sacc[j][0][0] + sacc[j][1][0]) + (sacc[j][0][2] + sacc[j][1][2]);
        const float d1 = (sacc[j][0][1] + sacc[j][1][1]) + (sacc[j][0][3] + sacc[j][1][3]);
        sc[2 * j] = fmaf(sk.x, d0, zk.x * zq);
        sc[2 * j + 1] = fmaf(sk.y, d1, zk.y * zq);
      }
      if (ntok < kBlockSize) {  // the last block of a sequence: drop the empty rows
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (8 * (q >> 1) + 2 * c + (q & 1) >= ntok) sc[q] = -CUDART_INF_F;
      }
      // Lazy running max: rescale only when a score exceeds the reference by
      // more than 8 (base 2).  Probabilities are taken relative to m_ref + 8,
      // p = 2^(s - m_ref - 8) <= 1, so p' = p S_V <= S_V always fits fp16;
      // o, l and zeta all carry the same factor, which the final o / l
      // cancels.  One warp vote decides; the head max (shuffles) and the
      // rescale run only when some lane needs them.
      const float mloc = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
      if (__any_sync(0xffffffffu, mloc > m_ref + kRescaleLog2)) {
        float mx = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        if (mx > m_ref + kRescaleLog2) {
          const float alpha = m_ref == -CUDART_INF_F ? 0.0f : ex2(m_ref - mx);
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
      }
      const float m8 = m_ref + kRescaleLog2;
      // probabilities with the value scale folded in: p' = p S_V
      float pv[4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float2 sv = half2_at(sg + kOffSV + 4 * (4 * j + c));
        float2 zv = half2_at(sg + kOffZV + 4 * (4 * j + c));
        if (ntok < kBlockSize) {  // rows past the end may hold NaN metadata
          if (8 * j + 2 * c >= ntok) sv.x = zv.x = 0.0f;
          if (8 * j + 2 * c + 1 >= ntok) sv.y = zv.y = 0.0f;
        }
        const float p0 = ex2(sc[2 * j] - m8);
        const float p1 = ex2(sc[2 * j + 1] - m8);
        l_part += p0 + p1;
        z_part = fmaf(p0, zv.x, fmaf(p1, zv.y, z_part));
        pv[2 * j] = p0 * sv.x;
        pv[2 * j + 1] = p1 * sv.y;
      }
      uint32_t pa[4];
      split_pair(pv[0], pv[1], pa[0], pa[1]);
      split_pair(pv[2], pv[3], pa[2], pa[3]);

      // p'.c_V: one ldmatrix.x4.trans gives this lane's value operands
      uint32_t vr[4];
      {
        const uint32_t addr = smem_u32(sg + kOffV + ld_tok * kVRowBytes + 16 * ld_half);
        asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                     : "=r"(vr[0]), "=r"(vr[1]), "=r"(vr[2]), "=r"(vr[3])
                     : "r"(addr));
      }
      const uint32_t vs[4] = {vr[0] >> 10, vr[1] >> 10, vr[2] >> 10, vr[3] >> 10};
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        mma16816(o[8 * h2 + 0], pa, codes_f16<0x00030003u>(vr[h2], bias), codes_f16<0x00030003u>(vr[2 + h2], bias));
        mma16816(o[8 * h2 + 1], pa, codes_f16<0x000C000Cu>(vr[h2], bias), codes_f16<0x000C000Cu>(vr[2 + h2], bias));
        mma16816(o[8 * h2 + 2], pa, codes_f16<0x00300030u>(vr[h2], bias), codes_f16<0x00300030u>(vr[2 + h2], bias));
        mma16816(o[8 * h2 + 3], pa, codes_f16<0x00C000C0u>(vr[h2], bias), codes_f16<0x00C000C0u>(vr[2 + h2], bias));
        mma16816(o[8 * h2 + 4], pa, codes_f16<0x03000300u>(vr[h2], bias), codes_f16<0x03000300u>(vr[2 + h2], bias));
        mma16816(o[8 * h2 + 5], pa, codes_f16<0x00030003u>(vs[h2], bias), codes_f16<0x00030003u>(vs[2 + h2], bias));
        mma16816(o[8 * h2 + 6], pa, codes_f16<0x000C000Cu>(vs[h2], bias), codes_f16<0x000C000Cu>(vs[2 + h2], bias));
        mma16816(o[8 * h2 + 7], pa, codes_f16<0x00300030u>(vs[h2], bias), codes_f16<0x00300030u>(vs[2 + h2], bias));
      }
    } else if (lane == 0 && i >= kStages) {
      record_status(a.status, KVQ_ERR_OUT_OF_RANGE);
    }
    __syncwarp();  // every lane is done reading the slot before it is refilled
    // refill this slot with the warp's block j = i + kStages
    const int j = i + kStages;
    valid_bits &= ~(1u << slot);
    if (j < nmine) {
      if (j >= wbase + 32) {  // slide the block-table window by 32 entries
        win0 = win1;
        wbase += 32;
        win1 = wbase + 32 + lane < nmine ? bt_row[W * (wbase + 32 + lane)] : -1;
      }
      const int32_t p = __shfl_sync(0xffffffffu, win0, j - wbase);
      if (p >= 0 && p < a.num_blocks) {
        bulk_load_segment_if(lane == 0, sm.stage[warp][slot], pool_h + p * pstride, &sm.bar[warp][slot]);
        valid_bits |= 1u << slot;
      }
    }
  }
  if (timed_out) {
    // a copy never landed: report it, give the others a bounded chance to
    // finish, and leave this warp's contribution empty
    if (lane == 0) record_status(a.status, KVQ_ERR_DEVICE_TIMEOUT);
    for (int s2 = 0; s2 < kStages; ++s2)
      if (valid_bits & (1u << s2)) mbar_wait(&sm.bar[warp][s2], (phase_bits >> s2) & 1u);
    m_ref = -CUDART_INF_F;
    l_part = z_part = 0.0f;
  }

  // ---- 4. merge: lanes of a head, then warps, then splits
  l_part += __shfl_xor_sync(0xffffffffu, l_part, 1);
  l_part += __shfl_xor_sync(0xffffffffu, l_part, 2);
  z_part += __shfl_xor_sync(0xffffffffu, z_part, 1);
  z_part += __shfl_xor_sync(0xffffffffu, z_part, 2);
  __syncthreads();  // every warp is done with its stages: reuse them
  float(*wo)[8][kHeadDim] = reinterpret_cast<float(*)[8][kHeadDim]>(&sm.stage[0][0][0]);
  {
    // n-tile (h, k) column n is dim 64h + 8n + k; its codes carry 4^k
    // (k <= 4) or 4^(k-5) (k >= 5)
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float f = 1.0f / static_cast<float>(1 << (2 * (k < 5 ? k : k - 5)));
        const int nt = 8 * h2 + k;
        wo[warp][g][64 * h2 + 16 * c + k] = fmaf(o[nt][0] + o[nt][2], f, z_part);
        wo[warp][g][64 * h2 + 16 * c + 8 + k] = fmaf(o[nt][1] + o[nt][3], f, z_part);
      }
    }
    if (c == 0) {
      sm.wm[warp][g] = m_ref;
      sm.wl[warp][g] = l_part;
    }
  }
  __syncthreads();
  // per head: the warps' common max, their weights 2^(m_w - M), and l
  if (tid < G) {
    const int gg = tid;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < W; ++w)
      if (sm.wl[w][gg] > 0.0f) M = fmaxf(M, sm.wm[w][gg]);
    float lsum = 0.0f;
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const float f = sm.wl[w][gg] > 0.0f ? ex2(sm.wm[w][gg] - M) : 0.0f;
      sm.wf[gg][w] = f;
      lsum = fmaf(sm.wl[w][gg], f, lsum);
    }
    sm.hm[gg] = M;
    sm.hl[gg] = lsum;
  }
  __syncthreads();
  for (int t = tid; t < G * kHeadDim; t += kThreads) {
    const int gg = t / kHeadDim, d = t % kHeadDim;
    float acc = 0.0f;
#pragma unroll
    for (int w = 0; w < W; ++w) acc = fmaf(wo[w][gg][d], sm.wf[gg][w], acc);
    const float M = sm.hm[gg], lsum = sm.hl[gg];
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
    for (int gg = warp; gg < G; gg += W) {
      float M = -CUDART_INF_F;
      for (int s = lane; s < ns; s += 32)
        if (mls[G * ns + gg * ns + s] > 0.0f) M = fmaxf(M, mls[gg * ns + s]);
#pragma unroll
      for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
      float lsum = 0.0f;
      for (int s = lane; s < ns; s += 32) {
        const float l = mls[G * ns + gg * ns + s];
        if (l > 0.0f) lsum = fmaf(l, ex2(mls[gg * ns + s] - M), lsum);
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
      const float inv = lsum > 0.0f ? 1.0f / lsum : 0.0f;
      for (int s = lane; s < ns; s += 32) {
        const float l = mls[G * ns + gg * ns + s];
        mls[2 * G * ns + gg * ns + s] = l > 0.0f ? ex2(mls[gg * ns + s] - M) * inv : 0.0f;
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
  __syncthreads();

  // rotate back once (warp w owns heads w, w+W, ...) and store
  for (int gg = warp; gg < G; gg += W) {
    float x[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) x[k] = sm.q[gg][lane + 32 * k];
    fwht_warp(x, lane, 1.0f);
    const int64_t o0 = (static_cast<int64_t>(b) * a.num_q_heads + h * G + gg) * kHeadDim;
#pragma unroll
    for (int k = 0; k < 4; ++k) store_from_f32(a.out, a.out_dtype, o0 + lane + 32 * k, x[k]);
  }
}

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
