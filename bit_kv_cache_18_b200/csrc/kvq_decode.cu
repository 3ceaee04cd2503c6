// kvq_decode.cu -- decode attention over the packed paged cache on the
// fifth-generation tensor cores (tcgen05), warp-specialised, in exact
// integer arithmetic.
//
// One CTA owns one (sequence b, kv head h, split of the context) and walks
// the split in chunks of 8 blocks = 128 tokens.  Three kinds of warps work on
// different chunks at the same time and hand buffers to each other through
// mbarrier rings of depth kNV:
//   * loader warps 0-3 (thread t <-> token t of a chunk <-> TMEM lane t):
//     bring their two segments of each chunk into a private kNV-slot
//     shared-memory ring with bulk copies (TMA, one instruction per segment)
//     kNV chunks ahead (the first ones after an L2 prefetch issued before
//     the dependency wait on the previous kernel); read them
//     with conflict-free 16-byte loads; spread the key codes (4 bits in the
//     default k4v2 preset, 2 or 8 in others) to one byte each into tensor
//     memory (A of QK, 16x256b stores whose fragment layout matches the
//     16-byte pieces) and the value codes (2 or 4 bits) to one byte each
//     into shared memory (A of PV), and publish the per-token factors as
//     stored (fp16; the softmax warps convert them);
//   * one MMA warp (tensor-memory owner) whose lane 0 issues, in order,
//     QK(0), QK(1), PV(0), QK(2), PV(1), ... as tcgen05.mma (M = 128, N = 32):
//       QK:  S  = codes_K (128 tok x 128) . digits(q~)^T  (u8 x s8 -> s32)
//       PV:  O += codes_V^T (128 pos x 128 tok) . digits(P') (u8 x u8 -> s32)
//   * softmax warps 4-7 (thread t <-> token t of S, value position t of O):
//     read a token's row of S, form the base-2 score of each of the G heads
//       s_g = S_K,t c1 (S0 + S1/254 + S2/254^2) + Z_K,t sum(q~_g),
//     the probability p = 2^(s_g - m_g) and P'_g = p S_V,t as a 32-bit fixed
//     point whose four bytes are four u8 digit columns of the PV operand,
//     and keep l_g = sum p and zeta_g = sum p Z_V in registers.
// For the fused decode step the MMA warp of the CTA whose split holds
// position L-1 quantizes the new token's K and V into that position during
// the set-up, while the query is rotated; the loaders copy that block after
// the set-up barrier.
// Before the scan the softmax warps rotate the G query heads once (warp
// FWHT, softmax scale times log2(e) folded in) and write q~ as three signed
// 8-bit digits, q~/c1 = Q0 + Q1/254 + Q2/254^2 with c1 = max|q~|/127.  After
// it they convert O to fp32 (o~ = sum P' c_V + zeta), write the split's
// partial (o~, m, l); the last CTA of (b, h) to take a ticket merges the
// splits and rotates back once, o = R o~ / l.  Scale folding at read time and
// the single rotations of the query and the output follow the KVarN pipeline
// list ("KVarN vs TurboQuant", dothoosh.com, fourth stage) and the
// definitions in include/kvq.h.  No CTA ever waits for another.
//
// Why integers: a tcgen05.mma with M = 128 costs about as much for N = 32
// as for N = 16, so each one should carry as much work as it can: u8 codes
// times 8-bit digits give K = 32 per instruction, the digits of q~ and P'
// fill the N columns a GQA group of 8 heads would leave empty, spreading a
// packed word to bytes is one or two logic operations per four codes, and
// every product and sum is exact.  The only roundings are the digit
// expansion of q~ (about 2^-22 of max|q~|) and the fixed point of P'
// (a step of 2^-29, with P' < 2^3).  The step must be that fine: tokens
// whose P' rounds to zero drop their S_V c_V but keep their p Z_V and p, and
// since codes are never negative that loss is a bias, not noise.
//
// Lazy running max.  m_g bounds s_g + E_t, E_t the exponent bound of
// S_V,t (S_V,t < 2^E_t, floored at -24), loosely: it only moves when some
// token has s_g + E_t > m_g + 2.9 (so P' < 2^3 always fits the fixed point),
// and then to the chunk's max of s_g + E_t plus a headroom of 2, which
// makes later moves rarer at the price of two bits of P' (the fixed point
// has them to spare).  A move is decided by one vote of the softmax warps
// per chunk (the scores are formed again from S for it, exactly).  The PVs
// then switch to the second integer accumulator, and the first is folded
// into fp32 registers with the factor 2^(m_old - m_new) one chunk later,
// when the PVs that ran into it are complete, so no warp waits for a PV.
// A split is at most 128 chunks (the block ids a CTA stages), which keeps
// every s32 sum of an accumulator below 2^31 (128 chunks x 128 tokens x 255
// x 255 < 2^31) without a restart.
//
// Code order.  The byte spreading permutes the 128 positions of a row (for
// k4v2 keys: position 32j + 8m + 4h + b holds dim 32m + 8j + 2b + h; values:
// position 16i + 4k + j holds dim 16i + 4j + k, times 4^k; the other
// presets' maps are given with key_pos_of_dim and value_dim_of_pos).  The
// query digits are written in the key order, so S is exact, and the output
// rows are put back in dim order, and divided by the spread's factor, when
// O is read.
#include <math_constants.h>

#include <type_traits>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

// Warp roles.  The default kernel has 4 loader warps (two segments of a
// chunk each), 4 softmax warps (one token each thread, all G heads) and the
// MMA warp: 288 threads, two CTAs per SM.  The wide kernel, for grids that
// fill the SMs once at one CTA per SM (small batches, where one CTA's chunk
// latency bounds the whole call), doubles the loader and softmax warps: a
// loader warp takes one segment, and two softmax threads share a token, four
// heads each (G = 8).
template <bool kWide>
struct Roles {
  static constexpr int kLoad = kWide ? 8 : 4;      // warps 0 .. kLoad-1
  static constexpr int kSoft = kWide ? 8 : 4;      // warps kLoad .. kMma-1
  static constexpr int kMma = kLoad + kSoft;       // tensor memory owner, MMA issue
  static constexpr int kThreads = 32 * (kMma + 1);  // 288 or 544
  static constexpr int kSegs = 8 / kLoad;          // segments a loader warp takes per chunk
};
constexpr int kChunkBlocks = 8;
constexpr int kChunkTokens = kChunkBlocks * kBlockSize;  // 128
constexpr int kMaxSplits = 256;    // the plan never cuts a sequence finer
constexpr int kTblBlocks = 1024;   // block ids a CTA stages in shared memory: no split is longer
// an integer accumulator of O takes at most this many chunks of u8 x u8 sums
static_assert(kTblBlocks / 8 * 128 * 255 * 255 < 2147483647ll, "s32 sums of one split stay below 2^31");
constexpr int kNS = 2;             // score buffers in tensor memory
constexpr int kNV = 3;             // key-code buffers in tensor memory; value / P' / factor buffers in smem
constexpr float kFix = 536870912.0f;  // P'_int = rne(P' 2^29) < 2^32
constexpr float kFixInv = 1.0f / 536870912.0f;
constexpr float kTrigger = 2.9f;    // move the max when s + E > m + kTrigger
// The running max before any token: far below every score (|s| stays far
// below 2^20 for fp16 factors), so the first token moves it and
// 2^(kNoMax - m) = 0, yet finite, so that s - m + m loses only the bits that
// the lazy max can spare.
constexpr float kNoMax = -1048576.0f;
constexpr float kHeadroom = 2.0f;  // a move sets m to the chunk's max of s + E plus this
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColA = 0;    // key codes of chunk c: kColA + 32 (c % 3)
constexpr uint32_t kColS = 96;   // S of chunk c: kColS + 32 (c % 2)
constexpr uint32_t kColO = 160;  // O accumulators: kColO + 32 k, k = 0, 1
constexpr uint32_t kColAcc = 224;  // per value position (lane): o~ so far in fp32, column g for head g
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // a device-side wait gives up after one second
constexpr int kBarSoftSync = 1;  // named barrier of the softmax threads
constexpr int kBarSoftVote = 2;  // named barrier for their vote

// Instruction descriptors (kind::i8, D = s32, M = 128, N = 32):
//   QK: A = u8 key codes (TMEM, K-major), B = s8 query digits (smem, K-major)
//   PV: A = u8 value codes (smem, MN-major), B = u8 P' digits (smem, MN-major)
constexpr uint32_t kIdescQK = (2u << 4) | (0u << 7) | (1u << 10) | ((32u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV =
    (2u << 4) | (0u << 7) | (0u << 10) | (1u << 15) | (1u << 16) | ((32u >> 3) << 17) | ((128u >> 4) << 24);

// Shared memory.  Operand tiles use the no-swizzle canonical layouts of
// 8-row x 16-byte core matrices:
//   vt (A of PV, MN-major): byte (tok, pos) at (tok/8)*1024 + (pos/16)*128 + (tok%8)*16 + pos%16
//   pm (B of PV, MN-major): byte (tok, n)   at (tok/8)*256  + (n/16)*128   + (tok%8)*16 + n%16
//   qb (B of QK, K-major):  byte (n, pos)   at (pos/16)*512 + (n/8)*128    + (n%8)*16   + pos%16
// S column n = 8j + g holds digit j of head g (rows 24..31 of qb are zero);
// P' and O column n = 4g + j hold byte j of head g.
template <int kSeg, bool kWide>  // segment bytes of the preset; the role layout
struct __align__(1024) Smem {
  using R = Roles<kWide>;
  uint8_t vt[kNV][kChunkTokens * kHeadDim];  // 3 x 16 KB
  uint8_t pm[kNV][kChunkTokens * 32];        // 3 x 4 KB
  uint8_t qb[32 * kHeadDim];                 // 4 KB
  uint16_t meta[kNV][4][kChunkTokens];       // per token, fp16 bits: S_K, Z_K, S_V (-1: segment absent), Z_V
  union {
    uint8_t stg[R::kLoad][kNV][R::kSegs * kSeg];  // loader warp w: its segments of chunk c in slot c % 3
    float obuf[8][kHeadDim];                      // o~ (epilogue, after the scan)
  };
  int32_t tbl[kTblBlocks];                   // the split's block ids, -1 where absent (outside the split,
                                             // the sequence or the pool)
  float2 hq[8];                              // per head: sum(q~), max|q~|
  float red[R::kSoft][8][2];                 // cross-warp reductions
  float palpha[R::kSoft][8];                 // per softmax warp: factor of the pending O buffer
  float c1;                                  // max|q~| / 127: the unit of the query digits
  uint64_t kv_ready[kNV];  // loaders -> MMA warp, softmax: codes and factors of chunk c written
  uint64_t qk_done[kNS];   // QK(c) complete -> softmax: S of chunk c ready (and PV(c-3) complete)
  uint64_t s_free[kNS];    // softmax -> MMA warp: S of chunk c read
  uint64_t p_ready[kNV];   // softmax -> MMA warp: P' of chunk c written
  uint64_t pv_done[kNV];   // PV(c) complete -> loaders, softmax (and QK(c+1) complete)
  uint64_t full[R::kLoad][kNV];  // TMA -> loader warp w: segments of chunk c in slot c % 3
  uint64_t fin;            // every MMA issued is complete
  uint32_t tmem_base;
  int fresh[kNV];          // PV of chunk c: bit 0 starts the accumulator afresh, bit 1 its O buffer
  int is_last;
  int abort;              // a wait ran out: every other wait gives up at once
};
template <int kSeg, bool kWide = false>
constexpr int kSmemBytesOf = static_cast<int>((sizeof(Smem<kSeg, kWide>) + 1023) / 1024 * 1024);
static_assert(kSmemBytesOf<Fmt<4, 2>::kSegBytes> <= 113 * 1024, "two CTAs per SM (k4v2)");
static_assert(kSmemBytesOf<Fmt<2, 2>::kSegBytes> <= 113 * 1024, "two CTAs per SM (k2v2)");
static_assert(kSmemBytesOf<Fmt<8, 4>::kSegBytes> <= 227 * 1024, "one CTA per SM (k8v4)");
// The tensor-memory rule of kvq_internal.cuh: no SM holds three of these
// CTAs (each allocates 256 of the 512 columns), since three never fit in the
// SM's 228 KB of shared memory (1 KB per CTA is reserved by the hardware).
static_assert(3 * (kSmemBytesOf<Fmt<2, 2>::kSegBytes> + 1024) > 228 * 1024, "at most two decode CTAs per SM");

// Position in a ring of three buffers and the parity of its current use.
struct Ring3 {
  int i;
  uint32_t ph;
  __device__ __forceinline__ void next() {
    if (++i == 3) {
      i = 0;
      ph ^= 1u;
    }
  }
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// sm_100 shared-memory matrix descriptor: start address, leading and stride
// byte offsets in 16-byte units, version 1, no swizzle.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(smem_u32(bar)) : "memory");
}
// Arrive once and expect `bytes` more from the bulk copies tracked here.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
// Bulk copy (TMA, no tensor map) of `bytes` from global to this CTA's shared
// memory, completing on `bar`; both addresses 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
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
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded, warp-uniform wait for a barrier phase.  False if it did not come
// within `limit_ns` nanoseconds (the global timer decides; a try_wait may
// suspend the thread for a while, so a count of polls would bound nothing)
// or another warp already gave up (then every later wait returns at once
// and the kernel runs to its end on void data, which it reports; the loaders
// stop issuing copies and wait for those in flight before the CTA exits).
// The slow loop is a call, one copy per preset (kTag), which keeps the wait
// sites small.
template <int kTag>
__device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, volatile int* abort, uint64_t limit_ns) {
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    if ((it & 15u) == 0u) {
      if (__any_sync(0xffffffffu, *abort != 0)) return false;
      if (__any_sync(0xffffffffu, global_ns() - t0 > limit_ns)) break;
    }
  }
  *abort = 1;
  return false;
}
template <int kTag>
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  return mbar_wait_slow<kTag>(bar, parity, abort, kWaitLimitNs);
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void async_proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
template <int kN>  // the softmax threads
__device__ __forceinline__ void soft_sync() { asm volatile("bar.sync %0, %1;" ::"n"(kBarSoftSync), "n"(kN) : "memory"); }
template <int kN>
__device__ __forceinline__ bool soft_vote_any(bool x) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.or.pred q, %2, %3, p; selp.u32 %0, 1, 0, q; }"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(x)), "n"(kBarSoftVote), "n"(kN)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void mma_qk(uint32_t d, uint32_t a, uint64_t bdesc, bool acc) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %3, 0;\n"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %4, p; }" ::"r"(d),
      "r"(a), "l"(bdesc), "r"(static_cast<uint32_t>(acc)), "r"(kIdescQK)
      : "memory");
}
__device__ __forceinline__ void mma_pv(uint32_t d, uint64_t adesc, uint64_t bdesc, bool acc) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %3, 0;\n"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %4, p; }" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(static_cast<uint32_t>(acc)), "r"(kIdescPV)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 16 lanes x 256 bits, 4 repetitions: registers 4j, 4j+1 go to lane
// (addr lane) + t/4, columns 8j + 2(t%4) + {0, 1}; registers 4j+2, 4j+3 to
// lane + 8 + t/4, same columns (t = thread in the warp).
__device__ __forceinline__ void tmem_st16x256(uint32_t addr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          addr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t addr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(addr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld8(uint32_t addr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t addr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(addr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// The 128-byte line holding p into L2.
__device__ __forceinline__ void prefetch_line_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
  return r;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 r;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr));
  return r;
}
__device__ __forceinline__ void sts64(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.b32 [%0], {%1,%2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

typedef unsigned long long u64x;
__device__ __forceinline__ u64x pk2(float a, float b) {
  u64x r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk2(u64x v, float& a, float& b) { asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v)); }
__device__ __forceinline__ u64x add2(u64x a, u64x b) {
  u64x d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ u64x mul2(u64x a, u64x b) {
  u64x d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ u64x fma2(u64x a, u64x b, u64x c) {
  u64x d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float ex2(float x) {  // 2^x (MUFU.EX2); ex2(-inf) = 0
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float h2f(uint32_t bits) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(bits)));
}
// Exact int -> float for |v| < 2^22 without the conversion unit: the
// integer added to the bits of 1.5 * 2^23 lands in the mantissa.
__device__ __forceinline__ float small_i2f(uint32_t v) {
  return __uint_as_float(v + 0x4B400000u) - 12582912.0f;
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

// The same transform of a 128-vector held with element 4 lane + k in x[k]:
// strides 1 and 2 in registers, strides 4 .. 64 by shuffles (lane xor
// stride / 4), then the 1/sqrt(128) factor.
__device__ __forceinline__ void fwht_warp_blocked(float (&x)[4], int lane) {
  const float y0 = x[0] + x[1], y1 = x[0] - x[1], y2 = x[2] + x[3], y3 = x[2] - x[3];
  x[0] = y0 + y2;
  x[1] = y1 + y3;
  x[2] = y0 - y2;
  x[3] = y1 - y3;
#pragma unroll
  for (int st = 1; st < 32; st <<= 1) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float o = __shfl_xor_sync(0xffffffffu, x[k], st);
      x[k] = (lane & st) ? o - x[k] : x[k] + o;
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) x[k] *= 0.088388347648318440550f;
}

// Position of dim d in a spread key row of KB-bit codes (with 32m + 8j + 4h
// + b the byte b of column 8j + 2(l%4) + h written by lane l, m = l%4):
//   KB = 4: position 32j + 8m + 4h + b holds dim 32m + 8j + 2b + h
//   KB = 8: position 32j + 8m + e holds dim 32m + 8j + e (the raw bytes)
//   KB = 2: position 32j + 8m + 4h + b holds dim 32m + 16(j/2) + 4b + 2(j%2) + h
template <int KB>
__device__ __forceinline__ int key_pos_of_dim(int d) {
  const int m = d >> 5, r = d & 31;
  if (KB == 4) return ((r >> 3) & 3) << 5 | m << 3 | (r & 1) << 2 | ((r >> 1) & 3);
  if (KB == 8) return ((r >> 3) & 3) << 5 | m << 3 | (r & 7);
  const int j = 2 * (r >> 4) + ((r >> 1) & 1);
  return j << 5 | m << 3 | (r & 1) << 2 | ((r >> 2) & 3);
}
// Dim of position p in a spread value row and log2 of the factor the spread
// multiplied its code by:
//   VB = 2: position 16i + 4k + b holds dim 16i + 4b + k, times 4^k
//   VB = 4: position 32m + 16h + 4w + b holds dim 32m + 8w + 2b + h, times 16^h
template <int VB>
__device__ __forceinline__ int value_dim_of_pos(int p) {
  if (VB == 2) return (p & ~15) | ((p & 3) << 2) | ((p >> 2) & 3);
  return (p & ~31) | (((p >> 2) & 3) << 3) | ((p & 3) << 1) | ((p >> 4) & 1);
}
template <int VB>
__device__ __forceinline__ uint32_t value_scale_log2(int p) {
  return VB == 2 ? 2u * ((p >> 2) & 3) : 4u * ((p >> 4) & 1);
}

// Raw key codes of one segment row pair for lane l (rows l/4 and 8 + l/4,
// dims 32(l%4) .. +31 of each) and their spread into the 16 words of a
// tcgen05.st.16x256b.x4 (registers 4j, 4j+1: row l/4, columns
// 8j + 2(l%4) + 0/1; registers 4j+2, 4j+3: row 8 + l/4).
template <int KB>
struct KeyRaw;
template <>
struct KeyRaw<4> {
  uint4 a, b;
  __device__ __forceinline__ void load(uint32_t k, int lane);
  __device__ __forceinline__ void spread(uint32_t (&w)[16]) const;
};
template <>
struct KeyRaw<8> {
  uint4 a0, a1, b0, b1;
  __device__ __forceinline__ void load(uint32_t k, int lane);
  __device__ __forceinline__ void spread(uint32_t (&w)[16]) const;
};
template <>
struct KeyRaw<2> {
  uint2 a, b;
  __device__ __forceinline__ void load(uint32_t k, int lane);
  __device__ __forceinline__ void spread(uint32_t (&w)[16]) const;
};
// 4-bit: 16 bytes of each row; nibbles to bytes (even dims, odd dims)
__device__ __forceinline__ void KeyRaw<4>::load(uint32_t k, int lane) {
  a = lds128(k + 16 * lane);
  b = lds128(k + 512 + 16 * lane);
}
__device__ __forceinline__ void KeyRaw<4>::spread(uint32_t (&w)[16]) const {
  const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    w[4 * j] = wa[j] & 0x0F0F0F0Fu;
    w[4 * j + 1] = (wa[j] >> 4) & 0x0F0F0F0Fu;
    w[4 * j + 2] = wb[j] & 0x0F0F0F0Fu;
    w[4 * j + 3] = (wb[j] >> 4) & 0x0F0F0F0Fu;
  }
}
// 8-bit: 32 bytes of each row, already one code per byte
__device__ __forceinline__ void KeyRaw<8>::load(uint32_t k, int lane) {
  a0 = lds128(k + 32 * lane);
  a1 = lds128(k + 32 * lane + 16);
  b0 = lds128(k + 1024 + 32 * lane);
  b1 = lds128(k + 1024 + 32 * lane + 16);
}
__device__ __forceinline__ void KeyRaw<8>::spread(uint32_t (&w)[16]) const {
  const uint32_t wa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
  const uint32_t wb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    w[4 * j] = wa[2 * j];
    w[4 * j + 1] = wa[2 * j + 1];
    w[4 * j + 2] = wb[2 * j];
    w[4 * j + 3] = wb[2 * j + 1];
  }
}
// 2-bit: 8 bytes of each row; word u, shift 2k -> register 4(2u + k/2) + k%2
__device__ __forceinline__ void KeyRaw<2>::load(uint32_t k, int lane) {
  a = lds64(k + 8 * lane);
  b = lds64(k + 256 + 8 * lane);
}
__device__ __forceinline__ void KeyRaw<2>::spread(uint32_t (&w)[16]) const {
  const uint32_t wa[2] = {a.x, a.y}, wb[2] = {b.x, b.y};
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int j = 2 * u + (k >> 1), hh = k & 1;
      w[4 * j + hh] = (wa[u] >> (2 * k)) & 0x03030303u;
      w[4 * j + 2 + hh] = (wb[u] >> (2 * k)) & 0x03030303u;
    }
}

// Bounded wait that ignores the abort flag: the issuer's last wait for its
// own MMAs, so tensor memory is never released under a running MMA.
__device__ __forceinline__ bool mbar_wait_final(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    if ((it & 15u) == 0u && __any_sync(0xffffffffu, global_ns() - t0 > kWaitLimitNs)) return false;
  }
}
// CTAs per SM the shared memory of a preset allows (two for k4v2 and k2v2).
template <int KB, int VB>
constexpr int kMinCtasOf = kSmemBytesOf<Fmt<KB, VB>::kSegBytes> <= 113 * 1024 ? 2 : 1;

// Segment (block) s of a chunk of 8 that loader warp w takes as its sg-th:
// TMEM lanes 16 s .. 16 s + 15 lie in the warp's lane quarter w % 4.
template <bool kWide>
__device__ __forceinline__ int seg_of(int w, int sg) {
  return kWide ? 2 * (w & 3) + (w >> 2) : 2 * w + sg;
}

// Split-K ticket of (b, h): one acquire-release add by thread 0 after the
// CTA barrier that published every thread's record stores (they happen
// before the add); in the last CTA, the barrier after the add makes every
// record visible to every thread's loads.  True in the last CTA.
__device__ __forceinline__ bool take_ticket(const DecodeArgs& a, int b, int h, int* is_last) {
  if (threadIdx.x == 0) {
    int t;
    asm volatile("atom.add.acq_rel.gpu.global.s32 %0, [%1], 1;"
                 : "=r"(t)
                 : "l"(a.tickets + b * a.num_kv_heads + h)
                 : "memory");
    *is_last = (t == a.nrec - 1);
  }
  __syncthreads();
  return *is_last != 0;
}

// The last CTA of (b, h) merges the a.nrec records of each of its G heads
// and writes the outputs.
template <int G, int kThreads>
__device__ __forceinline__ void merge_records(const DecodeArgs& a, int b, int h) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the last CTA of (b, h) merges the splits: warp g takes head g, lane l
  // dims 4l .. 4l+3 of every split and, in lane s, (m, l) of split s; all
  // loads of a batch of 16 splits are in flight at once, the weights go
  // round by shuffles, and batches merge online (max, rescale, sum)
  const int ns = a.nrec;
  const float* base = a.partials + (static_cast<int64_t>(b) * a.num_q_heads + h * G) * ns * kPartialFloats;
  for (int g = warp; g < G; g += kThreads / 32) {
    const float* hb = base + static_cast<int64_t>(g) * ns * kPartialFloats;
    float M = -CUDART_INF_F, lsum = 0.0f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < ns; s0 += 16) {
      float4 v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u)
        v[u] = s0 + u < ns ? __ldcg(reinterpret_cast<const float4*>(hb + static_cast<int64_t>(s0 + u) * kPartialFloats) + lane)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
      const float2 ml = lane < 16 && s0 + lane < ns
                            ? __ldcg(reinterpret_cast<const float2*>(hb + static_cast<int64_t>(s0 + lane) * kPartialFloats + kHeadDim))
                            : make_float2(0.f, 0.f);
      const bool has = ml.y > 0.0f;  // (an empty split has l = 0)
      float Mb = has ? ml.x : -CUDART_INF_F;
#pragma unroll
      for (int o = 16; o; o >>= 1) Mb = fmaxf(Mb, __shfl_xor_sync(0xffffffffu, Mb, o));
      Mb = fmaxf(Mb, M);
      const float f = M == -CUDART_INF_F ? 0.0f : ex2(M - Mb);
      const float w = has ? ex2(ml.x - Mb) : 0.0f;  // weight of split s0 + lane
      float lw = w * ml.y;
#pragma unroll
      for (int o = 16; o; o >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
      lsum = fmaf(lsum, f, lw);
      acc.x *= f;
      acc.y *= f;
      acc.z *= f;
      acc.w *= f;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float wu = __shfl_sync(0xffffffffu, w, u);
        acc.x = fmaf(wu, v[u].x, acc.x);
        acc.y = fmaf(wu, v[u].y, acc.y);
        acc.z = fmaf(wu, v[u].z, acc.z);
        acc.w = fmaf(wu, v[u].w, acc.w);
      }
      M = Mb;
    }
    // normalise and rotate back once, in the layout the merge left (lane l
    // holds dims 4l .. 4l+3), and store
    const float inv = lsum > 0.0f ? 1.0f / lsum : 0.0f;
    float x[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
    fwht_warp_blocked(x, lane);
    const int64_t o0 = (static_cast<int64_t>(b) * a.num_q_heads + h * G + g) * kHeadDim + 4 * lane;
#pragma unroll
    for (int k = 0; k < 4; ++k) store_from_f32(a.out, a.out_dtype, o0 + k, x[k]);
  }
  if (tid == 0) a.tickets[b * a.num_kv_heads + h] = 0;  // ready for the next call
}

// ---- bf16 window of sink and recent tokens --------------------------------
// With a window ("Kompresja pamięci podręcznej KV..." (encorp.ai), OSCAR
// section: the sink and the most recent tokens are kept in BF16), CTA x =
// nsplit of each (b, h) attends over the window rows of sequence b in fp32
// and hands its partial to the split-K merge as record nsplit; the split
// CTAs skip these positions of the pool.  Scores are formed in the original
// domain (q.k times the softmax scale and log2 e equals the cache's rotated
// q~.k~), then m = max s, p = 2^(s - m), l = sum p, o = sum p v, and o is
// rotated once into the cache's domain (R o; R = R^T = R^-1), which is the
// domain of every other record.  Window position i is sink row i for i <
// nsink, else position rec_lo + i - nsink in ring row sink + t % recent.
constexpr int kWinRowsMax = kMaxWindowSink + kMaxWindowRecent;
constexpr int kWinInFlight = 8;  // rows a warp loads ahead
// warps that walk the window rows: 8, or 16 in the wide layout
template <int kThreads>
constexpr int kWinWarpsOf = kThreads / 32 > 16 ? 16 : 8;
template <int G, int kThreads>
constexpr int kWindowSmemBytes = (kWinRowsMax * G + kWinWarpsOf<kThreads> * G * kHeadDim + 2 * G + 4) * 4;

// Sum over the warp of G values per lane, G = 1, 2, 4 or 8: log2 G halving
// exchanges (a lane keeps the half of its values that its lane bit selects
// and adds the other lane's copy of that half), then plain butterflies over
// the remaining lane bits.  Lane l returns the sum of value
// (l >> (5 - log2 G)) & (G - 1).
template <int G>
__device__ __forceinline__ float warp_sum_heads(float (&v)[G], int lane) {
  constexpr int kLog = G == 8 ? 3 : G == 4 ? 2 : G == 2 ? 1 : 0;
#pragma unroll
  for (int st = 0; st < kLog; ++st) {
    const int s = 16 >> st;
    const int n = G >> (st + 1);
    const bool up = (lane & s) != 0;
#pragma unroll
    for (int j = 0; j < n; ++j) {
      const float send = up ? v[j] : v[j + n];
      const float keep = up ? v[j + n] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  float x = v[0];
#pragma unroll
  for (int s = 16 >> kLog; s >= 1; s >>= 1) x += __shfl_xor_sync(0xffffffffu, x, s);
  return x;
}

template <int G, int kThreads>
__device__ __forceinline__ void window_part(const DecodeArgs& a, uint8_t* smem) {
  constexpr int kWinWarps = kWinWarpsOf<kThreads>;
  static_assert(kThreads / 32 >= kWinWarps && kWinWarps >= G, "enough warps for the window's rows and heads");
  const int h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* pw = reinterpret_cast<float*>(smem);                             // [kWinRowsMax][G]: s, then p
  float* part = pw + kWinRowsMax * G;                                     // [kWinWarps][G][128]: sums of p v
  float2* ml = reinterpret_cast<float2*>(part + kWinWarps * G * kHeadDim);  // [G]: (m, l)
  int* is_last = reinterpret_cast<int*>(ml + G);
  const int wrows = a.win_sink + a.win_recent;
  const uint16_t* wb = a.win + (static_cast<int64_t>(b) * a.num_kv_heads + h) * wrows * (2 * kHeadDim);
  pdl_trigger();  // this CTA holds no tensor memory
  // L2 prefetch of this (b, h)'s window rows, before the dependency wait (a
  // row written by the previous kernel is read after the wait, from L2, the
  // point of coherence)
  for (int r = tid; r < wrows; r += kThreads) prefetch_l2(wb + static_cast<int64_t>(r) * (2 * kHeadDim), 4 * kHeadDim);
  pdl_wait();
  // the length, cut as the split CTAs cut it (they record a bad one)
  int L = a.seq_lens[b];
  L = max(L, 0);
  L = min(L, a.max_seq_len);
  L = min(L, a.max_blocks_per_seq * kBlockSize);
  const int nsink = min(a.win_sink, L);
  const int rec_lo = a.win_recent > 0 ? max(L - a.win_recent, nsink) : L;
  const int nw = nsink + (L - rec_lo);  // <= sink + recent <= kWinRowsMax
  auto row_of = [&](int i) { return i < nsink ? i : a.win_sink + (rec_lo + i - nsink) % a.win_recent; };
  if (warp < kWinWarps) {
    // s: a warp per row (lane l: dims 4l .. 4l+3 of K and of every head's q)
    float qr[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int64_t q0 = (static_cast<int64_t>(b) * a.num_q_heads + h * G + g) * kHeadDim + 4 * lane;
#pragma unroll
      for (int k = 0; k < 4; ++k) qr[g][k] = load_as_f32(a.q, a.q_dtype, q0 + k) * a.scale_log2;
    }
    for (int i0 = warp; i0 < nw; i0 += kWinWarps * kWinInFlight) {
      uint2 kr[kWinInFlight];
#pragma unroll
      for (int u = 0; u < kWinInFlight; ++u) {
        const int i = i0 + u * kWinWarps;
        kr[u] = i < nw ? __ldg(reinterpret_cast<const uint2*>(wb + static_cast<int64_t>(row_of(i)) * (2 * kHeadDim)) + lane)
                       : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kWinInFlight; ++u) {
        const int i = i0 + u * kWinWarps;
        if (i >= nw) break;  // (warp-uniform)
        const float k0 = __uint_as_float(kr[u].x << 16), k1 = __uint_as_float(kr[u].x & 0xFFFF0000u);
        const float k2 = __uint_as_float(kr[u].y << 16), k3 = __uint_as_float(kr[u].y & 0xFFFF0000u);
        float d[G];
#pragma unroll
        for (int g = 0; g < G; ++g) d[g] = fmaf(qr[g][0], k0, fmaf(qr[g][1], k1, fmaf(qr[g][2], k2, qr[g][3] * k3)));
        const float sum = warp_sum_heads<G>(d, lane);
        constexpr int kShift = G == 8 ? 2 : G == 4 ? 3 : G == 2 ? 4 : 5;
        if ((lane & ((1 << kShift) - 1)) == 0) pw[i * G + (lane >> kShift)] = sum;
      }
    }
  }
  // the first rows of V go out now, under the barrier and the softmax below
  uint2 vr[kWinInFlight];
  auto load_v = [&](int i0) {
#pragma unroll
    for (int u = 0; u < kWinInFlight; ++u) {
      const int i = i0 + u * kWinWarps;
      vr[u] = i < nw ? __ldg(reinterpret_cast<const uint2*>(wb + static_cast<int64_t>(row_of(i)) * (2 * kHeadDim) +
                                                            kHeadDim) + lane)
                     : make_uint2(0u, 0u);
    }
  };
  if (warp < kWinWarps) load_v(warp);
  __syncthreads();
  // per head (warp g): m, p = 2^(s - m) in place, l
  if (warp < G) {
    const int g = warp;
    float m = -CUDART_INF_F;
    for (int i = lane; i < nw; i += 32) m = fmaxf(m, pw[i * G + g]);
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.0f;
    for (int i = lane; i < nw; i += 32) {
      const float pv = ex2(pw[i * G + g] - m);
      pw[i * G + g] = pv;
      l += pv;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) ml[g] = nw > 0 ? make_float2(m, l) : make_float2(0.0f, 0.0f);
  }
  __syncthreads();
  if (warp < kWinWarps) {
    // sum p v: a warp per row again (lane l: dims 4l .. 4l+3 of V), the G
    // probabilities of a row read at one shared-memory address by every lane
    float acc[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g) acc[g][0] = acc[g][1] = acc[g][2] = acc[g][3] = 0.0f;
    for (int i0 = warp; i0 < nw; i0 += kWinWarps * kWinInFlight) {
      if (i0 != warp) load_v(i0);
#pragma unroll
      for (int u = 0; u < kWinInFlight; ++u) {
        const int i = i0 + u * kWinWarps;
        if (i >= nw) break;
        const float v0 = __uint_as_float(vr[u].x << 16), v1 = __uint_as_float(vr[u].x & 0xFFFF0000u);
        const float v2 = __uint_as_float(vr[u].y << 16), v3 = __uint_as_float(vr[u].y & 0xFFFF0000u);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float pg = pw[i * G + g];
          acc[g][0] = fmaf(pg, v0, acc[g][0]);
          acc[g][1] = fmaf(pg, v1, acc[g][1]);
          acc[g][2] = fmaf(pg, v2, acc[g][2]);
          acc[g][3] = fmaf(pg, v3, acc[g][3]);
        }
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g)
      *reinterpret_cast<float4*>(part + (warp * G + g) * kHeadDim + 4 * lane) =
          make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
  }
  __syncthreads();
  // o over the warps, rotated once into the cache's domain (R o; R = R^T),
  // written as record nsplit (warp g: dims 4 lane + k)
  if (warp < G) {
    const int g = warp;
    float x[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int w = 0; w < kWinWarps; ++w) {
      const float4 t = *reinterpret_cast<const float4*>(part + (w * G + g) * kHeadDim + 4 * lane);
      x[0] += t.x;
      x[1] += t.y;
      x[2] += t.z;
      x[3] += t.w;
    }
    fwht_warp_blocked(x, lane);
    float* rg = a.partials + ((static_cast<int64_t>(b) * a.num_q_heads + h * G + g) * a.nrec + a.nsplit) * kPartialFloats;
    *reinterpret_cast<float4*>(rg + 4 * lane) = make_float4(x[0], x[1], x[2], x[3]);
    if (lane == 0) *reinterpret_cast<float2*>(rg + kHeadDim) = ml[g];
  }
  __syncthreads();
  if (take_ticket(a, b, h, is_last)) merge_records<G, kThreads>(a, b, h);
}

// kWin: the instantiation that takes a bf16 window (a.win set); the others
// carry no window code at all.
template <int G, int KB, int VB, bool kWide, bool kWin>
__global__ void __launch_bounds__(Roles<kWide>::kThreads, kWide ? 1 : kMinCtasOf<KB, VB>)
    decode_kernel(DecodeArgs a) {
  using F = Fmt<KB, VB>;
  using R = Roles<kWide>;
  constexpr int kLoadWarps = R::kLoad, kSoftWarps = R::kSoft, kMmaWarp = R::kMma, kThreads = R::kThreads;
  constexpr int kSegs = R::kSegs;                  // segments per loader warp and chunk
  constexpr int kSoftThreads = 32 * kSoftWarps;
  constexpr int kHeads = kWide ? G / 2 : G;        // heads a softmax thread takes (the wide layout: two threads a token)
  constexpr int kQHeads = 8 / kSoftWarps;          // query heads a softmax warp rotates at set-up (at most)
  static_assert(!kWide || G == 8, "the wide layout splits 8 heads over two threads");
  constexpr int kSeg = F::kSegBytes;
  constexpr int kWaitTag = 16 * KB + VB + (kWide ? 256 : 0);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem<kSeg, kWide>& sm = *reinterpret_cast<Smem<kSeg, kWide>*>(smem_raw);
  volatile int* abort = &sm.abort;
  const int split = blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const bool is_loader = warp < kLoadWarps;
  const bool is_soft = warp >= kLoadWarps && warp < kMmaWarp;
  static_assert(kWindowSmemBytes<G, kThreads> <= kSmemBytesOf<kSeg, kWide>, "the window part fits the CTA's shared memory");
  if constexpr (kWin) {
    if (split == a.nsplit) {  // the window's CTA of (b, h)
      window_part<G, kThreads>(a, smem_raw);
      return;
    }
  }

  // tensor memory and barriers touch no global memory: set up before
  // waiting for the previous kernel in the stream
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                 "n"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    if (lane == 0) {
#pragma unroll
      for (int i = 0; i < kNV; ++i) {
        mbar_init(&sm.kv_ready[i], kLoadWarps);  // one elected lane per warp arrives
        mbar_init(&sm.p_ready[i], kSoftWarps);
        mbar_init(&sm.pv_done[i], 1);
      }
#pragma unroll
      for (int i = 0; i < kNS; ++i) {
        mbar_init(&sm.qk_done[i], 1);
        mbar_init(&sm.s_free[i], kSoftWarps);
      }
      mbar_init(&sm.fin, 1);
      sm.abort = 0;
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
  } else if (warp < kLoadWarps) {
    // my staging ring's barriers (used by this warp only)
    if (lane == 0) {
#pragma unroll
      for (int i = 0; i < kNV; ++i) mbar_init(&sm.full[warp][i], 1);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    // Before the dependency wait: L2 prefetches only.  Nothing read here is
    // used for anything else (every real read comes after the wait, which
    // orders it after the previous kernel's writes; a stale line prefetched
    // now is updated in L2, the point of coherence, by any later write): the
    // split's block-table slice, the sequence length and, by the block ids
    // as they read now, the first three chunks' segments.
    const int pblk0 = blockIdx.x * a.blocks_per_split;
    const int pn = min(a.blocks_per_split, a.max_blocks_per_seq - pblk0);
    const int32_t* prow = a.block_table + static_cast<int64_t>(blockIdx.z) * a.max_blocks_per_seq + pblk0;
    for (int ln = tid; ln * 32 < pn; ln += 32 * kLoadWarps) prefetch_line_l2(prow + ln * 32);
    if (tid == 0) prefetch_line_l2(a.seq_lens + blockIdx.z);
    if (lane < kSegs * kNV) {
      const int blk = kChunkBlocks * (lane / kSegs) + seg_of<kWide>(warp, lane % kSegs);
      if (blk < pn) {
        int32_t p;
        asm volatile("ld.global.cg.s32 %0, [%1];" : "=r"(p) : "l"(prow + blk));
        if (p >= 0 && p < a.num_blocks)
          prefetch_l2(a.pool + (static_cast<int64_t>(p) * a.num_kv_heads + blockIdx.y) * Fmt<KB, VB>::kSegBytes,
                      Fmt<KB, VB>::kSegBytes);
      }
    }
  } else {
    // the query rows of this CTA's G heads (L2 prefetch, as above)
    const int sw = warp - kLoadWarps;
    const int esz = a.q_dtype == KVQ_F32 ? 4 : 2;  // a row is esz 128-byte lines
    const int g = sw + kSoftWarps * (lane >> 2);
    if (g < G && (lane & 3) < esz) {
      const char* qrow = static_cast<const char*>(a.q) +
                         ((static_cast<int64_t>(blockIdx.z) * a.num_q_heads + blockIdx.y * G + g) * kHeadDim) * esz;
      prefetch_line_l2(qrow + 128 * (lane & 3));
    }
  }
  pdl_wait();

  // The loads that need no sequence length go out first: softmax warp sw's
  // query heads sw, sw + kSoftWarps, ... and, in a fused step, the MMA
  // warp's lanes' 8 bytes of the new token's K and V rows.
  float x[kQHeads][4];
  uint2 new_k = make_uint2(0u, 0u), new_v = make_uint2(0u, 0u);
  if (is_soft) {
    const int sw = warp - kLoadWarps;
#pragma unroll
    for (int i = 0; i < kQHeads; ++i) {
      const int g = sw + kSoftWarps * i;
      if (g < G) {
        const int64_t q0 = (static_cast<int64_t>(b) * a.num_q_heads + h * G + g) * kHeadDim;
#pragma unroll
        for (int k = 0; k < 4; ++k) x[i][k] = load_as_f32(a.q, a.q_dtype, q0 + lane + 32 * k);
      }
    }
  } else if (warp == kMmaWarp && a.k_new != nullptr) {
    const int64_t off = static_cast<int64_t>(b) * a.new_stride_bytes + static_cast<int64_t>(h) * (kHeadDim * 2) + 8 * lane;
    new_k = *reinterpret_cast<const uint2*>(a.k_new + off);
    new_v = *reinterpret_cast<const uint2*>(a.v_new + off);
  }

  // ---- the split: blocks [blk0, blk1) of sequence b, in chunks of 8 -------
  // Loader warp w owns segment(s) seg_of(w, sg) of every chunk (tokens 16 s
  // .. 16 s + 15 = TMEM lanes of its quarter).  Before the sequence length is
  // known (every entry read is inside the table row), lanes sg < kSegs read
  // the block ids of their segment of chunks 0 .. 2; the split's whole slice
  // of the row goes to shared memory in the set-up below, cut to the split
  // and the pool.
  const int blk0 = split * a.blocks_per_split;
  const int32_t* bt_row = a.block_table + static_cast<int64_t>(b) * a.max_blocks_per_seq;
  constexpr int kTblPer = kTblBlocks / (32 * kLoadWarps);
  int32_t bfirst[kNV];  // loaders, lanes sg < kSegs: block ids of chunks 0 .. 2
  if (is_loader) {
    const int nload = min(a.blocks_per_split, a.max_blocks_per_seq - blk0);
#pragma unroll
    for (int i = 0; i < kNV; ++i) {
      const int j = kChunkBlocks * i + seg_of<kWide>(warp, lane % kSegs);
      bfirst[i] = lane < kSegs && j < nload ? __ldg(bt_row + blk0 + j) : -1;
    }
  }
  int L = a.seq_lens[b];
  // a length outside [0, max_seq_len] or beyond the table row is recorded
  // and the read is truncated to what the row covers; the fused append is
  // then skipped (its position would be a clamped one, not seq_lens[b] - 1)
  const bool l_bad = L < 0 || L > a.max_seq_len || L > a.max_blocks_per_seq * kBlockSize;
  if (l_bad) {
    if (tid == 0) record_status(a.status, KVQ_ERR_OUT_OF_RANGE);
    L = max(L, 0);
    L = min(L, a.max_seq_len);
    L = min(L, a.max_blocks_per_seq * kBlockSize);
  }
  const int nb = (L + kBlockSize - 1) / kBlockSize;
  // the positions read from the pool: [qlo, qhi) = [0, L) but, with a
  // window, its sink and recent positions; the split ends at the last block
  // that holds any
  int qlo = 0, qhi = L;
  if constexpr (kWin) {
    qlo = min(a.win_sink, L);
    qhi = a.win_recent > 0 ? max(L - a.win_recent, qlo) : L;
  }
  const int blk1 = min(min(nb, blk0 + a.blocks_per_split), (qhi + kBlockSize - 1) / kBlockSize);
  // a block holds positions read from the pool
  auto needed = [&](int blk) { return blk * kBlockSize < qhi && (blk + 1) * kBlockSize > qlo; };
  const int nchunks = blk1 > blk0 ? (blk1 - blk0 + kChunkBlocks - 1) / kChunkBlocks : 0;
  bool bad = false;      // a wait ran out: the results are void, the control flow is kept
  bool bad_blk = false;  // a block-table entry outside the pool (its tokens are skipped)

  const uint8_t* pool_h = a.pool + static_cast<int64_t>(h) * kSeg;
  const int64_t pstride = static_cast<int64_t>(a.num_kv_heads) * kSeg;
  const int mseg = lane >> 4;  // my factor bytes: those of the loader warp's mseg-th segment (< kSegs)

  const uint32_t my_stg = smem_u32(sm.stg[warp < kLoadWarps ? warp : 0][0]);
  // Bulk copies of the loader warp's segments of a chunk into staging slot
  // `slot`: lanes sg < kSegs pass their segment's block id (-1: absent,
  // nothing copied; the factors mark its tokens absent), every lane calls.
  // The expected byte count is posted before any copy is issued.
  auto issue = [&](int32_t p, int slot) {
    uint64_t* bar = &sm.full[warp][slot];
    const uint32_t okm = __ballot_sync(0xffffffffu, lane < kSegs && p >= 0);
    if (lane == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(__popc(okm)) * kSeg);
    __syncwarp();
    if (lane < kSegs && p >= 0)
      bulk_g2s(my_stg + slot * (kSegs * kSeg) + lane * kSeg, pool_h + static_cast<int64_t>(p) * pstride, kSeg, bar);
  };

  // ---- 0. set-up: barriers and tensor memory; first loads; query digits ----
  // the chunk holding the block that the fused append writes is copied only
  // after the set-up barrier (-1: none)
  int c_defer = -1;
  if (a.k_new != nullptr && L > 0 && !l_bad) {
    const int bn = (L - 1) / kBlockSize;
    if (bn >= blk0 && bn < blk1) c_defer = (bn - blk0) / kChunkBlocks;
  }

  if (is_loader) {
    // my block ids of chunks 0 .. 2, cut to the split and the pool
    const int nblk = blk1 - blk0;
#pragma unroll
    for (int i = 0; i < kNV; ++i) {
      const int j = kChunkBlocks * i + seg_of<kWide>(warp, lane % kSegs);
      if (!(j < nblk && needed(blk0 + j) && bfirst[i] >= 0 && bfirst[i] < a.num_blocks)) bfirst[i] = -1;
    }
    // the first three chunks' copies go out while the query is rotated (each
    // warp set up its staging ring's barriers before the dependency wait)
#pragma unroll
    for (int i = 0; i < kNV; ++i)
      if (i < nchunks && i != c_defer) issue(bfirst[i], i);
    // the split's slice of the block table, cut to the split and the pool
    // (an entry inside the sequence that names no block of the pool is
    // recorded and its tokens skipped); the set-up barrier publishes it
#pragma unroll 4
    for (int i = 0; i < kTblPer; ++i) {
      const int j = tid + 32 * kLoadWarps * i;
      const bool inside = j < nblk && needed(blk0 + j);
      const int32_t p = inside ? __ldg(bt_row + blk0 + j) : -1;
      const bool okp = inside && p >= 0 && p < a.num_blocks;
      bad_blk |= inside && !okp;
      sm.tbl[j] = okp ? p : -1;
    }
  } else if (is_soft) {
    const int sw = warp - kLoadWarps;
    const int st = tid - 32 * kLoadWarps;  // 0 .. kSoftThreads-1
    // rotate the G query heads, then write their digits with one c1 for all
    // heads
    for (int i = st; i < 32 * kHeadDim / 16; i += kSoftThreads) reinterpret_cast<uint4*>(sm.qb)[i] = make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int i = 0; i < kQHeads; ++i) {
      const int g = sw + kSoftWarps * i;
      if (g < G) {
        fwht_warp(x[i], lane, a.scale_log2);
        float s4 = (x[i][0] + x[i][1]) + (x[i][2] + x[i][3]);
        float mx = fmaxf(fmaxf(fabsf(x[i][0]), fabsf(x[i][1])), fmaxf(fabsf(x[i][2]), fabsf(x[i][3])));
#pragma unroll
        for (int o = 16; o; o >>= 1) {
          s4 += __shfl_xor_sync(0xffffffffu, s4, o);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        if (lane == 0) sm.hq[g] = make_float2(s4, mx);
      }
    }
    soft_sync<kSoftThreads>();
    float mx = 0.0f;
#pragma unroll
    for (int g = 0; g < G; ++g) mx = fmaxf(mx, sm.hq[g].y);
    const float inv = mx > 0.0f ? 127.0f / mx : 0.0f;
    if (st == 0) sm.c1 = mx * (1.0f / 127.0f);
#pragma unroll
    for (int i = 0; i < kQHeads; ++i) {
      const int g = sw + kSoftWarps * i;
      if (g < G) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int pos = key_pos_of_dim<KB>(lane + 32 * k);
          const float y = x[i][k] * inv;
          const float q1 = rintf(y);
          const float r1 = (y - q1) * 254.0f;
          const float q2 = rintf(r1);
          const float q3 = rintf((r1 - q2) * 254.0f);
          const float dig[3] = {q1, q2, q3};
#pragma unroll
          for (int j = 0; j < 3; ++j) {
            const int n = 8 * j + g;
            const int v = max(-127, min(127, static_cast<int>(dig[j])));
            sm.qb[(pos >> 4) * 512 + (n >> 3) * 128 + (n & 7) * 16 + (pos & 15)] = static_cast<uint8_t>(v & 0xFF);
          }
        }
      }
    }
    async_proxy_fence();
  } else if (c_defer >= 0) {
    // fused one-token append: the MMA warp (idle until the first chunk
    // lands) of the split holding position L-1 writes the new token's K and
    // V of kv head h into that position, in parallel with the query
    // rotation; the proxy fence and the set-up barrier order the writes
    // before the loaders' bulk copy of that block
    const int32_t p = __ldg(bt_row + (L - 1) / kBlockSize);
    if (p >= 0 && p < a.num_blocks) {
      uint8_t* seg = const_cast<uint8_t*>(pool_h) + static_cast<int64_t>(p) * pstride;
      const int row = (L - 1) % kBlockSize;
      if (a.new_bf16) {
        quantize_vector_warp_raw<true, KB, VB>(new_k, seg, row, false, lane);
        quantize_vector_warp_raw<true, KB, VB>(new_v, seg, row, true, lane);
      } else {
        quantize_vector_warp_raw<false, KB, VB>(new_k, seg, row, false, lane);
        quantize_vector_warp_raw<false, KB, VB>(new_v, seg, row, true, lane);
      }
      asm volatile("fence.proxy.async.global;" ::: "memory");
    } else if (lane == 0) {
      record_status(a.status, KVQ_ERR_OUT_OF_RANGE);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;
  const float c1 = sm.c1;

  // ---- 1. the paged scan ------------------------------------------------------
  if (is_loader) {
    // TMEM lanes of my segment sg: 16 seg_of(warp, sg) + [0, 16)
    auto seg_lanes = [&](int sg) { return tbase + (static_cast<uint32_t>(16 * seg_of<kWide>(warp, sg)) << 16); };
    // my value rows of segment sg (token base tb = 16 s).  VB = 2: row lane/2
    // of the segment, positions 64 (lane%2) + [0, 64); VB = 4: rows lane/4
    // and (+ 1024) 8 + lane/4, positions 32 (lane%4) + [0, 32)
    auto seg_vt = [&](int sg) -> uint32_t {
      const int tb = 16 * seg_of<kWide>(warp, sg);
      return VB == 2 ? smem_u32(sm.vt[0]) + ((tb + (lane >> 1)) >> 3) * 1024 + (lane & 1) * 512 + (lane >> 1 & 7) * 16
                     : smem_u32(sm.vt[0]) + (tb >> 3) * 1024 + (lane >> 2) * 16 + 2 * (lane & 3) * 128;
    };
    const int mrow0 = 4 * (lane & 3);    // my factor rows mrow0 .. mrow0+3 of my factor segment
    const int mkind = (lane >> 2) & 3;  // S_K, Z_K, S_V, Z_V
    const bool mlive = mseg < kSegs;    // (a one-segment loader warp: lanes 16-31 have no factors)
    const int mslot = mlive ? mseg : 0;
    const int mblk = seg_of<kWide>(warp, mslot);  // my factor segment's block within a chunk
    const uint32_t mnone = mkind == 2 ? 0xBC00BC00u : 0u;  // the factors of an absent segment (S_V = -1)
    // the blocks holding the ends of [qlo, qhi), for the lanes holding S_V
    // (-2: none; without a window only the block of position L-1)
    const int blk_hi = mkind == 2 ? (qhi - 1) / kBlockSize : -2;
    const int blk_lo = mkind == 2 && (qlo & (kBlockSize - 1)) != 0 ? qlo / kBlockSize : -2;
    const uint32_t my_meta = smem_u32(&sm.meta[0][mkind][16 * mblk + mrow0]);
#pragma unroll
    for (int i = 0; i < kNV; ++i)  // the deferred chunk, if it is one of the first three
      if (i == c_defer) issue(bfirst[i], i);
    Ring3 r{0, 0u};  // chunk c: staging slot, key-code, value and factor buffers r.i
    // staging slots whose bulk copy is still in flight after a failed wait:
    // bit i, and its phase parity in bit 4 + i
    uint32_t pend = 0u;
#pragma unroll 1
    for (int c = 0; c < nchunks; ++c) {
      if (!mbar_wait<kWaitTag>(&sm.full[warp][r.i], r.ph, abort)) {
        bad = true;
        pend |= (1u << r.i) | (r.ph << (4 + r.i));
      }
      const uint32_t sb = my_stg + r.i * (kSegs * kSeg);
      KeyRaw<KB> kr[kSegs];
      uint4 vr[kSegs][VB / 2];  // VB = 2: one 16-byte piece per segment; VB = 4: two
#pragma unroll
      for (int sg = 0; sg < kSegs; ++sg) {
        kr[sg].load(sb + sg * kSeg + F::kOffK, lane);
#pragma unroll
        for (int i = 0; i < VB / 2; ++i) vr[sg][i] = lds128(sb + sg * kSeg + F::kOffV + 512 * i + 16 * lane);
      }
      const uint2 mr2 = lds64(sb + mslot * kSeg + F::kOffSK + 8 * (lane & 15));
      const bool seg_ok = sm.tbl[kChunkBlocks * c + mblk] >= 0;  // my factor segment is present
      // the slot is read: refill it with chunk c+3 (the reads above are
      // ordered before the copy's writes by the proxy fence).  (After a
      // failed wait no copy is issued any more: see the drain below.)  An
      // L2 prefetch further ahead bought nothing here: three chunks in
      // flight cover the latency, and the extra instructions sit on this
      // warp's path, which sets the chunk rate.
      async_proxy_fence();
      __syncwarp();
      if (!bad && c + kNV < nchunks)
        issue(lane < kSegs ? sm.tbl[kChunkBlocks * (c + kNV) + seg_of<kWide>(warp, lane)] : -1, r.i);

      if (c >= kNV) {  // buffers r.i are free once PV(c-3) (issued after QK(c-2)) is done
        if (!mbar_wait<kWaitTag>(&sm.pv_done[r.i], r.ph ^ 1u, abort)) bad = true;
        tc_fence_after();
      }
#pragma unroll
      for (int sg = 0; sg < kSegs; ++sg) {  // key codes of segment sg -> its 16 TMEM lanes
        uint32_t w[16];
        kr[sg].spread(w);
        tmem_st16x256(seg_lanes(sg) + kColA + 32 * r.i, w);
      }
#pragma unroll
      for (int sg = 0; sg < kSegs; ++sg) {  // value codes, one byte each
        const uint32_t va = seg_vt(sg) + r.i * (kChunkTokens * kHeadDim);
        if (VB == 2) {  // crumb k of each byte -> position 16i + 4k + b, times 4^k
          const uint32_t vw[4] = {vr[sg][0].x, vr[sg][0].y, vr[sg][0].z, vr[sg][0].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t x = vw[i];
            sts128(va + 128 * i, x & 0x03030303u, x & 0x0C0C0C0Cu, x & 0x30303030u, x & 0xC0C0C0C0u);
          }
        } else {  // nibble h of byte b of word w -> position 16h + 4w + b, times 16^h
#pragma unroll
          for (int i = 0; i < VB / 2; ++i) {  // rows lane/4 and 8 + lane/4
            const uint4 x = vr[sg][i];
            sts128(va + 1024 * i, x.x & 0x0F0F0F0Fu, x.y & 0x0F0F0F0Fu, x.z & 0x0F0F0F0Fu, x.w & 0x0F0F0F0Fu);
            sts128(va + 1024 * i + 128, x.x & 0xF0F0F0F0u, x.y & 0xF0F0F0F0u, x.z & 0xF0F0F0F0u, x.w & 0xF0F0F0F0u);
          }
        }
      }
      {  // factors of my four rows, as stored; S_V = -1 marks an absent token
         // (a segment outside the split or the pool, a row past the end of
         // the sequence: only in the block holding position L-1)
        uint32_t m0 = seg_ok ? mr2.x : mnone, m1 = seg_ok ? mr2.y : mnone;
        const int blk = blk0 + kChunkBlocks * c + mblk;
        if (blk == blk_hi || blk == blk_lo) {
          // my rows k with position p0 + k outside [qlo, qhi): k < nlo or k >= nhi
          const int p0 = blk * kBlockSize + mrow0;
          const int nlo = qlo - p0, nhi = qhi - p0;
          if (0 < nlo || 0 >= nhi) m0 = (m0 & 0xFFFF0000u) | 0xBC00u;
          if (1 < nlo || 1 >= nhi) m0 = (m0 & 0x0000FFFFu) | 0xBC000000u;
          if (2 < nlo || 2 >= nhi) m1 = (m1 & 0xFFFF0000u) | 0xBC00u;
          if (3 < nlo || 3 >= nhi) m1 = (m1 & 0x0000FFFFu) | 0xBC000000u;
        }
        if (mlive) sts64(my_meta + r.i * (4 * kChunkTokens * 2), m0, m1);
      }
      tmem_wait_st();
      tc_fence_before();
      async_proxy_fence();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.kv_ready[r.i]);
      r.next();
    }
    // Exit ordering after a wait gave up: this warp issued no copy since, and
    // every copy it issued before lands in its own staging ring, so it waits
    // (bounded, ignoring the abort flag) for the ones still in flight; the
    // CTA barrier below then orders this before the CTA releases its shared
    // memory.
#pragma unroll
    for (int i = 0; i < kNV; ++i)
      if ((pend >> i) & 1u) mbar_wait_final(&sm.full[warp][i], (pend >> (4 + i)) & 1u);
  } else if (warp == kMmaWarp) {
    // one lane issues, in this order: QK(0), QK(1), PV(0), QK(2), PV(1), ...
    const uint32_t qb0 = smem_u32(sm.qb);
    const uint32_t vt0 = smem_u32(sm.vt[0]);
    const uint32_t pm0 = smem_u32(sm.pm[0]);
    Ring3 rq{0, 0u};  // QK(c)
    Ring3 rp{0, 0u};  // PV(c - 1)
#pragma unroll 1
    for (int c = 0; c <= nchunks; ++c) {
      if (c < nchunks) {  // QK(c): its codes are in, and S buffer c % 2 was read (chunk c-2)
        const int P = c & 1;
        if (!mbar_wait<kWaitTag>(&sm.kv_ready[rq.i], rq.ph, abort)) bad = true;
        if (c >= kNS && !mbar_wait<kWaitTag>(&sm.s_free[P], static_cast<uint32_t>(((c - kNS) >> 1) & 1), abort)) bad = true;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t acol = tbase + kColA + 32 * rq.i, scol = tbase + kColS + 32 * P;
#pragma unroll
          for (int s = 0; s < 4; ++s) mma_qk(scol, acol + 8 * s, sdesc(qb0 + 1024 * s, 512, 128), s > 0);
          mma_commit(&sm.qk_done[P]);
        }
        __syncwarp();
        rq.next();
      }
      if (c >= 1) {  // PV(c-1) once its P' is written
        if (!mbar_wait<kWaitTag>(&sm.p_ready[rp.i], rp.ph, abort)) bad = true;
        tc_fence_after();
        if (lane == 0) {
          const int fr = sm.fresh[rp.i];
          const bool fresh = (fr & 1) != 0;
          const uint32_t ocol = tbase + kColO + 16 * (fr & 2);
          const uint32_t va = vt0 + rp.i * (kChunkTokens * kHeadDim), pa = pm0 + rp.i * (kChunkTokens * 32);
#pragma unroll
          for (int s = 0; s < 4; ++s)
            mma_pv(ocol, sdesc(va + 4096 * s, 1024, 128), sdesc(pa + 1024 * s, 256, 128), !fresh || s > 0);
          mma_commit(&sm.pv_done[rp.i]);
        }
        __syncwarp();
        rp.next();
      }
    }
    if (lane == 0) mma_commit(&sm.fin);
    __syncwarp();
    if (!mbar_wait_final(&sm.fin, 0u)) bad = true;
  } else {
    // softmax warps: thread st <-> token stok = st % 128 of S and value
    // position stok of O, heads hb .. hb + kHeads - 1 (hb = 0 but in the
    // wide layout, where the second 128 threads take heads 4 .. 7)
    const int sw = warp - kLoadWarps;
    const int st = tid - 32 * kLoadWarps;
    const int stok = st & 127;
    const int hf = kWide ? st >> 7 : 0;
    const int hb = hf * kHeads;
    const int wg = sw & ~3;  // the four warps of my heads: wg .. wg + 3
    const uint32_t my_lanes = tbase + (static_cast<uint32_t>((sw & 3) * 32) << 16);
    const uint32_t my_acc = my_lanes + kColAcc + 8 * hf;  // o~ so far of my heads (fp32, column per head)
    const uint32_t my_pm = smem_u32(sm.pm[0]) + (stok >> 3) * 256 + (stok & 7) * 16;
    // the three S digits of my heads, by fixed register indices (a register
    // array indexed by the run-time hb would go to local memory)
    auto pick_digits = [&](const uint32_t (&a)[16], const uint32_t (&b)[8], uint32_t (&e0)[kHeads],
                           uint32_t (&e1)[kHeads], uint32_t (&e2)[kHeads]) {
#pragma unroll
      for (int g = 0; g < kHeads; ++g) {
        const int hi = kWide ? kHeads + g : g;
        e0[g] = hf ? a[hi] : a[g];
        e1[g] = hf ? a[8 + hi] : a[8 + g];
        e2[g] = hf ? b[hi] : b[g];
      }
    };
    // (o~ so far, in units of the output scale below, lives in tensor memory
    // at my_acc: it is touched only when the running max moves and at the
    // end, and registers are the scarce resource of this loop)
    float qs[kHeads], mr[kHeads], lr[kHeads], zr[kHeads];
#pragma unroll
    for (int g = 0; g < kHeads; ++g) {
      qs[g] = sm.hq[hb + g].x;
      mr[g] = kNoMax;
      lr[g] = zr[g] = 0.0f;
    }
    int fresh_c = 0;  // the chunk whose PV started the integer accumulator
    int ob = 0;       // the O buffer the PVs of chunks fresh_c .. run into
    // A max move switches the PVs to the other O buffer and leaves the old
    // one (chunks up to c-1, in units of the old max) pending with the factor
    // palpha: it is folded at the next chunk, when QK(c+1) is done and so are
    // the PVs issued before it; nothing waits for a PV at the move.
    bool pend = false;  // (its per-head factor is in sm.palpha[sw], one copy per warp)

    {  // o~ so far: 0
      const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      tmem_st8(my_acc, z);
      tmem_wait_st();
    }
    // fold O buffer k (my lane = value position stok; my heads' columns
    // 4 hb .. 4 hb + 4 kHeads - 1) into o~ so far, with the pending factor of
    // each head (scaled) or 1
    auto fold_o = [&](int k, bool scaled) {
      uint32_t r[16], r2[16], oa[8];
      tmem_ld16(my_lanes + kColO + 32 * k + 4 * hb, r);
      if (kHeads > 4) tmem_ld16(my_lanes + kColO + 32 * k + 16, r2);
      tmem_ld8(my_acc, oa);
      tmem_wait_ld();
#pragma unroll
      for (int g = 0; g < kHeads; ++g) {
        const uint32_t* q = g < 4 ? r + 4 * g : r2 + 4 * g - 16;
        const float v = fmaf(static_cast<float>(static_cast<int>(q[3])), 16777216.0f,
                             fmaf(static_cast<float>(static_cast<int>(q[2])), 65536.0f,
                                  fmaf(static_cast<float>(static_cast<int>(q[1])), 256.0f,
                                       static_cast<float>(static_cast<int>(q[0])))));
        const float o = __uint_as_float(oa[g]);
        oa[g] = __float_as_uint(scaled ? fmaf(v, sm.palpha[sw][hb + g], o) : o + v);
      }
      tmem_st8(my_acc, oa);
      tmem_wait_st();
    };

    Ring3 r{0, 0u};  // chunk c: buffers r.i
#pragma unroll 1
    for (int c = 0; c < nchunks; ++c) {
      const int P = c & 1;
      if (!mbar_wait<kWaitTag>(&sm.qk_done[P], static_cast<uint32_t>((c >> 1) & 1), abort)) bad = true;
      tc_fence_after();
      if (pend) {  // the PVs into the pending buffer (up to chunk c-2) are done
        fold_o(ob ^ 1, true);
        pend = false;
      }
      uint32_t sr[16], sr2[8];
      tmem_ld16(my_lanes + kColS + 32 * P, sr);
      tmem_ld8(my_lanes + kColS + 32 * P + 16, sr2);
      if (!mbar_wait<kWaitTag>(&sm.kv_ready[r.i], r.ph, abort)) bad = true;
      const uint32_t hsv = sm.meta[r.i][2][stok];
      const bool valid = (hsv & 0x8000u) == 0;  // a token (not marked absent by the loaders)
      // S_K c1, Z_K, S_V 2^29, Z_V (0 for an absent token); a flat value row
      // (S_V = 0: every code 0) takes 2^29 instead, so that its P' still
      // stands for p (its codes add nothing to O, its p Z_V goes to zeta)
      const float sv = h2f(hsv);
      const float4 mt = make_float4(h2f(sm.meta[r.i][0][stok]) * c1, h2f(sm.meta[r.i][1][stok]),
                                    (sv == 0.0f ? 1.0f : sv) * kFix, valid ? h2f(sm.meta[r.i][3][stok]) : 0.0f);
      float pinv;  // 1 / (S_V 2^29)
      asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(pinv) : "f"(mt.z));
      // E with S_V < 2^E, from the fp16 exponent of S_V (-14 for subnormals and 0)
      const float e = static_cast<float>(static_cast<int>((hsv >> 10) & 31u) - 14);
      tmem_wait_ld();
      // S column g holds digit 0 of head g, column 8 + g digit 1, 16 + g digit 2
      uint32_t d0[kHeads], d1[kHeads], d2[kHeads];
      pick_digits(sr, sr2, d0, d1, d2);
      float dg[kHeads];
      float dmax = -CUDART_INF_F;
      if (kHeads == 1) {
        const int e12 = static_cast<int>(d1[0]) * 254 + static_cast<int>(d2[0]);
        const float xg = fmaf(__int2float_rn(e12), 1.0f / 64516.0f, small_i2f(d0[0]));
        dg[0] = fmaf(mt.x, xg, fmaf(mt.y, qs[0], -mr[0]));
        dmax = dg[0];
      } else {
        const u64x mx2 = pk2(mt.x, mt.x), my2 = pk2(mt.y, mt.y);
        const u64x k2 = pk2(1.0f / 64516.0f, 1.0f / 64516.0f), m2 = pk2(-12582912.0f, -12582912.0f);
#pragma unroll
        for (int g = 0; g < (kHeads > 1 ? kHeads : 2); g += 2) {
          const float xe0 = __int2float_rn(static_cast<int>(d1[g]) * 254 + static_cast<int>(d2[g]));
          const float xe1 = __int2float_rn(static_cast<int>(d1[g + 1]) * 254 + static_cast<int>(d2[g + 1]));
          const u64x s0 = add2(pk2(__uint_as_float(d0[g] + 0x4B400000u), __uint_as_float(d0[g + 1] + 0x4B400000u)), m2);
          const u64x xg = fma2(pk2(xe0, xe1), k2, s0);
          const u64x d = fma2(mx2, xg, fma2(my2, pk2(qs[g], qs[g + 1]), pk2(-mr[g], -mr[g + 1])));
          upk2(d, dg[g], dg[g + 1]);
          dmax = max3f(dmax, dg[g], dg[g + 1]);
        }
      }
      const bool flag = valid && (dmax + e > kTrigger);
      // (one vote over all softmax threads, the wide layout's two halves
      // included: a move switches the O buffer that every head's PV runs into)
      const bool any = soft_vote_any<kSoftThreads>(flag);
      if (any) {
        // rare: move the running max of each head to the chunk's max of
        // s + E plus the headroom; the scores are formed again from S (still
        // in tensor memory: it is released below), exactly, without the
        // running max
        tmem_ld16(my_lanes + kColS + 32 * P, sr);
        tmem_ld8(my_lanes + kColS + 32 * P + 16, sr2);
        tmem_wait_ld();
        pick_digits(sr, sr2, d0, d1, d2);
        float sg[kHeads];
#pragma unroll
        for (int g = 0; g < kHeads; ++g) {
          const int gh = hb + g;
          const int e12 = static_cast<int>(d1[g]) * 254 + static_cast<int>(d2[g]);
          const float xg = fmaf(__int2float_rn(e12), 1.0f / 64516.0f, small_i2f(d0[g]));
          sg[g] = fmaf(mt.x, xg, mt.y * qs[g]);
          float u = valid ? sg[g] + e : -CUDART_INF_F;
#pragma unroll
          for (int o = 16; o; o >>= 1) u = fmaxf(u, __shfl_xor_sync(0xffffffffu, u, o));
          if (lane == 0) sm.red[sw][gh][0] = u;
        }
        soft_sync<kSoftThreads>();
        float alpha[kHeads];
#pragma unroll
        for (int g = 0; g < kHeads; ++g) {
          const int gh = hb + g;
          const float M = fmaxf(fmaxf(sm.red[wg][gh][0], sm.red[wg + 1][gh][0]),
                                fmaxf(sm.red[wg + 2][gh][0], sm.red[wg + 3][gh][0]));
          const float mn = fmaxf(mr[g], M + kHeadroom);
          alpha[g] = ex2(mr[g] - mn);
          lr[g] *= alpha[g];
          zr[g] *= alpha[g];
          dg[g] = sg[g] - mn;
          mr[g] = mn;
        }
        {  // o~ so far in units of the new max
          uint32_t oa[8];
          tmem_ld8(my_acc, oa);
          tmem_wait_ld();
#pragma unroll
          for (int g = 0; g < kHeads; ++g) oa[g] = __float_as_uint(__uint_as_float(oa[g]) * alpha[g]);
          tmem_st8(my_acc, oa);
          tmem_wait_st();
        }
        if (c > fresh_c) {  // PVs of chunks fresh_c .. c-1 ran into buffer ob: pending
          if (lane == 0) {
#pragma unroll
            for (int g = 0; g < kHeads; ++g) sm.palpha[sw][hb + g] = alpha[g];
          }
          __syncwarp();
          pend = true;
          ob ^= 1;
        }
        fresh_c = c;
        // the reductions above read sm.red: none writes it again before the next vote
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.s_free[P]);
      // P' of chunk c -> pm[r.i] (free: PV(c-3) was issued before QK(c), which is done)
      uint32_t pw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      if (kHeads == 1) {
        const float p = valid ? ex2(dg[0]) : 0.0f;
        pw[0] = __float2uint_rn(p * mt.z);
        const float pt = __uint2float_rn(pw[0]) * pinv;
        lr[0] += pt;
        zr[0] = fmaf(pt, mt.w, zr[0]);
      } else {
        const u64x z2 = pk2(mt.z, mt.z), i2 = pk2(pinv, pinv), w2 = pk2(mt.w, mt.w);
#pragma unroll
        for (int g = 0; g < (kHeads > 1 ? kHeads : 2); g += 2) {
          float x0, x1, l0, l1, q0, q1;
          upk2(mul2(pk2(valid ? ex2(dg[g]) : 0.0f, valid ? ex2(dg[g + 1]) : 0.0f), z2), x0, x1);
          pw[g] = __float2uint_rn(x0);  // rne(P' 2^29) < 2^32
          pw[g + 1] = __float2uint_rn(x1);
          // l and zeta take the p that the rounded P' stands for
          const u64x pt = mul2(pk2(__uint2float_rn(pw[g]), __uint2float_rn(pw[g + 1])), i2);
          upk2(add2(pk2(lr[g], lr[g + 1]), pt), l0, l1);
          upk2(fma2(pt, w2, pk2(zr[g], zr[g + 1])), q0, q1);
          lr[g] = l0;
          lr[g + 1] = l1;
          zr[g] = q0;
          zr[g + 1] = q1;
        }
      }
      // (P' column n = 4 g + j: my heads' bytes are 16-byte piece hf, and the
      // next one when I take all eight)
      const uint32_t pa = my_pm + r.i * (kChunkTokens * 32) + 128 * hf;
      sts128(pa, pw[0], pw[1], pw[2], pw[3]);
      if (kHeads > 4) sts128(pa + 128, pw[4], pw[5], pw[6], pw[7]);
      if (st == 0) sm.fresh[r.i] = (fresh_c == c ? 1 : 0) | (ob << 1);
      async_proxy_fence();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_ready[r.i]);
      r.next();
    }
    if (nchunks > 0) {  // the last PV, then the accumulator
      const int pi = r.i == 0 ? 2 : r.i - 1;
      const uint32_t pph = r.i == 0 ? r.ph ^ 1u : r.ph;
      if (!mbar_wait<kWaitTag>(&sm.pv_done[pi], pph, abort)) bad = true;
      tc_fence_after();
      if (pend) fold_o(ob ^ 1, true);
      fold_o(ob, false);
    }
    // l and zeta over the 128 tokens' threads of my heads; o~ in dim order
#pragma unroll
    for (int g = 0; g < kHeads; ++g) {
      float l = lr[g], z = zr[g];
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        l += __shfl_xor_sync(0xffffffffu, l, o);
        z += __shfl_xor_sync(0xffffffffu, z, o);
      }
      if (lane == 0) {
        sm.red[sw][hb + g][0] = l;
        sm.red[sw][hb + g][1] = z;
      }
    }
    soft_sync<kSoftThreads>();
    const int d = value_dim_of_pos<VB>(stok);
    // output scale of my value position: the fixed point and the factor of the spread
    const float oscale = kFixInv * __uint_as_float((127u - value_scale_log2<VB>(stok)) << 23);
    // With several splits, every thread writes its dim of the split's record
    // (o~[128], m, l per head) straight to the workspace; with one, the
    // normalised o~ goes to shared memory for the output rotation.
    float* rec = a.partials + ((static_cast<int64_t>(b) * a.num_q_heads + h * G) * a.nrec + split) * kPartialFloats;
    uint32_t oacc[8];
    tmem_ld8(my_acc, oacc);
    tmem_wait_ld();
#pragma unroll
    for (int g = 0; g < kHeads; ++g) {
      const int gh = hb + g;
      const float z = (sm.red[wg][gh][1] + sm.red[wg + 1][gh][1]) + (sm.red[wg + 2][gh][1] + sm.red[wg + 3][gh][1]);
      const float lsum = (sm.red[wg][gh][0] + sm.red[wg + 1][gh][0]) + (sm.red[wg + 2][gh][0] + sm.red[wg + 3][gh][0]);
      const float o = fmaf(__uint_as_float(oacc[g]), oscale, z);
      if (a.nrec > 1) {
        float* rg = rec + static_cast<int64_t>(gh) * a.nrec * kPartialFloats;
        rg[d] = o;
        if (stok == gh) *reinterpret_cast<float2*>(rg + kHeadDim) = make_float2(mr[g], lsum);
      } else {
        sm.obuf[gh][d] = lsum > 0.0f ? o / lsum : 0.0f;
      }
    }
  }
  if (bad) record_status(a.status, KVQ_ERR_DEVICE_TIMEOUT);
  // (any loader thread may have met a bad entry of the block table)
  if (__any_sync(0xffffffffu, bad_blk) && lane == 0) record_status(a.status, KVQ_ERR_OUT_OF_RANGE);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp)  // every MMA and tensor-memory load is complete
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "n"(kTmemCols));
  pdl_trigger();  // this CTA holds no tensor memory any more

  // ---- 2. output rotation (one record), or ticket and merge ---------------------
  if (a.nrec == 1) {
    // rotate back once (warp w owns heads w, w + 9, ...) and store; the CTA
    // barrier above published obuf
    for (int g = warp; g < G; g += kThreads / 32) {
      float x[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) x[k] = sm.obuf[g][lane + 32 * k];
      fwht_warp(x, lane, 1.0f);
      const int64_t o0 = (static_cast<int64_t>(b) * a.num_q_heads + h * G + g) * kHeadDim;
#pragma unroll
      for (int k = 0; k < 4; ++k) store_from_f32(a.out, a.out_dtype, o0 + lane + 32 * k, x[k]);
    }
    return;
  }
  if (take_ticket(a, b, h, &sm.is_last)) merge_records<G, kThreads>(a, b, h);
}

template <int G, int KB, int VB, bool kWide, bool kWin>
cudaError_t launch_gw(const DecodeArgs& a, cudaStream_t stream) {
  constexpr int kBytes = kSmemBytesOf<Fmt<KB, VB>::kSegBytes, kWide>;
  const cudaError_t e = ensure_smem_limit<decode_kernel<G, KB, VB, kWide, kWin>>(kBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid(a.nsplit + (kWin ? 1 : 0), a.num_kv_heads, a.batch);  // (+ the window's CTA)
  return launch_pdl(decode_kernel<G, KB, VB, kWide, kWin>, grid, dim3(Roles<kWide>::kThreads), kBytes, stream, a);
}
template <int G, int KB, int VB, bool kWide>
cudaError_t launch_g(const DecodeArgs& a, cudaStream_t stream) {
  return a.win != nullptr ? launch_gw<G, KB, VB, kWide, true>(a, stream) : launch_gw<G, KB, VB, kWide, false>(a, stream);
}

template <int KB, int VB>
cudaError_t launch_p(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.num_q_heads / a.num_kv_heads) {
    case 1: return launch_g<1, KB, VB, false>(a, stream);
    case 2: return launch_g<2, KB, VB, false>(a, stream);
    case 4: return launch_g<4, KB, VB, false>(a, stream);
    case 8:
      // a grid that the SMs hold at once, one CTA each: the wide role layout
      // (its chunks pass each role in about half the time)
      if (static_cast<int64_t>(a.nsplit + (a.win != nullptr ? 1 : 0)) * a.num_kv_heads * a.batch <= device_sm_count())
        return launch_g<8, KB, VB, true>(a, stream);
      return launch_g<8, KB, VB, false>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

// Failure-detection self-test: one warp waits, through the decode kernel's
// bounded wait (the same slow loop), on a barrier that nothing arrives at.
// Nothing else is issued (no bulk copy, no MMA, no tensor memory), so
// nothing is in flight when the wait gives up after limit_ns; the kernel
// records KVQ_ERR_DEVICE_TIMEOUT and the time the wait took.
__global__ void __launch_bounds__(32) wait_timeout_probe_kernel(int* status, uint64_t limit_ns, uint64_t* elapsed_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  const int lane = threadIdx.x;
  if (lane == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  const uint64_t t0 = global_ns();
  const bool ok = mbar_wait_slow<0>(&bar, 0u, &abort_flag, limit_ns);
  const uint64_t t1 = global_ns();
  if (lane == 0) {
    if (!ok) record_status(status, KVQ_ERR_DEVICE_TIMEOUT);
    if (elapsed_ns != nullptr) *elapsed_ns = t1 - t0;
  }
}

}  // namespace

cudaError_t launch_wait_probe(int* status, uint64_t limit_ns, uint64_t* elapsed_ns, cudaStream_t stream) {
  wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(status, limit_ns, elapsed_ns);
  return cudaGetLastError();
}
uint64_t wait_limit_ns() { return kWaitLimitNs; }

int decode_ctas_per_sm() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
  if (cached[dev] > 0) return cached[dev];
  int n = 0;
  constexpr int kBytes = kSmemBytesOf<Fmt<4, 2>::kSegBytes>;
  if (ensure_smem_limit<decode_kernel<8, 4, 2, false, false>>(kBytes) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_kernel<8, 4, 2, false, false>, Roles<false>::kThreads, kBytes) !=
          cudaSuccess ||
      n < 1)
    n = 1;
  cached[dev] = n < 2 ? n : 2;  // two CTAs' tensor memory (2 x 256 columns) fills an SM
  return cached[dev];
}

int decode_max_splits() { return kMaxSplits; }
int decode_max_split_blocks() { return kTblBlocks; }
int decode_chunk_blocks() { return kChunkBlocks; }

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  if (a.k_bits == 4 && a.v_bits == 2) return launch_p<4, 2>(a, stream);
  if (a.k_bits == 4 && a.v_bits == 4) return launch_p<4, 4>(a, stream);
  if (a.k_bits == 2 && a.v_bits == 2) return launch_p<2, 2>(a, stream);
  if (a.k_bits == 8 && a.v_bits == 4) return launch_p<8, 4>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace kvq
