// kvq_quantize.cu -- cache write path: rotate, normalise, quantise, pack.
//
// Bulk appends (prefill): the rotation of a tile of 128 head vectors is one
// matrix product on the fifth-generation tensor cores, Y = X H with H the
// 128 x 128 Sylvester Hadamard matrix (entries +-1, exact in bf16 and fp16,
// accumulated in fp32), written as two N = 64 halves over the Sylvester
// blocks, Y0 = X0 H64 + X1 H64 and Y1 = X0 H64 - X1 H64 (16 MMAs of K = 16).
// Each warp copies its 32 rows of a tile two tiles ahead with 16-byte
// cp.async straight into a 3-slot ring of A operands in the 128-byte
// swizzled K-major layout (conflict free, nothing moves twice); one thread
// issues tile k's MMAs into accumulator k % 2 of tensor memory, so tile k's
// rotation runs while the CTA reads tile k-1's accumulator.  Thread t owns
// vector t (tensor-memory lane t): one read of its 128 columns gives the
// moments, range, (S, Z) and codes, packed with fp32x2 arithmetic and written
// as 16-byte stores into the paged segment plus two fp16 stores.  Two CTAs
// per SM overlap each other's barriers and waits.
//
// Small appends (decode steps): one warp per vector (quantize_vector_warp in
// kvq_internal.cuh), butterflies in registers and shuffles.
//
// Method ("Трюк Huawei с KV-кэшем", section "Заявка, которая ломает
// привычный компромисс"; "KVarN vs TurboQuant", pipeline list): Hadamard
// rotation, variance normalisation, asymmetric round-to-nearest; the exact
// definition and pool layout are stated in include/kvq.h.
#include <math_constants.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

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

// ---- tensor-core pieces -------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
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
// Wait for a barrier phase, at most about a second (false: it never came).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1; it < (1u << 26); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0 && global_ns() - t0 > 1000000000ull) return false;
  }
  return false;
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void async_proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// sm_100 shared-memory matrix descriptor: start address, leading (K) and
// stride (M/N) byte offsets in 16-byte units, version 1, no swizzle.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// The 128 fp32 columns at addr of this thread's tensor-memory lane, one
// load and one wait.
__device__ __forceinline__ void tmem_ld128(uint32_t addr, float (&v)[128]) {
  uint32_t r[128];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 {"
      "%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,"
      "%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,"
      "%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,"
      "%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,"
      "%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127"
      "}, [%128];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]),
        "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]),
        "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]),
        "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]),
        "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]),
        "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]),
        "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]),
        "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]),
        "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(addr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 128; ++i) v[i] = __uint_as_float(r[i]);
}

// ---- bulk path ------------------------------------------------------------------
// A CTA of 128 threads walks tiles of 128 head vectors (one tensor, K or V);
// thread t owns vector t of a tile and tensor-memory lane t.  Warp w stages
// its 32 rows (vectors 32w .. 32w+31 of the tile), two tiles ahead, with
// coalesced 16-byte cp.async copies straight into the A operand of the
// rotation: a 128-byte-swizzled K-major tile in shared memory (three such
// tiles rotate: one being staged, one read by the tensor cores, one whose
// staging is in flight).  The rotation y = x H (H the 128 x 128 Sylvester
// Hadamard matrix, unnormalised, exact in 16-bit floats) runs on the tensor
// cores into one of two 128-column fp32 accumulators, so that the MMAs of
// tile i run while every thread computes the moments, range and codes of
// its vector of tile i-1 from the other accumulator.  H is applied through
// its Sylvester halves, H = [[H64, H64], [H64, -H64]]: with x = (x0, x1),
// y0 = x0 H64 + x1 H64 and y1 = x0 H64 - x1 H64, sixteen MMAs of N = 64
// (B = H64 and -H64, 16 KB of shared memory instead of 32).
constexpr int kTileVecs = 128;
constexpr int kBulkThreads = 128;
constexpr int kWarpRows = 32;   // rows a warp stages per tile
constexpr int kNA = 3;          // A tiles in shared memory
constexpr uint32_t kBulkTmemCols = 256;  // two accumulators of 128 fp32 columns
constexpr int kHalfBytes = kTileVecs * 128;  // one K-half (64 elements) of a tile: 128 rows of 128 B

// Shared memory, every operand tile in the 128-byte-swizzled K-major layout
// (8-row x 128-byte atoms, 16-byte chunk c of row r stored at chunk c ^ (r %
// 8) of that row; atoms 1024 B apart along M):
//   a[i][h]: elements 64h .. 64h+63 of the 128 rows of a tile
//   hb[0] = H64, hb[1] = -H64 (row n = output column n, 64 elements)
struct __align__(1024) BulkSmem {
  uint8_t a[kNA][2][kHalfBytes];   // 96 KB
  uint8_t hb[2][64 * 128];         // 16 KB
  uint64_t mma_done[2];            // the MMAs into accumulator j are complete
  uint32_t tmem_base;
  int abort;                       // a wait ran out: every other wait gives up at once
};
constexpr int kBulkSmemBytes = static_cast<int>(sizeof(BulkSmem));
static_assert(kBulkSmemBytes <= 113 * 1024, "two CTAs per SM");
// The tensor-memory rule of kvq_internal.cuh: three CTAs that allocate 256
// columns each (this kernel's and the decode kernel's) never fit on one SM's
// 228 KB.
static_assert(3 * (kBulkSmemBytes + 1024) > 228 * 1024, "at most two tensor-memory CTAs per SM");

// Byte offset of 16-byte chunk c of row r in a 128-byte-swizzled K-major
// operand whose atoms start at 1024-byte boundaries.
__device__ __forceinline__ uint32_t sw128(int r, int c) {
  return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}
// sm_100 shared-memory matrix descriptor of a 128-byte-swizzled K-major
// operand: start address, stride offset 1024 B between 8-row atoms, version
// 1, layout type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t addr) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1u) << 16) |
         (static_cast<uint64_t>(1024u >> 4) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor, kind::f16: D f32, A and B f16 or bf16, both
// K-major, N = 64, M = 128.
template <bool kBF16>
__host__ __device__ constexpr uint32_t idesc_h64() {
  return (1u << 4) | ((kBF16 ? 1u : 0u) << 7) | ((kBF16 ? 1u : 0u) << 10) | ((64u >> 3) << 17) | ((128u >> 4) << 24);
}
__device__ __forceinline__ void mma_f16_ss(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, bool acc) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %3, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p; }" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(static_cast<uint32_t>(acc)), "r"(idesc)
      : "memory");
}

// Token of vector n (n < n_vec): 32-bit division whenever the indices fit.
__device__ __forceinline__ int64_t token_of(int64_t n, int64_t n_vec, int hkv) {
  return n_vec <= 0xFFFFFFFFll ? static_cast<int64_t>(static_cast<uint32_t>(n) / static_cast<uint32_t>(hkv))
                               : n / hkv;
}

// Stage rows row0 .. row0+31 (vector n = token n / Hkv, head n % Hkv) into
// rows 32w .. 32w+31 of an A tile (a0: its first K-half): in copy j lane l
// moves 16-byte chunk l % 16 of row 2j + l/16 (two whole rows per
// instruction, conflict free in the swizzled layout); the row addresses are
// computed once per lane (its own row) and handed round by shuffles.  Rows
// past the tensor are zero filled.
__device__ __forceinline__ void stage_rows(uint32_t a0, const uint8_t* src, int64_t n_vec, int hkv,
                                           int64_t stride_bytes, int64_t row0, int w, int lane) {
  const int64_t n = row0 + lane;
  const bool mine = n < n_vec;
  const int64_t tok = mine ? token_of(n, n_vec, hkv) : 0;
  const int hh = mine ? static_cast<int>(n - tok * hkv) : 0;
  const uint8_t* my_row = src + tok * stride_bytes + static_cast<int64_t>(hh) * (kHeadDim * 2);
  const int col = lane & 15;
  const uint32_t half = a0 + static_cast<uint32_t>(col >> 3) * kHalfBytes;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int row = 2 * j + (lane >> 4);
    const uint8_t* row_ptr = reinterpret_cast<const uint8_t*>(
        __shfl_sync(0xffffffffu, static_cast<unsigned long long>(reinterpret_cast<uintptr_t>(my_row)), row));
    const bool valid = row0 + row < n_vec;
    cp_async16(half + sw128(32 * w + row, col & 7), valid ? row_ptr + col * 16 : src, valid);
  }
}

// Code of pair element with the integer in the low mantissa bits: the value
// t = q + 1.5*2^23 has ulp 1, so its low bits hold rne(q) (ties to even).
constexpr float kMagic = 12582912.0f;

// Codes rne(y a + b) (clamped to [0, L] if kClamp) of the 128 elements of
// y, packed: 8 four-bit codes or 16 two-bit codes per word, element 0 in
// the low bits.
template <int kBits, bool kClamp>
__device__ __forceinline__ void codes_to_words(const float (&y)[kHeadDim], u64 a2, u64 b2,
                                               uint32_t (&words)[kHeadDim * kBits / 32]) {
  constexpr float kLevels = static_cast<float>((1 << kBits) - 1);
  const u64 m2 = pk(kMagic, kMagic);
#pragma unroll
  for (int c0 = 0; c0 < kHeadDim; c0 += 32) {
    uint32_t c[32];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      u64 t = fma2(pk(y[c0 + 2 * j], y[c0 + 2 * j + 1]), a2, b2);
      if (kClamp) {
        float ta, tb;
        upk(t, ta, tb);
        t = pk(fminf(fmaxf(ta, 0.0f), kLevels), fminf(fmaxf(tb, 0.0f), kLevels));
      }
      upk_u(add2(t, m2), c[2 * j], c[2 * j + 1]);
    }
    if (kBits == 8) {
#pragma unroll
      for (int m = 0; m < 8; ++m) {  // word c0/4 + m = elements c0 + 4m .. +3
        const uint32_t* e = c + 4 * m;
        words[c0 / 4 + m] = prmt(prmt(e[0], e[1], 0x0040u), prmt(e[2], e[3], 0x0040u), 0x5410u);
      }
    } else if (kBits == 4) {
#pragma unroll
      for (int m = 0; m < 4; ++m) {  // word c0/8 + m = elements c0 + 8m .. +7
        const uint32_t* e = c + 8 * m;
        const uint32_t b0 = e[0] + 16u * e[1], b1 = e[2] + 16u * e[3];
        const uint32_t bb2 = e[4] + 16u * e[5], b3 = e[6] + 16u * e[7];
        words[c0 / 8 + m] = prmt(prmt(b0, b1, 0x0040u), prmt(bb2, b3, 0x0040u), 0x5410u);
      }
    } else {
#pragma unroll
      for (int m = 0; m < 2; ++m) {  // word c0/16 + m = elements c0 + 16m .. +15
        const uint32_t* e = c + 16 * m;
        uint32_t by[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) by[q] = e[4 * q] + 4u * e[4 * q + 1] + 16u * e[4 * q + 2] + 64u * e[4 * q + 3];
        words[c0 / 16 + m] = prmt(prmt(by[0], by[1], 0x0040u), prmt(by[2], by[3], 0x0040u), 0x5410u);
      }
    }
  }
}

// Moments, range, (S, Z) and codes of the vector whose y = x H sits in 128
// fp32 columns of tensor memory at taddr (read once, into registers); the
// packed row, S and Z go to row `row_in_block` of the segment (seg ==
// nullptr: not stored).  Every thread of the warp runs it: the
// tensor-memory load is warp-collective.
template <int kBits, bool kIsV, class F>
__device__ __forceinline__ void quantize_lane(uint32_t taddr, float x0, uint8_t* seg, int row_in_block) {
  constexpr float kLevels = static_cast<float>((1 << kBits) - 1);
  constexpr float kInvSqrtD = 0.088388347648318440550f;  // 1/sqrt(128)
  float y[kHeadDim];  // y = x H of my vector (r = y / sqrt(128))
  tmem_ld128(taddr, y);
  // moments and range; the mean of y is x0 (every column of H but the first
  // sums to zero), the rest is summed here
  u64 acc_q[4] = {0ull, 0ull, 0ull, 0ull};
  float mn[4], mx[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    mn[i] = CUDART_INF_F;
    mx[i] = -CUDART_INF_F;
  }
#pragma unroll
  for (int j = 0; j < kHeadDim / 2; ++j) {
    const u64 p = pk(y[2 * j], y[2 * j + 1]);
    acc_q[j & 3] = fma2(p, p, acc_q[j & 3]);
    mn[j & 3] = min3(mn[j & 3], y[2 * j], y[2 * j + 1]);
    mx[j & 3] = max3(mx[j & 3], y[2 * j], y[2 * j + 1]);
  }
  const u64 q2 = add2(add2(acc_q[0], acc_q[1]), add2(acc_q[2], acc_q[3]));
  float qa, qb;
  upk(q2, qa, qb);
  const float ymin = fminf(fminf(mn[0], mn[1]), fminf(mn[2], mn[3]));
  const float ymax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
  const float mean = x0;
  const float var = fmaxf((qa + qb) * (1.0f / kHeadDim) - mean * mean, 0.0f);
  float sigma = sqrtf(var);
  if (sigma == 0.0f) sigma = 1.0f;
  // (min/max of u = (y - mean)/sigma sit at the same elements as those of y)
  const float lo = (ymin - mean) / sigma;
  const float hi = (ymax - mean) / sigma;
  const __half Sh = __float2half_rn(kInvSqrtD * (sigma * (hi - lo)) / kLevels);
  const __half Zh = __float2half_rn(kInvSqrtD * (mean + sigma * lo));
  const float Sf = __half2float(Sh);
  const float Zf = __half2float(Zh);

  // codes: q = (r - Z)/S = y (c/S) - Z/S, rounded to nearest even, clamped
  // (S == 0: a = b = 0 gives code 0 everywhere)
  constexpr int kWords = kHeadDim * kBits / 32;  // 16 (K) or 8 (V)
  uint32_t words[kWords];
  {
    const bool flat = Sf == 0.0f;
    const float a = flat ? 0.0f : kInvSqrtD / Sf;
    const float b = flat ? 0.0f : -Zf / Sf;
    const u64 a2 = pk(a, a), b2 = pk(b, b);
    // q is monotone in y, so clamping is needed only if the code of an
    // extreme leaves [0, L]: rne(q) < 0 iff q < -1/2, rne(q) > L iff
    // q >= L + 1/2 (the same fused multiply-add as below); clamping to the
    // integers 0 and L commutes with the rounding
    const bool clamp = (fmaf(ymin, a, b) < -0.5f) || (fmaf(ymax, a, b) >= kLevels + 0.5f);
    // (two copies of the loop, so that the common unclamped one carries no
    // clamping work)
    if (clamp)
      codes_to_words<kBits, true>(y, a2, b2, words);
    else
      codes_to_words<kBits, false>(y, a2, b2, words);
  }
  if (seg == nullptr) return;
  uint4* dst = reinterpret_cast<uint4*>(
      seg + (kIsV ? F::kOffV + row_in_block * F::kVRowBytes : F::kOffK + row_in_block * F::kKRowBytes));
#pragma unroll
  for (int m = 0; m < kBits; ++m)  // (a row is 16 kBits bytes)
    dst[m] = make_uint4(words[4 * m], words[4 * m + 1], words[4 * m + 2], words[4 * m + 3]);
  reinterpret_cast<__half*>(seg + (kIsV ? F::kOffSV : F::kOffSK))[row_in_block] = Sh;
  reinterpret_cast<__half*>(seg + (kIsV ? F::kOffZV : F::kOffZK))[row_in_block] = Zh;
}

// Wait for a barrier phase, at most about a second, giving up at once once
// another thread of the CTA has given up (false: it never came).
__device__ __forceinline__ bool mbar_wait_ab(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (global_ns() - t0 > 1000000000ull) {
        *abort = 1;
        return false;
      }
    }
  }
}

template <bool kBF16, int KB, int VB>
__global__ void __launch_bounds__(kBulkThreads, 2)
    quantize_kernel(uint8_t* __restrict__ pool, int32_t num_blocks, int32_t hkv,
                    const uint8_t* __restrict__ k, const uint8_t* __restrict__ v,
                    int32_t n_tokens, int64_t stride_bytes, const int32_t* __restrict__ slots, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  BulkSmem& sm = *reinterpret_cast<BulkSmem*>(smem_raw);
  volatile int* abort = &sm.abort;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;

  // tensor memory, the barriers and H need no global memory: before the wait
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                 "n"(kBulkTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    mbar_init(&sm.mma_done[0], 1);
    mbar_init(&sm.mma_done[1], 1);
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  {  // B: H64 (table 0) and -H64 (table 1); row n: entries (-1)^popcount(n & k), k < 64, as 16-bit +-1
    const uint32_t one = kBF16 ? 0x3F80u : 0x3C00u;
    const int tb = tid >> 6, n = tid & 63;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int k0 = 8 * cc + 2 * e;
        const uint32_t h0 = one | (((__popc(n & k0) + tb) & 1u) << 15);
        const uint32_t h1 = one | (((__popc(n & (k0 + 1)) + tb) & 1u) << 15);
        w[e] = h0 | (h1 << 16);
      }
      *reinterpret_cast<uint4*>(sm.hb[tb] + sw128(n, cc)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  async_proxy_fence();  // (H is read by the tensor cores)
  // Release the dependent grid only once this CTA holds its tensor memory
  // (the barrier orders warp 0's allocation before every thread's trigger):
  // a dependent CTA that lands on this SM may allocate before its own
  // dependency wait, and must then never take columns this CTA still needs.
  // (The grid is persistent: every CTA is resident at once.)
  __syncthreads();
  pdl_trigger();
  pdl_wait();

  const int64_t n_vec = static_cast<int64_t>(n_tokens) * hkv;
  const int64_t tiles_per_tensor = (n_vec + kTileVecs - 1) / kTileVecs;
  // (the swizzle is a function of the shared address: the operand tiles must
  // start on 1024-byte boundaries; never seen otherwise, checked all the same)
  const bool aligned = (smem_u32(smem_raw) & 1023u) == 0;
  if (!aligned && tid == 0) record_status(status, KVQ_ERR_UNSUPPORTED);
  const int64_t total_tiles = aligned ? 2 * tiles_per_tensor : 0;  // K tiles, then V tiles
  const int64_t grid = gridDim.x;
  // my warp's rows of tile t into A buffer `buf` (a group is committed even
  // when there is nothing to copy, which keeps the counting uniform)
  auto stage = [&](int64_t t, int buf) {
    if (t < total_tiles) {
      const bool isv = t >= tiles_per_tensor;
      stage_rows(smem_u32(sm.a[buf][0]), isv ? v : k, n_vec, hkv, stride_bytes,
                 (isv ? t - tiles_per_tensor : t) * kTileVecs + kWarpRows * warp, warp, lane);
    }
    cp_async_commit();
  };
  const int64_t tile0 = blockIdx.x;
  stage(tile0, 0);
  stage(tile0 + grid, 1);
  const uint32_t tbase = sm.tmem_base;
  const uint32_t tlane = tbase + (static_cast<uint32_t>(32 * warp) << 16);  // my lane
  uint32_t issued = 0;  // thread 0: MMA batches committed (batch k to mma_done[k & 1])

  // my vector of the tile whose epilogue runs next: its slot, block row,
  // head and tensor
  int32_t e_slot = -1;
  int e_head = 0;
  bool e_isv = false;
  // epilogue of tile kk (A buffer kk % 3, accumulator kk & 1)
  auto epilogue = [&](int64_t kk, float x0) {
    if (!mbar_wait_ab(&sm.mma_done[kk & 1], static_cast<uint32_t>((kk >> 1) & 1), abort)) return;
    tc_fence_after();
    uint8_t* seg = nullptr;
    if (e_slot >= 0) {
      const int32_t p = e_slot / kBlockSize;
      if (p >= num_blocks)
        record_status(status, KVQ_ERR_OUT_OF_RANGE);
      else
        seg = pool + (static_cast<int64_t>(p) * hkv + e_head) * Fmt<KB, VB>::kSegBytes;
    }
    const uint32_t dcol = tlane + 128u * static_cast<uint32_t>(kk & 1);
    if (e_isv)  // (uniform over the tile)
      quantize_lane<VB, true, Fmt<KB, VB>>(dcol, x0, seg, e_slot >= 0 ? e_slot % kBlockSize : 0);
    else
      quantize_lane<KB, false, Fmt<KB, VB>>(dcol, x0, seg, e_slot >= 0 ? e_slot % kBlockSize : 0);
  };
  auto first_elem = [&](int buf) -> float {  // element 0 of my row in A buffer buf
    const uint16_t u = *reinterpret_cast<const uint16_t*>(sm.a[buf][0] + sw128(tid, 0));
    return kBF16 ? __uint_as_float(static_cast<uint32_t>(u) << 16) : __half2float(__ushort_as_half(u));
  };

  int64_t kk = 0;  // tiles of this CTA walked so far
  for (int64_t tile = tile0; tile < total_tiles; tile += grid, ++kk) {
    // my vector of this tile: its slot load overlaps the copies and the MMAs
    const bool is_v = tile >= tiles_per_tensor;
    const int64_t n = (is_v ? tile - tiles_per_tensor : tile) * kTileVecs + tid;
    const int64_t tok = n < n_vec ? token_of(n, n_vec, hkv) : 0;
    const int32_t pslot = n < n_vec ? __ldg(slots + tok) : -1;
    // element 0 of my row of the previous tile, read before its A buffer is
    // staged again below (the barrier completes the read)
    const float x0_prev = kk >= 1 ? first_elem(static_cast<int>((kk - 1) % kNA)) : 0.0f;

    cp_async_wait<1>();  // my copies of this tile are done
    async_proxy_fence();  // (the tensor cores read them)
    tc_fence_before();
    __syncthreads();  // every row of this tile is in; the accumulator of tile kk-2 is read
    tc_fence_after();
    if (tid == 0 && !*abort) {
      // y0 = x0 H64 + x1 H64, y1 = x0 H64 - x1 H64 (N = 64 each, K in steps of 16)
      const int ab = static_cast<int>(kk % kNA);
      const uint32_t d = tbase + 128u * static_cast<uint32_t>(kk & 1);
      const uint32_t a0 = smem_u32(sm.a[ab][0]), a1 = smem_u32(sm.a[ab][1]);
      const uint32_t h0 = smem_u32(sm.hb[0]), h1 = smem_u32(sm.hb[1]);
      constexpr uint32_t id = idesc_h64<kBF16>();
#pragma unroll
      for (int st = 0; st < 4; ++st) mma_f16_ss(d, sdesc_sw128(a0 + 32 * st), sdesc_sw128(h0 + 32 * st), id, st > 0);
#pragma unroll
      for (int st = 0; st < 4; ++st) mma_f16_ss(d, sdesc_sw128(a1 + 32 * st), sdesc_sw128(h0 + 32 * st), id, true);
#pragma unroll
      for (int st = 0; st < 4; ++st)
        mma_f16_ss(d + 64, sdesc_sw128(a0 + 32 * st), sdesc_sw128(h0 + 32 * st), id, st > 0);
#pragma unroll
      for (int st = 0; st < 4; ++st) mma_f16_ss(d + 64, sdesc_sw128(a1 + 32 * st), sdesc_sw128(h1 + 32 * st), id, true);
      mma_commit(&sm.mma_done[kk & 1]);
      ++issued;
    }
    if (kk >= 1) {
      // tile kk-1: wait for its MMAs (then its A buffer is free for tile
      // kk+2), stage tile kk+2 there, then its epilogue from its accumulator
      epilogue(kk - 1, x0_prev);
      stage(tile + 2 * grid, static_cast<int>((kk + 2) % kNA));
    } else {
      stage(tile + 2 * grid, 2);
    }
    tc_fence_before();
    e_slot = pslot;
    e_head = static_cast<int>(n - tok * hkv);
    e_isv = is_v;
  }
  if (kk >= 1) epilogue(kk - 1, first_elem(static_cast<int>((kk - 1) % kNA)));
  cp_async_wait<0>();
  if (*abort) {
    if (tid == 0) {
      record_status(status, KVQ_ERR_DEVICE_TIMEOUT);
      // tensor memory is released only once every MMA batch issued is complete
      // (bounded waits that ignore the abort flag)
      int zero = 0;
      for (uint32_t j = issued >= 2 ? issued - 2 : 0; j < issued; ++j)
        mbar_wait_ab(&sm.mma_done[j & 1], (j >> 1) & 1u, &zero);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "n"(kBulkTmemCols));
}


// ---- small appends (a few tokens per call, as in decode) --------------------
// One warp per head vector (quantize_vector_warp in kvq_internal.cuh).
constexpr int kSmallWarps = 4;
constexpr int64_t kSmallMaxVecs = 1024;  // at most this many head vectors per tensor

template <bool kBF16, int KB, int VB>
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
  uint8_t* seg = pool + (static_cast<int64_t>(p) * hkv + h) * Fmt<KB, VB>::kSegBytes;

  quantize_vector_warp<kBF16, KB, VB>((is_v ? v : k) + tok * stride_bytes + static_cast<int64_t>(h) * (kHeadDim * 2),
                                      seg, row_in_block, is_v, lane);
}

template <bool kBF16, int KB, int VB>
cudaError_t launch_quantize_t(const QuantizeArgs& a, cudaStream_t stream) {
  const int64_t n_vec = static_cast<int64_t>(a.n_tokens) * a.num_kv_heads;
  const int64_t stride_bytes = a.token_stride * 2;
  const uint8_t* k = static_cast<const uint8_t*>(a.k);
  const uint8_t* v = static_cast<const uint8_t*>(a.v);
  if (n_vec <= kSmallMaxVecs) {
    const unsigned grid = static_cast<unsigned>((2 * n_vec + kSmallWarps - 1) / kSmallWarps);
    return launch_pdl(quantize_small_kernel<kBF16, KB, VB>, dim3(grid), dim3(kSmallWarps * 32), 0, stream, a.pool,
                      a.num_blocks, a.num_kv_heads, k, v, a.n_tokens, stride_bytes, a.slots, a.status);
  }
  const int64_t tiles = 2 * ((n_vec + kTileVecs - 1) / kTileVecs);
  const int smem = kBulkSmemBytes;
  int64_t grid = tiles;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 2;  // two CTAs per SM, all resident
  if (grid > cap) grid = cap;
  const cudaError_t e = ensure_smem_limit<quantize_kernel<kBF16, KB, VB>>(smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(quantize_kernel<kBF16, KB, VB>, dim3(static_cast<unsigned>(grid)), dim3(kBulkThreads), smem,
                    stream, a.pool, a.num_blocks, a.num_kv_heads, k, v, a.n_tokens, stride_bytes, a.slots, a.status);
}

template <int KB, int VB>
cudaError_t launch_quantize_p(const QuantizeArgs& a, cudaStream_t stream) {
  return a.in_dtype == KVQ_BF16 ? launch_quantize_t<true, KB, VB>(a, stream)
                                : launch_quantize_t<false, KB, VB>(a, stream);
}

}  // namespace

cudaError_t launch_quantize(const QuantizeArgs& a, cudaStream_t stream) {
  if (a.n_tokens == 0) return cudaSuccess;
  if (a.k_bits == 4 && a.v_bits == 2) return launch_quantize_p<4, 2>(a, stream);
  if (a.k_bits == 4 && a.v_bits == 4) return launch_quantize_p<4, 4>(a, stream);
  if (a.k_bits == 2 && a.v_bits == 2) return launch_quantize_p<2, 2>(a, stream);
  if (a.k_bits == 8 && a.v_bits == 4) return launch_quantize_p<8, 4>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace kvq
