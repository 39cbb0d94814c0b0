// Long query runs (prefill, chunked prefill) on the 5th-generation tensor cores.
//
// Same computation as the mma.sync kernels of pa_extend.cu (query i of sequence s at
// position L_s - Q_s + i attends causally to the paged context; page 2, sections
// "2.1 核心组件交互流程" and "2.2 关键数据结构剖析"), with 128-row tiles on tcgen05:
//   * a work unit is (sequence, kv head, tile of 128 rows, chunk of the context); a row
//     is a (query, q head of the kv head's group) pair; the chunk is a multiple of the
//     512-token partition, chosen by the host so that there are enough units to fill
//     the GPU (the whole context when there are, then no merge pass at all); the plan
//     kernel writes one record per (sequence, tile, chunk);
//   * one persistent CTA per SM runs two independent pipelines ("sets") that share the
//     tensor core: each set takes its own units from the global queue and has its own
//     Q, K and V buffers in shared memory and its own S and O accumulators in TMEM
//     (S of set c in columns [128 c, 128 c + 128), O in [256 + 128 c, ...)). While one
//     set's softmax works on its scores, the tensor core runs the other set's MMAs;
//   * warps: 4 softmax warps per set (thread = one row of the tile, all 128 columns, so
//     no two warps ever combine a row), one MMA-issue warp for both sets, and one
//     producer warp per set that takes its units, loads Q (one 3-D TMA box per 64-dim
//     half: 64 dims x G heads x 128 / G queries) and streams K and V tiles (2-D TMA,
//     one box per (cache block, 64-dim half), 128B swizzle, no multicast);
//   * S = Q K^T (both operands K-major in shared memory). The softmax writes P over its
//     own scores in TMEM as 16-bit pairs, and O += P V takes P from TMEM (A operand)
//     and V in its [token][dim] cache layout (MN-major B operand). Per set the issue
//     order is S(g), P(g) V(g), S(g + 1) (which waits for P(g) V(g): it overwrites the
//     P it reads); the MMA warp alternates S(set 0), S(set 1), P V(set 0), P V(set 1);
//   * the softmax keeps a reference maximum that moves only when the row maximum passes
//     it by more than 2^8 (O and the running sum are then rescaled; every p stays below
//     2^8). For bf16, p rounded to bf16 can leave the parity tolerance when a few
//     weights dominate and their V values cancel, so the rounded remainder
//     p - bf16(p) goes into the other 64 columns of S and a second P V product adds it
//     (hi + lo carries p to within 2^-16): for every tile, or only for tiles where some
//     row has a weight above 1/8 of its running sum (a later tile can only lower that
//     share, so every unadjusted weight ends below 1/8 of the row's total);
//   * a unit that covers a row's whole context writes the output row; otherwise it
//     writes (max, sum, unnormalised row) for the log-sum-exp merge kernel.
// Every wait is bounded; on a timeout the kernel records it, every role stops, the MMA
// and load issuers drain what they issued, and the TMEM is freed.
#include <cstdlib>
#include <cstring>

namespace pa {

constexpr int kTcRows = 128;            // query rows per unit (TMEM lanes)
constexpr int kTcTok = 128;             // tokens per K/V tile
constexpr int kTcD = 128;               // head_dim of this path
constexpr uint32_t kTcTmemCols = 512;   // S of the two sets in [0, 256), their O in [256, 512)
constexpr int kTcSets = 2;              // independent pipelines sharing the tensor core
constexpr int kTcSetWarps = 4;          // softmax warps per set: one thread per row
constexpr int kTcSoftmaxWarps = kTcSets * kTcSetWarps;
constexpr int kTcMmaWarp = kTcSoftmaxWarps;           // followed by one producer warp per set
constexpr int kTcThreads = (kTcSoftmaxWarps + 1 + kTcSets) * 32;
constexpr float kTcRescale = 8.f;       // log2 units

// P V precision modes (ExtendParams::lo_mode)
constexpr int kLoNone = 0;      // P rounded to the 16-bit type only (f16: rounding up to 2^-11 of p)
constexpr int kLoAlways = 1;    // the bf16 remainder for every tile
constexpr int kLoAdaptive = 2;  // the bf16 remainder for tiles with a weight above kLoShare (pa_extend.cu)

struct TcSmem {
  static constexpr int kTile = kTcRows * kTcD * 2;   // 32 KB: two 64-column halves of 16 KB
  static constexpr int kQ = 0, kK = kTile, kV = 2 * kTile;
  static constexpr int kSet = 3 * kTile;             // Q, K and V of one set
  static constexpr int kBytes = kTcSets * kSet + 1024;   // 193 KB with the alignment slack
};
static_assert(kTcRows == kTcTok, "Q, K and V tiles share one swizzled layout");

// Shared-memory matrix descriptor: 128B swizzle, sm_100 descriptor version.
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr, uint32_t sbo, uint32_t lbo) {
  uint64_t d = uint64_t((saddr >> 4) & 0x3FFF);
  d |= uint64_t((lbo >> 4) & 0x3FFF) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFF) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

// Instruction descriptor of kind::f16: f32 accumulate, A and B both bf16 or both f16,
// A K-major, B K-major (b_mn = 0) or MN-major (b_mn = 1), M = N = 128.
template <int QD>
__device__ __forceinline__ uint32_t tc_idesc(uint32_t b_mn) {
  constexpr uint32_t fmt = QD == PA_BF16 ? 1u : 0u;
  return (1u << 4) | (fmt << 7) | (fmt << 10) | (b_mn << 16) | (uint32_t(kTcTok >> 3) << 17) |
         (uint32_t(kTcRows >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  const uint32_t z = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(z)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive columns of this warp's 32 lanes (warp-collective).
__device__ __forceinline__ void tc_ld32(uint32_t addr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(addr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// The same load without its wait: issue several, then one tc_wait_ld(), then read the
// registers through pin_after_wait() so that no use is scheduled before the wait.
__device__ __forceinline__ void tc_ld32_async(uint32_t addr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(addr));
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ uint32_t pin_after_wait(uint32_t x) {
  asm volatile("" : "+r"(x));
  return x;
}

__device__ __forceinline__ void tc_st32(uint32_t addr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(addr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// max(a, b, c) in one instruction (sm_100 three-input max; a NaN operand is ignored as by fmaxf).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x on the special-function unit (flushes subnormal results to zero).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed binary32 pairs (sm_100 f32x2 arithmetic): a * b + c and a + b, lane-wise.
__device__ __forceinline__ float2 fma2(float2 a, float b, float c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\t"
      "mov.b64 rc, {%5, %5};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// 3-D tiled TMA load.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
      : "memory");
}

// 2-D tiled TMA store shared -> global (bulk async-group of the issuing thread).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int x, int y, const void* src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(map), "r"(x),
               "r"(y), "r"(smem_addr(src))
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Byte offset of 16-byte chunk c (0..15) of row r in a [128 x 128] 16-bit tile kept
// as two 128B-swizzled K-major halves of 64 columns (8-row atoms of 1 KB).
__device__ __forceinline__ uint32_t tc_swz(int r, int c) {
  return uint32_t((c >> 3) * (kTcRows * 128) + (r >> 3) * 1024 + (r & 7) * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Geometry of one work unit as every role of the CTA computes it.
struct TcUnit {
  int s, hk, t, part;
  int Q, base, row0;
  int t0, nvis, ntiles;     // first context token of the chunk, visible tokens, K/V tiles
};

// Unit u = pair * Hkv + kv head; the pair's record was written by the plan kernel.
__device__ __forceinline__ TcUnit tc_unit(const ExtendParams& p, int u) {
  const int pair = u / p.num_kv_heads;
  const int4 a = __ldg(p.units + 2 * size_t(pair)), b = __ldg(p.units + 2 * size_t(pair) + 1);
  TcUnit t;
  t.s = a.x;
  t.hk = u - pair * p.num_kv_heads;
  t.t = a.y;
  t.part = a.z;
  t.row0 = a.w;
  t.Q = b.x;
  t.base = b.y;
  t.t0 = b.z;
  t.nvis = b.w;
  t.ntiles = (t.nvis + kTcTok - 1) / kTcTok;
  return t;
}

// Bounded wait that also gives up as soon as another role of the CTA has aborted.
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int where, int u) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_timer_ns() - t0 > 2000000000ull) {
      record_error(PA_DEV_WAIT_TIMEOUT, where, u, int(parity));
      *abort = 1;
      return false;
    }
  }
}

// Warp-uniform form: true only if every lane's wait succeeded.
__device__ __forceinline__ bool tc_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort, int where, int u) {
  return __all_sync(kFull, tc_wait(bar, parity, abort, where, u));
}


// O += P V with P (the A operand) in TMEM: M = 128 lanes, K = 16 per instruction (8
// columns of bf16 / f16 pairs), B from shared memory.
__device__ __forceinline__ void tc_mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// 16 consecutive 32-bit columns of this warp's 32 lanes, without the wait (the registers
// are read at issue; one tc_wait_st() orders all of them before the next barrier).
__device__ __forceinline__ void tc_st16(uint32_t addr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          addr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// 16 consecutive 32-bit columns of this warp's 32 lanes, without the wait.
__device__ __forceinline__ void tc_ld16_async(uint32_t addr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(addr));
}

// 8 consecutive 32-bit columns of this warp's 32 lanes, without the wait.
__device__ __forceinline__ void tc_st8(uint32_t addr, const uint32_t* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(addr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

// Two values rounded to the 16-bit type and packed (lo in the low half).
template <int QD>
__device__ __forceinline__ uint32_t pack16x2(float lo, float hi) {
  if constexpr (QD == PA_BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
  }
}

// The binary32 values of a packed bf16 pair (bf16 is the upper half of a binary32).
__device__ __forceinline__ float2 bf16x2_value(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// Keeps the compiler from moving the computation of v past this point (an empty asm that
// reads it): the work on one TMEM chunk then overlaps the load of the next one.
__device__ __forceinline__ void keep8(const float (&v)[8]) {
  asm volatile("" ::"f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
}

// Folds 32 scores (columns c0 .. c0 + 31 of the tile; with kMask those past `vis` masked)
// into 8 maxima.
template <bool kMask>
__device__ __forceinline__ void tc_fold_max(const uint32_t (&r)[32], int c0, int vis, float (&m8)[8]) {
  auto at = [&](int i) {
    const float v = __uint_as_float(pin_after_wait(r[i]));
    return kMask && c0 + i > vis ? -INFINITY : v;
  };
#pragma unroll
  for (int i = 0; i < 32; i += 16)
#pragma unroll
    for (int e = 0; e < 8; ++e) m8[e] = fmax3(m8[e], at(i + e), at(i + 8 + e));
}

// Pass 1 of the softmax: the maximum of one row's 128 scores in TMEM (this thread's lane;
// with kMask those past `vis` masked), 32 columns at a time with the next 32 in flight.
template <bool kMask>
__device__ __forceinline__ float tc_row_max(uint32_t addr, int vis) {
  float m8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m8[e] = -INFINITY;
  uint32_t ra[32], rb[32];
  tc_ld32_async(addr, ra);
  tc_wait_ld();
  tc_ld32_async(addr + 32, rb);
  tc_fold_max<kMask>(ra, 0, vis, m8);
  keep8(m8);
  tc_wait_ld();
  tc_ld32_async(addr + 64, ra);
  tc_fold_max<kMask>(rb, 32, vis, m8);
  keep8(m8);
  tc_wait_ld();
  tc_ld32_async(addr + 96, rb);
  tc_fold_max<kMask>(ra, 64, vis, m8);
  keep8(m8);
  tc_wait_ld();
  tc_fold_max<kMask>(rb, 96, vis, m8);
  return fmaxf(fmax3(m8[0], m8[1], m8[2]), fmax3(fmax3(m8[3], m8[4], m8[5]), m8[6], m8[7]));
}

// Pass 2 on 16 scores (tokens 16 t .. 16 t + 15 of the tile, columns [16 t, 16 t + 16) of
// S; with kMask those past `vis` masked): p = 2^(s * s_mul + nmb) written over them as
// 16-bit pairs, P in columns [16 t, 16 t + 8) and, with kLo, the rounded remainder
// p - bf16(p) in [16 t + 8, 16 t + 16); the binary32 p are added to l2 (four pair chains).
template <int QD, bool kMask, bool kLo>
__device__ __forceinline__ void tc_make_p16(uint32_t addr, const uint32_t (&r)[16], int t, int vis, float s_mul,
                                            float nmb, float2 (&l2)[4]) {
  uint32_t wh[8], wl[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int col = t * 16 + 2 * e;
    float s0 = __uint_as_float(pin_after_wait(r[2 * e]));
    float s1 = __uint_as_float(pin_after_wait(r[2 * e + 1]));
    if (kMask) {
      s0 = col > vis ? -INFINITY : s0;
      s1 = col + 1 > vis ? -INFINITY : s1;
    }
    const float2 a = fma2(make_float2(s0, s1), s_mul, nmb);
    const float p0 = ex2(a.x), p1 = ex2(a.y);
    wh[e] = pack16x2<QD>(p0, p1);
    l2[e & 3] = add2(l2[e & 3], make_float2(p0, p1));
    if constexpr (kLo) {
      const float2 hv = bf16x2_value(wh[e]);
      wl[e] = pack16x2<QD>(p0 - hv.x, p1 - hv.y);
    }
  }
  tc_st8(addr + t * 16, wh);
  if constexpr (kLo) tc_st8(addr + t * 16 + 8, wl);
}

// Pass 2 over the row's 128 scores, 16 columns at a time with the next 16 in flight.
template <int QD, bool kMask, bool kLo>
__device__ __forceinline__ void tc_make_p(uint32_t addr, int vis, float s_mul, float nmb, float2 (&l2)[4]) {
  uint32_t ra[16], rb[16];
  tc_ld16_async(addr, ra);
  tc_wait_ld();
#pragma unroll 1
  for (int t = 0; t < kTcTok / 16; t += 2) {
    tc_ld16_async(addr + (t + 1) * 16, rb);
    tc_make_p16<QD, kMask, kLo>(addr, ra, t, vis, s_mul, nmb, l2);
    tc_wait_ld();
    if (t + 2 < kTcTok / 16) tc_ld16_async(addr + (t + 2) * 16, ra);
    tc_make_p16<QD, kMask, kLo>(addr, rb, t + 1, vis, s_mul, nmb, l2);
    tc_wait_ld();
  }
}

// One CTA per SM. The register file is split between the SM's four sub-partitions and a
// warp takes its registers from its own: with 11 warps, three share one sub-partition's
// 16384 registers, so a thread may hold at most 170 (the compiler takes 168).
template <int QD, int BS, int G>
__global__ void __launch_bounds__(kTcThreads, 1)
    extend_tc_kernel(const ExtendParams p, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tq,
                     const __grid_constant__ CUtensorMap tkn, const __grid_constant__ CUtensorMap tvn) {
  using QT = typename Q<QD>::T;
  constexpr int QPT = kTcRows / G;                    // queries per unit
  constexpr int BPT = kTcTok / BS;                    // cache blocks per K/V tile
  constexpr uint32_t kBlockTx = BS * kTcD * 2;        // bytes of one cache block of K (or V)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // per set: S(g) landed, P(g) written (one arrival per softmax warp), P(g) V(g) done;
  // K(g) / V(g) landed, K buffer free; Q of unit k landed / free; O of unit k complete /
  // read (one arrival per softmax warp); the unit ring
  __shared__ uint64_t s_full[kTcSets], p_full[kTcSets], pv_done[kTcSets], k_full[kTcSets], v_full[kTcSets];
  __shared__ uint64_t k_empty[kTcSets], q_full[kTcSets], q_empty[kTcSets], o_full[kTcSets], o_empty[kTcSets];
  __shared__ uint64_t uq_full[kTcSets][4], uq_empty[kTcSets][4], bar_fin;
  __shared__ int uq[kTcSets][4];               // unit k of set c in slot k % 4
  __shared__ int lo_tile[kTcSets];             // adaptive remainder: the set's latest tile that needs it
  __shared__ uint64_t vote_bar[kTcSets];       // the set's warps agree on the remainder of each tile
  __shared__ int vote_word[kTcSets][3];        // ... through one word per tile, three in rotation
  __shared__ uint32_t tmem_slot;
  __shared__ int s_abort;
  volatile int* abort = &s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&tmem_slot)),
                 "r"(kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 32) {
    for (int c = 0; c < kTcSets; ++c) {
      mbar_init(&s_full[c], 1);
      mbar_init(&p_full[c], kTcSetWarps);
      mbar_init(&pv_done[c], 1);
      mbar_init(&k_full[c], 1);
      mbar_init(&v_full[c], 1);
      mbar_init(&k_empty[c], 1);
      mbar_init(&q_full[c], 1);
      mbar_init(&q_empty[c], 1);
      mbar_init(&o_full[c], 1);
      mbar_init(&o_empty[c], kTcSetWarps);
      for (int i = 0; i < 4; ++i) {
        mbar_init(&uq_full[c][i], 1);
        mbar_init(&uq_empty[c][i], kTcSetWarps + 1);   // the set's softmax warps and the MMA warp
      }
      lo_tile[c] = -1;
      mbar_init(&vote_bar[c], kTcSetWarps);
      vote_word[c][0] = vote_word[c][1] = vote_word[c][2] = 0;
    }
    mbar_init(&bar_fin, 1);
    s_abort = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dependency_launch_dependents();
  grid_dependency_wait();

  const uint32_t tmem = tmem_slot;
  const int Hq = p.num_q_heads, Hkv = p.num_kv_heads;
  const int total = p.plan[p.num_seqs] * Hkv;
  uint32_t k_loads = 0, v_loads = 0, q_loads = 0;   // producer: loads issued (for the drain after an abort)

  // Dynamic scheduling: each set's producer takes the set's unit k from the global queue
  // (the plan kernel lists each sequence's longest row tile first) and publishes it in
  // the set's ring; the set's softmax warps and the MMA warp read the same sequence. -1
  // ends the set's work. False on an abort.
  auto next_unit = [&](int c, uint32_t k, bool taker, int& u) -> bool {
    const int slot = k & 3;
    const uint32_t ph = (k >> 2) & 1;
    if (taker) {
      if (!tc_wait_warp(&uq_empty[c][slot], ph ^ 1, abort, 28, int(k))) return false;
      int v = 0;
      if (lane == 0) {
        v = atomicAdd(p.queue, 1);
        if (v >= total) v = -1;
        uq[c][slot] = v;
        mbar_arrive(&uq_full[c][slot]);
      }
      u = __shfl_sync(kFull, v, 0);
      return true;
    }
    if (!tc_wait_warp(&uq_full[c][slot], ph, abort, 29, int(k))) return false;
    u = *reinterpret_cast<volatile int*>(&uq[c][slot]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&uq_empty[c][slot]);
    return true;
  };

  if (warp > kTcMmaWarp) {
    // ---------------- producer of set c: its units, their Q, K and V tiles ----------------
    const int c = warp - kTcMmaWarp - 1;
    uint8_t* sQ = sm + c * TcSmem::kSet + TcSmem::kQ;
    uint8_t* sK = sm + c * TcSmem::kSet + TcSmem::kK;
    uint8_t* sV = sm + c * TcSmem::kSet + TcSmem::kV;
    uint32_t g = 0;
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      int u;
      if (!(ok = next_unit(c, k, true, u)) || u < 0) break;
      const TcUnit x = tc_unit(p, u);
      // the unit's q rows, once the last S of the set's previous unit has read the buffer
      if (!(ok = tc_wait_warp(&q_empty[c], (k & 1) ^ 1, abort, 26, u))) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&q_full[c], TcSmem::kTile);
        tma_load_3d(sQ, &tq, 0, x.hk * G, x.row0 + x.t * QPT, &q_full[c]);
        tma_load_3d(sQ + kTcRows * 128, &tq, 64, x.hk * G, x.row0 + x.t * QPT, &q_full[c]);
      }
      __syncwarp();
      q_loads = k + 1;
      const int32_t* trow = p.block_tables + size_t(x.s) * p.max_blocks;
      auto blocks = [&](int j) { return min(BPT, (x.nvis - j * kTcTok + BS - 1) / BS); };
      auto fetch = [&](int lb, int n) {   // block id of this lane's block (lane < n), checked
        int id = 0;
        if (lane < n) {
          id = trow[lb + lane];
          if (id < 0 || id >= p.num_blocks) {
            record_error(PA_DEV_BAD_BLOCK_ID, x.s, lb + lane, id);
            id = 0;
          }
        }
        return id;
      };
      for (int j = 0; j < x.ntiles; ++j, ++g) {
        const int p0 = x.t0 + j * kTcTok;
        const int nb = blocks(j);
        const int id = p.fresh ? 0 : fetch(p0 / BS, nb);
        // K(g) once S(g-1) has read the buffer (and, for whole prompts, once the cache
        // stores of the previous tile have read both buffers)
        if (!(ok = tc_wait_warp(&k_empty[c], (g & 1) ^ 1, abort, 10, u))) break;
        if (p.fresh) bulk_wait_read_all();
        __syncwarp();
        if (p.fresh) {   // whole prompts: the prompt's own rows, 128 per box
          if (lane == 0) {
            mbar_arrive_expect_tx(&k_full[c], TcSmem::kTile);
            tma_load_3d(sK, &tkn, 0, x.hk, x.row0 + p0, &k_full[c]);
            tma_load_3d(sK + kTcTok * 128, &tkn, 64, x.hk, x.row0 + p0, &k_full[c]);
          }
        } else {
          if (lane == 0) mbar_arrive_expect_tx(&k_full[c], uint32_t(nb) * kBlockTx);
          __syncwarp();
          if (lane < nb) {
            const int y = (id * Hkv + x.hk) * BS;
            tma_load_2d(sK + lane * (BS * 128), &tk, 0, y, &k_full[c]);
            tma_load_2d(sK + kTcTok * 128 + lane * (BS * 128), &tk, 64, y, &k_full[c]);
          }
        }
        __syncwarp();
        k_loads = g + 1;
        // V(g) once P(g-1) V(g-1) has read the buffer
        if (!(ok = tc_wait_warp(&pv_done[c], (g & 1) ^ 1, abort, 11, u))) break;
        if (p.fresh) {
          if (lane == 0) {
            mbar_arrive_expect_tx(&v_full[c], TcSmem::kTile);
            tma_load_3d(sV, &tvn, 0, x.hk, x.row0 + p0, &v_full[c]);
            tma_load_3d(sV + kTcTok * 128, &tvn, 64, x.hk, x.row0 + p0, &v_full[c]);
          }
        } else {
          if (lane == 0) mbar_arrive_expect_tx(&v_full[c], uint32_t(nb) * kBlockTx);
          __syncwarp();
          if (lane < nb) {
            const int y = (id * Hkv + x.hk) * BS;
            tma_load_2d(sV + lane * (BS * 128), &tv, 0, y, &v_full[c]);
            tma_load_2d(sV + kTcTok * 128 + lane * (BS * 128), &tv, 64, y, &v_full[c]);
          }
        }
        __syncwarp();
        v_loads = g + 1;
        // whole prompts: the row tile that sees every prompt position of this K/V tile
        // writes the tile into its cache blocks, once both loads have landed
        if (p.fresh && x.t == min((p0 + kTcTok - 1) / QPT, (x.Q - 1) / QPT)) {
          if (!(ok = tc_wait_warp(&k_full[c], g & 1, abort, 27, u) && tc_wait_warp(&v_full[c], g & 1, abort, 27, u)))
            break;
          const int nbw = (min(p0 + kTcTok, x.Q) - p0 + BS - 1) / BS;
          const int idw = fetch(p0 / BS, nbw);
          if (lane < nbw) {
            const int y = (idw * Hkv + x.hk) * BS;
            tma_store_2d(&tk, 0, y, sK + lane * (BS * 128));
            tma_store_2d(&tk, 64, y, sK + kTcTok * 128 + lane * (BS * 128));
            tma_store_2d(&tv, 0, y, sV + lane * (BS * 128));
            tma_store_2d(&tv, 64, y, sV + kTcTok * 128 + lane * (BS * 128));
            bulk_commit();
          }
          __syncwarp();
        }
      }
    }
    bulk_wait_all();   // this thread's cache stores are complete before the kernel ends
  } else if (warp == kTcMmaWarp) {
    // ---------------- MMA issue for both sets ----------------
    // Per set the products form a chain S(g), P(g) V(g), S(g + 1), ...: S(g + 1) overwrites
    // the P that P(g) V(g) reads, so it waits for that product to complete. The sets are
    // served in turn -- P V(set 0), S(set 0), P V(set 1), S(set 1), ... -- so that each
    // set's next S follows its own P V as soon as possible while the other set's softmax
    // runs, and the tensor core alternates between the two chains.
    const uint32_t idS = tc_idesc<QD>(0), idO = tc_idesc<QD>(1);
    TcUnit x[kTcSets];
    int j[kTcSets];
    uint32_t g[kTcSets], k[kTcSets];
    bool live[kTcSets], fresh_unit[kTcSets];
#pragma unroll
    for (int c = 0; c < kTcSets; ++c) {
      j[c] = 0;
      g[c] = k[c] = 0;
      live[c] = fresh_unit[c] = true;
    }
    bool ok = true;
    // S(g) of set c (taking the set's next unit first when the last one is done); false
    // when the set has no more work (live[c] cleared) or on an abort (ok cleared)
    auto issue_s = [&](int c) {
      if (fresh_unit[c]) {
        int u;
        if (!(ok = next_unit(c, k[c], false, u))) return false;
        if (u < 0) {
          live[c] = false;
          return false;
        }
        x[c] = tc_unit(p, u);
        j[c] = 0;
        fresh_unit[c] = false;
        if (!(ok = tc_wait_warp(&q_full[c], k[c] & 1, abort, 14, u))) return false;
      }
      // once K(g) has landed and P(g-1) V(g-1), which reads P from the S columns, completed
      if (!(ok = tc_wait_warp(&k_full[c], g[c] & 1, abort, 16, int(g[c])) &&
                 tc_wait_warp(&pv_done[c], (g[c] & 1) ^ 1, abort, 17, int(g[c]))))
        return false;
      if (lane == 0) {
        tc_fence_after();
        const uint32_t qa = smem_addr(sm + c * TcSmem::kSet + TcSmem::kQ);
        const uint32_t ka = smem_addr(sm + c * TcSmem::kSet + TcSmem::kK);
#pragma unroll
        for (int kk = 0; kk < kTcD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kTcRows * 128) + (kk & 3) * 32;
          tc_mma(tmem + c * 128, tc_desc(qa + off, 1024, 16), tc_desc(ka + off, 1024, 16), idS, kk > 0);
        }
        tc_commit(&s_full[c]);
        tc_commit(&k_empty[c]);
        if (j[c] + 1 == x[c].ntiles) tc_commit(&q_empty[c]);   // the Q buffer is free once this S completes
      }
      __syncwarp();
      return true;
    };
    // O += P(g) V(g) (+ the remainder) of set c, once P is in TMEM and V(g) has landed; a
    // unit's first product overwrites O, so it waits until the previous unit's O was read
    auto issue_pv = [&](int c) {
      if (!(ok = tc_wait_warp(&p_full[c], g[c] & 1, abort, 12, int(g[c])) &&
                 tc_wait_warp(&v_full[c], g[c] & 1, abort, 13, int(g[c]))))
        return;
      if (j[c] == 0 && k[c] > 0 && !(ok = tc_wait_warp(&o_empty[c], (k[c] & 1) ^ 1, abort, 15, int(k[c])))) return;
      const bool lo = p.lo_mode == kLoAlways ||
                      (p.lo_mode == kLoAdaptive && *reinterpret_cast<volatile int*>(&lo_tile[c]) == int(g[c]));
      if (lane == 0) {
        tc_fence_after();
        const uint32_t va = smem_addr(sm + c * TcSmem::kSet + TcSmem::kV);
        const uint32_t d = tmem + 256 + c * 128, a = tmem + c * 128;
#pragma unroll
        for (int kk = 0; kk < kTcTok / 16; ++kk)   // P of tokens 16 kk .. 16 kk + 15
          tc_mma_ts(d, a + 16 * kk, tc_desc(va + kk * 2048, 1024, kTcTok * 128), idO, (j[c] > 0 || kk > 0) ? 1u : 0u);
        if (lo) {
#pragma unroll
          for (int kk = 0; kk < kTcTok / 16; ++kk)   // their remainders, 8 columns further
            tc_mma_ts(d, a + 16 * kk + 8, tc_desc(va + kk * 2048, 1024, kTcTok * 128), idO, 1u);
        }
        tc_commit(&pv_done[c]);
        if (j[c] + 1 == x[c].ntiles) tc_commit(&o_full[c]);
      }
      __syncwarp();
      ++g[c];
      if (++j[c] == x[c].ntiles) {
        fresh_unit[c] = true;
        ++k[c];
      }
    };
    bool pend[kTcSets];
#pragma unroll
    for (int c = 0; c < kTcSets; ++c) pend[c] = ok && issue_s(c);
    while (ok && (pend[0] || pend[1])) {
#pragma unroll
      for (int c = 0; c < kTcSets; ++c) {
        if (!ok || !pend[c]) continue;
        issue_pv(c);
        pend[c] = ok && issue_s(c);
      }
    }
  } else {
    // ---------------- softmax warps: set c, rows 32 rw .. 32 rw + 31 of the tile ----------------
    const int c = warp / kTcSetWarps, rw = warp % kTcSetWarps, row = rw * 32 + lane;
    const uint32_t t_row = tmem + (uint32_t(rw * 32) << 16);
    const uint32_t c_s = c * 128, c_o = 256 + c * 128;
    uint8_t* sV = sm + c * TcSmem::kSet + TcSmem::kV;
    uint32_t g = 0;
    for (uint32_t k = 0;; ++k) {
      int u;
      if (!next_unit(c, k, false, u) || u < 0) break;
      const TcUnit x = tc_unit(p, u);
      const int qi = x.t * QPT + row / G;
      const int head = x.hk * G + row % G;
      const bool has_q = qi < x.Q;
      const int qpos = has_q ? x.base + qi : -1;
      const int tok = has_q ? x.row0 + qi : -1;
      float m_ref = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < x.ntiles; ++j, ++g) {
        if (!(ok = tc_wait_warp(&s_full[c], g & 1, abort, 18, u))) break;
        tc_fence_after();
        // pass 1: the row maximum of the causally masked scores (8 independent chains); the
        // mask costs work only in tiles where some row of the warp ends
        const int tp0 = x.t0 + j * kTcTok;
        const int vis = qpos - tp0;   // columns 0 .. vis of this tile are visible to the row
        const bool masked = !__all_sync(kFull, vis >= kTcTok - 1);
        const float mx = (masked ? tc_row_max<true>(t_row + c_s, vis) : tc_row_max<false>(t_row + c_s, vis)) * p.s_mul;
        const bool up = mx > m_ref + kTcRescale;
        const float corr = up ? ex2(m_ref - mx) : 1.f;   // 0 while nothing was accumulated
        if (up) {
          l *= corr;
          m_ref = mx;
        }
        if (j > 0 && __any_sync(kFull, up)) {
          // O holds every earlier P V of the unit: S(g) was issued after P(g-1) V(g-1) completed
#pragma unroll 1
          for (int i = 0; i < kTcD / 32; ++i) {
            float o[32];
            tc_ld32(t_row + c_o + i * 32, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= corr;
            tc_st32(t_row + c_o + i * 32, o);
          }
        }
        const float nmb = m_ref == -INFINITY ? 0.f : -m_ref;
        // bf16: does this tile need P's remainder? Adaptive: when some row of the set has a
        // weight above kLoShare of its running sum -- tested, before the sum of this tile is
        // known, against the running sum plus the tile's largest weight (a lower bound of the
        // final sum, so the test flags at least the tiles that need it). The set's four warps
        // agree through one word and a 4-arrival barrier, since the product covers all rows.
        bool lo = false;
        if (QD == PA_BF16 && p.lo_mode == kLoAlways) {
          lo = true;
        } else if (QD == PA_BF16 && p.lo_mode == kLoAdaptive) {
          const float pmax = ex2(mx + nmb);   // the row's largest weight in this tile (0: none visible)
          const bool need = __any_sync(kFull, pmax > kLoShare * (l + pmax));
          volatile int* vw = vote_word[c];
          if (lane == 0) {
            if (rw == 0) vw[(g + 1) % 3] = 0;   // the next tile's word: every warp read it two tiles ago
            if (need) atomicOr(const_cast<int*>(&vw[g % 3]), 1);
            mbar_arrive(&vote_bar[c]);
          }
          if (!(ok = tc_wait_warp(&vote_bar[c], g & 1, abort, 24, u))) break;
          lo = vw[g % 3] != 0;
          if (lo && rw == 0 && lane == 0) *reinterpret_cast<volatile int*>(&lo_tile[c]) = int(g);
        }
        // pass 2, 16 columns at a time: P = 2^(s * scale - ref) as 16-bit pairs over the
        // scores it was made from (tokens 16 t ..: P in columns [16 t, 16 t + 8), with the
        // remainder p - bf16(p) in [16 t + 8, 16 t + 16))
        float2 l2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        if (masked) {
          if (lo) tc_make_p<QD, true, QD == PA_BF16>(t_row + c_s, vis, p.s_mul, nmb, l2);
          else tc_make_p<QD, true, false>(t_row + c_s, vis, p.s_mul, nmb, l2);
        } else {
          if (lo) tc_make_p<QD, false, QD == PA_BF16>(t_row + c_s, vis, p.s_mul, nmb, l2);
          else tc_make_p<QD, false, false>(t_row + c_s, vis, p.s_mul, nmb, l2);
        }
        l += ((l2[0].x + l2[0].y) + (l2[1].x + l2[1].y)) + ((l2[2].x + l2[2].y) + (l2[3].x + l2[3].y));
        // V rows past the visible tokens (cache bytes beyond the context, or stale rows of
        // blocks not loaded) are zeroed, so that 0-weighted rows cannot bring a NaN into O
        const int rem = x.nvis - j * kTcTok;
        if (rem < kTcTok) {
          if (!(ok = tc_wait_warp(&v_full[c], g & 1, abort, 21, u))) break;
          if (row >= rem) {
#pragma unroll
            for (int i = 0; i < kTcD / 8; ++i) *reinterpret_cast<uint4*>(sV + tc_swz(row, i)) = make_uint4(0, 0, 0, 0);
          }
          fence_async_smem();
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[c]);
      }
      if (!ok) break;
      // this unit's O, 64 columns at a time: the output row (the row's whole context was in
      // this unit) or the chunk's partial (unnormalised row, then max and sum); the
      // accumulator is released once all of it is read
      if (!tc_wait_warp(&o_full[c], k & 1, abort, 22, u)) break;
      tc_fence_after();
      const int P = has_q ? (qpos + 1 + p.chunk - 1) / p.chunk : 0;
      const bool wr = has_q && x.part < P, fin = wr && P == 1;
      const float inv = fin ? 1.f / l : 0.f;
      const size_t slot = (size_t(max(tok, 0)) * Hq + head) * p.max_parts + x.part;
      uint4* orow = reinterpret_cast<uint4*>(static_cast<QT*>(p.out) + (size_t(max(tok, 0)) * Hq + head) * kTcD);
      float4* acc = reinterpret_cast<float4*>(p.part_acc + slot * kTcD);
#pragma unroll
      for (int h = 0; h < kTcD / 64; ++h) {
        uint32_t r[64];
        tc_ld32_async(t_row + c_o + h * 64, r);
        tc_ld32_async(t_row + c_o + h * 64 + 32, r + 32);
        tc_wait_ld();
        auto o = [&](int i) { return __uint_as_float(pin_after_wait(r[i])); };
        if (fin) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            orow[h * 8 + i] = make_uint4(pack16x2<QD>(o(8 * i) * inv, o(8 * i + 1) * inv),
                                         pack16x2<QD>(o(8 * i + 2) * inv, o(8 * i + 3) * inv),
                                         pack16x2<QD>(o(8 * i + 4) * inv, o(8 * i + 5) * inv),
                                         pack16x2<QD>(o(8 * i + 6) * inv, o(8 * i + 7) * inv));
        } else if (wr) {
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[h * 16 + i] = make_float4(o(4 * i), o(4 * i + 1), o(4 * i + 2), o(4 * i + 3));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_empty[c]);
      if (wr && !fin) {
        p.part_ml[slot * 2] = m_ref;
        p.part_ml[slot * 2 + 1] = l;
      }
    }
  }

  __syncthreads();
  if (*abort) {   // drain what this CTA issued: MMAs (their thread), then each set's last loads
    if (warp == kTcMmaWarp && lane == 0) {
      tc_commit(&bar_fin);
      mbar_wait_bounded(&bar_fin, 0);
    }
    if (warp > kTcMmaWarp && lane == 0) {
      const int c = warp - kTcMmaWarp - 1;
      if (k_loads > 0) mbar_wait_bounded(&k_full[c], (k_loads - 1) & 1, 100000000ull);
      if (v_loads > 0) mbar_wait_bounded(&v_full[c], (v_loads - 1) & 1, 100000000ull);
      if (q_loads > 0) mbar_wait_bounded(&q_full[c], (q_loads - 1) & 1, 100000000ull);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols) : "memory");
}

// --------------------------------------------------------------------------
// host side: tensor maps over the cache viewed as [blocks * kv heads * block_size][head_dim]
// --------------------------------------------------------------------------
// q viewed as [tokens][q heads][head_dim]; box = 64 dims x G heads x 128 / G queries,
// i.e. one 64-column half of a unit's 128 rows in (query, head) order.
bool q_tmap(TmapEncodeFn enc, CUtensorMap* m, const void* q, int qd, int num_tokens, int Hq, int G) {
  const cuuint64_t dims[3] = {cuuint64_t(kTcD), cuuint64_t(Hq), cuuint64_t(num_tokens)};
  const cuuint64_t strides[2] = {cuuint64_t(kTcD) * 2, cuuint64_t(Hq) * kTcD * 2};
  const cuuint32_t box[3] = {64, cuuint32_t(G), cuuint32_t(kTcRows / G)};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, qd == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
             const_cast<void*>(q), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The prompts' own K / V ([tokens][kv heads][head_dim]); box = 64 dims x 1 head x 128 tokens.
bool kv_in_tmap(TmapEncodeFn enc, CUtensorMap* m, const void* kv, int qd, int num_tokens, int Hkv) {
  const cuuint64_t dims[3] = {cuuint64_t(kTcD), cuuint64_t(Hkv), cuuint64_t(num_tokens)};
  const cuuint64_t strides[2] = {cuuint64_t(kTcD) * 2, cuuint64_t(Hkv) * kTcD * 2};
  const cuuint32_t box[3] = {64, 1, cuuint32_t(kTcTok)};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, qd == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
             const_cast<void*>(kv), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

using TcKernel = void (*)(const ExtendParams, const CUtensorMap, const CUtensorMap, const CUtensorMap,
                          const CUtensorMap, const CUtensorMap);

template <int QD, int BS>
TcKernel tc_pick_g(int G) {
  switch (G) {
    case 1: return extend_tc_kernel<QD, BS, 1>;
    case 2: return extend_tc_kernel<QD, BS, 2>;
    case 4: return extend_tc_kernel<QD, BS, 4>;
    case 8: return extend_tc_kernel<QD, BS, 8>;
  }
  return nullptr;
}

TcKernel tc_pick(int qd, int BS, int G) {
  if (qd == PA_BF16) return BS == 16 ? tc_pick_g<PA_BF16, 16>(G) : BS == 32 ? tc_pick_g<PA_BF16, 32>(G) : nullptr;
  if (qd == PA_F16) return BS == 16 ? tc_pick_g<PA_F16, 16>(G) : BS == 32 ? tc_pick_g<PA_F16, 32>(G) : nullptr;
  return nullptr;
}

// How the bf16 remainder of P enters P V on this path: for the tiles that need it
// (default), or for every tile when PA_BF16_REMAINDER=always is set in the environment
// (read once). Both keep every weight to within the parity tolerance's needs.
int tc_bf16_lo_mode() {
  static const int mode = [] {
    const char* e = std::getenv("PA_BF16_REMAINDER");
    return (e && std::strcmp(e, "always") == 0) ? kLoAlways : kLoAdaptive;
  }();
  return mode;
}

bool extend_tc_supported(int qd, int D, int BS, int G) {
  return D == kTcD && tc_pick(qd, BS, G) != nullptr && tmap_encoder() != nullptr;
}

// Resident-CTA cap of the tcgen05 kernel (one CTA per SM).
cudaError_t extend_tc_grid_cap(int qd, int BS, int G, int* cap) {
  Launch l;
  l.fn = reinterpret_cast<KernelFn>(tc_pick(qd, BS, G));
  l.smem = TcSmem::kBytes;
  l.threads = kTcThreads;
  return occupancy(l, cap);
}

// Launch after the plan kernel (programmatic dependent launch). The cache base pointers
// are 16-byte aligned and the rows 256 bytes, as the tensor maps require.
pa_status extend_tc_launch(const ExtendParams& p, const pa_cache_desc* c, int qd, int G, int grid,
                           cudaStream_t s, const void* k_new, const void* v_new) {
  TcKernel fn = tc_pick(qd, c->block_size, G);
  TmapEncodeFn enc = tmap_encoder();
  if (!fn || !enc) return PA_ERR_ARG;
  CUtensorMap tk, tv, tq;
  const long long rows = (long long)c->num_blocks * c->num_kv_heads * c->block_size;
  if (!cache_tmap(enc, &tk, c->k_cache, qd, rows, c->block_size, kTcD) ||
      !cache_tmap(enc, &tv, c->v_cache, qd, rows, c->block_size, kTcD) ||
      !q_tmap(enc, &tq, p.q, qd, p.num_tokens, p.num_q_heads, G))
    return PA_ERR_ARG;
  CUtensorMap tkn = tk, tvn = tv;   // used only for whole prompts
  if (p.fresh && (!kv_in_tmap(enc, &tkn, k_new, qd, p.num_tokens, c->num_kv_heads) ||
                  !kv_in_tmap(enc, &tvn, v_new, qd, p.num_tokens, c->num_kv_heads)))
    return PA_ERR_ARG;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = TcSmem::kBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, p, tk, tv, tq, tkn, tvn) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace pa
