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
//   * one persistent CTA per SM takes units from a global queue. Its TMEM holds three S
//     buffers (tile g of the CTA's sequence of K/V tiles in buffer g % 3, columns
//     [128 b, 128 b + 128)) and O (columns [384, 512)); shared memory holds the unit's Q
//     and two buffers each for K and V tiles (tile g in buffer g % 2);
//   * warps: 8 softmax warps in pairs -- warp w owns the 32 rows of TMEM lane quarter
//     w % 4 (a warp can only reach its own quarter) and columns [64 h, 64 h + 64) of each
//     tile, h = w / 4; the two warps of a quarter exchange their row maxima (and running
//     sums) through shared memory and a two-arrival barrier -- one MMA-issue warp, a K
//     producer (takes the units, loads Q: one 3-D TMA box per 64-dim half, 64 dims x G
//     heads x 128 / G queries, and streams K) and a V producer (2-D TMA, one box per
//     (cache block, 64-dim half), 128B swizzle, no multicast);
//   * S = Q K^T (both operands K-major in shared memory). The softmax writes P over its
//     own scores in TMEM as 16-bit pairs, and O += P V takes P from TMEM (A operand)
//     and V in its [token][dim] cache layout (MN-major B operand). S(g) is issued once
//     K(g) has landed and P(g - 3) V(g - 3), which read its buffer, completed, so the
//     scores of the next tiles are ready while the softmax works on tile g; P(g) V(g) once
//     the softmax has written P(g). One thread of the MMA warp tests the barriers without
//     blocking and issues each product's 8 MMAs from one block of instructions;
//   * the softmax keeps a reference maximum that moves only when the row maximum passes
//     it by more than 2^8 (O and the running sum are then rescaled; every p stays below
//     2^8). For bf16, p rounded to bf16 can leave the parity tolerance when a few
//     weights dominate and their V values cancel, so the rounded remainder
//     p - bf16(p) goes into the other 64 columns of each token group of S and a second
//     P V product adds it (hi + lo carries p to within 2^-16): for every tile, or only
//     for tiles where some row has a weight above 1/8 of its running sum (a later tile
//     can only lower that share, so every unadjusted weight ends below 1/8 of the row's
//     total) -- the warps whose rows do not need it write zeros there;
//   * a unit that covers a row's whole context writes the output row (staged through
//     shared memory so that each store covers whole 128-byte row segments); otherwise it
//     writes (max, sum, unnormalised row) for the log-sum-exp merge kernel. A unit's O is
//     read after the first tile of the next unit, while the unit's last P V runs, and is
//     released before the rows are written.
// Every wait is bounded; on a timeout the kernel records it, every role stops, the MMA
// and load issuers drain what they issued, and the TMEM is freed.
#include <cstdlib>
#include <cstring>
#include <type_traits>

namespace pa {

constexpr int kTcRows = 128;            // query rows per unit (TMEM lanes)
constexpr int kTcTok = 128;             // tokens per K/V tile
constexpr int kTcHalf = kTcTok / 2;     // columns of a tile per softmax warp
constexpr int kTcD = 128;               // head_dim of this path
constexpr int kTcSBufs = 3;             // S buffers in TMEM (tile g in buffer g % 3)
constexpr int kTcKvBufs = 2;            // K and V buffers in shared memory (tile g in buffer g % 2)
constexpr uint32_t kTcOCol = kTcSBufs * kTcTok;   // O after the S buffers: 384 + 128 = 512 columns
constexpr uint32_t kTcTmemCols = 512;
constexpr int kTcQuarters = 4;          // row groups of 32 (a warp reads the TMEM lanes of its quarter)
constexpr int kTcSoftmaxWarps = 2 * kTcQuarters;      // warp w: rows of quarter w % 4, column half w / 4
constexpr int kTcMmaWarp = kTcSoftmaxWarps;           // then the K producer and the V producer
constexpr int kTcKWarp = kTcMmaWarp + 1, kTcVWarp = kTcMmaWarp + 2;
constexpr int kTcThreads = (kTcSoftmaxWarps + 3) * 32;
constexpr float kTcRescale = 8.f;       // log2 units
static_assert(kTcOCol + kTcD == kTcTmemCols, "three S buffers and O fill the TMEM");

// P V precision modes (ExtendParams::lo_mode)
constexpr int kLoNone = 0;      // P rounded to the 16-bit type only (f16: rounding up to 2^-11 of p)
constexpr int kLoAlways = 1;    // the bf16 remainder for every tile
constexpr int kLoAdaptive = 2;  // the bf16 remainder for tiles with a weight above kLoShare (pa_extend.cu)

// Shared memory: the Q tile and two buffers each for K and V tiles, every tile kept as two
// 128B-swizzled halves of 64 columns (dims); then the softmax warps' output staging rows.
struct TcSmem {
  static constexpr int kQTile = kTcRows * kTcD * 2;    // 32 KB: two halves of 16 KB
  static constexpr int kKvTile = kTcTok * kTcD * 2;    // 32 KB: two halves of 16 KB
  static constexpr int kQ = 0, kK = kQTile, kV = kQTile + kTcKvBufs * kKvTile;
  static constexpr int kStageWarp = 32 * kTcHalf * 2;  // 4 KB: a softmax warp's 32 output rows (its 64 dims)
  static constexpr int kStage = kV + kTcKvBufs * kKvTile;
  static constexpr int kBytes = kStage + kTcSoftmaxWarps * kStageWarp + 1024;   // 193 KB with the alignment slack
};

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
// A K-major, B K-major (b_mn = 0) or MN-major (b_mn = 1), M = 128, N = n.
template <int QD>
__device__ __forceinline__ uint32_t tc_idesc(uint32_t b_mn, uint32_t n) {
  constexpr uint32_t fmt = QD == PA_BF16 ? 1u : 0u;
  return (1u << 4) | (fmt << 7) | (fmt << 10) | (b_mn << 16) | ((n >> 3) << 17) | (uint32_t(kTcRows >> 4) << 24);
}

// S = Q K^T of one tile: the 8 MMAs of K = 16 over head_dim 128, issued from one block
// (descriptors advanced by immediates: a separately computed descriptor per MMA costs the
// issuing thread more time than the MMA takes). a0 / b0 describe dims 0 .. 15 of Q and K;
// dims 16 k .. lie 32 k bytes into the first 64-column half (k < 4) or one half (16 KB)
// further -- descriptor addresses count 16-byte units.
static_assert(kTcRows * 128 / 16 == 1024 && kTcTok * 128 / 16 == 1024, "descriptor steps of tc_mma_s8");
__device__ __forceinline__ void tc_mma_s8(uint32_t tmem_d, uint64_t a0, uint64_t b0, uint32_t idesc) {
  const uint32_t zero = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 a, b;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
      "add.s64 a, %1, 2;\n\tadd.s64 b, %2, 2;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, 1;\n\t"
      "add.s64 a, %1, 4;\n\tadd.s64 b, %2, 4;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, 1;\n\t"
      "add.s64 a, %1, 6;\n\tadd.s64 b, %2, 6;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, 1;\n\t"
      "add.s64 a, %1, 1024;\n\tadd.s64 b, %2, 1024;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, 1;\n\t"
      "add.s64 a, %1, 1026;\n\tadd.s64 b, %2, 1026;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, 1;\n\t"
      "add.s64 a, %1, 1028;\n\tadd.s64 b, %2, 1028;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, 1;\n\t"
      "add.s64 a, %1, 1030;\n\tadd.s64 b, %2, 1030;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, 1;\n\t}" ::"r"(tmem_d),
      "l"(a0), "l"(b0), "r"(idesc), "r"(zero)
      : "memory");
}

// O += P V of one tile with P (the A operand) in TMEM: 8 MMAs of K = 16 tokens, A at TMEM
// columns tmem_a + 16 t (8 columns of 16-bit pairs each), B = V rows 16 t .. 16 t + 15,
// 2 KB apart (128 descriptor units). acc0 = 0 makes the first product overwrite O.
static_assert(kTcTok == 128, "tc_mma_pv8 covers one 128-token tile");
__device__ __forceinline__ void tc_mma_pv8(uint32_t tmem_d, uint32_t tmem_a, uint64_t b0, uint32_t idesc,
                                           uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 b;\n\t.reg .b32 t;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "add.s32 t, %1, 16;\n\tadd.s64 b, %2, 128;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %3, 1;\n\t"
      "add.s32 t, %1, 32;\n\tadd.s64 b, %2, 256;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %3, 1;\n\t"
      "add.s32 t, %1, 48;\n\tadd.s64 b, %2, 384;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %3, 1;\n\t"
      "add.s32 t, %1, 64;\n\tadd.s64 b, %2, 512;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %3, 1;\n\t"
      "add.s32 t, %1, 80;\n\tadd.s64 b, %2, 640;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %3, 1;\n\t"
      "add.s32 t, %1, 96;\n\tadd.s64 b, %2, 768;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %3, 1;\n\t"
      "add.s32 t, %1, 112;\n\tadd.s64 b, %2, 896;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %3, 1;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(b0), "r"(idesc), "r"(acc0)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive columns of this warp's 32 lanes (warp-collective), without the wait:
// issue several, then one tc_wait_ld(), then read the registers through pin_after_wait()
// so that no use is scheduled before the wait.
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

// Byte offset of 16-byte chunk c (0..15) of row r in a K / V tile ([128 tokens x 128]
// 16-bit values kept as two 128B-swizzled halves of 64 columns, 8-row atoms of 1 KB).
__device__ __forceinline__ uint32_t tc_swz_kv(int r, int c) {
  return uint32_t((c >> 3) * (kTcTok * 128) + (r >> 3) * 1024 + (r & 7) * 128 + (((c & 7) ^ (r & 7)) << 4));
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

// As tc_wait, polling with the non-blocking test: for the short waits between the two
// softmax warps of a row quarter, where a suspended thread would wake later than the
// phase completes.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity);
__device__ __forceinline__ bool tc_spin(uint64_t* bar, uint32_t parity, volatile int* abort, int where, int u) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_test(bar, parity)) return true;
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

// As mbar_try_wait, with a bound on how long the hardware may suspend the thread while
// the phase is incomplete (nanoseconds; it resumes earlier when the phase completes).
__device__ __forceinline__ bool mbar_try_wait_for(uint64_t* bar, uint32_t parity, uint32_t suspend_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(suspend_ns)
      : "memory");
  return ok != 0;
}

// Non-blocking test: has the phase with this parity completed (as this thread sees it)?
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
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

// Pass 1 of the softmax: the maximum of one row's 64 scores of this warp's half of the
// tile in TMEM (this thread's lane; with kMask those past `vis` masked), both 32-column
// loads in flight at once.
static_assert(kTcHalf == 64, "tc_row_max reads one half tile");
template <bool kMask>
__device__ __forceinline__ float tc_row_max(uint32_t addr, int vis) {
  float m8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m8[e] = -INFINITY;
  uint32_t ra[32], rb[32];
  tc_ld32_async(addr, ra);
  tc_ld32_async(addr + 32, rb);
  tc_wait_ld();
  tc_fold_max<kMask>(ra, 0, vis, m8);
  tc_fold_max<kMask>(rb, 32, vis, m8);
  return fmaxf(fmax3(m8[0], m8[1], m8[2]), fmax3(fmax3(m8[3], m8[4], m8[5]), m8[6], m8[7]));
}

// The binary32 values of a packed bf16 pair (bf16 is the upper half of a binary32).
__device__ __forceinline__ float2 bf16x2_value(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// What pass 2 writes beside P (bf16 only): nothing, the rounded remainder, or zeros (the
// remainder product may cover these rows because another warp's rows need it).
constexpr int kRemNone = 0, kRemValue = 1, kRemZero = 2;

// Pass 2 on 16 scores (tokens 16 t .. 16 t + 15 of the tile, columns [16 t, 16 t + 16) of
// S; with kMask those past `vis` masked): p = 2^(s * s_mul + nmb) written over them as
// 16-bit pairs, P in columns [16 t, 16 t + 8) and, per kRem, the rounded remainder
// p - bf16(p) (or zeros) in [16 t + 8, 16 t + 16); the binary32 p are added to l2 (four pair
// chains).
template <int QD, bool kMask, int kRem>
__device__ __forceinline__ void tc_make_p16(uint32_t addr, const uint32_t (&r)[16], int t, int vis, float s_mul,
                                            float nmb, float2 (&l2)[4]) {
  static_assert(kRem == kRemNone || QD == PA_BF16, "the remainder is for bf16 P");
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
    if constexpr (kRem == kRemValue) {
      const float2 hv = bf16x2_value(wh[e]);
      wl[e] = pack16x2<QD>(p0 - hv.x, p1 - hv.y);
    } else if constexpr (kRem == kRemZero) {
      wl[e] = 0u;
    }
  }
  tc_st8(addr + t * 16, wh);
  if constexpr (kRem != kRemNone) tc_st8(addr + t * 16 + 8, wl);
}

// Pass 2 over the row's 64 scores of this warp's half, 16 columns at a time with the next
// 16 in flight.
template <int QD, bool kMask, int kRem>
__device__ __forceinline__ void tc_make_p(uint32_t addr, int vis, float s_mul, float nmb, float2 (&l2)[4]) {
  uint32_t ra[16], rb[16];
  tc_ld16_async(addr, ra);
  tc_wait_ld();
#pragma unroll 1
  for (int t = 0; t < kTcHalf / 16; t += 2) {
    tc_ld16_async(addr + (t + 1) * 16, rb);
    tc_make_p16<QD, kMask, kRem>(addr, ra, t, vis, s_mul, nmb, l2);
    tc_wait_ld();
    if (t + 2 < kTcHalf / 16) tc_ld16_async(addr + (t + 2) * 16, ra);
    tc_make_p16<QD, kMask, kRem>(addr, rb, t + 1, vis, s_mul, nmb, l2);
    tc_wait_ld();
  }
}

// One CTA per SM. The register file is split between the SM's four sub-partitions and a
// warp takes its registers from its own: with 11 warps, three share one sub-partition's
// 16384 registers, so a thread may hold at most 170.
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
  // tile g: S buffer g % 3 (phase g / 3 of its barriers), K / V buffer g % 2 (phase g / 2).
  // S(g) landed, P(g) written (one arrival per softmax warp), P(g) V(g) done; K(g) / V(g)
  // landed; Q of unit k landed / free; O of unit k complete / read (one arrival per
  // softmax warp); the two warps of a row quarter exchanged; the unit ring.
  __shared__ uint64_t s_full[kTcSBufs], p_full[kTcSBufs], pv_done[kTcSBufs], k_full[kTcKvBufs], v_full[kTcKvBufs];
  __shared__ uint64_t q_full, q_empty, o_full, o_empty, xchg[kTcQuarters];
  __shared__ uint64_t uq_full[4], uq_empty[4], bar_fin;
  __shared__ int uq[4], uq_nt[4];                                // unit k in slot k % 4, and its K/V tiles
  __shared__ __align__(8) char lo_need[kTcSBufs][kTcSoftmaxWarps];   // adaptive remainder: the warps' flags
  __shared__ float2 xval[2][kTcSoftmaxWarps][32];                // row maxima and sums exchanged, two in rotation
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
    for (int b = 0; b < kTcSBufs; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], kTcSoftmaxWarps);
      mbar_init(&pv_done[b], 1);
      for (int w = 0; w < kTcSoftmaxWarps; ++w) lo_need[b][w] = 0;
    }
    for (int b = 0; b < kTcKvBufs; ++b) {
      mbar_init(&k_full[b], 1);
      mbar_init(&v_full[b], 1);
    }
    mbar_init(&q_full, 1);
    mbar_init(&q_empty, 1);
    mbar_init(&o_full, 1);
    mbar_init(&o_empty, kTcSoftmaxWarps);
    for (int q = 0; q < kTcQuarters; ++q) mbar_init(&xchg[q], 2);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&uq_full[i], 1);
      mbar_init(&uq_empty[i], kTcSoftmaxWarps + 2);   // softmax warps, the MMA warp, the V producer
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
  uint32_t kv_loads = 0, q_loads = 0;   // producers: loads issued (for the drain after an abort)

  // Dynamic scheduling: the K producer takes unit k from the global queue (the plan kernel
  // lists each sequence's longest row tile first) and publishes it in slot k % 4 of the
  // ring; the V producer, the softmax warps and the MMA warp read the same sequence. -1
  // ends the work.
  auto read_unit = [&](uint32_t k, int& u) -> bool {   // reads slot k % 4 and releases it
    const int slot = k & 3;
    if (!tc_wait_warp(&uq_full[slot], (k >> 2) & 1, abort, 29, int(k))) return false;
    u = *reinterpret_cast<volatile int*>(&uq[slot]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&uq_empty[slot]);
    return true;
  };

  if (warp == kTcKWarp || warp == kTcVWarp) {
    // ---------------- producers: the K warp takes the units and loads Q and K, the V warp V ----------------
    const bool isk = warp == kTcKWarp;
    uint8_t* sQ = sm + TcSmem::kQ;
    uint32_t g = 0;
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      int u = -1;
      TcUnit x{};
      if (isk) {
        const int slot = k & 3;
        if (!(ok = tc_wait_warp(&uq_empty[slot], ((k >> 2) & 1) ^ 1, abort, 28, int(k)))) break;
        int v = 0;
        if (lane == 0) {
          v = atomicAdd(p.queue, 1);
          if (v >= total) v = -1;
        }
        u = __shfl_sync(kFull, v, 0);
        if (u >= 0) x = tc_unit(p, u);
        if (lane == 0) {
          uq[slot] = u;
          uq_nt[slot] = u < 0 ? 0 : x.ntiles;
          mbar_arrive(&uq_full[slot]);
        }
      } else {
        if (!(ok = read_unit(k, u))) break;
        if (u >= 0) x = tc_unit(p, u);
      }
      if (u < 0) break;
      if (isk) {
        // the unit's q rows, once the last S of the previous unit has read the buffer
        if (!(ok = tc_wait_warp(&q_empty, (k & 1) ^ 1, abort, 26, u))) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&q_full, TcSmem::kQTile);
          tma_load_3d(sQ, &tq, 0, x.hk * G, x.row0 + x.t * QPT, &q_full);
          tma_load_3d(sQ + kTcRows * 128, &tq, 64, x.hk * G, x.row0 + x.t * QPT, &q_full);
        }
        __syncwarp();
        q_loads = k + 1;
      }
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
      const CUtensorMap* cache_map = isk ? &tk : &tv;
      const CUtensorMap* new_map = isk ? &tkn : &tvn;
      for (int j = 0; j < x.ntiles; ++j, ++g) {
        const int xb = g & 1;
        uint64_t* full = isk ? &k_full[xb] : &v_full[xb];
        uint8_t* dst = sm + (isk ? TcSmem::kK : TcSmem::kV) + xb * TcSmem::kKvTile;
        const int p0 = x.t0 + j * kTcTok;
        const int nb = blocks(j);
        const int id = p.fresh ? 0 : fetch(p0 / BS, nb);
        // K(g) once S(g - 2), V(g) once P(g - 2) V(g - 2) has read the buffer (and, for
        // whole prompts, once this warp's cache stores have read theirs)
        if (g >= 2) {
          const uint32_t gr = g - 2;
          if (!(ok = tc_wait_warp(isk ? &s_full[gr % kTcSBufs] : &pv_done[gr % kTcSBufs], (gr / kTcSBufs) & 1, abort,
                                  isk ? 10 : 11, u)))
            break;
        }
        if (p.fresh) bulk_wait_read_all();
        __syncwarp();
        if (p.fresh) {   // whole prompts: the prompt's own rows, 128 per box
          if (lane == 0) {
            mbar_arrive_expect_tx(full, TcSmem::kKvTile);
            tma_load_3d(dst, new_map, 0, x.hk, x.row0 + p0, full);
            tma_load_3d(dst + kTcTok * 128, new_map, 64, x.hk, x.row0 + p0, full);
          }
        } else {
          if (lane == 0) mbar_arrive_expect_tx(full, uint32_t(nb) * kBlockTx);
          __syncwarp();
          if (lane < nb) {
            const int y = (id * Hkv + x.hk) * BS;
            tma_load_2d(dst + lane * (BS * 128), cache_map, 0, y, full);
            tma_load_2d(dst + kTcTok * 128 + lane * (BS * 128), cache_map, 64, y, full);
          }
        }
        __syncwarp();
        kv_loads = g + 1;
        // whole prompts: the row tile that sees every prompt position of this K/V tile
        // writes the tile into its cache blocks, once the load has landed
        if (p.fresh && x.t == min((p0 + kTcTok - 1) / QPT, (x.Q - 1) / QPT)) {
          if (!(ok = tc_wait_warp(full, (g >> 1) & 1, abort, 27, u))) break;
          const int nbw = (min(p0 + kTcTok, x.Q) - p0 + BS - 1) / BS;
          const int idw = fetch(p0 / BS, nbw);
          if (lane < nbw) {
            const int y = (idw * Hkv + x.hk) * BS;
            tma_store_2d(cache_map, 0, y, dst + lane * (BS * 128));
            tma_store_2d(cache_map, 64, y, dst + kTcTok * 128 + lane * (BS * 128));
            bulk_commit();
          }
          __syncwarp();
        }
      }
    }
    bulk_wait_all();   // this thread's cache stores are complete before the kernel ends
  } else if (warp == kTcMmaWarp) {
    // ---------------- MMA issue ----------------
    // S(g) into S buffer g % 3 once its unit's Q and K(g) have landed and P(g - 3) V(g - 3),
    // which reads the buffer, completed -- so S runs up to three tiles (and units) ahead of
    // the softmax; P V(g) once the softmax has written P(g) and V(g) has landed. Both
    // cursors read the units from the ring; the slot is released when the P V cursor is
    // done with the unit. One thread (lane 0) runs the issuer: it tests the barriers
    // without blocking and issues whatever is ready; the other lanes wait for it.
    if (lane == 0) {
      const uint32_t idS = tc_idesc<QD>(0, kTcTok), idO = tc_idesc<QD>(1, kTcD);
      const uint64_t dq = tc_desc(smem_addr(sm + TcSmem::kQ), 1024, 16);
      const uint64_t dk0 = tc_desc(smem_addr(sm + TcSmem::kK), 1024, 16);
      const uint64_t dv0 = tc_desc(smem_addr(sm + TcSmem::kV), 1024, kTcTok * 128);
      constexpr uint64_t kKvDesc = TcSmem::kKvTile >> 4;   // one K / V buffer in descriptor units
      int s_nt = 0, p_nt = 0;   // K/V tiles of the S cursor's and of the P V cursor's unit
      int js = 0, jp = 0;
      uint32_t gs = 0, gp = 0, ks = 0, kp = 0;
      bool s_live = true, s_fresh = true, p_fresh = true;
      auto try_s = [&]() -> bool {
        if (!s_live || gs >= gp + kTcSBufs) return false;
        if (s_fresh) {
          const int slot = ks & 3;
          if (!mbar_test(&uq_full[slot], (ks >> 2) & 1)) return false;
          const int u = *reinterpret_cast<volatile int*>(&uq[slot]);
          if (u < 0) {
            s_live = false;
            return true;
          }
          s_nt = *reinterpret_cast<volatile int*>(&uq_nt[slot]);
          js = 0;
          s_fresh = false;
        }
        const int b = gs % kTcSBufs, xb = gs & 1;
        if (!((js > 0 || mbar_test(&q_full, ks & 1)) && mbar_test(&k_full[xb], (gs >> 1) & 1) &&
              mbar_test(&pv_done[b], ((gs / kTcSBufs) & 1) ^ 1)))
          return false;
        tc_fence_after();
        tc_mma_s8(tmem + b * kTcTok, dq, dk0 + xb * kKvDesc, idS);
        tc_commit(&s_full[b]);
        if (js + 1 == s_nt) tc_commit(&q_empty);   // the Q buffer is free once this S completes
        ++gs;
        if (++js == s_nt) {
          s_fresh = true;
          ++ks;
        }
        return true;
      };
      // a unit's first P V overwrites O, so it also waits until the previous unit's O was read
      auto try_pv = [&]() -> bool {
        if (gp >= gs) return false;
        if (p_fresh) {   // the unit of this tile: the S cursor has read its slot already
          p_nt = *reinterpret_cast<volatile int*>(&uq_nt[kp & 3]);
          jp = 0;
          p_fresh = false;
        }
        const int b = gp % kTcSBufs, xb = gp & 1;
        if (!(mbar_test(&p_full[b], (gp / kTcSBufs) & 1) && mbar_test(&v_full[xb], (gp >> 1) & 1) &&
              (jp > 0 || kp == 0 || mbar_test(&o_empty, (kp & 1) ^ 1))))
          return false;
        // the remainder product: every tile, or (adaptive) when a softmax warp flagged it
        const bool lo = p.lo_mode == kLoAlways ||
                        (p.lo_mode == kLoAdaptive && *reinterpret_cast<volatile unsigned long long*>(lo_need[b]) != 0);
        tc_fence_after();
        const uint32_t d = tmem + kTcOCol, a = tmem + b * kTcTok;
        const uint64_t dv = dv0 + xb * kKvDesc;
        tc_mma_pv8(d, a, dv, idO, jp > 0 ? 1u : 0u);   // P of tokens 16 t .. 16 t + 15 at a + 16 t
        if (lo) tc_mma_pv8(d, a + 8, dv, idO, 1u);      // their remainders, 8 columns further
        tc_commit(&pv_done[b]);
        if (jp + 1 == p_nt) tc_commit(&o_full);
        ++gp;
        if (++jp == p_nt) {   // the unit is done: release its ring slot
          mbar_arrive(&uq_empty[kp & 3]);
          p_fresh = true;
          ++kp;
        }
        return true;
      };
      uint64_t t_idle = 0;   // since when nothing was ready
      while (s_live || gp < gs) {
        bool moved = try_pv();
        moved |= try_s();
        if (moved) {
          t_idle = 0;
          continue;
        }
        // nothing ready: sleep in the blocking test of the barrier the next P V needs (it
        // returns when the phase completes or after at most 20 us), or briefly when no P V
        // is pending, so that the polling takes no issue slots from the softmax warps of
        // this sub-partition; give up after 2 s without progress, or once another role
        // aborted
        if (gp < gs) mbar_try_wait_for(&p_full[gp % kTcSBufs], (gp / kTcSBufs) & 1, 20000u);
        else __nanosleep(200);
        const uint64_t now = global_timer_ns();
        if (t_idle == 0) t_idle = now;
        if (*abort) break;
        if (now - t_idle > 2000000000ull) {
          record_error(PA_DEV_WAIT_TIMEOUT, 30, int(gs), int(gp));
          *abort = 1;
          break;
        }
      }
    }
    __syncwarp();
  } else {
    // ---------------- softmax warps: rows of quarter rq, columns [64 h, 64 h + 64) of each tile ----------------
    const int rq = warp % kTcQuarters, h = warp / kTcQuarters, row = rq * 32 + lane;
    const int partner = warp ^ kTcQuarters;
    const uint32_t t_row = tmem + (uint32_t(rq * 32) << 16);
    uint32_t g = 0, xn = 0;
    // the partner's values for this lane's row, after both wrote theirs (exchange xn)
    auto exchange = [&](float2 v, float2& other) -> bool {
      xval[xn & 1][warp][lane] = v;
      __syncwarp();
      if (lane == 0) mbar_arrive(&xchg[rq]);
      if (!__all_sync(kFull, tc_spin(&xchg[rq], xn & 1, abort, 23, int(xn)))) return false;
      volatile float* o = reinterpret_cast<volatile float*>(&xval[xn & 1][partner][lane]);
      other = make_float2(o[0], o[1]);
      ++xn;
      return true;
    };
    // Unit kk's O (this warp's 64 columns), once the unit's last P V completed: the output
    // row (the row's whole context was in this unit) or the chunk's partial (unnormalised
    // row, then max and sum). The accumulator is released as soon as it is in registers.
    // Called after the next unit's first tile, so that the last P V runs meanwhile.
    auto epilogue = [&](const TcUnit& x, uint32_t kk, float l, float m_ref) -> bool {
      if (!tc_wait_warp(&o_full, kk & 1, abort, 22, int(kk))) return false;
      tc_fence_after();
      float2 other;
      if (!exchange(make_float2(l, 0.f), other)) return false;
      l += other.x;   // the row sum
      // a row whose context reaches into this unit's chunk writes now: its output row when
      // the chunk is the row's only one (position below the chunk length), else a partial
      const int qi = x.t * QPT + row / G, qpos = x.base + qi;
      const bool wr = qi < x.Q && qpos >= x.part * p.chunk, fin = wr && qpos < p.chunk;
      uint4* stage = reinterpret_cast<uint4*>(sm + TcSmem::kStage + warp * TcSmem::kStageWarp);
      const size_t slot = (size_t(x.row0 + qi) * Hq + x.hk * G + row % G) * p.max_parts + x.part;
      float4* acc = reinterpret_cast<float4*>(p.part_acc + slot * kTcD + h * kTcHalf);
      const float inv = fin ? 1.f / l : 0.f;
      // 32 columns at a time; the accumulator is released once both halves are in registers
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t r[32];
        tc_ld32_async(t_row + kTcOCol + h * kTcHalf + hh * 32, r);
        tc_wait_ld();
        if (hh == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&o_empty);
        }
        auto o = [&](int i) { return __uint_as_float(pin_after_wait(r[i])); };
        if (fin) {
          // the 16-bit row into this warp's staging rows (16-byte chunk c of row `lane` at
          // chunk c ^ (lane & 7), so that 8 consecutive lanes cover every bank) ...
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int cc = hh * 4 + i;
            stage[lane * 8 + (cc ^ (lane & 7))] = make_uint4(pack16x2<QD>(o(8 * i) * inv, o(8 * i + 1) * inv),
                                                             pack16x2<QD>(o(8 * i + 2) * inv, o(8 * i + 3) * inv),
                                                             pack16x2<QD>(o(8 * i + 4) * inv, o(8 * i + 5) * inv),
                                                             pack16x2<QD>(o(8 * i + 6) * inv, o(8 * i + 7) * inv));
          }
        } else if (wr) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            acc[hh * 8 + i] = make_float4(o(4 * i), o(4 * i + 1), o(4 * i + 2), o(4 * i + 3));
        }
      }
      if (wr && !fin && h == 0) {
        p.part_ml[slot * 2] = m_ref;
        p.part_ml[slot * 2 + 1] = l;
      }
      __syncwarp();
      // ... then out, 4 rows of 128 bytes per instruction: lane j writes chunk j % 8 of
      // staging row 4 i + j / 8
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int rr = 4 * i + (lane >> 3), c = lane & 7;
        const int row_r = rq * 32 + rr, qi_r = x.t * QPT + row_r / G;
        if (x.part == 0 && qi_r < x.Q && x.base + qi_r < p.chunk) {   // that row's output row was staged
          QT* out_r = static_cast<QT*>(p.out) + (size_t(x.row0 + qi_r) * Hq + x.hk * G + row_r % G) * kTcD +
                      h * kTcHalf;
          reinterpret_cast<uint4*>(out_r)[c] = stage[rr * 8 + (c ^ (rr & 7))];
        }
      }
      __syncwarp();
      return true;
    };
    TcUnit xprev;
    uint32_t kprev = 0;
    float lprev = 0.f, mprev = 0.f;
    bool pend = false, ok = true;   // pend: the previous unit's O is still to be read
    for (uint32_t k = 0; ok; ++k) {
      int u;
      if (!(ok = read_unit(k, u)) || u < 0) break;
      const TcUnit x = tc_unit(p, u);
      const int qi = x.t * QPT + row / G;
      const bool has_q = qi < x.Q;
      const int qpos = has_q ? x.base + qi : -1;
      float m_ref = -INFINITY, l = 0.f;   // l: this warp's columns' share of the row sum
      for (int j = 0; j < x.ntiles; ++j, ++g) {
        const int b = g % kTcSBufs;
        const uint32_t c_s = b * kTcTok + h * kTcHalf;   // this half of S(g), then of P(g)
        if (!(ok = tc_wait_warp(&s_full[b], (g / kTcSBufs) & 1, abort, 18, u))) break;
        tc_fence_after();
        // pass 1: the maximum of this half's causally masked scores (8 independent chains;
        // the mask costs work only in tiles where some row of the warp ends), then the
        // row's maximum from both halves (and the other half's running sum)
        const int vis = qpos - (x.t0 + j * kTcTok + h * kTcHalf);   // columns 0 .. vis of the half are visible
        const bool masked = !__all_sync(kFull, vis >= kTcHalf - 1);
        const float mh = masked ? tc_row_max<true>(t_row + c_s, vis) : tc_row_max<false>(t_row + c_s, vis);
        float2 other;
        if (!(ok = exchange(make_float2(mh, l), other))) break;
        const float mx = fmaxf(mh, other.x) * p.s_mul;
        const bool up = mx > m_ref + kTcRescale;
        const float corr = up ? ex2(m_ref - mx) : 1.f;   // 0 while nothing was accumulated
        float l_row = l + other.y;                       // the row's running sum
        if (up) {
          l *= corr;
          l_row *= corr;
          m_ref = mx;
        }
        if (j > 0 && __any_sync(kFull, up)) {
          // O holds every earlier P V of the unit once P(g-1) V(g-1) has completed; this
          // warp rescales its half of the row's O
          const uint32_t gr = g - 1;
          if (!(ok = tc_wait_warp(&pv_done[gr % kTcSBufs], (gr / kTcSBufs) & 1, abort, 19, u))) break;
          tc_fence_after();
#pragma unroll 1
          for (int i = 0; i < kTcHalf / 16; ++i) {   // 16 columns at a time (the scores stay live)
            uint32_t o[16];
            tc_ld16_async(t_row + kTcOCol + h * kTcHalf + i * 16, o);
            tc_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(pin_after_wait(o[e])) * corr);
            tc_st16(t_row + kTcOCol + h * kTcHalf + i * 16, o);
          }
          tc_wait_st();
        }
        const float nmb = m_ref == -INFINITY ? 0.f : -m_ref;
        // bf16: the remainder p - bf16(p) goes beside P. Adaptive: the MMA issuer multiplies it
        // only if some softmax warp flags the tile -- when a row has a weight above kLoShare
        // of its running sum, tested before the sum of this tile is known against the running
        // sum plus the tile's largest weight (a lower bound of the row's final sum, so the
        // test flags at least the tiles that need it); a warp that does not flag the tile
        // writes zeros there. A warp writes its flag before it signals P; the issuer reads all
        // flags once all have signalled.
        int rem_mode = kRemNone;   // bf16: the remainder of every tile, or (adaptive) of flagged rows
        if (QD == PA_BF16 && p.lo_mode == kLoAlways) rem_mode = kRemValue;
        if (QD == PA_BF16 && p.lo_mode == kLoAdaptive) {
          const float pmax = ex2(mx + nmb);   // the row's largest weight in this tile (0: none visible)
          const bool need = __any_sync(kFull, pmax > kLoShare * (l_row + pmax));
          if (lane == 0) reinterpret_cast<volatile char*>(lo_need[b])[warp] = need ? 1 : 0;
          rem_mode = need ? kRemValue : kRemZero;
        }
        // pass 2, 16 columns at a time: P = 2^(s * scale - ref) as 16-bit pairs over the
        // scores it was made from (tokens 16 t ..: P in columns [16 t, 16 t + 8), with the
        // remainder p - bf16(p), or zeros, in [16 t + 8, 16 t + 16))
        float2 l2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        auto pass2 = [&](auto mask_c) {
          constexpr bool kM = decltype(mask_c)::value;
          if constexpr (QD == PA_BF16) {
            if (rem_mode == kRemValue) tc_make_p<QD, kM, kRemValue>(t_row + c_s, vis, p.s_mul, nmb, l2);
            else if (rem_mode == kRemZero) tc_make_p<QD, kM, kRemZero>(t_row + c_s, vis, p.s_mul, nmb, l2);
            else tc_make_p<QD, kM, kRemNone>(t_row + c_s, vis, p.s_mul, nmb, l2);
          } else {
            tc_make_p<QD, kM, kRemNone>(t_row + c_s, vis, p.s_mul, nmb, l2);
          }
        };
        if (masked) pass2(std::true_type{});
        else pass2(std::false_type{});
        l += ((l2[0].x + l2[0].y) + (l2[1].x + l2[1].y)) + ((l2[2].x + l2[2].y) + (l2[3].x + l2[3].y));
        // V rows past the visible tokens (cache bytes beyond the context, or stale rows of
        // blocks not loaded) are zeroed by the first-half warps (one V row per thread), so
        // that 0-weighted rows cannot bring a NaN into O
        const int rem = x.nvis - j * kTcTok;
        if (h == 0 && rem < kTcTok) {
          if (!(ok = tc_wait_warp(&v_full[g & 1], (g >> 1) & 1, abort, 21, u))) break;
          if (row >= rem) {
            uint8_t* sV = sm + TcSmem::kV + (g & 1) * TcSmem::kKvTile;
#pragma unroll
            for (int i = 0; i < kTcD / 8; ++i) *reinterpret_cast<uint4*>(sV + tc_swz_kv(row, i)) = make_uint4(0, 0, 0, 0);
          }
          fence_async_smem();
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[b]);
        if (j == 0 && pend) {
          pend = false;
          if (!(ok = epilogue(xprev, kprev, lprev, mprev))) break;
        }
      }
      if (!ok) break;
      xprev = x;
      kprev = k;
      lprev = l;
      mprev = m_ref;
      pend = true;
    }
    if (ok && pend) epilogue(xprev, kprev, lprev, mprev);
  }

  __syncthreads();
  if (*abort) {   // drain what this CTA issued: MMAs (their thread), then the producers' last loads
    if (warp == kTcMmaWarp && lane == 0) {
      tc_commit(&bar_fin);
      mbar_wait_bounded(&bar_fin, 0);
    }
    if ((warp == kTcKWarp || warp == kTcVWarp) && lane == 0) {
      uint64_t* full = warp == kTcKWarp ? k_full : v_full;
      for (uint32_t i = kv_loads > 2 ? kv_loads - 2 : 0; i < kv_loads; ++i)
        mbar_wait_bounded(&full[i & 1], (i >> 1) & 1, 100000000ull);
      if (warp == kTcKWarp && q_loads > 0) mbar_wait_bounded(&q_full, (q_loads - 1) & 1, 100000000ull);
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
