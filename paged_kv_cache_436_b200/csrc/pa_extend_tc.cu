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
//   * one persistent CTA per SM with warp-specialised roles: 8 softmax warps (warps w and
//     w + 4 share TMEM lanes 32 (w % 4) .. + 31, i.e. rows of the tile, and split the 128
//     columns into slices of 64: more slices put more warps in lockstep on the same SM
//     sub-partition and measured slower), one MMA-issue warp, one K and one V producer warp;
//   * TMEM: S of two consecutive 128-token K/V tiles in columns [0, 256), the output
//     accumulators O of two consecutive units in [256, 512);
//   * the unit's Q rows come by one 3-D TMA box per 64-column half (64 dims x G heads x
//     128 / G queries: the rows in (query, head) order) into a 128B-swizzled K-major
//     tile, loaded as soon as the previous unit's last S has completed; K and V tiles
//     come by 2-D TMA (cp.async.bulk.tensor, 128B swizzle, no multicast) straight from
//     the paged cache, one box per (cache block, 64-column half), into 2-deep K and V
//     rings;
//   * S = Q K^T (both K-major) and O += P V (P K-major; V MN-major, i.e. left in its
//     [token][dim] cache layout) are issued by one thread; order S(g), P(g-1) V(g-1),
//     S(g+1), ... so that the next S runs while the softmax works on the current one;
//   * the softmax reads its half of the S row from TMEM, masks causally and keeps a
//     reference maximum that moves only when the row maximum passes it by more than 2^8
//     (O and the running sum are then rescaled; every p stays below 2^8, so nothing is
//     lost). The group's maximum is combined through TMEM columns and a kTcSplit-arrival
//     mbarrier; P is computed speculatively with the current reference meanwhile and
//     recomputed only when the reference moves. P goes to a swizzled K-major shared
//     tile in the query's 16-bit type; the running sum adds the binary32 values;
//   * a unit that covers a row's whole context writes the output row; otherwise it
//     writes (max, sum, unnormalised row) for the log-sum-exp merge kernel.
// Every wait is bounded; on a timeout the kernel records it, every role stops, the MMA
// and load issuers drain what they issued, and the TMEM is freed.
namespace pa {

constexpr int kTcRows = 128;            // query rows per unit (TMEM lanes)
constexpr int kTcTok = 128;             // tokens per K/V tile
constexpr int kTcD = 128;               // head_dim of this path
constexpr uint32_t kTcTmemCols = 512;   // S double buffer [0, 256), O double buffer [256, 512)
constexpr int kTcSplit = 2;             // softmax warps per 32-row group (column slices)
constexpr int kTcSoftmaxWarps = 4 * kTcSplit;   // + an MMA-issue warp + K and V producer warps
constexpr int kTcThreads = (kTcSoftmaxWarps + 3) * 32;
constexpr float kTcRescale = 8.f;       // log2 units

struct TcSmem {
  static constexpr int kTile = kTcRows * kTcD * 2;   // 32 KB: two 64-column halves of 16 KB
  static constexpr int kQ = 0;
  static constexpr int kP = kQ + kTile;              // P buffers 0, 1
  static constexpr int kK = kP + 2 * kTile;          // K buffers 0, 1
  static constexpr int kV = kK + 2 * kTile;          // V buffers 0, 1
  static constexpr int kBytes = kV + 2 * kTile + 1024;   // 225 KB with the alignment slack
};
static_assert(kTcRows == kTcTok, "Q, P, K and V tiles share one swizzled layout");

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

// Two values rounded to the 16-bit type and packed (lo in the low half); `sum` adds the
// rounded values.
template <int QD>
__device__ __forceinline__ uint32_t pack2_sum(float lo, float hi, float& sum) {
  if constexpr (QD == PA_BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    const uint32_t w = *reinterpret_cast<const uint32_t*>(&v);
    sum += __uint_as_float(w << 16) + __uint_as_float(w & 0xffff0000u);
    return w;
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    const float2 f = __half22float2(v);
    sum += f.x + f.y;
    return *reinterpret_cast<const uint32_t*>(&v);
  }
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

// One 32-bit column of this warp's 32 lanes (warp-collective), with its wait.
__device__ __forceinline__ void tc_st1(uint32_t addr, uint32_t v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(addr), "r"(v) : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t tc_ld1(uint32_t addr) {
  uint32_t v;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(v) : "r"(addr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  return pin_after_wait(v);
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

// p = 2^a for a pair, rounded to the 16-bit type and packed (lo in the low half); the
// binary32 values are added to `sum` as a pair (the weights in P differ from them by at
// most one 16-bit rounding each).
template <int QD>
__device__ __forceinline__ uint32_t exp2_pack(float2 a, float2& sum) {
  const float p0 = ex2(a.x), p1 = ex2(a.y);
  uint32_t w;
  if constexpr (QD == PA_BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(p0, p1);
    w = *reinterpret_cast<const uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(p0, p1);
    w = *reinterpret_cast<const uint32_t*>(&v);
  }
  sum = add2(sum, make_float2(p0, p1));
  return w;
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
  uint8_t* sQ = sm + TcSmem::kQ;
  // per-tile ring barriers (index = tile & 1); per-unit ones (q_full, o_full/o_empty by unit & 1)
  __shared__ uint64_t k_full[2], v_full[2], k_empty[2], pv_done[2], s_full[2], s_empty[2], p_full[2];
  __shared__ uint64_t q_full, q_empty, o_full[2], o_empty[2], bar_fin, grp_bar[4];
  __shared__ int uq[4];                        // unit ring: unit k of this CTA in slot k % 4
  __shared__ uint64_t uq_full[4], uq_empty[4];
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
    for (int b = 0; b < 2; ++b) {
      mbar_init(&k_full[b], 1);
      mbar_init(&v_full[b], 1);
      mbar_init(&k_empty[b], 1);
      mbar_init(&pv_done[b], 1);
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], kTcSoftmaxWarps);
      mbar_init(&p_full[b], kTcSoftmaxWarps);
      mbar_init(&o_full[b], 1);
      mbar_init(&o_empty[b], kTcSoftmaxWarps);
    }
    mbar_init(&q_full, 1);
    mbar_init(&q_empty, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&uq_full[i], 1);
      mbar_init(&uq_empty[i], kTcSoftmaxWarps + 2);   // V producer, MMA warp, softmax warps
    }
    for (int i = 0; i < 4; ++i) mbar_init(&grp_bar[i], kTcSplit);
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
  uint32_t last_load = 0;           // producer: tiles issued (for the drain after an abort)
  uint32_t q_loads = 0;             // V producer: Q tiles issued (likewise)
  // Dynamic scheduling: the K producer takes unit k of this CTA from the global queue (the
  // plan kernel lists each sequence's longest row tile first) and publishes it in the
  // ring; every other role reads the same sequence. -1 ends the work. False on an abort.
  auto next_unit = [&](uint32_t k, bool taker, int& u) -> bool {
    const int slot = k & 3;
    const uint32_t ph = (k >> 2) & 1;
    if (taker) {
      if (!tc_wait_warp(&uq_empty[slot], ph ^ 1, abort, 28, int(k))) return false;
      int v = 0;
      if (lane == 0) {
        v = atomicAdd(p.queue, 1);
        if (v >= total) v = -1;
        uq[slot] = v;
        mbar_arrive(&uq_full[slot]);
      }
      u = __shfl_sync(kFull, v, 0);
      return true;
    }
    if (!tc_wait_warp(&uq_full[slot], ph, abort, 29, int(k))) return false;
    u = *reinterpret_cast<volatile int*>(&uq[slot]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&uq_empty[slot]);
    return true;
  };

  if (warp > kTcSoftmaxWarps) {
    // ---------------- producers: warp kTcSoftmaxWarps + 1 streams K, the next one V, by 2-D
    // TMA, lane i loading cache block i of a tile; separate warps, so that a K tile never
    // waits behind the V tile before it (which waits for an older P V) ----------------
    const bool is_v = warp == kTcSoftmaxWarps + 2;
    uint64_t* full = is_v ? v_full : k_full;
    uint64_t* empty = is_v ? pv_done : k_empty;   // V(g) after P(g-2) V(g-2); K(g) after S(g-2)
    const CUtensorMap* map = is_v ? &tv : &tk;
    uint8_t* ring = sm + (is_v ? TcSmem::kV : TcSmem::kK);
    const CUtensorMap* in_map = is_v ? &tvn : &tkn;   // whole prompts: the prompt's K or V rows
    int pend_g = -1, pend_nbw = 0, pend_y = 0;        // a loaded tile still to be written to the cache
    auto flush_store = [&]() {
      if (pend_g < 0) return true;
      const int b = pend_g & 1;
      if (!tc_wait_warp(&full[b], (uint32_t(pend_g) >> 1) & 1, abort, 27, pend_g)) return false;
      if (lane < pend_nbw) {
        const uint8_t* src = ring + b * TcSmem::kTile + lane * (BS * 128);
        tma_store_2d(map, 0, pend_y, src);
        tma_store_2d(map, 64, pend_y, src + kTcTok * 128);
        bulk_commit();
      }
      pend_g = -1;
      return true;
    };
    uint32_t g = 0;
    for (uint32_t k = 0;; ++k) {
      int u;
      if (!next_unit(k, !is_v, u) || u < 0) break;
      const TcUnit x = tc_unit(p, u);
      if (is_v) {   // the unit's q rows: box {64 dims, G heads, QPT queries} per 64-dim half
        if (k > 0 && !tc_wait_warp(&q_empty, (k - 1) & 1, abort, 26, u)) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&q_full, TcSmem::kTile);
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
            if (!is_v) record_error(PA_DEV_BAD_BLOCK_ID, x.s, lb + lane, id);
            id = 0;
          }
        }
        return id;
      };
      if (p.fresh) {
        // whole prompts: tiles come from the prompt's own K / V rows, 128 rows per box;
        // the row tile that sees all of a K/V tile's prompt positions also writes that
        // tile into its cache blocks (TMA stores, once its load has landed)
        bool ok = true;
        for (int j = 0; j < x.ntiles; ++j, ++g) {
          const int b = g & 1, p0 = x.t0 + j * kTcTok;
          if (!(ok = tc_wait_warp(&empty[b], ((g >> 1) & 1) ^ 1, abort, is_v ? 11 : 10, u))) break;
          bulk_wait_read_all();   // the stores that read this buffer two tiles ago
          if (lane == 0) {
            mbar_arrive_expect_tx(&full[b], TcSmem::kTile);
            tma_load_3d(ring + b * TcSmem::kTile, in_map, 0, x.hk, x.row0 + p0, &full[b]);
            tma_load_3d(ring + b * TcSmem::kTile + kTcTok * 128, in_map, 64, x.hk, x.row0 + p0, &full[b]);
          }
          __syncwarp();
          last_load = g + 1;
          if (!(ok = flush_store())) break;
          if (x.t == min((p0 + kTcTok - 1) / QPT, (x.Q - 1) / QPT)) {
            pend_nbw = (min(p0 + kTcTok, x.Q) - p0 + BS - 1) / BS;
            pend_y = (fetch(p0 / BS, pend_nbw) * Hkv + x.hk) * BS;
            pend_g = int(g);
          }
        }
        if (!ok) break;
        continue;
      }
      int id = fetch(x.t0 / BS, blocks(0));
      for (int j = 0; j < x.ntiles; ++j, ++g) {
        const int b = g & 1, nb = blocks(j);
        const int next = j + 1 < x.ntiles ? fetch((x.t0 + (j + 1) * kTcTok) / BS, blocks(j + 1)) : 0;
        const int y = (id * Hkv + x.hk) * BS;
        uint8_t* dst = ring + b * TcSmem::kTile + lane * (BS * 128);
        if (!tc_wait_warp(&empty[b], ((g >> 1) & 1) ^ 1, abort, is_v ? 11 : 10, u)) break;
        if (lane == 0) mbar_arrive_expect_tx(&full[b], uint32_t(nb) * kBlockTx);
        __syncwarp();
        if (lane < nb) {
          tma_load_2d(dst, map, 0, y, &full[b]);
          tma_load_2d(dst + kTcTok * 128, map, 64, y, &full[b]);
        }
        last_load = g + 1;
        id = next;
      }
    }
    if (p.fresh && !*abort) flush_store();
    bulk_wait_all();   // this thread's cache stores are complete before the kernel ends
  } else if (warp == kTcSoftmaxWarps) {
    // ---------------- MMA issue: S(g) then O += P(g-1) V(g-1) ----------------
    const uint32_t idS = tc_idesc<QD>(0), idO = tc_idesc<QD>(1);
    uint32_t g = 0, k = 0;
    auto pv = [&](uint32_t h, bool first, uint32_t ob, int u) {
      const int b = h & 1;
      if (!tc_wait_warp(&p_full[b], (h >> 1) & 1, abort, 12, u)) return false;
      if (!tc_wait_warp(&v_full[b], (h >> 1) & 1, abort, 13, u)) return false;
      if (lane == 0) {
        tc_fence_after();
        const uint32_t pa_ = smem_addr(sm + TcSmem::kP + b * TcSmem::kTile);
        const uint32_t va = smem_addr(sm + TcSmem::kV + b * TcSmem::kTile);
#pragma unroll
        for (int kk = 0; kk < kTcTok / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * (kTcRows * 128) + (kk & 3) * 32;
          tc_mma(tmem + 256 + ob * 128, tc_desc(pa_ + aoff, 1024, 16), tc_desc(va + kk * 2048, 1024, kTcTok * 128),
                 idO, (first && kk == 0) ? 0u : 1u);
        }
        tc_commit(&pv_done[b]);
      }
      __syncwarp();
      return true;
    };
    for (;; ++k) {
      int u;
      if (!next_unit(k, false, u) || u < 0) break;
      const TcUnit x = tc_unit(p, u);
      const uint32_t ob = k & 1;
      if (!tc_wait_warp(&q_full, k & 1, abort, 14, u)) break;
      if (!tc_wait_warp(&o_empty[ob], ((k >> 1) & 1) ^ 1, abort, 15, u)) break;
      bool ok = true;
      for (int j = 0; j < x.ntiles && ok; ++j, ++g) {
        const int b = g & 1;
        ok = tc_wait_warp(&k_full[b], (g >> 1) & 1, abort, 16, u) &&
             tc_wait_warp(&s_empty[b], ((g >> 1) & 1) ^ 1, abort, 17, u);
        if (!ok) break;
        if (lane == 0) {
          tc_fence_after();
          const uint32_t qa = smem_addr(sQ), ka = smem_addr(sm + TcSmem::kK + b * TcSmem::kTile);
#pragma unroll
          for (int kk = 0; kk < kTcD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * (kTcRows * 128) + (kk & 3) * 32;
            tc_mma(tmem + b * 128, tc_desc(qa + off, 1024, 16), tc_desc(ka + off, 1024, 16), idS, kk > 0);
          }
          tc_commit(&s_full[b]);
          tc_commit(&k_empty[b]);
          if (j + 1 == x.ntiles) tc_commit(&q_empty);   // sQ is free once this S completes
        }
        __syncwarp();
        if (j > 0) ok = pv(g - 1, j == 1, ob, u);
      }
      if (!ok || !pv(g - 1, x.ntiles == 1, ob, u)) break;
      if (lane == 0) tc_commit(&o_full[ob]);
      __syncwarp();
    }
  } else {
    // ---------------- softmax warps ----------------
    // Warps w, w + 4, w + 8, ... share TMEM lanes 32 (w % 4) .. + 31 (rows of the tile) and
    // split the columns: slice q = w / 4 holds score / P / O columns [kCW q, kCW q + kCW).
    // The group combines its row maxima and sums through one TMEM column each has already
    // read (its own first column of the S or O buffer) and a kTcSplit-arrival mbarrier.
    constexpr int kCW = kTcTok / kTcSplit;             // columns per warp
    const int qs_ = warp >> 2, rw = warp & 3, row = rw * 32 + lane;
    const uint32_t t_row = tmem + (uint32_t(rw * 32) << 16);
    uint32_t xc = 0;   // group exchanges so far
    auto publish = [&](uint32_t col_own, float v) {
      tc_st1(t_row + col_own, __float_as_uint(v));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&grp_bar[rw]);
    };
    // all slices' values in slice order (identical in every warp of the group)
    auto gather = [&](uint32_t col0, float own, int u, float* all) {
      const bool ok = tc_wait_warp(&grp_bar[rw], xc & 1, abort, 23, u);
      ++xc;
      if (!ok) return false;
      tc_fence_after();
#pragma unroll
      for (int q = 0; q < kTcSplit; ++q)
        all[q] = q == qs_ ? own : __uint_as_float(tc_ld1(t_row + col0 + q * kCW));
      return true;
    };
    uint32_t g = 0, k = 0;
    for (;; ++k) {
      int u;
      if (!next_unit(k, false, u) || u < 0) break;
      const TcUnit x = tc_unit(p, u);
      const uint32_t ob = k & 1, c_o = 256 + ob * 128 + qs_ * kCW;   // this slice of the O buffer
      const int qi = x.t * QPT + row / G;
      const int head = x.hk * G + row % G;
      const bool has_q = qi < x.Q;
      const int qpos = has_q ? x.base + qi : -1;
      const int tok = has_q ? x.row0 + qi : -1;
      float m_ref = -INFINITY, l = 0.f;   // l: this slice's share of the row sum
      bool ok = true;
      for (int j = 0; j < x.ntiles; ++j, ++g) {
        const int b = g & 1;
        const uint32_t c_s = b * 128 + qs_ * kCW;                    // this slice of S(g)
        if (!(ok = tc_wait_warp(&s_full[b], (g >> 1) & 1, abort, 18, u))) break;
        tc_fence_after();
        float s[kCW];
        {
          uint32_t r[kCW];
#pragma unroll
          for (int c = 0; c < kCW / 32; ++c) tc_ld32_async(t_row + c_s + c * 32, r + c * 32);
          tc_wait_ld();
#pragma unroll
          for (int c = 0; c < kCW; ++c) s[c] = __uint_as_float(pin_after_wait(r[c]));
        }
        // causal mask, this slice's maximum (8 independent chains)
        const int tp0 = x.t0 + j * kTcTok + qs_ * kCW;
        if (tp0 + kCW - 1 > qpos) {
#pragma unroll
          for (int c = 0; c < kCW; ++c) s[c] = tp0 + c > qpos ? -INFINITY : s[c];
        }
        float m8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) m8[e] = s[e];
#pragma unroll
        for (int c = 8; c + 8 < kCW; c += 16)
#pragma unroll
          for (int e = 0; e < 8; ++e) m8[e] = fmax3(m8[e], s[c + e], s[c + 8 + e]);
        if constexpr ((kCW - 8) % 16 != 0) {
#pragma unroll
          for (int e = 0; e < 8; ++e) m8[e] = fmaxf(m8[e], s[kCW - 8 + e]);
        }
        const float pm = fmaxf(fmax3(m8[0], m8[1], m8[2]), fmax3(fmax3(m8[3], m8[4], m8[5]), m8[6], m8[7]));
        publish(c_s, pm);
        // P(g) goes into buffer b once P(g-2) V(g-2) has finished reading it
        if (!(ok = tc_wait_warp(&pv_done[b], ((g >> 1) & 1) ^ 1, abort, 20, u))) break;
        uint8_t* sP = sm + TcSmem::kP + b * TcSmem::kTile;
        auto make_p = [&](float ref) {   // P = 2^(s * scale - ref) into sP; returns its rounded sum
          const float nmb = -ref;
          float2 l2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
          for (int c = 0; c < kCW / 8; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w[e] = exp2_pack<QD>(fma2(make_float2(s[c * 8 + 2 * e], s[c * 8 + 2 * e + 1]), p.s_mul, nmb), l2[e]);
            *reinterpret_cast<uint4*>(sP + tc_swz(row, qs_ * (kCW / 8) + c)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
          return ((l2[0].x + l2[0].y) + (l2[1].x + l2[1].y)) + ((l2[2].x + l2[2].y) + (l2[3].x + l2[3].y));
        };
        // speculatively with the current reference while the others' maxima are in flight:
        // it stands unless the row maximum passes the reference by more than 2^8
        const bool spec = m_ref != -INFINITY && pm * p.s_mul <= m_ref + kTcRescale;
        float lt = spec ? make_p(m_ref) : 0.f;
        float pms[kTcSplit];
        if (!(ok = gather(b * 128, pm, u, pms))) break;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[b]);
        float rmax = pms[0];
#pragma unroll
        for (int q = 1; q < kTcSplit; ++q) rmax = fmaxf(rmax, pms[q]);
        const float mx = rmax * p.s_mul;
        const bool up = mx > m_ref + kTcRescale;
        const float corr = up ? ex2(m_ref - mx) : 1.f;   // 0 while nothing was accumulated
        if (up) {
          l *= corr;
          m_ref = mx;
        }
        if (j > 0 && __any_sync(kFull, up)) {
          // O must hold P(g-1) V(g-1) before it is rescaled
          if (!(ok = tc_wait_warp(&pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, abort, 19, u))) break;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < kCW / 32; ++c) {
            float o[32];
            tc_ld32(t_row + c_o + c * 32, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= corr;
            tc_st32(t_row + c_o + c * 32, o);
          }
        }
        if (!spec || up) lt = make_p(m_ref == -INFINITY ? 0.f : m_ref);
        l += lt;
        // V rows past the visible tokens (cache bytes beyond the context, or stale rows
        // of blocks not loaded) are zeroed, this slice of each, so that 0-weighted rows
        // cannot bring a NaN into O
        const int rem = x.nvis - j * kTcTok;
        if (rem < kTcTok) {
          if (!(ok = tc_wait_warp(&v_full[b], (g >> 1) & 1, abort, 21, u))) break;
          if (row >= rem) {
            uint8_t* vt = sm + TcSmem::kV + b * TcSmem::kTile;
#pragma unroll
            for (int c = 0; c < kCW / 8; ++c)
              *reinterpret_cast<uint4*>(vt + tc_swz(row, qs_ * (kCW / 8) + c)) = make_uint4(0, 0, 0, 0);
          }
        }
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[b]);
      }
      if (!ok) break;
      // this unit's O
      if (!tc_wait_warp(&o_full[ob], (k >> 1) & 1, abort, 22, u)) break;
      tc_fence_after();
      float o[kCW];
      {
        uint32_t r[kCW];
#pragma unroll
        for (int c = 0; c < kCW / 32; ++c) tc_ld32_async(t_row + c_o + c * 32, r + c * 32);
        tc_wait_ld();
#pragma unroll
        for (int c = 0; c < kCW; ++c) o[c] = __uint_as_float(pin_after_wait(r[c]));
      }
      publish(c_o, l);
      float ls[kTcSplit];
      if (!gather(256 + ob * 128, l, u, ls)) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_empty[ob]);
      float lsum = ls[0];   // slice order: the same sum in every warp of the group
#pragma unroll
      for (int q = 1; q < kTcSplit; ++q) lsum += ls[q];
      const int P = has_q ? (qpos + 1 + p.chunk - 1) / p.chunk : 0;
      const bool wr = has_q && x.part < P;
      const bool fin = wr && P == 1;
      if (fin) {   // this slice of the row, rounded, staged in P buffer 0 (every P V has completed)
        const float inv = 1.f / lsum;
#pragma unroll
        for (int i = 0; i < kCW / 8; ++i) {
          float dummy = 0.f;
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) w[e] = pack2_sum<QD>(o[i * 8 + 2 * e] * inv, o[i * 8 + 2 * e + 1] * inv, dummy);
          *reinterpret_cast<uint4*>(sm + TcSmem::kP + tc_swz(row, qs_ * (kCW / 8) + i)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      __syncwarp();
      {   // coalesced: each store instruction writes (32 / kLPR) rows x kCW * 2 contiguous bytes
        constexpr int kLPR = kCW / 8;               // lanes per row (16 bytes each)
        constexpr int kRPI = 32 / kLPR;             // rows per instruction
#pragma unroll
        for (int i = 0; i < 32 / kRPI; ++i) {
          const int rr = rw * 32 + i * kRPI + lane / kLPR, c = lane % kLPR;
          const int rqi = x.t * QPT + rr / G;
          if (x.part == 0 && rqi < x.Q && x.base + rqi + 1 <= p.chunk) {   // that row's whole context is here
            QT* orow =
                static_cast<QT*>(p.out) + (size_t(x.row0 + rqi) * Hq + x.hk * G + rr % G) * kTcD + qs_ * kCW;
            *reinterpret_cast<uint4*>(orow + c * 8) =
                *reinterpret_cast<const uint4*>(sm + TcSmem::kP + tc_swz(rr, qs_ * kLPR + c));
          }
        }
      }
      __syncwarp();
      if (wr && !fin) {   // this chunk's partial: unnormalised row slice, (max, sum) once
        const size_t slot = (size_t(tok) * Hq + head) * p.max_parts + x.part;
        float4* acc = reinterpret_cast<float4*>(p.part_acc + slot * kTcD + qs_ * kCW);
#pragma unroll
        for (int i = 0; i < kCW / 4; ++i) acc[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        if (qs_ == 0) {
          p.part_ml[slot * 2] = m_ref;
          p.part_ml[slot * 2 + 1] = lsum;
        }
      }
    }
  }

  __syncthreads();
  if (*abort) {   // drain what this CTA issued: MMAs (their thread), then loads (their warp)
    if (warp == kTcSoftmaxWarps && lane == 0) {
      tc_commit(&bar_fin);
      mbar_wait_bounded(&bar_fin, 0);
    }
    if (warp > kTcSoftmaxWarps && lane == 0) {
      uint64_t* full = warp == kTcSoftmaxWarps + 2 ? v_full : k_full;
      for (uint32_t h = last_load >= 2 ? last_load - 2 : 0; h < last_load; ++h)
        mbar_wait_bounded(&full[h & 1], (h >> 1) & 1, 100000000ull);
      if (q_loads > 0) mbar_wait_bounded(&q_full, (q_loads - 1) & 1, 100000000ull);   // V producer only
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
