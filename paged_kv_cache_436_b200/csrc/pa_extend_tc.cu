// Long query runs (prefill, chunked prefill) on the 5th-generation tensor cores.
//
// Same computation as the mma.sync kernels of pa_extend.cu (query i of sequence s at
// position L_s - Q_s + i attends causally to the paged context; page 2, sections
// "2.1 核心组件交互流程" and "2.2 关键数据结构剖析"), with 128-row tiles on tcgen05:
//   * a work unit is (sequence, kv head, tile of 128 rows, chunk of the context); a row
//     is a (query, q head of the kv head's group) pair; the chunk is a multiple of the
//     512-token partition, chosen by the host so that there are enough units to fill
//     the GPU (the whole context when there are, then no merge pass at all);
//   * one CTA of 4 warps per unit (persistent); TMEM lane r holds row r and thread r
//     owns it; TMEM columns [0, 128) hold S of the current 128-token K/V tile,
//     [128, 256) the output accumulator O;
//   * Q rows are stored by their threads into a 128B-swizzled K-major shared tile;
//     K and V tiles come by 2-D TMA (cp.async.bulk.tensor, 128B swizzle, no
//     multicast) straight from the paged cache, one box per (cache block, 64-column
//     half); two K/V buffers, so tile j + 1 loads while tile j is in use;
//   * thread 0 issues S = Q K^T (both K-major) and O += P V (P K-major; V MN-major,
//     i.e. left in its [token][dim] cache layout) and commits each to an mbarrier;
//   * the softmax reads its S row from TMEM, masks causally and keeps a reference
//     maximum that moves only when the row maximum passes it by more than 2^8 (O and
//     the running sum are then rescaled; every p stays below 2^8, so nothing is lost);
//     P goes to a swizzled K-major shared tile in the query's 16-bit type and the
//     running sum adds those same rounded values;
//   * a unit that covers a row's whole context writes the output row; otherwise it
//     writes (max, sum, unnormalised row) for the log-sum-exp merge kernel.
// Every wait is bounded; on a timeout the kernel records it, drains what it issued,
// frees its TMEM and returns.
#include <cuda.h>

#include <mutex>

namespace pa {

constexpr int kTcRows = 128;            // query rows per unit (TMEM lanes)
constexpr int kTcTok = 128;             // tokens per K/V tile
constexpr int kTcD = 128;               // head_dim of this path
constexpr uint32_t kTcTmemCols = 256;   // S and O
constexpr float kTcRescale = 8.f;       // log2 units

struct TcSmem {
  static constexpr int kTile = kTcRows * kTcD * 2;   // 32 KB: two 64-column halves of 16 KB
  static constexpr int kQ = 0;
  static constexpr int kP = kQ + kTile;
  static constexpr int kK = kP + kTile;              // K buffers 0, 1
  static constexpr int kV = kK + 2 * kTile;          // V buffers 0, 1
  static constexpr int kBytes = kV + 2 * kTile + 1024;   // + alignment slack
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

// 2^x on the special-function unit (flushes subnormal results to zero).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2-D tiled TMA load (box given by the tensor map) signalling `bar` with its bytes.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

// Byte offset of 16-byte chunk c (0..15) of row r in a [128 x 128] 16-bit tile kept
// as two 128B-swizzled K-major halves of 64 columns (8-row atoms of 1 KB).
__device__ __forceinline__ uint32_t tc_swz(int r, int c) {
  return uint32_t((c >> 3) * (kTcRows * 128) + (r >> 3) * 1024 + (r & 7) * 128 + (((c & 7) ^ (r & 7)) << 4));
}

template <int QD, int BS, int G>
__global__ void __launch_bounds__(128, 1)
    extend_tc_kernel(const ExtendParams p, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv) {
  using QT = typename Q<QD>::T;
  constexpr int QPT = kTcRows / G;             // queries per unit
  constexpr int BPT = kTcTok / BS;             // cache blocks per K/V tile
  constexpr uint32_t kBlockTx = 2u * BS * kTcD * 2;   // K and V bytes of one cache block
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = sm + TcSmem::kQ;
  uint8_t* sP = sm + TcSmem::kP;
  __shared__ uint64_t bar_kv[2], bar_s, bar_o, bar_fin;
  __shared__ uint32_t tmem_slot;
  __shared__ int s_fail;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&tmem_slot)),
                 "r"(kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    mbar_init(&bar_kv[0], 1);
    mbar_init(&bar_kv[1], 1);
    mbar_init(&bar_s, 1);
    mbar_init(&bar_o, 1);
    mbar_init(&bar_fin, 1);
    s_fail = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dependency_launch_dependents();
  grid_dependency_wait();

  const uint32_t tmem = tmem_slot;
  const uint32_t t_row = tmem + (uint32_t(warp * 32) << 16);   // this warp's 32 lanes, column 0
  const int Hq = p.num_q_heads, Hkv = p.num_kv_heads;
  const int total = p.plan[p.num_seqs] * Hkv;
  const uint32_t idS = tc_idesc<QD>(0), idO = tc_idesc<QD>(1);
  uint32_t it = 0;                          // K/V tiles this CTA has used (buffer it & 1)
  uint32_t pending = 0, par[2] = {0, 0};    // thread 0: loads issued and not yet waited for

  for (int u = blockIdx.x; u < total; u += gridDim.x) {
    const ExtUnit x = ext_make_unit<16>(p, u, total, QPT, 64);   // geometry only (no block ids)
    const int qi = x.t * QPT + tid / G;
    const int head = x.hk * G + tid % G;
    const bool has_q = qi < x.Q;
    const int qpos = has_q ? x.base + qi : -1;
    const int tok = has_q ? x.row0 + qi : -1;
    const int last = x.base + min((x.t + 1) * QPT, x.Q) - 1;   // last position the unit's rows see
    const int t0 = x.part * p.chunk;
    const int nvis = min(p.chunk, last + 1 - t0);                // visible tokens of the chunk (>= 1)
    const int ntiles = (nvis + kTcTok - 1) / kTcTok;

    {   // this thread's Q row -> swizzled K-major tile (zero for rows without a query)
      const uint4* qrow =
          reinterpret_cast<const uint4*>(static_cast<const QT*>(p.q) + (size_t(has_q ? tok : 0) * Hq + head) * kTcD);
#pragma unroll
      for (int c = 0; c < 16; ++c)
        *reinterpret_cast<uint4*>(sQ + tc_swz(tid, c)) = has_q ? qrow[c] : make_uint4(0, 0, 0, 0);
    }
    fence_async_smem();
    __syncthreads();

    // K/V tile j of the unit into buffer g & 1, issued by warp 0: lane i loads cache
    // block i of the tile (only the blocks with visible tokens). The block ids are read
    // one tile ahead so that their latency hides behind the current tile's S = Q K^T.
    const int32_t* trow = p.block_tables + size_t(x.s) * p.max_blocks;
    auto tile_blocks = [&](int j) { return min(BPT, (nvis - j * kTcTok + BS - 1) / BS); };
    auto fetch_id = [&](int j) {
      const int lb = (t0 + j * kTcTok) / BS + lane;
      int id = 0;
      if (lane < tile_blocks(j)) {
        id = trow[lb];
        if (id < 0 || id >= p.num_blocks) {
          record_error(PA_DEV_BAD_BLOCK_ID, x.s, lb, id);
          id = 0;
        }
      }
      return id;
    };
    auto issue_tile = [&](int j, uint32_t g, int id) {
      const int b = g & 1;
      const int nb = tile_blocks(j);
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar_kv[b], uint32_t(nb) * kBlockTx);
        pending |= 1u << b;
        par[b] = (g >> 1) & 1;
      }
      __syncwarp();
      if (lane < nb) {
        uint8_t* dk = sm + TcSmem::kK + b * TcSmem::kTile + lane * (BS * 128);
        uint8_t* dv = sm + TcSmem::kV + b * TcSmem::kTile + lane * (BS * 128);
        const int y = (id * Hkv + x.hk) * BS;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          tma_load_2d(dk + h * (kTcTok * 128), &tk, h * 64, y, &bar_kv[b]);
          tma_load_2d(dv + h * (kTcTok * 128), &tv, h * 64, y, &bar_kv[b]);
        }
      }
    };
    if (warp == 0) issue_tile(0, it, fetch_id(0));

    float m_ref = -INFINITY, l = 0.f;
    for (int j = 0; j < ntiles; ++j, ++it) {
      const int b = it & 1;
      int next_id = 0;
      if (warp == 0 && j + 1 < ntiles) next_id = fetch_id(j + 1);
      if (tid == 0) {   // S = Q K^T into columns [0, 128)
        if (!mbar_wait_bounded(&bar_kv[b], (it >> 1) & 1)) {
          record_error(PA_DEV_WAIT_TIMEOUT, 5, u, j);
          s_fail = 1;
        } else {
          pending &= ~(1u << b);
          tc_fence_after();
          const uint32_t qa = smem_addr(sQ), ka = smem_addr(sm + TcSmem::kK + b * TcSmem::kTile);
#pragma unroll
          for (int kk = 0; kk < kTcD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * (kTcRows * 128) + (kk & 3) * 32;
            tc_mma(tmem, tc_desc(qa + off, 1024, 16), tc_desc(ka + off, 1024, 16), idS, kk > 0);
          }
          tc_commit(&bar_s);
        }
      }
      __syncthreads();
      if (s_fail) break;
      // S is in TMEM; the previous tile's P V is done too (P, O and that K/V buffer are free)
      bool ok = mbar_wait_bounded(&bar_s, it & 1);
      if (it > 0) ok = ok && mbar_wait_bounded(&bar_o, (it - 1) & 1);
      if (!__all_sync(kFull, ok) && (tid & 31) == 0) {
        record_error(PA_DEV_WAIT_TIMEOUT, 6, u, j);
        s_fail = 1;
      }
      __syncthreads();
      if (s_fail) break;
      tc_fence_after();
      if (warp == 0 && j + 1 < ntiles) issue_tile(j + 1, it + 1, next_id);

      // V rows past the visible tokens (cache bytes beyond the context, or stale rows of
      // blocks not loaded) are zeroed so that 0-weighted rows cannot carry a NaN into O
      const int rem = nvis - j * kTcTok;
      if (tid >= rem) {
        uint8_t* vrow = sm + TcSmem::kV + b * TcSmem::kTile + (tid >> 3) * 1024 + (tid & 7) * 128;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(vrow + h * (kTcTok * 128) + c * 16) = make_uint4(0, 0, 0, 0);
      }

      // softmax of this thread's row (base 2; scale * log2(e) applied here)
      float s[kTcTok];
#pragma unroll
      for (int c = 0; c < kTcTok / 32; ++c) tc_ld32(t_row + c * 32, s + c * 32);
      const int tp0 = t0 + j * kTcTok;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kTcTok; ++c) {
        const float v = tp0 + c > qpos ? -INFINITY : s[c] * p.s_mul;
        s[c] = v;
        mx = fmaxf(mx, v);
      }
      const bool up = mx > m_ref + kTcRescale;
      const float corr = up ? ex2(m_ref - mx) : 1.f;   // 0 while nothing was accumulated
      if (up) {
        l *= corr;
        m_ref = mx;
      }
      if (j > 0 && __any_sync(kFull, up)) {   // rescale the O rows of this warp that moved
#pragma unroll 1
        for (int c = 0; c < kTcD / 32; ++c) {
          float o[32];
          tc_ld32(t_row + 128 + c * 32, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= corr;
          tc_st32(t_row + 128 + c * 32, o);
        }
      }
      const float mb = m_ref == -INFINITY ? 0.f : m_ref;
#pragma unroll
      for (int c = 0; c < kTcTok / 8; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float r0, r1;
          w[e] = pack2<QD>(ex2(s[c * 8 + 2 * e] - mb), ex2(s[c * 8 + 2 * e + 1] - mb), r0, r1);
          l += r0 + r1;
        }
        *reinterpret_cast<uint4*>(sP + tc_swz(tid, c)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {   // O += P V into columns [128, 256)
        tc_fence_after();
        const uint32_t pa_ = smem_addr(sP), va = smem_addr(sm + TcSmem::kV + b * TcSmem::kTile);
#pragma unroll
        for (int kk = 0; kk < kTcTok / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * (kTcRows * 128) + (kk & 3) * 32;
          tc_mma(tmem + 128, tc_desc(pa_ + aoff, 1024, 16), tc_desc(va + kk * 2048, 1024, kTcTok * 128), idO,
                 (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&bar_o);
      }
    }
    if (s_fail) break;
    {
      const bool ok = mbar_wait_bounded(&bar_o, (it - 1) & 1);
      if (!__all_sync(kFull, ok) && (tid & 31) == 0) {
        record_error(PA_DEV_WAIT_TIMEOUT, 7, u, 0);
        s_fail = 1;
      }
    }
    __syncthreads();
    if (s_fail) break;
    tc_fence_after();

    // the output row (whole context in this unit) or this chunk's partial
    const int P = has_q ? (qpos + 1 + p.chunk - 1) / p.chunk : 0;
    const bool wr = has_q && x.part < P;
    const bool fin = wr && P == 1;
    const float inv = fin ? 1.f / l : 0.f;
    const size_t slot = (size_t(has_q ? tok : 0) * Hq + head) * p.max_parts + x.part;
#pragma unroll 1
    for (int c = 0; c < kTcD / 32; ++c) {
      float o[32];
      tc_ld32(t_row + 128 + c * 32, o);
      if (fin) {
        uint4* orow = reinterpret_cast<uint4*>(static_cast<QT*>(p.out) + (size_t(tok) * Hq + head) * kTcD + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float a, b2;
            w[e] = pack2<QD>(o[i * 8 + 2 * e] * inv, o[i * 8 + 2 * e + 1] * inv, a, b2);
          }
          orow[i] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      } else if (wr) {
        float4* acc = reinterpret_cast<float4*>(p.part_acc + slot * kTcD + c * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
      }
    }
    if (wr && !fin) {
      p.part_ml[slot * 2] = m_ref;
      p.part_ml[slot * 2 + 1] = l;
    }
    tc_fence_before();
    __syncthreads();
  }

  if (s_fail && tid == 0) {   // drain: MMAs issued so far, then outstanding loads
    tc_commit(&bar_fin);
    mbar_wait_bounded(&bar_fin, 0);
    for (int b = 0; b < 2; ++b)
      if (pending & (1u << b)) mbar_wait_bounded(&bar_kv[b], par[b]);
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
typedef CUresult (*TmapEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

TmapEncodeFn tmap_encoder() {
  static std::once_flag once;
  static TmapEncodeFn fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<TmapEncodeFn>(f);
  });
  return fn;
}

bool cache_tmap(TmapEncodeFn enc, CUtensorMap* m, const void* base, int qd, long long rows, int BS) {
  const cuuint64_t dims[2] = {cuuint64_t(kTcD), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(kTcD) * 2};
  const cuuint32_t box[2] = {64, cuuint32_t(BS)};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, qd == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
             const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

using TcKernel = void (*)(const ExtendParams, const CUtensorMap, const CUtensorMap);

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
  l.threads = 128;
  return occupancy(l, cap);
}

// Launch after the plan kernel (programmatic dependent launch). The cache base pointers
// are 16-byte aligned and the rows 256 bytes, as the tensor maps require.
pa_status extend_tc_launch(const ExtendParams& p, const pa_cache_desc* c, int qd, int G, int grid,
                           cudaStream_t s) {
  TcKernel fn = tc_pick(qd, c->block_size, G);
  TmapEncodeFn enc = tmap_encoder();
  if (!fn || !enc) return PA_ERR_ARG;
  CUtensorMap tk, tv;
  const long long rows = (long long)c->num_blocks * c->num_kv_heads * c->block_size;
  if (!cache_tmap(enc, &tk, c->k_cache, qd, rows, c->block_size) ||
      !cache_tmap(enc, &tv, c->v_cache, qd, rows, c->block_size))
    return PA_ERR_ARG;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = TcSmem::kBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, p, tk, tv) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace pa
