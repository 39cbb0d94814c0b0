// Multi-query causal attention over the paged cache ("extend": several new tokens per
// sequence -- speculative verification, chunked prefill -- attend to the whole context).
//
// Page 2 (untitled; first section "1. 为什么vLLM能实现24倍推理加速"), section
// "2.1 核心组件交互流程": the execution engine runs prefill, decode and extend modes;
// section "2.2 关键数据结构剖析": the attention metadata carries query lengths beside
// the context lengths. Query i of sequence s sits at position L_s - Q_s + i and
// attends to tokens 0 .. L_s - Q_s + i.
//
// With 16 query rows per K/V byte the work is a real contraction, so it runs on the
// tensor cores (mma.sync m16n8k16, 16-bit inputs, binary32 accumulation):
//   * a work unit is (sequence, kv head, tile of 16 rows, 512-token partition), read
//     from the record the plan kernel writes for it; a row is a (query, q head of the
//     kv head's group) pair, so a tile holds 16 / G queries;
//   * each warp is an independent persistent worker with a 2-stage ring of K/V blocks;
//     a cache block arrives as 128B-swizzled 2-D TMA boxes (one per 64-dim half, no
//     multicast) and ldmatrix reads it at swizzled addresses, free of bank conflicts;
//     V rows past the tile's last token are zeroed in shared memory;
//   * the 64-row cooperative kernel (long runs at head_dim 64) streams each token row
//     by its own 1-D bulk copy into a padded row (head_dim * 2 + 16 bytes) instead;
//   * long runs at head_dim 128 go to the tcgen05 kernel of pa_extend_tc.cu;
//   * S = Q K^T and O += P V per 16-token slice; the S accumulators are reused as the
//     P operand (rounded to the cache's 16-bit type; for bf16, in a slice where some
//     weight exceeds 1/8 of its running sum, the rounded remainder p - bf16(p) is a
//     second operand, so such weights enter P V to within 2^-16; the running sum adds
//     what enters the products); causal mask per row; online softmax in base 2;
//   * one partition writes the output row, several write (max, sum, unnormalised row)
//     for the log-sum-exp merge kernel, as in decode.
#include <cuda_runtime.h>

#include "pa.h"
#include "pa_device.cuh"
#include "pa_tmap.cuh"

namespace pa {

struct ExtendParams {
  const void* q;
  void* out;
  const uint8_t* k_cache;
  const uint8_t* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* query_start;   // [S + 1]; null: one query row per sequence, row s (decode)
  int32_t* plan;                // [S + 1] exclusive scan of units per sequence (one kv head)
  float* part_ml;               // [T][Hq][Pmax][2]
  float* part_acc;              // [T][Hq][Pmax][D]
  int num_seqs, num_tokens, num_q_heads, num_kv_heads, num_blocks, max_blocks, max_parts;
  int len_limit;
  float s_mul;                  // scale * log2(e)
  int out_row_bytes;            // Hq * D * 2
  int chunk;                    // context tokens per unit: a multiple of kPartitionTokens
  int4* units;                  // optional: two int4 per (seq, tile, chunk) pair, written by the plan
                                //   {s, tile, chunk index, row0}, {Q, base, first token, visible tokens}
  long long units_cap;          // pairs the records can hold
  int* queue;                   // next unit to hand out (zeroed by the plan kernel); null: round-robin
  int* row_parts;               // [T] chunks query row t's context spans (0: no valid query);
                                //   null when no merge pass follows
  int fresh;                    // whole prompts (pa_prefill): every L_s must equal Q_s
  int lo_mode;                  // tcgen05 path: how the bf16 remainder of P enters P V (kLoNone /
                                //   kLoAlways / kLoAdaptive in pa_extend_tc.cu)
  float k_scale, v_scale;       // E4M3 caches: per-tensor dequantisation scales (1 otherwise)
  const void* k_new;            // E4M3 prefill: the prompts' K / V rows [T][Hkv][D] of q's type,
  const void* v_new;            //   quantised into the cache before the attention reads it
};

constexpr int kTileRows = 16;

__device__ __forceinline__ int ext_clamp(int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); }

// Query rows q0 .. q1-1 of sequence s: from query_start, or -- decode through these
// kernels, query_start null -- the one query row s.
__device__ __forceinline__ void ext_rows(const ExtendParams& p, int s, int& q0, int& q1) {
  if (p.query_start) {
    q0 = p.query_start[s];
    q1 = p.query_start[s + 1];
  } else {
    q0 = s;
    q1 = s + 1;
  }
}

// Query count and position of query 0 of sequence s (validated the same way everywhere).
// Decode (query_start null): an empty context has no query, and its row is zero.
__device__ __forceinline__ void ext_seq(const ExtendParams& p, int s, int& Q, int& base) {
  const int L = ext_clamp(p.context_lens[s], 0, p.len_limit);
  int q0, q1;
  ext_rows(p, s, q0, q1);
  Q = p.query_start || L > 0 ? q1 - q0 : 0;
  if (Q < 0 || Q > L || q0 < 0 || q1 > p.num_tokens || (p.fresh && Q != L)) Q = 0;   // invalid: recorded, no work
  base = L - Q;
}

// Chunks tile t of a sequence touches: its last query sits at base + last index.
__device__ __forceinline__ int ext_tile_parts(int base, int Q, int qpt, int t, int chunk) {
  const int last = min((t + 1) * qpt, Q) - 1;
  return (base + last + 1 + chunk - 1) / chunk;
}

__global__ void __launch_bounds__(1024) extend_plan_kernel(const ExtendParams p, int qpt) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  grid_dependency_launch_dependents();
  if (threadIdx.x == 0) carry = 0;
  if (p.row_parts)
    for (int t = threadIdx.x; t < p.num_tokens; t += blockDim.x) p.row_parts[t] = 0;
  __syncthreads();
  for (int b = 0; b < p.num_seqs; b += blockDim.x) {
    const int s = b + threadIdx.x;
    int units = 0;
    if (s < p.num_seqs) {
      const int Lraw = p.context_lens[s];
      int q0, q1;
      ext_rows(p, s, q0, q1);
      const int Qraw = q1 - q0;
      if (Lraw < 0 || Lraw > p.len_limit) record_error(PA_DEV_BAD_CONTEXT_LEN, s, Lraw, p.len_limit);
      int Q, base;
      ext_seq(p, s, Q, base);
      if (Qraw != Q) {
        // decode of an empty context is no error; anything else is recorded
        if (p.query_start || ext_clamp(Lraw, 0, p.len_limit) > 0) record_error(PA_DEV_BAD_CONTEXT_LEN, s, Qraw, Lraw);
        // the rows of an invalid sequence (or of an empty decode context) are zero
        const int t0 = ext_clamp(q0, 0, p.num_tokens);
        const int t1 = ext_clamp(q1, t0, p.num_tokens);
        for (int t = t0; t < t1; ++t) {
          uint4* row = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) + size_t(t) * p.out_row_bytes);
          for (int i = 0; i < p.out_row_bytes / 16; ++i) row[i] = make_uint4(0, 0, 0, 0);
        }
      }
      const int tiles = (Q + qpt - 1) / qpt;
      for (int t = 0; t < tiles; ++t) units += ext_tile_parts(base, Q, qpt, t, p.chunk);
    }
    int incl = units;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(kFull, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int nw = blockDim.x >> 5;
      int v = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int x = __shfl_up_sync(kFull, v, off);
        if (lane >= off) v += x;
      }
      if (lane < nw) warp_tot[lane] = v;
    }
    __syncthreads();
    const int before = carry + (warp > 0 ? warp_tot[warp - 1] : 0) + incl - units;
    if (s < p.num_seqs) {
      p.plan[s] = before;
      if (p.units && units > 0) {   // the pair records of this sequence, in plan order
        int Q, base, row0, q1;
        ext_seq(p, s, Q, base);
        ext_rows(p, s, row0, q1);
        int idx = before;
        const int tiles = (Q + qpt - 1) / qpt;
        for (int t = tiles - 1; t >= 0; --t) {   // longest tile first (dynamic scheduling takes them in order)
          const int last = base + min((t + 1) * qpt, Q) - 1;
          const int P = ext_tile_parts(base, Q, qpt, t, p.chunk);
          for (int part = 0; part < P && idx < p.units_cap; ++part, ++idx) {
            const int t0 = part * p.chunk;
            p.units[2 * size_t(idx)] = make_int4(s, t, part, row0);
            p.units[2 * size_t(idx) + 1] = make_int4(Q, base, t0, min(p.chunk, last + 1 - t0));
          }
        }
      }
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = before + units;
    __syncthreads();
  }
  // chunks each query row spans (the merge kernel reads them): a warp per sequence
  for (int s = warp; p.row_parts && s < p.num_seqs; s += blockDim.x >> 5) {
    int Q, base, row0, q1;
    ext_seq(p, s, Q, base);
    ext_rows(p, s, row0, q1);
    for (int i = lane; i < Q; i += 32) p.row_parts[row0 + i] = (base + i + 1 + p.chunk - 1) / p.chunk;
  }
  if (threadIdx.x == 0) {
    if (p.queue) *p.queue = 0;   // the extend kernels' work queue
    // pairs past the records' capacity (only from inconsistent query_start) are dropped
    if (p.units && carry > p.units_cap) record_error(PA_DEV_BAD_CONTEXT_LEN, -1, carry, int(p.units_cap));
    p.plan[p.num_seqs] = p.units && carry > p.units_cap ? int(p.units_cap) : carry;
  }
}

// --------------------------------------------------------------------------
// tensor-core helpers
// --------------------------------------------------------------------------
template <int QD>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (QD == PA_BF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr(p)));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr(p)));
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

template <int QD>
__device__ __forceinline__ uint32_t pack2(float lo, float hi, float& lo_r, float& hi_r) {
  using T = typename Q<QD>::T;
  const T a = Q<QD>::from_float(lo), b = Q<QD>::from_float(hi);
  lo_r = Q<QD>::to_float(a);
  hi_r = Q<QD>::to_float(b);
  const uint16_t ua = *reinterpret_cast<const uint16_t*>(&a), ub = *reinterpret_cast<const uint16_t*>(&b);
  return uint32_t(ua) | (uint32_t(ub) << 16);
}

// The share of a row's running sum above which a weight's bf16 rounding is corrected: a
// later token can only lower a weight's share, so every weight left uncorrected ends
// below this share of its row's total, one of many small independent rounding terms.
constexpr float kLoShare = 0.125f;

// The P operands of one 16-token slice (the S accumulator layout reused as the A
// fragment): p = 2^(s - m) per element; hi = p rounded to the 16-bit type. For bf16 the
// rounding (up to 2^-8 of p) can move an output by more than the parity tolerance when a
// few weights dominate and their V values cancel, so the remainder p - hi (exact in
// binary32) is rounded again into lo, a second operand: hi + lo is p to within 2^-16 of
// p. lo is needed only where some weight exceeds kLoShare of its running sum; each lane
// tests its own elements against its share of the row's sum (the lane holding a row's
// largest weight sees at least the true share), and the returned warp-wide answer says
// whether the caller multiplies lo. For f16 (rounding up to 2^-11 of p) lo is never
// formed. l adds what enters the products.
template <int QD>
__device__ __forceinline__ bool make_p_operands(const float (&sc)[2][4], const float (&base_m)[2], uint32_t (&hi)[4],
                                                uint32_t (&lo)[4], float (&l)[2]) {
  float lh[2] = {0.f, 0.f}, ll[2] = {0.f, 0.f}, pm[2] = {0.f, 0.f};
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float p0 = exp2f(sc[nt][2 * h] - base_m[h]), p1 = exp2f(sc[nt][2 * h + 1] - base_m[h]);
      float r0, r1;
      hi[nt * 2 + h] = pack2<QD>(p0, p1, r0, r1);
      lh[h] += r0 + r1;
      pm[h] = fmaxf(pm[h], fmaxf(p0, p1));
      if constexpr (QD == PA_BF16) {
        float e0, e1;
        lo[nt * 2 + h] = pack2<QD>(p0 - r0, p1 - r1, e0, e1);
        ll[h] += e0 + e1;
      } else {
        lo[nt * 2 + h] = 0u;
      }
    }
  if constexpr (QD != PA_BF16) {
    l[0] += lh[0];
    l[1] += lh[1];
    return false;
  }
  const bool need = pm[0] > kLoShare * (l[0] + lh[0] + ll[0]) || pm[1] > kLoShare * (l[1] + lh[1] + ll[1]);
  const bool any = __any_sync(kFull, need);
  l[0] += lh[0] + (any ? ll[0] : 0.f);
  l[1] += lh[1] + (any ? ll[1] : 0.f);
  return any;
}

template <int D, int BS>
struct ExtCfg {
  static constexpr int kRowBytes = D * 2;
  static constexpr int kHalf = BS * 128;                // one 64-dim half of a block: BS rows of 128 B
  static constexpr int kStage = 2 * BS * kRowBytes;     // K block then V block, each D / 64 halves
  static constexpr int kStages = 2;
  static constexpr int kWarps = 4;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kSmem = kWarps * kStages * kStage + kWarps * kStages * 8 + 1024;   // + alignment
  static constexpr int kBlocksPerPartition = kPartitionTokens / BS;
  static_assert(BS % 16 == 0, "blocks hold whole 16-token slices");
  static_assert(kBlocksPerPartition <= 32, "block ids of a partition fit the lanes");
};

struct ExtUnit {
  int u;
  int s, hk, t, part;
  int Q, base, row0;        // row0: query row index of the sequence's first query
  int b0, nblk;             // first block and block count of the partition (causal)
  int last;                 // last position any row of the tile sees
  int bid;                  // lane i: physical block of the unit's i-th block
};

template <int BS>
__device__ __forceinline__ ExtUnit ext_make_unit(const ExtendParams& p, int u, int total, int qpt, int lane) {
  constexpr int BPP = kPartitionTokens / BS;
  ExtUnit x;
  x.u = u;
  x.nblk = 0;
  x.bid = 0;
  if (u >= total) return x;
  const int pair = u / p.num_kv_heads;   // the plan kernel's record of (sequence, tile, partition)
  x.hk = u - pair * p.num_kv_heads;
  const int4 a = __ldg(p.units + 2 * size_t(pair)), b = __ldg(p.units + 2 * size_t(pair) + 1);
  x.s = a.x;
  x.t = a.y;
  x.part = a.z;
  x.row0 = a.w;
  x.Q = b.x;
  x.base = b.y;
  const int last = x.base + min((x.t + 1) * qpt, x.Q) - 1;     // last position the tile sees
  x.last = last;
  x.b0 = x.part * BPP;
  x.nblk = min(BPP, (last + 1 + BS - 1) / BS - x.b0);
  if (lane < x.nblk) {
    const int lb = x.b0 + lane;
    int v = p.block_tables[size_t(x.s) * p.max_blocks + lb];
    if (v < 0 || v >= p.num_blocks) {
      record_error(PA_DEV_BAD_BLOCK_ID, x.s, lb, v);
      v = 0;
    }
    x.bid = v;
  }
  return x;
}

// Byte offset of the 16-byte chunk holding dims [8 c, 8 c + 8) of row r in a block tile
// laid down by the 128B-swizzled 2-D TMA boxes (one per 64-dim half).
template <int BS>
__device__ __forceinline__ uint32_t ext_swz(int r, int c) {
  return uint32_t((c >> 3) * (BS * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

template <int QD, int D, int BS, int G>
__global__ void __launch_bounds__(ExtCfg<D, BS>::kThreads)
    extend_kernel(const ExtendParams p, const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv) {
  using C = ExtCfg<D, BS>;
  using QT = typename Q<QD>::T;
  constexpr int NS = C::kStages, NW = C::kWarps, KK = D / 16, NT = D / 8;
  constexpr int QPT = kTileRows / G;                      // queries per tile

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NW * NS * C::kStage);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* ring = smem + warp * NS * C::kStage;
  uint64_t* bar = bars + warp * NS;
  if (lane == 0) {
    for (int i = 0; i < NS; ++i) mbar_init(&bar[i], 1);
    fence_mbar_init();
  }
  __syncwarp();
  grid_dependency_launch_dependents();
  grid_dependency_wait();

  const int Hq = p.num_q_heads, Hkv = p.num_kv_heads;
  const int total = p.plan[p.num_seqs] * Hkv;
  uint32_t consumed = 0;

  // rows of this lane: r0 = lane / 4 and r0 + 8 of the tile
  const int r0 = lane >> 2, cq = (lane & 3) * 2;

  // units from the plan's queue (lane 0 takes the next one), or round-robin without one
  auto next_unit = [&](int cur) -> int {
    if (!p.queue) return cur < 0 ? int(blockIdx.x) * NW + warp : cur + int(gridDim.x) * NW;
    int v = 0;
    if (lane == 0) v = atomicAdd(p.queue, 1);
    return __shfl_sync(kFull, v, 0);
  };
  for (int u = next_unit(-1); u < total; u = next_unit(u)) {
    const ExtUnit x = ext_make_unit<BS>(p, u, total, QPT, lane);
    // query index, position and output row of the lane's two rows (-1: no such query)
    int qpos[2], tok[2], head[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = r0 + 8 * h;
      const int qi = x.t * QPT + r / G;
      head[h] = x.hk * G + r % G;
      if (qi < x.Q) {
        qpos[h] = x.base + qi;
        tok[h] = x.row0 + qi;
      } else {
        qpos[h] = -1;
        tok[h] = -1;
      }
    }
    // Q fragments (A operand, 16 rows x D), zero for missing rows
    uint32_t qa[KK][4];
#pragma unroll
    for (int kk = 0; kk < KK; ++kk)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int h = e & 1, dim = kk * 16 + cq + (e >> 1) * 8;
        qa[kk][e] = tok[h] >= 0 ? *reinterpret_cast<const uint32_t*>(
                                      static_cast<const QT*>(p.q) + (size_t(tok[h]) * Hq + head[h]) * D + dim)
                                : 0u;
      }

    auto issue = [&](int i, uint32_t g) {   // cache block i of the unit: one 2-D box per (K / V, half)
      const int bid = __shfl_sync(kFull, x.bid, i);
      const int st = g % NS;
      uint8_t* dst = ring + st * C::kStage;
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar[st], C::kStage);
        const int y = (bid * Hkv + x.hk) * BS;
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          tma_load_2d(dst + h * C::kHalf, &tk, h * 64, y, &bar[st]);
          tma_load_2d(dst + BS * C::kRowBytes + h * C::kHalf, &tv, h * 64, y, &bar[st]);
        }
      }
      __syncwarp();
    };
    for (int i = 0; i < NS && i < x.nblk; ++i) issue(i, consumed + i);

    float o[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    bool failed = false;

    for (int i = 0; i < x.nblk; ++i) {
      const uint32_t n = consumed;
      const int st = n % NS;
      if (!__all_sync(kFull, mbar_wait_bounded(&bar[st], (n / NS) & 1))) {
        if (lane == 0) record_error(PA_DEV_WAIT_TIMEOUT, 2, u, st);
        failed = true;
        break;
      }
      uint8_t* Ks = ring + st * C::kStage;
      uint8_t* Vs = Ks + BS * C::kRowBytes;
      const int tok0 = (x.b0 + i) * BS;
      // V rows past the tile's last token (cache bytes beyond the context, possibly NaN)
      // are zeroed: their P is 0, but 0 * NaN would still reach O
      if (tok0 + BS - 1 > x.last) {
        const int keep = x.last + 1 - tok0;
        for (int j = keep * (D / 8) + lane; j < BS * (D / 8); j += 32)
          *reinterpret_cast<uint4*>(Vs + ext_swz<BS>(j / (D / 8), j % (D / 8))) = make_uint4(0, 0, 0, 0);
        fence_async_smem();
        __syncwarp();
      }
#pragma unroll
      for (int sb = 0; sb < BS / 16; ++sb) {
        // S = Q K^T for 16 tokens (two n-tiles of 8)
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < KK; ++kk) {
          uint32_t b[4];
          const int trow = sb * 16 + (lane >> 4) * 8 + (lane & 7);
          ldsm_x4(b, Ks + ext_swz<BS>(trow, kk * 2 + ((lane >> 3) & 1)));
          mma16816<QD>(sc[0], qa[kk], b[0], b[1]);
          mma16816<QD>(sc[1], qa[kk], b[2], b[3]);
        }
        // scale, causal mask, online softmax per row
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int h = e >> 1;
            const int tp = tok0 + sb * 16 + nt * 8 + cq + (e & 1);
            float v = sc[nt][e] * p.s_mul;
            if (tp > qpos[h]) v = -INFINITY;
            sc[nt][e] = v;
            mx[h] = fmaxf(mx[h], v);
          }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          mx[h] = fmaxf(mx[h], __shfl_xor_sync(kFull, mx[h], 1));
          mx[h] = fmaxf(mx[h], __shfl_xor_sync(kFull, mx[h], 2));
        }
        float base_m[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (mx[h] > m[h]) {
            const float corr = exp2f(m[h] - mx[h]);     // 0 while nothing was accumulated
            m[h] = mx[h];
            l[h] *= corr;
#pragma unroll
            for (int nn = 0; nn < NT; ++nn) {
              o[nn][2 * h] *= corr;
              o[nn][2 * h + 1] *= corr;
            }
          }
          base_m[h] = m[h] == -INFINITY ? 0.f : m[h];
        }
        // P as the A operand of P V: p rounded to the 16-bit type, and for bf16 also the
        // rounded remainder p - bf16(p) as a second operand (hi + lo carries p to about
        // 2^-16); l adds what enters the products
        uint32_t pa[4], pl[4];
        const bool with_lo = make_p_operands<QD>(sc, base_m, pa, pl, l);
        // O += P V (V rows through ldmatrix.trans: two n-tiles of 8 dims per x4)
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          uint32_t b[4];
          const int trow = sb * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
          ldsm_x4_trans(b, Vs + ext_swz<BS>(trow, np * 2 + (lane >> 4)));
          mma16816<QD>(o[2 * np], pa, b[0], b[1]);
          mma16816<QD>(o[2 * np + 1], pa, b[2], b[3]);
          if (with_lo) {
            mma16816<QD>(o[2 * np], pl, b[0], b[1]);
            mma16816<QD>(o[2 * np + 1], pl, b[2], b[3]);
          }
        }
      }
      __syncwarp();
      ++consumed;
      if (i + NS < x.nblk) issue(i + NS, consumed + NS - 1);
    }
    if (failed) {
      // let this unit's copies still in flight land before leaving
      for (uint32_t k = consumed; k < consumed + NS; ++k) mbar_wait_bounded(&bar[k % NS], (k / NS) & 1, 100000000ull);
      break;
    }

    // row sums over the quad, then the output row or the partition's partial
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      l[h] += __shfl_xor_sync(kFull, l[h], 1);
      l[h] += __shfl_xor_sync(kFull, l[h], 2);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (tok[h] < 0) continue;
      const int P = (qpos[h] + 1 + p.chunk - 1) / p.chunk;
      if (x.part >= P) continue;
      if (P == 1) {
        QT* orow = static_cast<QT*>(p.out) + (size_t(tok[h]) * Hq + head[h]) * D;
        const float inv = 1.f / l[h];
#pragma unroll
        for (int nn = 0; nn < NT; ++nn) {
          float a, b2;
          const uint32_t w = pack2<QD>(o[nn][2 * h] * inv, o[nn][2 * h + 1] * inv, a, b2);
          *reinterpret_cast<uint32_t*>(orow + nn * 8 + cq) = w;
        }
      } else {
        const size_t slot = (size_t(tok[h]) * Hq + head[h]) * p.max_parts + x.part;
        float* acc = p.part_acc + slot * D;
#pragma unroll
        for (int nn = 0; nn < NT; ++nn)
          *reinterpret_cast<float2*>(acc + nn * 8 + cq) = make_float2(o[nn][2 * h], o[nn][2 * h + 1]);
        if ((lane & 3) == 0) {
          p.part_ml[slot * 2] = m[h];
          p.part_ml[slot * 2 + 1] = l[h];
        }
      }
    }
  }
}

// --------------------------------------------------------------------------
// cooperative variant for long query runs (prefill, long extends)
// --------------------------------------------------------------------------
// A unit covers 64 rows (4 consumer warps x 16 rows) so that each K/V block is
// streamed once per 64 rows instead of once per 16. A fifth warp only produces: it
// walks the same unit sequence as the consumers and keeps the 2-stage ring full,
// running ahead into the next unit; full[st] completes when a block has landed,
// empty[st] when all four consumers are done with it. Every wait is bounded.
constexpr int kCoopRows = 64;

template <int D, int BS>
struct CoopCfg {
  static constexpr int kRowBytes = D * 2;
  static constexpr int kRowPad = kRowBytes + 16;
  static constexpr int kStage = 2 * BS * kRowPad;
  static constexpr int kStages = 2;
  static constexpr int kConsumers = 4;
  static constexpr int kThreads = (kConsumers + 1) * 32;
  static constexpr int kSmem = kStages * kStage + 2 * kStages * 8;
  static constexpr int kBlocksPerPartition = kPartitionTokens / BS;
};

template <int QD, int D, int BS, int G>
__global__ void __launch_bounds__(CoopCfg<D, BS>::kThreads) extend_coop_kernel(const ExtendParams p) {
  using C = CoopCfg<D, BS>;
  using QT = typename Q<QD>::T;
  constexpr int NS = C::kStages, NC = C::kConsumers, KK = D / 16, NT = D / 8;
  constexpr int QPT = kCoopRows / G;                   // queries per unit tile

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + NS * C::kStage);
  uint64_t* empty = full + NS;
  __shared__ int s_abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], NC);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < NS * C::kStage / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0, 0, 0, 0);
  fence_async_smem();
  __syncthreads();
  grid_dependency_launch_dependents();
  grid_dependency_wait();

  const int Hq = p.num_q_heads, Hkv = p.num_kv_heads;
  const int total = p.plan[p.num_seqs] * Hkv;
  const size_t head_stride = size_t(BS) * C::kRowBytes;
  const size_t block_stride = size_t(Hkv) * head_stride;

  if (warp == NC) {
    // ---------------- producer warp ----------------
    const uint64_t pol = l2_policy_evict_first();
    uint32_t g = 0;
    volatile int* abort_flag = &s_abort;
    auto drain = [&]() {   // after an abort: the copies of the last NS stages land before the warp leaves
      if (lane == 0)
        for (uint32_t k = g > NS ? g - NS : 0; k < g; ++k) mbar_wait_bounded(&full[k % NS], (k / NS) & 1, 100000000ull);
      __syncwarp();
    };
    for (int u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x) {
      const ExtUnit x = ext_make_unit<BS>(p, u, total, QPT, lane);
      for (int i = 0; i < x.nblk; ++i, ++g) {
        const int st = g % NS;
        // the consumers released this stage (a fresh barrier passes parity 1 at once)
        if (!__all_sync(kFull, mbar_wait_bounded(&empty[st], ((g / NS) & 1) ^ 1))) {
          if (lane == 0) {
            record_error(PA_DEV_WAIT_TIMEOUT, 3, u, st);
            s_abort = 1;
          }
          drain();
          return;
        }
        const int bid = __shfl_sync(kFull, x.bid, i);
        uint8_t* dst = smem + st * C::kStage;
        const int nrows = min(BS, x.last + 1 - (x.b0 + i) * BS);   // rows past it stay finite
        if (lane == 0) mbar_arrive_expect_tx(&full[st], 2 * nrows * C::kRowBytes);
        __syncwarp();
        const size_t off = size_t(bid) * block_stride + size_t(x.hk) * head_stride;
        for (int j = lane; j < 2 * nrows; j += 32) {
          const int which = j / nrows, row = j - which * nrows;
          const uint8_t* src = (which ? p.v_cache : p.k_cache) + off + size_t(row) * C::kRowBytes;
          bulk_g2s(dst + which * BS * C::kRowPad + row * C::kRowPad, src, C::kRowBytes, &full[st], pol);
        }
      }
    }
    if (*abort_flag) drain();   // without an abort the consumers wait for every stage themselves
    return;
  }

  // ---------------- consumer warps: 16 rows each ----------------
  const int r0 = lane >> 2, cq = (lane & 3) * 2;
  uint32_t g = 0;
  for (int u = blockIdx.x; u < total; u += gridDim.x) {
    const ExtUnit x = ext_make_unit<BS>(p, u, total, QPT, lane);
    int qpos[2], tok[2], head[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = warp * 16 + r0 + 8 * h;              // row of the 64-row tile
      const int qi = x.t * QPT + r / G;
      head[h] = x.hk * G + r % G;
      if (qi < x.Q) {
        qpos[h] = x.base + qi;
        tok[h] = x.row0 + qi;
      } else {
        qpos[h] = -1;
        tok[h] = -1;
      }
    }
    uint32_t qa[KK][4];
#pragma unroll
    for (int kk = 0; kk < KK; ++kk)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int h = e & 1, dim = kk * 16 + cq + (e >> 1) * 8;
        qa[kk][e] = tok[h] >= 0 ? *reinterpret_cast<const uint32_t*>(
                                      static_cast<const QT*>(p.q) + (size_t(tok[h]) * Hq + head[h]) * D + dim)
                                : 0u;
      }
    float o[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    // a warp whose rows all lie before this partition's first token still consumes the
    // blocks (it must release the stages) but skips the math
    const bool active = max(qpos[0], qpos[1]) >= x.b0 * BS;
    const bool warp_active = __any_sync(kFull, active);

    for (int i = 0; i < x.nblk; ++i, ++g) {
      const int st = g % NS;
      if (!__all_sync(kFull, mbar_wait_bounded(&full[st], (g / NS) & 1))) {
        if (lane == 0) {
          record_error(PA_DEV_WAIT_TIMEOUT, 4, u, st);
          s_abort = 1;
        }
        return;
      }
      const uint8_t* Ks = smem + st * C::kStage;
      const uint8_t* Vs = Ks + BS * C::kRowPad;
      const int tok0 = (x.b0 + i) * BS;
      if (warp_active) {
#pragma unroll
        for (int sb = 0; sb < BS / 16; ++sb) {
          float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
          for (int kk = 0; kk < KK; ++kk) {
            uint32_t b[4];
            const int trow = sb * 16 + (lane >> 4) * 8 + (lane & 7);
            ldsm_x4(b, Ks + trow * C::kRowPad + (kk * 16 + ((lane >> 3) & 1) * 8) * 2);
            mma16816<QD>(sc[0], qa[kk], b[0], b[1]);
            mma16816<QD>(sc[1], qa[kk], b[2], b[3]);
          }
          float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int h = e >> 1;
              const int tp = tok0 + sb * 16 + nt * 8 + cq + (e & 1);
              float v = sc[nt][e] * p.s_mul;
              if (tp > qpos[h]) v = -INFINITY;
              sc[nt][e] = v;
              mx[h] = fmaxf(mx[h], v);
            }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(kFull, mx[h], 1));
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(kFull, mx[h], 2));
          }
          float base_m[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (mx[h] > m[h]) {
              const float corr = exp2f(m[h] - mx[h]);
              m[h] = mx[h];
              l[h] *= corr;
#pragma unroll
              for (int nn = 0; nn < NT; ++nn) {
                o[nn][2 * h] *= corr;
                o[nn][2 * h + 1] *= corr;
              }
            }
            base_m[h] = m[h] == -INFINITY ? 0.f : m[h];
          }
          uint32_t pa[4], pl[4];
          const bool with_lo = make_p_operands<QD>(sc, base_m, pa, pl, l);
#pragma unroll
          for (int np = 0; np < NT / 2; ++np) {
            uint32_t b[4];
            const int trow = sb * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
            ldsm_x4_trans(b, Vs + trow * C::kRowPad + (np * 16 + (lane >> 4) * 8) * 2);
            mma16816<QD>(o[2 * np], pa, b[0], b[1]);
            mma16816<QD>(o[2 * np + 1], pa, b[2], b[3]);
            if (with_lo) {
              mma16816<QD>(o[2 * np], pl, b[0], b[1]);
              mma16816<QD>(o[2 * np + 1], pl, b[2], b[3]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);          // this warp is done with the stage
    }
    if (*static_cast<volatile int*>(&s_abort)) return;

#pragma unroll
    for (int h = 0; h < 2; ++h) {
      l[h] += __shfl_xor_sync(kFull, l[h], 1);
      l[h] += __shfl_xor_sync(kFull, l[h], 2);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (tok[h] < 0) continue;
      const int P = (qpos[h] + 1 + p.chunk - 1) / p.chunk;
      if (x.part >= P) continue;
      if (P == 1) {
        QT* orow = static_cast<QT*>(p.out) + (size_t(tok[h]) * Hq + head[h]) * D;
        const float inv = 1.f / l[h];
#pragma unroll
        for (int nn = 0; nn < NT; ++nn) {
          float a, b2;
          *reinterpret_cast<uint32_t*>(orow + nn * 8 + cq) =
              pack2<QD>(o[nn][2 * h] * inv, o[nn][2 * h + 1] * inv, a, b2);
        }
      } else {
        const size_t slot = (size_t(tok[h]) * Hq + head[h]) * p.max_parts + x.part;
        float* acc = p.part_acc + slot * D;
#pragma unroll
        for (int nn = 0; nn < NT; ++nn)
          *reinterpret_cast<float2*>(acc + nn * 8 + cq) = make_float2(o[nn][2 * h], o[nn][2 * h + 1]);
        if ((lane & 3) == 0) {
          p.part_ml[slot * 2] = m[h];
          p.part_ml[slot * 2 + 1] = l[h];
        }
      }
    }
  }
}

// --------------------------------------------------------------------------
// E4M3 caches: the 16-row warp kernel with each cache block converted in shared memory
// --------------------------------------------------------------------------
// Every (cache block, kv head) chunk of K and of V is contiguous in the cache layout and
// arrives by one 1-D bulk copy (TMA engine, no multicast) into the warp's ring. Before use
// it is converted to f16 -- the hardware E4M3 -> f16 conversion, exact: every E4M3 value
// is an f16 value -- into a staging tile laid out as the 16-bit kernel's swizzled boxes, so
// the same ldmatrix fragment code reads it. The products then run in f16: q is scaled by
// 2^-8 into f16 when it is bf16 (exact for |q| in [2^-6, 1.6e7], within 2^-25 below,
// saturating above), P is f16 (rounding up to 2^-11 of p: no remainder term is needed),
// and the per-tensor scales multiply the scores (k_scale) and the output (v_scale). The K
// block is converted and every score of the block formed first; then the V block takes
// the same staging tile (rows past the tile's last token zero) for the P V products.
template <int D, int BS>
struct Fp8Cfg {
  static constexpr int kChunk = BS * D;           // one (block, kv head) chunk of K (or V), bytes
  static constexpr int kStage = 2 * kChunk;       // K then V
  static constexpr int kStages = 2;
  static constexpr int kStaging = BS * D * 2;     // one block of K or V as f16
  static constexpr int kWarps = 4;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kPerWarp = kStages * kStage + kStaging;
  static constexpr int kSmem = kWarps * kPerWarp + kWarps * kStages * 8 + 1024;
  static_assert(BS % 16 == 0, "blocks hold whole 16-token slices");
};

// Two values to f16, rounded to nearest and saturating to +-65504, packed (lo in the low half).
__device__ __forceinline__ uint32_t f16x2_satfinite(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Four E4M3 codes (byte i = code i) as two f16 pairs (codes 0, 1 in lo; 2, 3 in hi), exact:
// the hardware e4m3x2 -> f16x2 conversion on each 16-bit half of the word, the halves
// taken apart by a register unpack rather than shifts.
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t four, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 c01, c23;\n\tmov.b32 {c01, c23}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, c01;\n\tcvt.rn.f16x2.e4m3x2 %1, c23;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(four));
}

// One block of E4M3 rows (BS x D bytes, row-major) into the f16 staging tile, rows from
// `keep` on set to zero. Each lane converts 16-byte chunks (16 codes into two 16-byte f16
// chunks); every 8-lane phase of the reads and of the stores touches all 32 banks once.
template <int D, int BS>
__device__ __forceinline__ void fp8_block_to_f16(const uint8_t* src, uint8_t* dst, int keep, int lane) {
  constexpr int CPR = D / 16;   // 16-byte chunks (16 codes) per row
#pragma unroll
  for (int idx = lane; idx < BS * CPR; idx += 32) {
    int r = idx / CPR, cb = idx - r * CPR;
    if constexpr (CPR >= 8) {
      // rows in pairs, each 8-lane phase four chunks of the even row and four of the odd
      // row, taken from different 64-byte halves: the reads cover all 32 banks and the two
      // rows' swizzled destinations fill complementary bank groups
      const int w = idx % (2 * CPR), g = w >> 3, k = w & 7, rb = k >> 2;
      r = (idx / (2 * CPR)) * 2 + rb;
      cb = 4 * (g ^ rb) + (k & 3);
    }
    uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
    if (r < keep) {
      const uint4 raw = *reinterpret_cast<const uint4*>(src + r * D + cb * 16);
      e4m3x4_to_f16x4(raw.x, a.x, a.y);
      e4m3x4_to_f16x4(raw.y, a.z, a.w);
      e4m3x4_to_f16x4(raw.z, b.x, b.y);
      e4m3x4_to_f16x4(raw.w, b.z, b.w);
    }
    *reinterpret_cast<uint4*>(dst + ext_swz<BS>(r, 2 * cb)) = a;
    *reinterpret_cast<uint4*>(dst + ext_swz<BS>(r, 2 * cb + 1)) = b;
  }
}

// P of one 16-token slice as f16 A operands. Rows r0 + 8 (h = 1) only when some row of the
// tile's upper half is a real query row (else their operands are left zero: those rows'
// outputs are never read); l adds what enters the products.
__device__ __forceinline__ void make_p_f16(const float (&sc)[2][4], const float (&base_m)[2], uint32_t (&pa)[4],
                                           float (&l)[2], bool hi_rows) {
  float lh[2] = {0.f, 0.f};
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (h == 1 && !hi_rows) {
        pa[nt * 2 + h] = 0u;
        continue;
      }
      float p0, p1;   // 2^x on the special-function unit (results below 2^-126 are 0)
      asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(p0) : "f"(sc[nt][2 * h] - base_m[h]));
      asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(p1) : "f"(sc[nt][2 * h + 1] - base_m[h]));
      float r0, r1;
      pa[nt * 2 + h] = pack2<PA_F16>(p0, p1, r0, r1);
      lh[h] += r0 + r1;
    }
  l[0] += lh[0];
  l[1] += lh[1];
}

template <int QD, int D, int BS, int G>
__global__ void __launch_bounds__(Fp8Cfg<D, BS>::kThreads) extend_fp8_kernel(const ExtendParams p) {
  using C = Fp8Cfg<D, BS>;
  using QT = typename Q<QD>::T;
  constexpr int NS = C::kStages, NW = C::kWarps, KK = D / 16, NT = D / 8, SB = BS / 16;
  constexpr int QPT = kTileRows / G;                      // queries per tile
  constexpr float kQScale = QD == PA_BF16 ? 1.f / 256.f : 1.f;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* ring = smem + warp * C::kPerWarp;
  uint8_t* stg = ring + NS * C::kStage;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + NW * C::kPerWarp) + warp * NS;
  if (lane == 0) {
    for (int i = 0; i < NS; ++i) mbar_init(&bar[i], 1);
    fence_mbar_init();
  }
  __syncwarp();
  grid_dependency_launch_dependents();
  grid_dependency_wait();

  const int Hq = p.num_q_heads, Hkv = p.num_kv_heads;
  const int total = p.plan[p.num_seqs] * Hkv;
  const uint64_t pol = l2_policy_evict_first();
  const size_t head_stride = size_t(BS) * D, block_stride = size_t(Hkv) * head_stride;
  const float s_mul = p.s_mul * p.k_scale / kQScale;      // scores: the f16 products times this
  uint32_t consumed = 0;
  const int r0 = lane >> 2, cq = (lane & 3) * 2;

  // units from the plan's queue (lane 0 takes the next one), or round-robin without one
  auto next_unit = [&](int cur) -> int {
    if (!p.queue) return cur < 0 ? int(blockIdx.x) * NW + warp : cur + int(gridDim.x) * NW;
    int v = 0;
    if (lane == 0) v = atomicAdd(p.queue, 1);
    return __shfl_sync(kFull, v, 0);
  };
  for (int u = next_unit(-1); u < total; u = next_unit(u)) {
    const ExtUnit x = ext_make_unit<BS>(p, u, total, QPT, lane);
    int qpos[2], tok[2], head[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = r0 + 8 * h;
      const int qi = x.t * QPT + r / G;
      head[h] = x.hk * G + r % G;
      if (qi < x.Q) {
        qpos[h] = x.base + qi;
        tok[h] = x.row0 + qi;
      } else {
        qpos[h] = -1;
        tok[h] = -1;
      }
    }
    // whether any of the tile's rows 8 .. 15 is a query row (a warp-uniform skip of their
    // softmax otherwise: with few queries per tile only the first rows are real)
    const bool hi = __any_sync(kFull, tok[1] >= 0);
    // Q fragments as f16 pairs (scaled by 2^-8 from bf16), zero for missing rows
    uint32_t qa[KK][4];
#pragma unroll
    for (int kk = 0; kk < KK; ++kk)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int h = e & 1, dim = kk * 16 + cq + (e >> 1) * 8;
        uint32_t v = 0u;
        if (tok[h] >= 0) {
          const QT* qp = static_cast<const QT*>(p.q) + (size_t(tok[h]) * Hq + head[h]) * D + dim;
          if constexpr (QD == PA_F16) v = *reinterpret_cast<const uint32_t*>(qp);
          else v = f16x2_satfinite(Q<QD>::to_float(qp[0]) * kQScale, Q<QD>::to_float(qp[1]) * kQScale);
        }
        qa[kk][e] = v;
      }

    auto issue = [&](int i, uint32_t g) {   // cache block i of the unit: one bulk copy each of K and V
      const int bid = __shfl_sync(kFull, x.bid, i);
      const int st = g % NS;
      if (lane == 0) {
        uint8_t* dst = ring + st * C::kStage;
        const size_t off = size_t(bid) * block_stride + size_t(x.hk) * head_stride;
        mbar_arrive_expect_tx(&bar[st], C::kStage);
        bulk_g2s(dst, p.k_cache + off, C::kChunk, &bar[st], pol);
        bulk_g2s(dst + C::kChunk, p.v_cache + off, C::kChunk, &bar[st], pol);
      }
      __syncwarp();
    };
    for (int i = 0; i < NS && i < x.nblk; ++i) issue(i, consumed + i);

    float o[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    bool failed = false;

    for (int i = 0; i < x.nblk; ++i) {
      const uint32_t n = consumed;
      const int st = n % NS;
      if (!__all_sync(kFull, mbar_wait_bounded(&bar[st], (n / NS) & 1))) {
        if (lane == 0) record_error(PA_DEV_WAIT_TIMEOUT, 5, u, st);
        failed = true;
        break;
      }
      const uint8_t* Ke = ring + st * C::kStage;
      const int tok0 = (x.b0 + i) * BS;
      // the K block as f16, then every score of the block
      fp8_block_to_f16<D, BS>(Ke, stg, BS, lane);
      __syncwarp();
      float sc[SB][2][4];
#pragma unroll
      for (int sb = 0; sb < SB; ++sb) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) sc[sb][nt][0] = sc[sb][nt][1] = sc[sb][nt][2] = sc[sb][nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KK; ++kk) {
          uint32_t b[4];
          const int trow = sb * 16 + (lane >> 4) * 8 + (lane & 7);
          ldsm_x4(b, stg + ext_swz<BS>(trow, kk * 2 + ((lane >> 3) & 1)));
          mma16816<PA_F16>(sc[sb][0], qa[kk], b[0], b[1]);
          mma16816<PA_F16>(sc[sb][1], qa[kk], b[2], b[3]);
        }
      }
      __syncwarp();   // every lane has read K from the staging tile
      // the V block into the same tile; rows past the tile's last token (cache bytes beyond
      // the context, possibly NaN codes) are zero
      fp8_block_to_f16<D, BS>(Ke + C::kChunk, stg, x.last + 1 - tok0, lane);
      __syncwarp();
      ++consumed;     // both halves of the stage are read: it can be refilled
      if (i + NS < x.nblk) issue(i + NS, consumed + NS - 1);
#pragma unroll
      for (int sb = 0; sb < SB; ++sb) {
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int h = e >> 1;
            if (h == 1 && !hi) break;
            const int tp = tok0 + sb * 16 + nt * 8 + cq + (e & 1);
            float v = sc[sb][nt][e] * s_mul;
            if (tp > qpos[h]) v = -INFINITY;
            sc[sb][nt][e] = v;
            mx[h] = fmaxf(mx[h], v);
          }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (h == 1 && !hi) break;
          mx[h] = fmaxf(mx[h], __shfl_xor_sync(kFull, mx[h], 1));
          mx[h] = fmaxf(mx[h], __shfl_xor_sync(kFull, mx[h], 2));
        }
        float base_m[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (mx[h] > m[h]) {
            const float corr = exp2f(m[h] - mx[h]);     // 0 while nothing was accumulated
            m[h] = mx[h];
            l[h] *= corr;
#pragma unroll
            for (int nn = 0; nn < NT; ++nn) {
              o[nn][2 * h] *= corr;
              o[nn][2 * h + 1] *= corr;
            }
          }
          base_m[h] = m[h] == -INFINITY ? 0.f : m[h];
        }
        uint32_t pa[4];
        make_p_f16(sc[sb], base_m, pa, l, hi);
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          uint32_t b[4];
          const int trow = sb * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
          ldsm_x4_trans(b, stg + ext_swz<BS>(trow, np * 2 + (lane >> 4)));
          mma16816<PA_F16>(o[2 * np], pa, b[0], b[1]);
          mma16816<PA_F16>(o[2 * np + 1], pa, b[2], b[3]);
        }
      }
      __syncwarp();   // every lane has read V before the next block takes the tile
    }
    if (failed) {
      for (uint32_t k = consumed; k < consumed + NS; ++k) mbar_wait_bounded(&bar[k % NS], (k / NS) & 1, 100000000ull);
      break;
    }

#pragma unroll
    for (int h = 0; h < 2; ++h) {
      l[h] += __shfl_xor_sync(kFull, l[h], 1);
      l[h] += __shfl_xor_sync(kFull, l[h], 2);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (tok[h] < 0) continue;
      const int P = (qpos[h] + 1 + p.chunk - 1) / p.chunk;
      if (x.part >= P) continue;
      if (P == 1) {
        QT* orow = static_cast<QT*>(p.out) + (size_t(tok[h]) * Hq + head[h]) * D;
        const float inv = p.v_scale / l[h];
#pragma unroll
        for (int nn = 0; nn < NT; ++nn) {
          float a, b2;
          *reinterpret_cast<uint32_t*>(orow + nn * 8 + cq) = pack2<QD>(o[nn][2 * h] * inv, o[nn][2 * h + 1] * inv, a, b2);
        }
      } else {
        const size_t slot = (size_t(tok[h]) * Hq + head[h]) * p.max_parts + x.part;
        float* acc = p.part_acc + slot * D;
#pragma unroll
        for (int nn = 0; nn < NT; ++nn)
          *reinterpret_cast<float2*>(acc + nn * 8 + cq) =
              make_float2(o[nn][2 * h] * p.v_scale, o[nn][2 * h + 1] * p.v_scale);
        if ((lane & 3) == 0) {
          p.part_ml[slot * 2] = m[h];
          p.part_ml[slot * 2 + 1] = l[h];
        }
      }
    }
  }
}

// Whole prompts into an E4M3 cache (pa_prefill): token t of sequence s (rows query_start[s]
// ..) goes to slot bt[s][i / BS] * BS + i % BS, i = t - query_start[s], stored as
// e4m3_rne_satfinite(x / scale) as pa_reshape_and_cache stores it. Grid (tokens, K / V,
// 16-byte input chunks / 128).
template <int IN>
__global__ void __launch_bounds__(128) prefill_fp8_write_kernel(const ExtendParams p, int BS, int D) {
  const int t = blockIdx.x, which = blockIdx.y;
  const int i = blockIdx.z * blockDim.x + threadIdx.x;
  const int nvec = p.num_kv_heads * D / 8;
  if (i >= nvec) return;
  int lo = 0, hi = p.num_seqs;                 // query_start[lo] <= t < query_start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.query_start[mid] <= t) lo = mid; else hi = mid;
  }
  const int s = lo;
  int nq, base;
  ext_seq(p, s, nq, base);                     // an invalid sequence (recorded by the plan) has none
  const int pos = t - p.query_start[s];
  if (pos < 0 || pos >= nq) return;
  int bid = p.block_tables[size_t(s) * p.max_blocks + pos / BS];
  if (bid < 0 || bid >= p.num_blocks) {
    if (i == 0 && which == 0) record_error(PA_DEV_BAD_BLOCK_ID, s, pos / BS, bid);
    return;
  }
  const int e0 = i * 8, h = e0 / D, d = e0 - h * D;
  using IT = typename Q<IN>::T;
  const IT* src = static_cast<const IT*>(which ? p.v_new : p.k_new) + (size_t(t) * p.num_kv_heads) * D + e0;
  const uint4 raw = *reinterpret_cast<const uint4*>(src);
  uint8_t* dst = const_cast<uint8_t*>(which ? p.v_cache : p.k_cache) +
                 ((size_t(bid) * p.num_kv_heads + h) * BS + pos % BS) * D + d;
  *reinterpret_cast<uint2*>(dst) = encode_e4m3x8<IN>(raw, which ? p.v_scale : p.k_scale);
}

// Log-sum-exp merge of a query row's partitions: one 4-warp CTA per (query row, q head).
template <int QD, int D>
__global__ void __launch_bounds__(128) extend_reduce_kernel(const ExtendParams p) {
  using QT = typename Q<QD>::T;
  constexpr int NWARP = 4, NT = NWARP * 32, DPL = D / 32;
  extern __shared__ float wsm[];
  __shared__ float red[NWARP];
  __shared__ float wsum[NWARP][D];
  __shared__ float s_M;
  grid_dependency_wait();
  const int th = blockIdx.x;
  const int t = th / p.num_q_heads;
  const int P = p.row_parts[t];                       // written by the plan kernel
  if (P <= 1) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t sbase = size_t(th) * p.max_parts;
  const float* ml = p.part_ml + sbase * 2;
  float M = -INFINITY;
  for (int i = tid; i < P; i += NT) M = fmaxf(M, ml[2 * i]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, off));
  if (lane == 0) red[warp] = M;
  __syncthreads();
  if (tid == 0) s_M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  M = s_M;
  float ls = 0.f;
  for (int i = tid; i < P; i += NT) {
    const float w = exp2f(ml[2 * i] - M);
    wsm[i] = w;
    ls += ml[2 * i + 1] * w;
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) ls += __shfl_xor_sync(kFull, ls, off);
  __syncthreads();
  if (lane == 0) red[warp] = ls;
  const float* accp = p.part_acc + sbase * D + lane * DPL;
  float a[DPL];
#pragma unroll
  for (int k = 0; k < DPL; ++k) a[k] = 0.f;
  for (int i = warp; i < P; i += NWARP)
#pragma unroll
    for (int k = 0; k < DPL; ++k) a[k] = fmaf(wsm[i], accp[size_t(i) * D + k], a[k]);
#pragma unroll
  for (int k = 0; k < DPL; ++k) wsum[warp][lane * DPL + k] = a[k];
  __syncthreads();
  for (int d = tid; d < D; d += NT) {
    const float tot = (wsum[0][d] + wsum[1][d]) + (wsum[2][d] + wsum[3][d]);
    const float lsum = (red[0] + red[1]) + (red[2] + red[3]);
    static_cast<QT*>(p.out)[size_t(th) * D + d] = Q<QD>::from_float(tot / lsum);
  }
}

// --------------------------------------------------------------------------
// host side
// --------------------------------------------------------------------------
struct ExtWs {
  size_t plan, ml, acc, units, queue, rows, total;
};

// Unit records: a sequence with Q_s > 0 queries has at most Q_s row tiles (a tile holds at
// least one query), so there are at most T tiles (tile groups), each with at most
// max_parts chunks.
inline size_t ext_units_bound(int T, int Hq, int max_parts) {
  (void)Hq;
  return size_t(T > 0 ? T : 1) * size_t(max_parts);
}

inline ExtWs ext_ws(int S, int T, int Hq, int D, int max_parts) {
  ExtWs w;
  w.plan = 0;
  w.ml = align256(size_t(S + 1) * 4);
  w.acc = w.ml + align256(size_t(T) * Hq * max_parts * 2 * 4);
  w.units = w.acc + align256(size_t(T) * Hq * max_parts * D * 4);
  w.queue = w.units + align256(ext_units_bound(T, Hq, max_parts) * 32);
  w.rows = w.queue + 256;
  w.total = w.rows + align256(size_t(T > 0 ? T : 1) * 4);
  return w;
}

using ExtKernel = void (*)(const ExtendParams);
using ExtTmapKernel = void (*)(const ExtendParams, const CUtensorMap, const CUtensorMap);
struct ExtLaunch {
  ExtKernel fn = nullptr;          // the cooperative kernel
  ExtTmapKernel tfn = nullptr;     // the warp kernel (reads the cache through tensor maps)
  int smem = 0, threads = 0;
  const void* key() const { return tfn ? reinterpret_cast<const void*>(tfn) : reinterpret_cast<const void*>(fn); }
};

template <int QD, int D, int BS, int G>
ExtLaunch ext_get(bool coop) {
  if (coop) return ExtLaunch{extend_coop_kernel<QD, D, BS, G>, nullptr, CoopCfg<D, BS>::kSmem, CoopCfg<D, BS>::kThreads};
  return ExtLaunch{nullptr, extend_kernel<QD, D, BS, G>, ExtCfg<D, BS>::kSmem, ExtCfg<D, BS>::kThreads};
}
template <int QD, int D, int BS>
ExtLaunch ext_pick_g(int G, bool coop) {
  switch (G) {
    case 1: return ext_get<QD, D, BS, 1>(coop);
    case 2: return ext_get<QD, D, BS, 2>(coop);
    case 4: return ext_get<QD, D, BS, 4>(coop);
    case 8: return ext_get<QD, D, BS, 8>(coop);
  }
  return ExtLaunch{};
}
template <int QD, int D>
ExtLaunch ext_pick_bs(int BS, int G, bool coop) {
  if (BS == 16) return ext_pick_g<QD, D, 16>(G, coop);
  if (BS == 32) return ext_pick_g<QD, D, 32>(G, coop);
  return ExtLaunch{};
}
template <int QD>
ExtLaunch ext_pick_d(int D, int BS, int G, bool coop) {
  if (D == 64) return ext_pick_bs<QD, 64>(BS, G, coop);
  if (D == 128) return ext_pick_bs<QD, 128>(BS, G, coop);
  return ExtLaunch{};
}

template <int QD, int D, int BS>
ExtLaunch fp8_pick_g(int G) {
  using C = Fp8Cfg<D, BS>;
  switch (G) {
    case 1: return ExtLaunch{extend_fp8_kernel<QD, D, BS, 1>, nullptr, C::kSmem, C::kThreads};
    case 2: return ExtLaunch{extend_fp8_kernel<QD, D, BS, 2>, nullptr, C::kSmem, C::kThreads};
    case 4: return ExtLaunch{extend_fp8_kernel<QD, D, BS, 4>, nullptr, C::kSmem, C::kThreads};
    case 8: return ExtLaunch{extend_fp8_kernel<QD, D, BS, 8>, nullptr, C::kSmem, C::kThreads};
  }
  return ExtLaunch{};
}
template <int QD>
ExtLaunch fp8_pick_d(int D, int BS, int G) {
  if (D == 64) return BS == 16 ? fp8_pick_g<QD, 64, 16>(G) : BS == 32 ? fp8_pick_g<QD, 64, 32>(G) : ExtLaunch{};
  if (D == 128) return BS == 16 ? fp8_pick_g<QD, 128, 16>(G) : BS == 32 ? fp8_pick_g<QD, 128, 32>(G) : ExtLaunch{};
  return ExtLaunch{};
}

cudaError_t ext_launch(ExtKernel fn, int grid, int threads, size_t smem, cudaStream_t s, const ExtendParams& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, p);
}

// tcgen05 path for long query runs (pa_extend_tc.cu)
bool extend_tc_supported(int qd, int D, int BS, int G);
cudaError_t extend_tc_grid_cap(int qd, int BS, int G, int* cap);
pa_status extend_tc_launch(const ExtendParams& p, const pa_cache_desc* c, int qd, int G, int grid, cudaStream_t s,
                           const void* k_new, const void* v_new);
int tc_bf16_lo_mode();
constexpr int kTcUnitRows = 128;

}  // namespace pa

extern "C" {

size_t pa_extend_workspace_size(int32_t num_seqs, int32_t num_tokens, int32_t num_q_heads, int32_t head_dim,
                                int32_t max_context_len) {
  if (num_seqs < 0 || num_tokens < 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len < 0) return 0;
  const int mp = max_context_len > 0 ? (max_context_len + pa::kPartitionTokens - 1) / pa::kPartitionTokens : 1;
  return pa::ext_ws(num_seqs, num_tokens, num_q_heads, head_dim, mp).total;
}

}  // extern "C"

namespace pa {

// pa_extend (k_new = v_new = null) and pa_prefill (fresh: the prompts' K / V in k_new,
// v_new, written into the cache by the same kernel).
static pa_status extend_impl(const void* q, int32_t q_dtype, int32_t num_seqs, int32_t num_q_heads,
                             const int32_t* query_start, int32_t num_tokens, const pa_cache_desc* c,
                             const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                             int32_t max_context_len, float scale, void* out, void* workspace,
                             size_t workspace_bytes, void* stream, const void* k_new, const void* v_new, bool fresh) {
  pa_status st = validate_cache(c);
  if (st != PA_OK) return st;
  const bool fp8 = c->kv_dtype == PA_E4M3;
  if (q_dtype != PA_F16 && q_dtype != PA_BF16) return PA_ERR_ARG;
  if (!fp8 && q_dtype != c->kv_dtype) return PA_ERR_ARG;   // a 16-bit cache holds q's type
  if (c->block_size != 16 && c->block_size != 32) return PA_ERR_ARG;
  if (num_seqs < 0 || num_tokens < 0 || num_q_heads <= 0 || max_blocks_per_seq <= 0 || max_context_len < 0)
    return PA_ERR_ARG;
  if (num_q_heads % c->num_kv_heads != 0) return PA_ERR_ARG;
  const int G = num_q_heads / c->num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_ARG;
  if (!std::isfinite(scale)) return PA_ERR_ARG;
  if (num_seqs == 0 || num_tokens == 0) return PA_OK;
  if (!q || !out || !query_start || !block_tables || !context_lens || !workspace) return PA_ERR_ARG;
  if (!aligned16(q) || !aligned16(out) || (reinterpret_cast<uintptr_t>(workspace) & 255)) return PA_ERR_ARG;
  const int D = c->head_dim, BS = c->block_size;
  const int max_parts = max_context_len > 0 ? (max_context_len + kPartitionTokens - 1) / kPartitionTokens : 1;
  if (max_parts > kMaxPartitions) return PA_ERR_ARG;
  const ExtWs ws = ext_ws(num_seqs, num_tokens, num_q_heads, D, max_parts);
  if (workspace_bytes < ws.total) return PA_ERR_ARG;
  // Long query runs (at least half a 128-row tile per sequence on average) go to the
  // tcgen05 kernel (head_dim 128) or, otherwise, the cooperative 64-row kernel; short
  // ones (speculative drafts, decode) to the 16-row warp kernel. E4M3 caches take the
  // 16-row kernel that converts each block in shared memory, for runs of any length;
  // whole prompts into an E4M3 cache are first quantised into it by one more launch.
  const long long rows_total = (long long)num_tokens * G;
  const bool tc = !fp8 && (fresh || rows_total * 2 >= (long long)kTcUnitRows * num_seqs) && scale > 0.f &&
                  extend_tc_supported(q_dtype, D, BS, G);
  if (fresh && (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new) || (!tc && !fp8))) return PA_ERR_ARG;
  const bool coop = !fp8 && !tc && rows_total > (long long)kTileRows * num_seqs;
  ExtLaunch k;
  if (fp8) {
    k = q_dtype == PA_BF16 ? fp8_pick_d<PA_BF16>(D, BS, G) : fp8_pick_d<PA_F16>(D, BS, G);
    if (!k.key()) return PA_ERR_ARG;
  } else if (!tc) {
    k = q_dtype == PA_BF16 ? ext_pick_d<PA_BF16>(D, BS, G, coop) : ext_pick_d<PA_F16>(D, BS, G, coop);
    if (!k.key()) return PA_ERR_ARG;
  }

  ExtendParams p;
  p.q = q;
  p.out = out;
  p.k_cache = static_cast<const uint8_t*>(c->k_cache);
  p.v_cache = static_cast<const uint8_t*>(c->v_cache);
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.query_start = query_start;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  p.plan = reinterpret_cast<int32_t*>(w + ws.plan);
  p.part_ml = reinterpret_cast<float*>(w + ws.ml);
  p.part_acc = reinterpret_cast<float*>(w + ws.acc);
  p.units = reinterpret_cast<int4*>(w + ws.units);
  p.queue = reinterpret_cast<int*>(w + ws.queue);
  p.row_parts = nullptr;   // set below when a merge pass follows
  p.units_cap = (long long)ext_units_bound(num_tokens, num_q_heads, max_parts);
  p.fresh = fresh ? 1 : 0;
  p.lo_mode = q_dtype == PA_BF16 ? tc_bf16_lo_mode() : 0;
  p.k_scale = c->k_scale;
  p.v_scale = c->v_scale;
  p.k_new = k_new;
  p.v_new = v_new;
  p.num_seqs = num_seqs;
  p.num_tokens = num_tokens;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = c->num_kv_heads;
  p.num_blocks = c->num_blocks;
  p.max_blocks = max_blocks_per_seq;
  p.max_parts = max_parts;
  const long long lim_a = (long long)max_blocks_per_seq * BS, lim_b = (long long)max_parts * kPartitionTokens;
  p.len_limit = int(lim_a < lim_b ? lim_a : lim_b);
  p.s_mul = scale * 1.4426950408889634f;
  p.out_row_bytes = num_q_heads * D * 2;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  const int rows_per_unit = tc ? kTcUnitRows : coop ? kCoopRows : kTileRows;
  // upper bound of the row tiles: every sequence's queries plus one ragged tile each
  const long long tiles = (rows_total + rows_per_unit - 1) / rows_per_unit + num_seqs;
  int grid = 1;
  p.chunk = kPartitionTokens;
  if (tc) {
    // the whole context per unit when that already gives two units to each of a CTA's
    // two pipelines; otherwise the largest multiple of the partition length that does
    // (split-K + merge)
    int cap = 0;
    if (extend_tc_grid_cap(q_dtype, BS, G, &cap) != cudaSuccess) return PA_ERR_CUDA;
    int nchunks = 1;
    while (nchunks < max_parts && tiles * c->num_kv_heads * nchunks < 4LL * cap) ++nchunks;
    const int parts_per_chunk = (max_parts + nchunks - 1) / nchunks;
    p.chunk = parts_per_chunk * kPartitionTokens;
    const long long units = tiles * c->num_kv_heads * ((max_parts + parts_per_chunk - 1) / parts_per_chunk);
    grid = int(units < cap ? units : cap);
  } else {
    int cap = 0;
    Launch as_launch;
    as_launch.fn = reinterpret_cast<KernelFn>(const_cast<void*>(k.key()));
    as_launch.smem = k.smem;
    as_launch.threads = k.threads;
    if (occupancy(as_launch, &cap) != cudaSuccess) return PA_ERR_CUDA;
    const long long units = tiles * c->num_kv_heads * max_parts;
    // the warp kernels run 4 independent units per CTA, the cooperative one a unit per CTA
    const long long ctas = coop ? units : (units + ExtCfg<128, 16>::kWarps - 1) / ExtCfg<128, 16>::kWarps;
    static_assert(ExtCfg<128, 16>::kWarps == Fp8Cfg<128, 16>::kWarps, "both warp kernels run 4 units per CTA");
    grid = int(ctas < cap ? ctas : cap);
  }
  if (grid < 1) grid = 1;
  const bool merge = (long long)max_parts * kPartitionTokens > p.chunk;   // some row spans several chunks
  if (merge) p.row_parts = reinterpret_cast<int*>(w + ws.rows);

  extend_plan_kernel<<<1, 1024, 0, s>>>(p, rows_per_unit / G);
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  if (fp8 && fresh) {   // the prompts' K / V into the cache, before the attention reads it
    const int nvec = c->num_kv_heads * D / 8;
    const dim3 wgrid(num_tokens, 2, (nvec + 127) / 128);
    if (q_dtype == PA_BF16) prefill_fp8_write_kernel<PA_BF16><<<wgrid, 128, 0, s>>>(p, BS, D);
    else prefill_fp8_write_kernel<PA_F16><<<wgrid, 128, 0, s>>>(p, BS, D);
    if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  }
  if (tc) {
    st = extend_tc_launch(p, c, q_dtype, G, grid, s, k_new, v_new);
    if (st != PA_OK) return st;
  } else if (k.tfn) {
    TmapEncodeFn enc = tmap_encoder();
    CUtensorMap tk, tv;
    const long long rows = (long long)c->num_blocks * c->num_kv_heads * BS;
    if (!enc || !cache_tmap(enc, &tk, c->k_cache, q_dtype, rows, BS, D) ||
        !cache_tmap(enc, &tv, c->v_cache, q_dtype, rows, BS, D))
      return PA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(k.threads);
    cfg.dynamicSmemBytes = k.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k.tfn, p, tk, tv) != cudaSuccess) return PA_ERR_CUDA;
  } else if (ext_launch(k.fn, grid, k.threads, k.smem, s, p) != cudaSuccess) {
    return PA_ERR_CUDA;
  }
  if (merge) {
    const long long rows = (long long)num_tokens * num_q_heads;
    ExtKernel red = q_dtype == PA_BF16 ? (D == 64 ? extend_reduce_kernel<PA_BF16, 64> : extend_reduce_kernel<PA_BF16, 128>)
                                       : (D == 64 ? extend_reduce_kernel<PA_F16, 64> : extend_reduce_kernel<PA_F16, 128>);
    if (ext_launch(red, int(rows), 128, size_t(max_parts) * 4, s, p) != cudaSuccess) return PA_ERR_CUDA;
  }
  return PA_OK;
}

// Bytes of the workspace the extend kernels need for these sizes.
size_t ext_ws_total(int S, int T, int Hq, int D, int max_parts) { return ext_ws(S, T, Hq, D, max_parts).total; }

// Decode with grouped query heads on the tensor cores: the 16-row mma.sync kernel with one
// query row per sequence, so that a tile holds the G heads that share a kv head (padded
// to 16 rows) and each K / V element enters G products in one MMA instead of G FMAs. On
// B200 it beats the CUDA-core partition kernel for G >= 4 (GQA prefix workload: 54 vs
// 100 us; G = 8: 119 vs 398 us). Stages as pa_decode: 0 plans, 1 attends, 2 merges.
pa_status decode_grouped_mma(int stage_mask, const void* q, int32_t q_dtype, int32_t num_seqs, int32_t num_q_heads,
                             const pa_cache_desc* c, const int32_t* block_tables, int32_t max_blocks_per_seq,
                             const int32_t* context_lens, int32_t max_context_len, float scale, void* out,
                             void* workspace, size_t workspace_bytes, cudaStream_t s) {
  const int D = c->head_dim, BS = c->block_size, G = num_q_heads / c->num_kv_heads;
  const int max_parts = max_context_len > 0 ? (max_context_len + kPartitionTokens - 1) / kPartitionTokens : 1;
  const ExtWs ws = ext_ws(num_seqs, num_seqs, num_q_heads, D, max_parts);
  if (workspace_bytes < ws.total) return PA_ERR_ARG;
  const ExtLaunch k = q_dtype == PA_BF16 ? ext_pick_d<PA_BF16>(D, BS, G, false) : ext_pick_d<PA_F16>(D, BS, G, false);
  if (!k.tfn) return PA_ERR_ARG;
  ExtendParams p{};
  p.q = q;
  p.out = out;
  p.k_cache = static_cast<const uint8_t*>(c->k_cache);
  p.v_cache = static_cast<const uint8_t*>(c->v_cache);
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.query_start = nullptr;   // one query row per sequence
  uint8_t* w = static_cast<uint8_t*>(workspace);
  p.plan = reinterpret_cast<int32_t*>(w + ws.plan);
  p.part_ml = reinterpret_cast<float*>(w + ws.ml);
  p.part_acc = reinterpret_cast<float*>(w + ws.acc);
  p.units = reinterpret_cast<int4*>(w + ws.units);
  p.queue = nullptr;
  p.units_cap = (long long)ext_units_bound(num_seqs, num_q_heads, max_parts);
  p.fresh = 0;
  p.lo_mode = 0;
  p.k_scale = p.v_scale = 1.f;
  p.k_new = p.v_new = nullptr;
  p.num_seqs = p.num_tokens = num_seqs;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = c->num_kv_heads;
  p.num_blocks = c->num_blocks;
  p.max_blocks = max_blocks_per_seq;
  p.max_parts = max_parts;
  const long long lim_a = (long long)max_blocks_per_seq * BS, lim_b = (long long)max_parts * kPartitionTokens;
  p.len_limit = int(lim_a < lim_b ? lim_a : lim_b);
  p.s_mul = scale * 1.4426950408889634f;
  p.out_row_bytes = num_q_heads * D * 2;
  p.chunk = kPartitionTokens;
  const bool merge = max_parts > 1;
  p.row_parts = merge ? reinterpret_cast<int*>(w + ws.rows) : nullptr;
  if (stage_mask & 1) {
    extend_plan_kernel<<<1, 1024, 0, s>>>(p, kTileRows / G);
    if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  }
  if (stage_mask & 2) {
    int cap = 0;
    Launch as_launch;
    as_launch.fn = reinterpret_cast<KernelFn>(const_cast<void*>(k.key()));
    as_launch.smem = k.smem;
    as_launch.threads = k.threads;
    if (occupancy(as_launch, &cap) != cudaSuccess) return PA_ERR_CUDA;
    const long long units = (long long)num_seqs * c->num_kv_heads * max_parts;
    const long long ctas = (units + ExtCfg<128, 16>::kWarps - 1) / ExtCfg<128, 16>::kWarps;
    const int grid = int(ctas < cap ? (ctas > 0 ? ctas : 1) : cap);
    TmapEncodeFn enc = tmap_encoder();
    CUtensorMap tk, tv;
    const long long rows = (long long)c->num_blocks * c->num_kv_heads * BS;
    if (!enc || !cache_tmap(enc, &tk, c->k_cache, q_dtype, rows, BS, D) ||
        !cache_tmap(enc, &tv, c->v_cache, q_dtype, rows, BS, D))
      return PA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(k.threads);
    cfg.dynamicSmemBytes = k.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k.tfn, p, tk, tv) != cudaSuccess) return PA_ERR_CUDA;
  }
  if ((stage_mask & 4) && merge) {
    ExtKernel red = q_dtype == PA_BF16 ? (D == 64 ? extend_reduce_kernel<PA_BF16, 64> : extend_reduce_kernel<PA_BF16, 128>)
                                       : (D == 64 ? extend_reduce_kernel<PA_F16, 64> : extend_reduce_kernel<PA_F16, 128>);
    if (ext_launch(red, int((long long)num_seqs * num_q_heads), 128, size_t(max_parts) * 4, s, p) != cudaSuccess)
      return PA_ERR_CUDA;
  }
  return PA_OK;
}

}  // namespace pa

extern "C" {

pa_status pa_extend(const void* q, int32_t q_dtype, int32_t num_seqs, int32_t num_q_heads,
                    const int32_t* query_start, int32_t num_tokens, const pa_cache_desc* c,
                    const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                    int32_t max_context_len, float scale, void* out, void* workspace, size_t workspace_bytes,
                    void* stream) {
  return pa::extend_impl(q, q_dtype, num_seqs, num_q_heads, query_start, num_tokens, c, block_tables,
                         max_blocks_per_seq, context_lens, max_context_len, scale, out, workspace, workspace_bytes,
                         stream, nullptr, nullptr, false);
}

pa_status pa_prefill(const void* q, const void* k, const void* v, int32_t dtype, int32_t num_seqs,
                     int32_t num_q_heads, const int32_t* query_start, int32_t num_tokens, const pa_cache_desc* c,
                     const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                     int32_t max_context_len, float scale, void* out, void* workspace, size_t workspace_bytes,
                     void* stream) {
  return pa::extend_impl(q, dtype, num_seqs, num_q_heads, query_start, num_tokens, c, block_tables,
                         max_blocks_per_seq, context_lens, max_context_len, scale, out, workspace, workspace_bytes,
                         stream, k, v, true);
}

}  // extern "C"
