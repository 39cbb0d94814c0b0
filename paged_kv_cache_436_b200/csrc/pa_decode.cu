// Paged single-query decode attention for sm_100a.
//
// What it computes: page 2 (untitled; first section "1. 为什么vLLM能实现24倍推理加速"),
// section "1.1 PagedAttention的内存管理革命" -- paged_attention(queries, key_cache,
// value_cache, block_tables) in place of matmul(q, k^T)/sqrt(d); page 3
// «内存优化：KV Cache管理、PagedAttention原理与内存池配置», section "核心原理" -- each
// decode step scores the new token's query against every cached key and value.
// Long contexts: page 2, section "3.3 常见问题排查" names the v2 kernel as the fix
// for slow long text; here the context is cut into 512-token partitions whose
// partial softmax states are merged by a separate log-sum-exp kernel.
//
// Three launches on one stream:
//   plan      1 CTA: per-sequence partition counts (ceil(L/512)), exclusive scan into
//             the workspace, context-length checks, zero rows for empty sequences.
//   partition persistent grid (SMs x resident CTAs). A work unit is one (sequence,
//             kv head, partition). A CTA takes units blockIdx.x, +gridDim.x, ...; its 4
//             warps split the partition's blocks round-robin. Each warp streams its
//             blocks through a private ring of shared-memory stages filled by 1-D bulk
//             copies (the TMA engine; one (block, kv head) chunk of K and of V is
//             contiguous in the [NB, Hkv, BS, D] layout), completion on an mbarrier.
//             The G query heads of a kv head are computed together, so every KV byte
//             is read from HBM once. Online softmax in binary32 (base 2, the scale and
//             log2 e folded into q); warps merge through shared memory; one partition
//             writes the output directly, several write (max, sum, unnormalised acc).
//   reduce    one warp per (sequence, q head) with >1 partition: log-sum-exp merge.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <mutex>

#include "pa.h"
#include "pa_device.cuh"

namespace pa {

struct DecodeParams {
  const void* q;
  void* out;
  const uint8_t* k_cache;
  const uint8_t* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  int32_t* plan;      // [S + 1] exclusive scan of partitions per sequence
  float* part_ml;     // [S][Hq][Pmax][2]  (running max in log2 units, sum of exp2)
  float* part_acc;    // [S][Hq][Pmax][D]  unnormalised, v_scale applied
  int num_seqs, num_q_heads, num_kv_heads, num_blocks, max_blocks, max_parts;
  int len_limit;      // min(max_blocks * BS, max_parts * 512)
  float q_mul;        // scale * k_scale * log2(e)
  float v_scale;
  int out_row_bytes;  // Hq * D * sizeof(q element)
};

__device__ __forceinline__ int clamp_len(int L, int limit) { return L < 0 ? 0 : (L > limit ? limit : L); }

// --------------------------------------------------------------------------
// plan
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) plan_kernel(const DecodeParams p) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  grid_dependency_launch_dependents();       // the partition kernel may be scheduled now
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < p.num_seqs; base += blockDim.x) {
    const int s = base + threadIdx.x;
    int parts = 0;
    if (s < p.num_seqs) {
      const int L = p.context_lens[s];
      if (L < 0 || L > p.len_limit) record_error(PA_DEV_BAD_CONTEXT_LEN, s, L, p.len_limit);
      const int Lc = clamp_len(L, p.len_limit);
      parts = (Lc + kPartitionTokens - 1) / kPartitionTokens;
      if (Lc == 0) {  // empty context: all-zero output row
        uint4* row = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) + size_t(s) * p.out_row_bytes);
        for (int i = 0; i < p.out_row_bytes / 16; ++i) row[i] = make_uint4(0, 0, 0, 0);
      }
    }
    int incl = parts;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(kFull, incl, off);
      if (lane >= off) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int nw = blockDim.x >> 5;
      int v = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(kFull, v, off);
        if (lane >= off) v += t;
      }
      if (lane < nw) warp_tot[lane] = v;  // inclusive scan of warp totals
    }
    __syncthreads();
    const int before = carry + (warp > 0 ? warp_tot[warp - 1] : 0) + incl - parts;
    if (s < p.num_seqs) p.plan[s] = before;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = before + parts;
    __syncthreads();
  }
  if (threadIdx.x == 0) p.plan[p.num_seqs] = carry;
}

// --------------------------------------------------------------------------
// partition kernel
// --------------------------------------------------------------------------
template <int KV, int D, int BS, int G>
struct Cfg {
  static constexpr int kEB = Kv<KV>::kBytes;
  static constexpr int kRow = D * kEB;            // bytes of one token row of one head
  static constexpr int kLPR = kRow / 16;          // lanes covering one row (16 B each)
  static constexpr int kRPI = 32 / kLPR;          // rows a warp covers per iteration
  static constexpr int kEPL = 16 / kEB;           // elements per lane per row
  static constexpr int kIters = BS / kRPI;        // iterations per block
  static constexpr int kChunk = BS * kRow;        // one (block, kv head) chunk of K (or V)
  static constexpr int kStage = 2 * kChunk;       // K + V
  static constexpr int kBlocksPerPartition = kPartitionTokens / BS;
  // each warp streams about 8 blocks of a partition: 4 warps for BS 16, 2 for BS 32
  static constexpr int kWarps = kBlocksPerPartition / 8 < 2 ? 2 : (kBlocksPerPartition / 8 > 8 ? 8 : kBlocksPerPartition / 8);
  // 2 stages of K+V per warp: with 8 KB stages, 3 CTAs of 4 warps (or 6 of 2) share an
  // SM: 12 warps and 192 KB in flight per SM
  static constexpr int kStages = kStage >= 8192 ? 2 : 4;
  // the producer may run ahead into the warp's next unit. Measured on B200: +1-2 %
  // for E4M3 (more work per byte: the pipeline must stay full), -2 % for 16-bit
  // caches (already at the DRAM limit: more requests in flight only add queueing)
  static constexpr bool kLookahead = (KV == PA_E4M3);
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kMaxPerWarp = (kBlocksPerPartition + kWarps - 1) / kWarps;
  static constexpr int kStageBytes = kWarps * kStages * kStage;
  static constexpr int kBarBytes = kWarps * kStages * 8;
  static constexpr int kMergeFloats = kWarps * G * (D + 2);
  static constexpr int kSmem = kStageBytes + kBarBytes + kMergeFloats * 4;
  static_assert(kRow % 16 == 0 && kLPR >= 1 && kLPR <= 32, "row must be whole 16-byte vectors");
  static_assert(kIters >= 1 && kIters * kRPI == BS, "block size must be a multiple of rows/iter");
  static_assert(kMaxPerWarp <= 32, "block ids per warp must fit the lanes");
};

// One work unit (sequence, kv head, partition) as one warp of the CTA sees it.
struct Unit {
  int u;                 // unit index; >= total when there is no unit
  int s, hk, part;
  int L, nparts, b0;     // context length, partitions of the sequence, first block
  int mine;              // blocks of this unit this warp streams
  int bid;               // lane i: physical block of the warp's i-th block (i < mine)
};

template <int BS, int NW>
__device__ __forceinline__ Unit make_unit(const DecodeParams& p, int u, int total, int warp, int lane) {
  constexpr int BPP = kPartitionTokens / BS;
  Unit x;
  x.u = u;
  x.mine = 0;
  x.bid = 0;
  if (u >= total) return x;
  const int pair = u / p.num_kv_heads;
  x.hk = u - pair * p.num_kv_heads;
  int lo = 0, hi = p.num_seqs;       // plan[lo] <= pair < plan[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.plan[mid] <= pair) lo = mid; else hi = mid;
  }
  x.s = lo;
  x.part = pair - p.plan[lo];
  x.L = clamp_len(p.context_lens[lo], p.len_limit);
  x.nparts = (x.L + kPartitionTokens - 1) / kPartitionTokens;
  x.b0 = x.part * BPP;
  const int nblk = min(BPP, (x.L + BS - 1) / BS - x.b0);
  x.mine = nblk > warp ? (nblk - warp + NW - 1) / NW : 0;
  if (lane < x.mine) {
    const int lb = x.b0 + warp + lane * NW;
    int v = p.block_tables[size_t(x.s) * p.max_blocks + lb];
    if (v < 0 || v >= p.num_blocks) {
      record_error(PA_DEV_BAD_BLOCK_ID, x.s, lb, v);
      v = 0;
    }
    x.bid = v;
  }
  return x;
}

template <int QD, int KV, int D, int BS, int G>
__global__ void __launch_bounds__(Cfg<KV, D, BS, G>::kThreads) partition_kernel(const DecodeParams p) {
  using C = Cfg<KV, D, BS, G>;
  using QT = typename Q<QD>::T;
  constexpr int EPL = C::kEPL, LPR = C::kLPR, RPI = C::kRPI, IT = C::kIters;
  constexpr int NS = C::kStages, NW = C::kWarps, QV = EPL / 8;

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kStageBytes);
  float* mrg = reinterpret_cast<float*>(smem + C::kStageBytes + C::kBarBytes);
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = lane % LPR, r = lane / LPR;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NW * NS; ++i) mbar_init(&bars[i], 1);
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  grid_dependency_launch_dependents();       // the merge kernel may be scheduled early
  grid_dependency_wait();                    // the plan (and all earlier work) is complete

  const int Hkv = p.num_kv_heads, Hq = p.num_q_heads;
  const int total = p.plan[p.num_seqs] * Hkv;
  const uint64_t pol = l2_policy_evict_first();
  uint8_t* my_stage = smem + warp * NS * C::kStage;
  uint64_t* my_bar = bars + warp * NS;
  const size_t block_stride = size_t(Hkv) * C::kChunk;

  // The warp's blocks form one stream across its units: item g (a global count)
  // lives in stage g % NS and completes phase (g / NS) & 1 of that stage's barrier.
  // The producer (lane 0) keeps up to NS items in flight and runs ahead into the
  // next unit, so a unit boundary does not drain the pipeline.
  uint32_t consumed = 0;   // items consumed so far
  uint32_t issued = 0;     // items issued so far
  uint32_t base = 0;       // global number of cur's first item
  bool aborted = false;

  auto load_q = [&](const Unit& un, uint4 (&raw)[G][QV]) {
    const QT* qp = static_cast<const QT*>(p.q) + (size_t(un.s) * Hq + size_t(un.hk) * G) * D + j * EPL;
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int v = 0; v < QV; ++v) raw[g][v] = *reinterpret_cast<const uint4*>(qp + size_t(g) * D + v * 8);
  };
  auto issue = [&](const Unit& un, int idx, uint32_t g) {
    const int bid = __shfl_sync(kFull, un.bid, idx);
    if (lane == 0) {
      const int st = g % NS;
      uint8_t* dst = my_stage + st * C::kStage;
      mbar_arrive_expect_tx(&my_bar[st], C::kStage);
      const size_t off = size_t(bid) * block_stride + size_t(un.hk) * C::kChunk;
      bulk_g2s(dst, p.k_cache + off, C::kChunk, &my_bar[st], pol);
      bulk_g2s(dst + C::kChunk, p.v_cache + off, C::kChunk, &my_bar[st], pol);
    }
  };
  // issue every item whose stage is free: those of cur first, then of nxt
  auto top_up = [&](const Unit& cur, const Unit& nxt) {
    while (issued < consumed + NS) {
      const int k = int(issued - base);
      if (k < cur.mine) issue(cur, k, issued);
      else if (C::kLookahead && k - cur.mine < nxt.mine) issue(nxt, k - cur.mine, issued);
      else break;
      ++issued;
    }
  };

  Unit cur = make_unit<BS, NW>(p, blockIdx.x, total, warp, lane);
  uint4 qraw[G][QV];
  if (cur.u < total) load_q(cur, qraw);

  while (cur.u < total) {
    const Unit nxt = make_unit<BS, NW>(p, cur.u + gridDim.x, total, warp, lane);
    top_up(cur, nxt);
    uint4 qraw_next[G][QV];
    if (nxt.u < total) load_q(nxt, qraw_next);

    // q of the G heads, binary32, pre-multiplied by scale * k_scale * log2 e
    float qf[G][EPL];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int v = 0; v < QV; ++v) {
        const QT* e = reinterpret_cast<const QT*>(&qraw[g][v]);
#pragma unroll
        for (int x = 0; x < 8; ++x) qf[g][v * 8 + x] = Q<QD>::to_float(e[x]) * p.q_mul;
      }

    float m[G], l[G], acc[G][EPL];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m[g] = -INFINITY;
      l[g] = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[g][e] = 0.f;
    }

    for (int i = 0; i < cur.mine; ++i) {
      const uint32_t n = consumed;
      const int st = n % NS;
      const bool ok = mbar_wait_bounded(&my_bar[st], (n / NS) & 1);
      if (!__all_sync(kFull, ok)) {
        if (lane == 0) record_error(PA_DEV_WAIT_TIMEOUT, 1, cur.u, st);
        aborted = true;
        break;
      }
      const uint8_t* Ks = my_stage + st * C::kStage;
      const uint8_t* Vs = Ks + C::kChunk;
      const int lb = cur.b0 + warp + i * NW;
      const int valid = min(BS, cur.L - lb * BS);   // >= 1

      // scores of this lane's rows for the G heads
      float sc[G][IT];
#pragma unroll
      for (int it = 0; it < IT; ++it) {
        const int row = it * RPI + r;
        const uint4 raw = *reinterpret_cast<const uint4*>(Ks + row * C::kRow + j * 16);
        float kf[EPL];
        Kv<KV>::decode(raw, kf);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float a = 0.f;
#pragma unroll
          for (int e = 0; e < EPL; ++e) a = fmaf(qf[g][e], kf[e], a);
          sc[g][it] = a;
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int it = 0; it < IT; ++it) {
#pragma unroll
          for (int off = LPR / 2; off >= 1; off >>= 1) sc[g][it] += __shfl_xor_sync(kFull, sc[g][it], off);
          if (it * RPI + r >= valid) sc[g][it] = -INFINITY;
        }
      }
      // online softmax update (base 2); the accumulator is rescaled only when the
      // running maximum moves (a warp-uniform branch)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float mx = sc[g][0];
#pragma unroll
        for (int it = 1; it < IT; ++it) mx = fmaxf(mx, sc[g][it]);
#pragma unroll
        for (int off = LPR; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, off));
        if (mx > m[g]) {
          const float corr = exp2f(m[g] - mx);
          m[g] = mx;
          l[g] *= corr;
#pragma unroll
          for (int e = 0; e < EPL; ++e) acc[g][e] *= corr;
        }
        float ps = 0.f;
#pragma unroll
        for (int it = 0; it < IT; ++it) {
          sc[g][it] = exp2f(sc[g][it] - m[g]);
          ps += sc[g][it];
        }
        l[g] += ps;
      }
      // P . V over this lane's rows
#pragma unroll
      for (int it = 0; it < IT; ++it) {
        const int row = it * RPI + r;
        if (row < valid) {
          const uint4 raw = *reinterpret_cast<const uint4*>(Vs + row * C::kRow + j * 16);
          float vf[EPL];
          Kv<KV>::decode(raw, vf);
#pragma unroll
          for (int g = 0; g < G; ++g) {
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[g][e] = fmaf(sc[g][it], vf[e], acc[g][e]);
          }
        }
      }
      __syncwarp();          // every lane is done with this stage before it is refilled
      ++consumed;
      top_up(cur, nxt);
    }
    if (aborted && lane == 0) s_abort = 1;

    // combine the warp's row groups, then stage the warp's state for the merge
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int off = LPR; off < 32; off <<= 1) {
        l[g] += __shfl_xor_sync(kFull, l[g], off);
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[g][e] += __shfl_xor_sync(kFull, acc[g][e], off);
      }
    }
    if (r == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float* w = mrg + (warp * G + g) * (D + 2);
#pragma unroll
        for (int e = 0; e < EPL; ++e) w[2 + j * EPL + e] = acc[g][e];
        if (j == 0) {
          w[0] = m[g];
          w[1] = l[g];
        }
      }
    }
    __syncthreads();

    // merge the warps: out = sum_w acc_w 2^(m_w - M) / sum_w l_w 2^(m_w - M)
    for (int idx = threadIdx.x; idx < G * D; idx += C::kThreads) {
      const int g = idx / D, d = idx - g * D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW; ++w) M = fmaxf(M, mrg[(w * G + g) * (D + 2)]);
      float ls = 0.f, a = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float* ww = mrg + (w * G + g) * (D + 2);
        const float f = exp2f(ww[0] - M);   // 0 for a warp without blocks (m = -inf)
        ls += ww[1] * f;
        a += ww[2 + d] * f;
      }
      const int h = cur.hk * G + g;
      if (cur.nparts == 1) {
        QT* o = static_cast<QT*>(p.out) + (size_t(cur.s) * Hq + h) * D + d;
        *o = Q<QD>::from_float(a * p.v_scale / ls);
      } else {
        const size_t slot = (size_t(cur.s) * Hq + h) * p.max_parts + cur.part;
        p.part_acc[slot * D + d] = a * p.v_scale;
        if (d == 0) {
          p.part_ml[slot * 2] = M;
          p.part_ml[slot * 2 + 1] = ls;
        }
      }
    }
    __syncthreads();
    if (s_abort) break;
    base += cur.mine;
    cur = nxt;
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int v = 0; v < QV; ++v) qraw[g][v] = qraw_next[g][v];
  }
  // leave no copy in flight into this CTA's shared memory (bounded waits)
  for (uint32_t n = consumed; n < issued; ++n) mbar_wait_bounded(&my_bar[n % NS], (n / NS) & 1, 100000000ull);
}

// --------------------------------------------------------------------------
// log-sum-exp merge of partitions
// --------------------------------------------------------------------------
// One CTA of 4 warps per (sequence, q head); a row with one partition exits at once
// (the partition kernel wrote its output). Warp w merges partitions w, w + 4, ...;
// lane l owns D/32 consecutive output dims and keeps 8 partial rows in flight
// (coalesced: a warp reads one 4 B * D row per partition). The weights 2^(m_p - M)
// go through shared memory; the four warp sums meet in shared memory.
constexpr int kMergeWarps = 4;

template <int QD, int D>
__global__ void __launch_bounds__(kMergeWarps * 32) reduce_kernel(const DecodeParams p) {
  using QT = typename Q<QD>::T;
  constexpr int NT = kMergeWarps * 32, DPL = D / 32;
  extern __shared__ float wsm[];             // [max_parts] weights
  __shared__ float red[kMergeWarps];
  __shared__ float wsum[kMergeWarps][D];
  __shared__ float s_M;
  grid_dependency_wait();                    // partials of the partition kernel are complete
  const int sh = blockIdx.x;
  const int s = sh / p.num_q_heads;
  const int L = clamp_len(p.context_lens[s], p.len_limit);
  const int P = (L + kPartitionTokens - 1) / kPartitionTokens;
  if (P <= 1) return;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const size_t base = size_t(sh) * p.max_parts;
  const float* ml = p.part_ml + base * 2;
  float M = -INFINITY;
  for (int i = t; i < P; i += NT) M = fmaxf(M, ml[2 * i]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, off));
  if (lane == 0) red[warp] = M;
  __syncthreads();
  if (t == 0) {
    float v = red[0];
    for (int w = 1; w < kMergeWarps; ++w) v = fmaxf(v, red[w]);
    s_M = v;
  }
  __syncthreads();
  M = s_M;
  float ls = 0.f;
  for (int i = t; i < P; i += NT) {
    const float w = exp2f(ml[2 * i] - M);
    wsm[i] = w;
    ls += ml[2 * i + 1] * w;
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) ls += __shfl_xor_sync(kFull, ls, off);
  __syncthreads();                           // red[] reuse and wsm[] ready
  if (lane == 0) red[warp] = ls;
  const float* accp = p.part_acc + base * D + lane * DPL;
  float a[DPL];
#pragma unroll
  for (int k = 0; k < DPL; ++k) a[k] = 0.f;
  int i = warp;
  for (; i + 7 * kMergeWarps < P; i += 8 * kMergeWarps) {
    float x[8][DPL];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float* src = accp + size_t(i + u * kMergeWarps) * D;
      if constexpr (DPL == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        x[u][0] = v.x; x[u][1] = v.y; x[u][2] = v.z; x[u][3] = v.w;
      } else {
#pragma unroll
        for (int k = 0; k < DPL; ++k) x[u][k] = src[k];
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int k = 0; k < DPL; ++k) a[k] = fmaf(wsm[i + u * kMergeWarps], x[u][k], a[k]);
  }
  for (; i < P; i += kMergeWarps)
#pragma unroll
    for (int k = 0; k < DPL; ++k) a[k] = fmaf(wsm[i], accp[size_t(i) * D + k], a[k]);
#pragma unroll
  for (int k = 0; k < DPL; ++k) wsum[warp][lane * DPL + k] = a[k];
  __syncthreads();
  for (int d = t; d < D; d += NT) {
    float tot = 0.f, lsum = 0.f;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) {
      tot += wsum[w][d];
      lsum += red[w];
    }
    QT* o = static_cast<QT*>(p.out) + size_t(sh) * D + d;
    *o = Q<QD>::from_float(tot / lsum);
  }
}

// --------------------------------------------------------------------------
// host side
// --------------------------------------------------------------------------
constexpr int kMaxPartitions = 12288;   // max_context_len <= 12288 * 512 = 6,291,456 tokens

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
  size_t plan, ml, acc, total;
};

inline WsLayout ws_layout(int S, int Hq, int D, int max_parts) {
  WsLayout w;
  w.plan = 0;
  w.ml = align256(size_t(S + 1) * 4);
  w.acc = w.ml + align256(size_t(S) * Hq * max_parts * 2 * 4);
  w.total = w.acc + align256(size_t(S) * Hq * max_parts * D * 4);
  return w;
}

using KernelFn = void (*)(const DecodeParams);

struct Launch {
  KernelFn fn = nullptr;
  int smem = 0;
  int threads = 0;
};

template <int QD, int KV, int D, int BS, int G>
Launch get_partition() {
  Launch l;
  l.fn = partition_kernel<QD, KV, D, BS, G>;
  l.smem = Cfg<KV, D, BS, G>::kSmem;
  l.threads = Cfg<KV, D, BS, G>::kThreads;
  return l;
}

template <int QD, int KV, int D, int BS>
Launch pick_g(int G) {
  switch (G) {
    case 1: return get_partition<QD, KV, D, BS, 1>();
    case 2: return get_partition<QD, KV, D, BS, 2>();
    case 4: return get_partition<QD, KV, D, BS, 4>();
    case 8: return get_partition<QD, KV, D, BS, 8>();
  }
  return Launch{};
}

template <int QD, int KV, int D>
Launch pick_bs(int BS, int G) {
  switch (BS) {
    case 8: return pick_g<QD, KV, D, 8>(G);
    case 16: return pick_g<QD, KV, D, 16>(G);
    case 32: return pick_g<QD, KV, D, 32>(G);
  }
  return Launch{};
}

template <int QD, int KV>
Launch pick_d(int D, int BS, int G) {
  switch (D) {
    case 64: return pick_bs<QD, KV, 64>(BS, G);
    case 128: return pick_bs<QD, KV, 128>(BS, G);
  }
  return Launch{};
}

Launch pick_partition(int qd, int kv, int D, int BS, int G) {
  if (kv == PA_F16 && qd == PA_F16) return pick_d<PA_F16, PA_F16>(D, BS, G);
  if (kv == PA_BF16 && qd == PA_BF16) return pick_d<PA_BF16, PA_BF16>(D, BS, G);
  if (kv == PA_E4M3 && qd == PA_F16) return pick_d<PA_F16, PA_E4M3>(D, BS, G);
  if (kv == PA_E4M3 && qd == PA_BF16) return pick_d<PA_BF16, PA_E4M3>(D, BS, G);
  return Launch{};
}

KernelFn pick_reduce(int qd, int D) {
  if (qd == PA_F16) return D == 64 ? reduce_kernel<PA_F16, 64> : reduce_kernel<PA_F16, 128>;
  return D == 64 ? reduce_kernel<PA_BF16, 64> : reduce_kernel<PA_BF16, 128>;
}

// Resident CTAs per SM for one partition-kernel instantiation on the current device.
// Computed once per (device, kernel) and cached; the first call also raises the
// kernel's dynamic shared-memory limit.
constexpr int kMaxDevices = 64;
struct OccEntry {
  KernelFn fn;
  int blocks;
};
std::mutex g_occ_mu;
OccEntry g_occ[kMaxDevices][128];
int g_occ_n[kMaxDevices];
int g_num_sms[kMaxDevices];

cudaError_t occupancy(const Launch& l, int* grid_cap) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_occ_mu);
  if (g_num_sms[dev] == 0) {
    e = cudaDeviceGetAttribute(&g_num_sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  for (int i = 0; i < g_occ_n[dev]; ++i)
    if (g_occ[dev][i].fn == l.fn) {
      *grid_cap = g_occ[dev][i].blocks * g_num_sms[dev];
      return cudaSuccess;
    }
  e = cudaFuncSetAttribute(l.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, l.smem);
  if (e != cudaSuccess) return e;
  int blocks = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, l.fn, l.threads, l.smem);
  if (e != cudaSuccess) return e;
  if (blocks < 1) blocks = 1;
  if (g_occ_n[dev] < 128) g_occ[dev][g_occ_n[dev]++] = OccEntry{l.fn, blocks};
  *grid_cap = blocks * g_num_sms[dev];
  return cudaSuccess;
}

// Launch a kernel that may start while the previous kernel on the stream finishes
// (programmatic dependent launch). The kernel itself calls grid_dependency_wait()
// before it touches anything the earlier work produced; since every kernel launched
// this way waits on its predecessor, completion order stays transitive.
cudaError_t launch_dependent(KernelFn fn, int grid, int threads, size_t smem, cudaStream_t s,
                             const DecodeParams& p) {
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

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

pa_status validate_cache(const pa_cache_desc* c) {
  if (!c || !c->k_cache || !c->v_cache) return PA_ERR_ARG;
  if (c->num_blocks <= 0 || c->num_kv_heads <= 0) return PA_ERR_ARG;
  if (c->block_size != 8 && c->block_size != 16 && c->block_size != 32) return PA_ERR_ARG;
  if (c->head_dim != 64 && c->head_dim != 128) return PA_ERR_ARG;
  if (c->kv_dtype != PA_F16 && c->kv_dtype != PA_BF16 && c->kv_dtype != PA_E4M3) return PA_ERR_ARG;
  if (!aligned16(c->k_cache) || !aligned16(c->v_cache)) return PA_ERR_ARG;
  if (!(c->k_scale > 0.f) || !(c->v_scale > 0.f) || !std::isfinite(c->k_scale) ||
      !std::isfinite(c->v_scale))
    return PA_ERR_ARG;
  if (c->kv_dtype != PA_E4M3 && (c->k_scale != 1.f || c->v_scale != 1.f)) return PA_ERR_ARG;
  return PA_OK;
}

// Grouped query heads on the tensor cores (pa_extend.cu): the 16-row mma.sync kernel with one
// query row per sequence, and the size of its workspace.
pa_status decode_grouped_mma(int stage_mask, const void* q, int32_t q_dtype, int32_t num_seqs, int32_t num_q_heads,
                             const pa_cache_desc* c, const int32_t* block_tables, int32_t max_blocks_per_seq,
                             const int32_t* context_lens, int32_t max_context_len, float scale, void* out,
                             void* workspace, size_t workspace_bytes, cudaStream_t s);
size_t ext_ws_total(int S, int T, int Hq, int D, int max_parts);

// Whether decode runs on the tensor cores: grouped query heads (G >= 4) over a 16-bit cache
// in blocks of 16 or 32 tokens; otherwise the CUDA-core partition kernel.
inline bool decode_on_mma(const pa_cache_desc* c, int G) {
  return c->kv_dtype != PA_E4M3 && G >= 4 && (c->block_size == 16 || c->block_size == 32);
}

pa_status decode_impl(int stage_mask, const void* q, int32_t q_dtype, int32_t num_seqs,
                      int32_t num_q_heads, const pa_cache_desc* c, const int32_t* block_tables,
                      int32_t max_blocks_per_seq, const int32_t* context_lens,
                      int32_t max_context_len, float scale, void* out, void* workspace,
                      size_t workspace_bytes, void* stream) {
  pa_status st = validate_cache(c);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || num_q_heads <= 0 || max_blocks_per_seq <= 0 || max_context_len < 0)
    return PA_ERR_ARG;
  if (q_dtype != PA_F16 && q_dtype != PA_BF16) return PA_ERR_ARG;
  if (c->kv_dtype != PA_E4M3 && q_dtype != c->kv_dtype) return PA_ERR_ARG;
  if (num_q_heads % c->num_kv_heads != 0) return PA_ERR_ARG;
  const int G = num_q_heads / c->num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_ARG;
  if (!(std::isfinite(scale))) return PA_ERR_ARG;
  if (num_seqs == 0) return PA_OK;
  if (!q || !out || !block_tables || !context_lens || !workspace) return PA_ERR_ARG;
  if (!aligned16(q) || !aligned16(out) || (reinterpret_cast<uintptr_t>(workspace) & 255)) return PA_ERR_ARG;
  const int D = c->head_dim, BS = c->block_size;
  const int max_parts = max_context_len > 0 ? (max_context_len + kPartitionTokens - 1) / kPartitionTokens : 1;
  if (max_parts > kMaxPartitions) return PA_ERR_ARG;   // merge weights live in 48 KB of smem
  if (decode_on_mma(c, G))
    return decode_grouped_mma(stage_mask, q, q_dtype, num_seqs, num_q_heads, c, block_tables, max_blocks_per_seq,
                              context_lens, max_context_len, scale, out, workspace, workspace_bytes,
                              static_cast<cudaStream_t>(stream));
  const WsLayout ws = ws_layout(num_seqs, num_q_heads, D, max_parts);
  if (workspace_bytes < ws.total) return PA_ERR_ARG;
  const Launch part = pick_partition(q_dtype, c->kv_dtype, D, BS, G);
  if (!part.fn) return PA_ERR_ARG;

  DecodeParams p;
  p.q = q;
  p.out = out;
  p.k_cache = static_cast<const uint8_t*>(c->k_cache);
  p.v_cache = static_cast<const uint8_t*>(c->v_cache);
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  p.plan = reinterpret_cast<int32_t*>(w + ws.plan);
  p.part_ml = reinterpret_cast<float*>(w + ws.ml);
  p.part_acc = reinterpret_cast<float*>(w + ws.acc);
  p.num_seqs = num_seqs;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = c->num_kv_heads;
  p.num_blocks = c->num_blocks;
  p.max_blocks = max_blocks_per_seq;
  p.max_parts = max_parts;
  const long long lim_a = (long long)max_blocks_per_seq * BS, lim_b = (long long)max_parts * kPartitionTokens;
  p.len_limit = int(lim_a < lim_b ? lim_a : lim_b);
  p.q_mul = scale * c->k_scale * 1.4426950408889634f;
  p.v_scale = c->v_scale;
  p.out_row_bytes = num_q_heads * D * 2;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  if (stage_mask & 1) {
    plan_kernel<<<1, 1024, 0, s>>>(p);
    if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  }
  if (stage_mask & 2) {
    int cap = 0;
    if (occupancy(part, &cap) != cudaSuccess) return PA_ERR_CUDA;
    const long long units = (long long)num_seqs * c->num_kv_heads * max_parts;
    const int grid = int(units < cap ? units : cap);
    if (launch_dependent(part.fn, grid, part.threads, part.smem, s, p) != cudaSuccess) return PA_ERR_CUDA;
  }
  if ((stage_mask & 4) && max_parts > 1) {
    const long long rows = (long long)num_seqs * num_q_heads;
    if (launch_dependent(pick_reduce(q_dtype, D), int(rows), kMergeWarps * 32, size_t(max_parts) * 4, s, p) !=
        cudaSuccess)
      return PA_ERR_CUDA;
  }
  return PA_OK;
}

// ---------------------------------------------------------------------------
// Allocation-free decode: the workspace lives in a fixed device array
// ---------------------------------------------------------------------------
// Some callers may not allocate device memory at all: a plugin running inside a
// host framework that owns every device byte through its own caching allocator
// (a raw cudaMalloc would bypass that allocator's accounting, and cudaFree
// synchronises the whole device), or a latency-critical serving loop that forbids
// allocation calls because they can stall other streams. For them
// pa_decode_no_alloc uses this array as its workspace. It is part of the
// library's device image, so every GPU that loads the library holds these
// PA_NO_ALLOC_WORKSPACE_BYTES until the process exits.
static __device__ __align__(256) unsigned char g_no_alloc_ws[PA_NO_ALLOC_WORKSPACE_BYTES];

std::mutex g_no_alloc_mu;
void* g_no_alloc_ptr[kMaxDevices];

// Device address of g_no_alloc_ws on the current device. In host code the array's
// name only stands in for the symbol, so the address is looked up once per device
// (with that device current) and cached.
cudaError_t no_alloc_workspace(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_no_alloc_mu);
  if (!g_no_alloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_no_alloc_ws);
    if (e != cudaSuccess) return e;
    g_no_alloc_ptr[dev] = p;
  }
  *ptr = g_no_alloc_ptr[dev];
  return cudaSuccess;
}

}  // namespace pa

extern "C" {

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                int32_t max_context_len) {
  if (num_seqs < 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len < 0) return 0;
  const int max_parts =
      max_context_len > 0 ? (max_context_len + pa::kPartitionTokens - 1) / pa::kPartitionTokens : 1;
  // enough for either kernel: the grouped-head tensor-core path keeps a few more records
  const size_t a = pa::ws_layout(num_seqs, num_q_heads, head_dim, max_parts).total;
  const size_t b = pa::ext_ws_total(num_seqs, num_seqs, num_q_heads, head_dim, max_parts);
  return a > b ? a : b;
}

pa_status pa_decode(const void* q, int32_t q_dtype, int32_t num_seqs, int32_t num_q_heads,
                    const pa_cache_desc* cache, const int32_t* block_tables,
                    int32_t max_blocks_per_seq, const int32_t* context_lens,
                    int32_t max_context_len, float scale, void* out, void* workspace,
                    size_t workspace_bytes, void* stream) {
  return pa::decode_impl(7, q, q_dtype, num_seqs, num_q_heads, cache, block_tables,
                         max_blocks_per_seq, context_lens, max_context_len, scale, out, workspace,
                         workspace_bytes, stream);
}

pa_status pa_decode_stage(int32_t stage, const void* q, int32_t q_dtype, int32_t num_seqs,
                          int32_t num_q_heads, const pa_cache_desc* cache,
                          const int32_t* block_tables, int32_t max_blocks_per_seq,
                          const int32_t* context_lens, int32_t max_context_len, float scale,
                          void* out, void* workspace, size_t workspace_bytes, void* stream) {
  if (stage < 0 || stage > 2) return PA_ERR_ARG;
  return pa::decode_impl(1 << stage, q, q_dtype, num_seqs, num_q_heads, cache, block_tables,
                         max_blocks_per_seq, context_lens, max_context_len, scale, out, workspace,
                         workspace_bytes, stream);
}

pa_status pa_last_device_error(void* stream, int32_t* code, int32_t* info) {
  if (!code) return PA_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int host[4] = {0, 0, 0, 0};
  const int zero[4] = {0, 0, 0, 0};
  if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaMemcpyFromSymbol(host, pa::g_pa_error, sizeof(host)) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaMemcpyToSymbol(pa::g_pa_error, zero, sizeof(zero)) != cudaSuccess) return PA_ERR_CUDA;
  *code = host[0];
  if (info) {
    info[0] = host[1];
    info[1] = host[2];
    info[2] = host[3];
  }
  return host[0] ? PA_ERR_DEVICE_CHECK : PA_OK;
}

pa_status pa_decode_no_alloc(const void* q, int32_t q_dtype, int32_t num_seqs, int32_t num_q_heads,
                             const pa_cache_desc* cache, const int32_t* block_tables,
                             int32_t max_blocks_per_seq, const int32_t* context_lens,
                             int32_t max_context_len, float scale, void* out, void* stream) {
  if (!cache) return PA_ERR_ARG;
  const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, cache->head_dim, max_context_len);
  if (need == 0 || need > PA_NO_ALLOC_WORKSPACE_BYTES) return PA_ERR_ARG;
  void* ws = nullptr;
  if (pa::no_alloc_workspace(&ws) != cudaSuccess) return PA_ERR_CUDA;
  // Nothing in the workspace has to start at zero: every call rewrites the plan
  // and writes each partial result before reading it.
  return pa::decode_impl(7, q, q_dtype, num_seqs, num_q_heads, cache, block_tables, max_blocks_per_seq,
                         context_lens, max_context_len, scale, out, ws, PA_NO_ALLOC_WORKSPACE_BYTES,
                         stream);
}

const char* pa_version(void) { return "libpa 0.1 (sm_100a)"; }

}  // extern "C"
