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
  static constexpr int kWarps = 4;
  static constexpr int kStages = kStage >= 16384 ? 2 : (kStage >= 8192 ? 3 : 4);
  static constexpr int kBPP = kPartitionTokens / BS;             // blocks per partition
  static constexpr int kMaxPerWarp = (kBPP + kWarps - 1) / kWarps;
  static constexpr int kStageBytes = kWarps * kStages * kStage;
  static constexpr int kBarBytes = kWarps * kStages * 8;
  static constexpr int kMergeFloats = kWarps * G * (D + 2);
  static constexpr int kSmem = kStageBytes + kBarBytes + kMergeFloats * 4;
  static_assert(kRow % 16 == 0 && kLPR >= 1 && kLPR <= 32, "row must be whole 16-byte vectors");
  static_assert(kIters >= 1 && kIters * kRPI == BS, "block size must be a multiple of rows/iter");
  static_assert(kMaxPerWarp <= 32, "block ids per warp must fit the lanes");
};

template <int QD, int KV, int D, int BS, int G>
__global__ void __launch_bounds__(128) partition_kernel(const DecodeParams p) {
  using C = Cfg<KV, D, BS, G>;
  using QT = typename Q<QD>::T;
  constexpr int EPL = C::kEPL, LPR = C::kLPR, RPI = C::kRPI, IT = C::kIters;
  constexpr int NS = C::kStages, NW = C::kWarps;

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

  const int Hkv = p.num_kv_heads, Hq = p.num_q_heads;
  const int total_units = p.plan[p.num_seqs] * Hkv;
  const uint64_t pol = l2_policy_evict_first();
  uint8_t* my_stage = smem + warp * NS * C::kStage;
  uint64_t* my_bar = bars + warp * NS;
  uint32_t seq_no = 0;          // items this warp has consumed so far (all units)
  bool aborted = false;

  for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
    // ---- unit -> (sequence, kv head, partition) -------------------------------
    const int pair = u / Hkv, hk = u - pair * Hkv;
    int lo = 0, hi = p.num_seqs;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.plan[mid] <= pair) lo = mid; else hi = mid;
    }
    const int s = lo, part = pair - p.plan[s];
    const int L = clamp_len(p.context_lens[s], p.len_limit);
    const int nparts = (L + kPartitionTokens - 1) / kPartitionTokens;
    const int nblk_seq = (L + BS - 1) / BS;
    const int b0 = part * C::kBPP;
    const int nblk = min(C::kBPP, nblk_seq - b0);
    const int mine = nblk > warp ? (nblk - warp + NW - 1) / NW : 0;

    // this warp's block ids, one per lane, checked against the pool
    int bid_reg = 0;
    if (lane < mine) {
      const int lb = b0 + warp + lane * NW;
      int v = p.block_tables[size_t(s) * p.max_blocks + lb];
      if (v < 0 || v >= p.num_blocks) {
        record_error(PA_DEV_BAD_BLOCK_ID, s, lb, v);
        v = 0;
      }
      bid_reg = v;
    }

    // q for the G heads of this kv head, pre-multiplied by scale * k_scale * log2 e
    float qf[G][EPL];
    {
      const QT* qp = static_cast<const QT*>(p.q) + (size_t(s) * Hq + size_t(hk) * G) * D + j * EPL;
#pragma unroll
      for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int v = 0; v < EPL / 8; ++v) {
          const uint4 raw = *reinterpret_cast<const uint4*>(qp + size_t(g) * D + v * 8);
          const QT* e = reinterpret_cast<const QT*>(&raw);
#pragma unroll
          for (int t = 0; t < 8; ++t) qf[g][v * 8 + t] = Q<QD>::to_float(e[t]) * p.q_mul;
        }
      }
    }

    const size_t head_off = size_t(hk) * C::kChunk;
    const size_t block_stride = size_t(Hkv) * C::kChunk;
    auto issue = [&](int i) {
      const int bid = __shfl_sync(kFull, bid_reg, i);
      if (lane == 0) {
        const int st = (seq_no + i) % NS;
        uint8_t* dst = my_stage + st * C::kStage;
        mbar_arrive_expect_tx(&my_bar[st], C::kStage);
        const size_t off = size_t(bid) * block_stride + head_off;
        bulk_g2s(dst, p.k_cache + off, C::kChunk, &my_bar[st], pol);
        bulk_g2s(dst + C::kChunk, p.v_cache + off, C::kChunk, &my_bar[st], pol);
      }
    };
    const int pre = mine < NS ? mine : NS;
    for (int i = 0; i < pre; ++i) issue(i);

    float m[G], l[G], acc[G][EPL];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m[g] = -INFINITY;
      l[g] = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[g][e] = 0.f;
    }

    int consumed = 0;
    for (int i = 0; i < mine && !aborted; ++i) {
      const int n = seq_no + i;
      const int st = n % NS;
      const uint32_t parity = (n / NS) & 1;
      const bool ok = mbar_wait_bounded(&my_bar[st], parity);
      if (!__all_sync(kFull, ok)) {
        if (lane == 0) record_error(PA_DEV_WAIT_TIMEOUT, 1, u, st);
        aborted = true;
        break;
      }
      consumed = i + 1;
      const uint8_t* Ks = my_stage + st * C::kStage;
      const uint8_t* Vs = Ks + C::kChunk;
      const int lb = b0 + warp + i * NW;
      const int valid = min(BS, L - lb * BS);   // >= 1

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
      // online softmax update (base 2)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float mx = sc[g][0];
#pragma unroll
        for (int it = 1; it < IT; ++it) mx = fmaxf(mx, sc[g][it]);
#pragma unroll
        for (int off = LPR; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, off));
        const float mnew = fmaxf(m[g], mx);
        const float corr = exp2f(m[g] - mnew);
        m[g] = mnew;
        float ps = 0.f;
#pragma unroll
        for (int it = 0; it < IT; ++it) {
          sc[g][it] = exp2f(sc[g][it] - mnew);
          ps += sc[g][it];
        }
        l[g] = l[g] * corr + ps;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[g][e] *= corr;
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
      __syncwarp();
      if (i + NS < mine) issue(i + NS);
    }
    if (aborted) {
      // let the copies this warp still has in flight land before leaving
      for (int i = consumed; i < mine && i < consumed + NS; ++i) {
        const int n = seq_no + i;
        mbar_wait_bounded(&my_bar[n % NS], (n / NS) & 1, 100000000ull);
      }
      if (lane == 0) s_abort = 1;
    }
    seq_no += mine;

    // combine the row groups of the warp, then stage the warp's state for the merge
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
    for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
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
      const int h = hk * G + g;
      if (nparts == 1) {
        QT* o = static_cast<QT*>(p.out) + (size_t(s) * Hq + h) * D + d;
        *o = Q<QD>::from_float(a * p.v_scale / ls);
      } else {
        const size_t slot = (size_t(s) * Hq + h) * p.max_parts + part;
        p.part_acc[slot * D + d] = a * p.v_scale;
        if (d == 0) {
          p.part_ml[slot * 2] = M;
          p.part_ml[slot * 2 + 1] = ls;
        }
      }
    }
    __syncthreads();
    if (s_abort) break;
  }
}

// --------------------------------------------------------------------------
// log-sum-exp merge of partitions
// --------------------------------------------------------------------------
template <int QD, int D>
__global__ void __launch_bounds__(256) reduce_kernel(const DecodeParams p) {
  using QT = typename Q<QD>::T;
  constexpr int DPL = D / 32;   // dims per lane
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (gw >= p.num_seqs * p.num_q_heads) return;
  const int s = gw / p.num_q_heads, h = gw - s * p.num_q_heads;
  const int L = clamp_len(p.context_lens[s], p.len_limit);
  const int P = (L + kPartitionTokens - 1) / kPartitionTokens;
  if (P <= 1) return;
  const size_t base = (size_t(s) * p.num_q_heads + h) * p.max_parts;
  const float* ml = p.part_ml + base * 2;
  float M = -INFINITY;
  for (int i = lane; i < P; i += 32) M = fmaxf(M, ml[2 * i]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, off));
  float ls = 0.f;
  for (int i = lane; i < P; i += 32) ls += ml[2 * i + 1] * exp2f(ml[2 * i] - M);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) ls += __shfl_xor_sync(kFull, ls, off);
  float a[DPL];
#pragma unroll
  for (int k = 0; k < DPL; ++k) a[k] = 0.f;
  const float* accp = p.part_acc + base * D + lane * DPL;
  for (int i = 0; i < P; ++i) {
    const float w = exp2f(ml[2 * i] - M);
    if constexpr (DPL == 4) {
      const float4 v = *reinterpret_cast<const float4*>(accp + size_t(i) * D);
      a[0] = fmaf(w, v.x, a[0]);
      a[1] = fmaf(w, v.y, a[1]);
      a[2] = fmaf(w, v.z, a[2]);
      a[3] = fmaf(w, v.w, a[3]);
    } else {
#pragma unroll
      for (int k = 0; k < DPL; ++k) a[k] = fmaf(w, accp[size_t(i) * D + k], a[k]);
    }
  }
  QT* o = static_cast<QT*>(p.out) + (size_t(s) * p.num_q_heads + h) * D + lane * DPL;
#pragma unroll
  for (int k = 0; k < DPL; ++k) o[k] = Q<QD>::from_float(a[k] / ls);
}

// --------------------------------------------------------------------------
// host side
// --------------------------------------------------------------------------
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
};

template <int QD, int KV, int D, int BS, int G>
Launch get_partition() {
  Launch l;
  l.fn = partition_kernel<QD, KV, D, BS, G>;
  l.smem = Cfg<KV, D, BS, G>::kSmem;
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
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, l.fn, 128, l.smem);
  if (e != cudaSuccess) return e;
  if (blocks < 1) blocks = 1;
  if (g_occ_n[dev] < 128) g_occ[dev][g_occ_n[dev]++] = OccEntry{l.fn, blocks};
  *grid_cap = blocks * g_num_sms[dev];
  return cudaSuccess;
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
    part.fn<<<grid, 128, part.smem, s>>>(p);
    if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  }
  if ((stage_mask & 4) && max_parts > 1) {
    const long long warps = (long long)num_seqs * num_q_heads;
    const int grid = int((warps + 7) / 8);
    pick_reduce(q_dtype, D)<<<grid, 256, 0, s>>>(p);
    if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
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
  return pa::ws_layout(num_seqs, num_q_heads, head_dim, max_parts).total;
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
