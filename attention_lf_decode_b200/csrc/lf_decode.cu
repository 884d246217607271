// B200 (sm_100a) LongFlow fused decode step: single-query GQA attention,
// the zero-history / zero-cost importance score taken from the same softmax,
// and the in-place eviction of the least important unprotected slot, all in
// ONE launch.  The C ABI is declared in include/lf_decode.h.
//
// Method: "LongFlow: Efficient KV Cache Compression for Reasoning Models"
// (gist.science summary), §2A "Principios de Diseño", §2B "Derivación de la
// Métrica de Importancia", §2C "Implementación de Alto Rendimiento"; blog
// page "Долгая память: Оптимизация кэша для сложных рассуждений", section
// "Оптимизированная Реализация с Объединенными Ядрами" (attention output
// and score produced in one pass over KV blocks and a mask streamed from HBM
// into on-chip memory).
//
// Design (one row = one (batch, KV head) pair; its K and V slabs are each
// [budget, D] bf16, contiguous):
//   * A thread-block cluster of S CTAs splits the row's slots into S chunks
//     (flash-decoding split).  Each CTA has 4 consumer warps and 1 producer
//     warp.
//   * The producer streams the chunk's K tiles, then its V tiles (8 KB each,
//     contiguous), with 1-D bulk async copies into a 6-stage shared-memory
//     ring guarded by mbarriers.  Tiles whose slots are all free are never
//     loaded.  No multicast: every CTA fetches its own tiles.
//   * K phase: 8 lanes per slot, 16-byte conflict-free shared loads, fp32
//     FMAs against the pre-scaled query heads held in registers, then a
//     reduce-scatter over the 8 lanes.  Logits (log2 domain) stay in shared
//     memory: the exact normalised probabilities need the row-wide max and
//     sum, which only exist after every CTA of the cluster is done.
//   * V phase: p = 2^(s - m_cta) in place, o += p * v with one lane per 4
//     (D = 128) or 2 (D = 64) dims.
//   * Cluster exchange through distributed shared memory (no global
//     scratch, no second launch): row max / sum per head, newest position,
//     lowest free slot.  Each CTA then scores its own slots (exact
//     normalised probability averaged over the group's heads), reduces a
//     packed (fp32 score bits << 32 | slot) key to its two lowest values,
//     and combines its share of the output from all partial outputs.
//   * Near ties (two lowest scores within a relative 1e-4) are rescored in
//     fp64 from the cache, so the choice matches the exact ranking.
//   * CTA rank 0 writes k_new / v_new / t into the chosen slot, after a
//     cluster barrier that follows the last read of that slot.
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <limits.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "lf_decode.h"
#include "lf_ptx.cuh"

namespace cg = cooperative_groups;

namespace lf {

constexpr int kTileBytes = 8192;
constexpr int kStages = 6;
constexpr int kConsumerWarps = 4;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kWarps = kConsumerWarps + 1;
constexpr int kMaxSplit = 16;
constexpr int kMaxG = 8;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per barrier wait
constexpr float kTieRel = 1e-4f;                   // near-tie band rescored in fp64
constexpr unsigned long long kNoKey = ~0ull;

struct Params {
  const uint16_t* q;
  const uint16_t* k_new;
  const uint16_t* v_new;
  uint16_t* kcache;
  uint16_t* vcache;
  int32_t* pos;
  float* out;
  int32_t* evicted;
  int* status;
  int budget;
  int chunk;
  int sink;
  int window;
  int pos_vec4;
  float qscale2;     // log2(e) / sqrt(D)
  double qscale2_64;
};

// Per-CTA scalars; the fields marked "published" are read by the other CTAs
// of the cluster through distributed shared memory.
template <int GP>
struct alignas(16) Small {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  unsigned long long key1, key2;  // published: two lowest candidate keys
  double ref_score;               // published: fp64 rescoring result
  int ref_slot;                   // published
  int maxpos;                     // published: newest position in the chunk
  int first_free;                 // published: lowest free slot (global index)
  int err;                        // published: a bounded wait gave up
  float m[GP];                    // published: chunk max logit per head
  float l[GP];                    // published: chunk sum of 2^(s - m) per head
  float s_new[GP];                // new token logit per head (log2 domain)
  float Mg[GP], Lg[GP];           // row max / sum per head
  float cf[kMaxSplit][GP];        // 2^(m_r - M) per cluster rank and head
  float wmax[kConsumerWarps][GP];
  float wsum[kConsumerWarps][GP];
  unsigned long long wk1[kWarps], wk2[kWarps];
  double wref[kWarps];
  int wref_slot[kWarps];
  unsigned long long g_key1;       // row-wide lowest key (local copy)
  int g_t, g_free, g_err, g_refine, g_slot;
};

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ double bf16_to_f64(uint16_t b) {
  return static_cast<double>(__uint_as_float(static_cast<uint32_t>(b) << 16));
}

__device__ __forceinline__ void flag_error(int* err_smem, int* status) {
  *err_smem = 1;
  atomicOr(status, LF_STATUS_WAIT_TIMEOUT);
}

// keep the two smallest keys
__device__ __forceinline__ void top2_insert(unsigned long long& k1, unsigned long long& k2,
                                            unsigned long long k) {
  if (k < k1) {
    k2 = k1;
    k1 = k;
  } else if (k < k2) {
    k2 = k;
  }
}
__device__ __forceinline__ void top2_merge(unsigned long long& k1, unsigned long long& k2,
                                           unsigned long long o1, unsigned long long o2) {
  const unsigned long long lo = k1 < o1 ? k1 : o1;
  const unsigned long long hi = k1 < o1 ? o1 : k1;
  const unsigned long long s2 = k2 < o2 ? k2 : o2;
  k1 = lo;
  k2 = hi < s2 ? hi : s2;
}

// One step of the reduce-scatter over the 8 lanes of a slot: with C partial
// sums per lane, exchange half of them with the lane across `MASK` so that
// each lane keeps C/2 sums over twice as many lanes.  With C == 1 it is a
// plain butterfly step (both lanes end with the same sum).
template <int C, int MASK>
__device__ __forceinline__ void rs_step(float (&a)[kMaxG], int sub, int& head_base) {
  if constexpr (C > 1) {
    constexpr int H = C / 2;
    const bool hi = (sub & MASK) != 0;
#pragma unroll
    for (int i = 0; i < H; ++i) {
      const float send = hi ? a[i] : a[H + i];
      const float keep = hi ? a[H + i] : a[i];
      a[i] = keep + __shfl_xor_sync(0xffffffffu, send, MASK);
    }
    if (hi) head_base += H;
  } else {
    a[0] += __shfl_xor_sync(0xffffffffu, a[0], MASK);
  }
}

// Any slot of tile `tile` (chunk-local) filled?  Warp-uniform.
template <int T>
__device__ __forceinline__ bool tile_filled(const int* pos_s, int tile, int nvalid, int lane) {
  bool any = false;
#pragma unroll
  for (int k = 0; k < T / 32; ++k) {
    const int j = tile * T + k * 32 + lane;
    any |= (j < nvalid) && (pos_s[j] >= 0);
  }
  return __any_sync(0xffffffffu, any);
}

template <int D, int G>
struct Geometry {
  static constexpr int T = kTileBytes / (2 * D);  // slots per tile
  static constexpr int GP = G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8;
  static constexpr int CPL = D / 64;              // 16-byte chunks per lane (K phase)
  static constexpr int DPL = CPL * 8;             // dims per lane (K phase)
  static constexpr int GROUPS = T / 4;            // 4-slot groups per tile (K phase)
  static constexpr int DV = D / 32;               // dims per lane (V phase)
  static constexpr int TPW = T / kConsumerWarps;  // slots per warp per tile (V phase)
  static constexpr int RC = GP >= 8 ? GP / 8 : 1; // sums a lane holds after reduce-scatter
  static constexpr int BFLY = GP >= 8 ? 0 : GP == 4 ? 1 : GP == 2 ? 3 : 7;
  static size_t smem_bytes(int chunk) {
    return size_t(kStages) * kTileBytes + size_t(chunk) * GP * 4 + size_t(chunk) * 4 +
           size_t(G) * D * 4 + sizeof(Small<GP>);
  }
};

template <int D, int G, bool EVICT>
__global__ void __launch_bounds__(kThreads) fused_decode_kernel(const Params p) {
  using Geo = Geometry<D, G>;
  constexpr int T = Geo::T, GP = Geo::GP, CPL = Geo::CPL, DPL = Geo::DPL;
  constexpr int GROUPS = Geo::GROUPS, DV = Geo::DV, TPW = Geo::TPW, RC = Geo::RC;
  static_assert(G >= 1 && G <= kMaxG, "group size");
  static_assert(D == 64 || D == 128, "head dim");

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int S = static_cast<int>(cluster.num_blocks());
  const int row = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int N = p.budget, chunk = p.chunk;
  const int slot0 = rank * chunk;
  const int nvalid = max(0, min(chunk, N - slot0));
  const int ntiles = (nvalid + T - 1) / T;

  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* ring = smem;
  float* pl = reinterpret_cast<float*>(ring + kStages * kTileBytes);  // [chunk][GP]
  int* pos_s = reinterpret_cast<int*>(pl + size_t(chunk) * GP);        // [chunk]
  float* xo = reinterpret_cast<float*>(pos_s + chunk);                 // [G][D], published
  Small<GP>& sm = *reinterpret_cast<Small<GP>*>(xo + G * D);

  // ---------------------------------------------------------------- setup
  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    sm.maxpos = -1;
    sm.first_free = INT_MAX;
    sm.err = 0;
    fence_mbar_init();
  }
  __syncthreads();

  {  // position table of the chunk -> shared; newest position, lowest free slot
    int lmax = -1, lfree = INT_MAX;
    const int32_t* prow = p.pos + size_t(row) * N + slot0;
    const int nv4 = p.pos_vec4 ? (nvalid >> 2) : 0;
    for (int i = tid; i < nv4; i += kThreads) {
      const int4 v = reinterpret_cast<const int4*>(prow)[i];
      reinterpret_cast<int4*>(pos_s)[i] = v;
      const int vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (vv[k] >= 0) lmax = max(lmax, vv[k]);
        else lfree = min(lfree, 4 * i + k);
      }
    }
    for (int i = nv4 * 4 + tid; i < nvalid; i += kThreads) {
      const int v = prow[i];
      pos_s[i] = v;
      if (v >= 0) lmax = max(lmax, v);
      else lfree = min(lfree, i);
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) {
      lmax = max(lmax, __shfl_xor_sync(0xffffffffu, lmax, m));
      lfree = min(lfree, __shfl_xor_sync(0xffffffffu, lfree, m));
    }
    if (lane == 0) {
      if (lmax >= 0) atomicMax(&sm.maxpos, lmax);
      if (lfree != INT_MAX) atomicMin(&sm.first_free, slot0 + lfree);
    }
  }

  const uint16_t* qrow = p.q + size_t(row) * G * D;  // the G query heads of this KV head
  if (warp == 0) {  // logit of the new token, per head
    const uint16_t* kn = p.k_new + size_t(row) * D;
#pragma unroll
    for (int i = 0; i < G; ++i) {
      float a = 0.f;
#pragma unroll
      for (int d = 0; d < DV; ++d) {
        const int dd = lane * DV + d;
        a = fmaf(__uint_as_float(uint32_t(qrow[i * D + dd]) << 16),
                 __uint_as_float(uint32_t(kn[dd]) << 16), a);
      }
#pragma unroll
      for (int m = 16; m > 0; m >>= 1) a += __shfl_xor_sync(0xffffffffu, a, m);
      if (lane == 0) sm.s_new[i] = a * p.qscale2;
    }
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    int seq = 0;
    for (int phase = 0; phase < 2; ++phase) {
      const uint16_t* base = (phase == 0 ? p.kcache : p.vcache) + (size_t(row) * N + slot0) * D;
      for (int tile = 0; tile < ntiles; ++tile) {
        if (!tile_filled<T>(pos_s, tile, nvalid, lane)) continue;
        const int s = seq % kStages;
        const uint32_t par = uint32_t(seq / kStages) & 1u;
        if (lane == 0) {
          if (seq >= kStages && !mbar_wait_bounded(&sm.empty[s], par ^ 1u, kWaitLimitNs))
            flag_error(&sm.err, p.status);
          const int ns = min(T, nvalid - tile * T);
          const uint32_t bytes = uint32_t(ns) * D * 2;
          mbar_arrive_expect_tx(&sm.full[s], bytes);
          bulk_copy_g2s(ring + s * kTileBytes, base + size_t(tile) * T * D, bytes, &sm.full[s]);
        }
        __syncwarp();
        ++seq;
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int sub = lane & 7;   // lane within the slot's 8 lanes (K phase)
    const int sig = lane >> 3;  // slot within the warp's 4-slot group (K phase)

    float qf[G][DPL];  // query heads, pre-scaled to the log2 domain
#pragma unroll
    for (int i = 0; i < G; ++i) {
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        const uint4 w = *reinterpret_cast<const uint4*>(qrow + i * D + c * 64 + sub * 8);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          qf[i][c * 8 + 2 * k] = bf16lo(ww[k]) * p.qscale2;
          qf[i][c * 8 + 2 * k + 1] = bf16hi(ww[k]) * p.qscale2;
        }
      }
    }

    int head_base_lane = 0;  // first head whose sums this lane holds
    float rmax[RC];
#pragma unroll
    for (int k = 0; k < RC; ++k) rmax[k] = -INFINITY;
    const bool writer = (sub & Geo::BFLY) == 0;

    // K phase: logits of every filled slot of the chunk
    int seq = 0;
    for (int tile = 0; tile < ntiles; ++tile) {
      if (!tile_filled<T>(pos_s, tile, nvalid, lane)) continue;
      const int s = seq % kStages;
      const uint32_t par = uint32_t(seq / kStages) & 1u;
      if (!mbar_wait_bounded(&sm.full[s], par, kWaitLimitNs)) flag_error(&sm.err, p.status);
      const unsigned char* kt = ring + s * kTileBytes;
      const int ns = min(T, nvalid - tile * T);
#pragma unroll
      for (int grp = warp; grp < GROUPS; grp += kConsumerWarps) {
        const int si = grp * 4 + sig;
        float a[kMaxG];
#pragma unroll
        for (int i = 0; i < kMaxG; ++i) a[i] = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          const uint4 w = *reinterpret_cast<const uint4*>(kt + si * (2 * D) + c * 128 + sub * 16);
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float k0 = bf16lo(ww[k]), k1 = bf16hi(ww[k]);
#pragma unroll
            for (int i = 0; i < G; ++i) {
              a[i] = fmaf(qf[i][c * 8 + 2 * k], k0, a[i]);
              a[i] = fmaf(qf[i][c * 8 + 2 * k + 1], k1, a[i]);
            }
          }
        }
        int hb = 0;
        rs_step<GP, 4>(a, sub, hb);
        rs_step<(GP > 1 ? GP / 2 : 1), 2>(a, sub, hb);
        rs_step<(GP > 2 ? GP / 4 : 1), 1>(a, sub, hb);
        head_base_lane = hb;
        const int j = tile * T + si;
        const bool valid = (si < ns) && (pos_s[j] >= 0);
#pragma unroll
        for (int k = 0; k < RC; ++k) {
          const int h = hb + k;
          const float x = valid ? a[k] : -INFINITY;
          if (h < G) {
            if (writer) pl[j * GP + h] = x;
            rmax[k] = fmaxf(rmax[k], x);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
      ++seq;
    }

    // chunk max per head
    if (ntiles == 0) {  // no K tile processed: still define the lane's heads
      int hb = 0;
      if (GP >= 2 && (sub & 4)) hb += GP / 2;
      if (GP >= 4 && (sub & 2)) hb += GP / 4;
      if (GP >= 8 && (sub & 1)) hb += GP / 8;
      head_base_lane = hb;
    }
#pragma unroll
    for (int k = 0; k < RC; ++k) {
      rmax[k] = fmaxf(rmax[k], __shfl_xor_sync(0xffffffffu, rmax[k], 8));
      rmax[k] = fmaxf(rmax[k], __shfl_xor_sync(0xffffffffu, rmax[k], 16));
      const int h = head_base_lane + k;
      if (sig == 0 && writer && h < G) sm.wmax[warp][h] = rmax[k];
    }
    named_barrier(1, kConsumers);

    const int my_h = lane % GP;  // head of this lane in the probability pass
    float my_m = -INFINITY;
    if (my_h < G) {
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) my_m = fmaxf(my_m, sm.wmax[w][my_h]);
    }

    // V phase: p = 2^(s - m) in place, o += p v
    float o[G][DV];
#pragma unroll
    for (int i = 0; i < G; ++i)
#pragma unroll
      for (int d = 0; d < DV; ++d) o[i][d] = 0.f;
    float lsum = 0.f;
    for (int tile = 0; tile < ntiles; ++tile) {
      if (!tile_filled<T>(pos_s, tile, nvalid, lane)) continue;
      const int s = seq % kStages;
      const uint32_t par = uint32_t(seq / kStages) & 1u;
      if (!mbar_wait_bounded(&sm.full[s], par, kWaitLimitNs)) flag_error(&sm.err, p.status);
      const unsigned char* vt = ring + s * kTileBytes;
      const int ns = min(T, nvalid - tile * T);
#pragma unroll
      for (int idx = lane; idx < TPW * GP; idx += 32) {
        const int j = tile * T + warp * TPW + idx / GP;
        if (my_h < G) {
          const float x = pl[j * GP + my_h];
          const float pv = (x == -INFINITY) ? 0.f : exp2f(x - my_m);
          pl[j * GP + my_h] = pv;
          lsum += pv;
        }
      }
      __syncwarp();
#pragma unroll 4
      for (int u = 0; u < TPW; ++u) {
        const int si = warp * TPW + u;
        const int j = tile * T + si;
        if (si >= ns || pos_s[j] < 0) continue;  // warp-uniform
        float pv[GP];
        if constexpr (GP >= 4) {
#pragma unroll
          for (int h4 = 0; h4 < GP; h4 += 4) {
            const float4 f = *reinterpret_cast<const float4*>(pl + j * GP + h4);
            pv[h4] = f.x; pv[h4 + 1] = f.y; pv[h4 + 2] = f.z; pv[h4 + 3] = f.w;
          }
        } else if constexpr (GP == 2) {
          const float2 f = *reinterpret_cast<const float2*>(pl + j * GP);
          pv[0] = f.x; pv[1] = f.y;
        } else {
          pv[0] = pl[j];
        }
        float vf[DV];
        if constexpr (DV == 4) {
          const uint2 w = *reinterpret_cast<const uint2*>(vt + si * (2 * D) + lane * 8);
          vf[0] = bf16lo(w.x); vf[1] = bf16hi(w.x); vf[2] = bf16lo(w.y); vf[3] = bf16hi(w.y);
        } else {
          const uint32_t w = *reinterpret_cast<const uint32_t*>(vt + si * (2 * D) + lane * 4);
          vf[0] = bf16lo(w); vf[1] = bf16hi(w);
        }
#pragma unroll
        for (int i = 0; i < G; ++i)
#pragma unroll
          for (int d = 0; d < DV; ++d) o[i][d] = fmaf(pv[i], vf[d], o[i][d]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
      ++seq;
    }

    // chunk sums per head
#pragma unroll
    for (int m = GP; m < 32; m <<= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, m);
    if (lane < G) sm.wsum[warp][lane] = lsum;

    // partial outputs of the 4 warps -> xo (the ring is free: all tiles consumed)
    named_barrier(1, kConsumers);
    float* red = reinterpret_cast<float*>(ring);  // [warp][G][D]
#pragma unroll
    for (int i = 0; i < G; ++i)
#pragma unroll
      for (int d = 0; d < DV; ++d) red[(warp * G + i) * D + lane * DV + d] = o[i][d];
    named_barrier(1, kConsumers);
    for (int e = tid; e < G * D; e += kConsumers) {
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) acc += red[w * G * D + e];
      xo[e] = acc;
    }
    if (tid < G) {
      float mm = -INFINITY, ll = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        mm = fmaxf(mm, sm.wmax[w][tid]);
        ll += sm.wsum[w][tid];
      }
      sm.m[tid] = mm;
      sm.l[tid] = ll;
    }
  }
  __syncthreads();

  // -------------------------------------------- cluster exchange: max / sum
  cluster.sync();
  if (tid < G) {
    const int i = tid;
    float M = sm.s_new[i];
    for (int r = 0; r < S; ++r) M = fmaxf(M, cluster.map_shared_rank(&sm, r)->m[i]);
    float L = exp2f(sm.s_new[i] - M);
    for (int r = 0; r < S; ++r) {
      const Small<GP>* pr = cluster.map_shared_rank(&sm, r);
      const float cf = exp2f(pr->m[i] - M);  // 0 for an empty chunk (m = -inf)
      sm.cf[r][i] = cf;
      L += pr->l[i] * cf;
    }
    sm.Mg[i] = M;
    sm.Lg[i] = L;
  } else if (tid == 32) {
    int mx = -1, fr = INT_MAX, er = 0;
    for (int r = 0; r < S; ++r) {
      const Small<GP>* pr = cluster.map_shared_rank(&sm, r);
      mx = max(mx, pr->maxpos);
      fr = min(fr, pr->first_free);
      er |= pr->err;
    }
    sm.g_t = mx + 1;
    sm.g_free = fr;
    sm.g_err = er;
  }
  __syncthreads();

  // ----------------------------------------------- scores of own slots
  const bool full_row = (sm.g_free == INT_MAX);
  if (EVICT) {
    unsigned long long k1 = kNoKey, k2 = kNoKey;
    if (full_row && !sm.g_err) {
      float w[G];
#pragma unroll
      for (int i = 0; i < G; ++i) w[i] = sm.cf[rank][i] / sm.Lg[i] * (1.0f / G);
      const int lim = sm.g_t - p.window;
      for (int j = tid; j < nvalid; j += kThreads) {
        const int gj = slot0 + j;
        if (gj < p.sink || pos_s[j] >= lim) continue;
        float sc = 0.f;
#pragma unroll
        for (int i = 0; i < G; ++i) sc = fmaf(pl[j * GP + i], w[i], sc);
        top2_insert(k1, k2, (static_cast<unsigned long long>(__float_as_uint(sc)) << 32) |
                                static_cast<unsigned int>(gj));
      }
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) {
      const unsigned long long o1 = __shfl_xor_sync(0xffffffffu, k1, m);
      const unsigned long long o2 = __shfl_xor_sync(0xffffffffu, k2, m);
      top2_merge(k1, k2, o1, o2);
    }
    if (lane == 0) {
      sm.wk1[warp] = k1;
      sm.wk2[warp] = k2;
    }
  }

  // ------------------------------------------ output: this CTA's share
  {
    constexpr int E = G * D;
    const int per = (E + S - 1) / S;
    const int e0 = rank * per, e1 = min(E, e0 + per);
    const uint16_t* vn = p.v_new + size_t(row) * D;
    for (int e = e0 + tid; e < e1; e += kThreads) {
      const int i = e / D, d = e - i * D;
      float acc = exp2f(sm.s_new[i] - sm.Mg[i]) * __uint_as_float(uint32_t(vn[d]) << 16);
      for (int r = 0; r < S; ++r) acc = fmaf(cluster.map_shared_rank(xo, r)[e], sm.cf[r][i], acc);
      p.out[size_t(row) * E + e] = acc / sm.Lg[i];
    }
  }

  if (EVICT) {
    __syncthreads();
    if (tid == 0) {
      unsigned long long k1 = kNoKey, k2 = kNoKey;
      for (int w = 0; w < kWarps; ++w) top2_merge(k1, k2, sm.wk1[w], sm.wk2[w]);
      sm.key1 = k1;
      sm.key2 = k2;
    }
    cluster.sync();  // keys published
    if (tid == 0) {
      unsigned long long g1 = kNoKey, g2 = kNoKey;
      for (int r = 0; r < S; ++r) {
        const Small<GP>* pr = cluster.map_shared_rank(&sm, r);
        top2_merge(g1, g2, pr->key1, pr->key2);
      }
      int refine = 0;
      if (g1 != kNoKey && g2 != kNoKey) {
        const float s1 = __uint_as_float(uint32_t(g1 >> 32));
        const float s2 = __uint_as_float(uint32_t(g2 >> 32));
        refine = (s2 <= s1 * (1.0f + kTieRel)) ? 1 : 0;
      }
      sm.g_refine = refine;
      sm.g_slot = (g1 == kNoKey) ? -1 : int(uint32_t(g1 & 0xffffffffull));
      // the published key1/key2 stay untouched: peers may still be reading them
      sm.g_key1 = g1;
    }
    __syncthreads();

    if (sm.g_refine) {  // identical decision in every CTA of the cluster
      // fp64 rescoring of the candidates within the tie band
      const float s1 = __uint_as_float(uint32_t(sm.g_key1 >> 32));
      const float thr = s1 * (1.0f + kTieRel);
      float w[G];
#pragma unroll
      for (int i = 0; i < G; ++i) w[i] = sm.cf[rank][i] / sm.Lg[i] * (1.0f / G);
      const int lim = sm.g_t - p.window;
      double best = INFINITY;
      int bslot = INT_MAX;
      for (int j = tid; j < nvalid; j += kThreads) {
        const int gj = slot0 + j;
        if (gj < p.sink || pos_s[j] >= lim) continue;
        float sc = 0.f;
#pragma unroll
        for (int i = 0; i < G; ++i) sc = fmaf(pl[j * GP + i], w[i], sc);
        if (sc > thr) continue;
        const uint16_t* krow = p.kcache + (size_t(row) * N + gj) * D;
        double tot = 0.0;
        for (int i = 0; i < G; ++i) {
          double dot = 0.0;
          for (int d = 0; d < D; ++d) dot = fma(bf16_to_f64(qrow[i * D + d]), bf16_to_f64(krow[d]), dot);
          tot += exp2(dot * p.qscale2_64 - double(sm.Mg[i])) / double(sm.Lg[i]);
        }
        tot /= double(G);
        if (tot < best || (tot == best && gj < bslot)) {
          best = tot;
          bslot = gj;
        }
      }
#pragma unroll
      for (int m = 16; m > 0; m >>= 1) {
        const double ob = __shfl_xor_sync(0xffffffffu, best, m);
        const int os = __shfl_xor_sync(0xffffffffu, bslot, m);
        if (ob < best || (ob == best && os < bslot)) {
          best = ob;
          bslot = os;
        }
      }
      if (lane == 0) {
        sm.wref[warp] = best;
        sm.wref_slot[warp] = bslot;
      }
      __syncthreads();
      if (tid == 0) {
        double b = INFINITY;
        int bs = INT_MAX;
        for (int w2 = 0; w2 < kWarps; ++w2)
          if (sm.wref[w2] < b || (sm.wref[w2] == b && sm.wref_slot[w2] < bs)) {
            b = sm.wref[w2];
            bs = sm.wref_slot[w2];
          }
        sm.ref_score = b;
        sm.ref_slot = bs;
      }
      cluster.sync();  // rescoring results published
      if (tid == 0) {
        double b = INFINITY;
        int bs = INT_MAX;
        for (int r = 0; r < S; ++r) {
          const Small<GP>* pr = cluster.map_shared_rank(&sm, r);
          if (pr->ref_score < b || (pr->ref_score == b && pr->ref_slot < bs)) {
            b = pr->ref_score;
            bs = pr->ref_slot;
          }
        }
        if (bs != INT_MAX) sm.g_slot = bs;
      }
      __syncthreads();
    }

    // ------------------------------------------------ in-place eviction
    if (rank == 0) {
      int e, ev;
      if (sm.g_err) {
        e = -1;
        ev = -2;
      } else if (!full_row) {
        e = sm.g_free;
        ev = -1;
      } else if (sm.g_slot < 0) {
        e = -1;
        ev = -2;
        if (tid == 0) atomicOr(p.status, LF_STATUS_NO_CANDIDATE);
      } else {
        e = sm.g_slot;
        ev = e;
      }
      if (e >= 0) {
        constexpr int V16 = D / 8;  // 16-byte vectors per row
        if (tid < V16) {
          reinterpret_cast<uint4*>(p.kcache + (size_t(row) * N + e) * D)[tid] =
              reinterpret_cast<const uint4*>(p.k_new + size_t(row) * D)[tid];
        } else if (tid < 2 * V16) {
          reinterpret_cast<uint4*>(p.vcache + (size_t(row) * N + e) * D)[tid - V16] =
              reinterpret_cast<const uint4*>(p.v_new + size_t(row) * D)[tid - V16];
        } else if (tid == 2 * V16) {
          p.pos[size_t(row) * N + e] = sm.g_t;
        }
      }
      if (tid == 0) p.evicted[row] = ev;
    }
  }

  // after an error, do not leave with bulk copies still landing in shared memory
  if (sm.err && warp == kConsumerWarps && lane == 0) {
    int nseq = 0;
    for (int phase = 0; phase < 2; ++phase)
      for (int tile = 0; tile < ntiles; ++tile) {
        bool any = false;
        for (int k = 0; k < T; ++k) {
          const int j = tile * T + k;
          any |= (j < nvalid) && (pos_s[j] >= 0);
        }
        nseq += any ? 1 : 0;
      }
    for (int q = max(0, nseq - kStages); q < nseq; ++q)
      mbar_wait_bounded(&sm.full[q % kStages], uint32_t(q / kStages) & 1u, kWaitLimitNs);
  }
  cluster.sync();  // no CTA leaves while a peer may still read its shared memory
}

// --------------------------------------------------------------- prefill
__global__ void prefill_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, int n,
                               uint4* __restrict__ kc, uint4* __restrict__ vc,
                               int32_t* __restrict__ pos, int budget, int rows, int vec_per_row) {
  const size_t stride = size_t(gridDim.x) * blockDim.x;
  const size_t tid = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t per_row = size_t(n) * vec_per_row;
  const size_t total = per_row * rows;
  for (size_t i = tid; i < total; i += stride) {
    const size_t r = i / per_row, rest = i - r * per_row;
    const size_t dst = r * size_t(budget) * vec_per_row + rest;
    kc[dst] = k[i];
    vc[dst] = v[i];
  }
  const size_t ptotal = size_t(rows) * budget;
  for (size_t i = tid; i < ptotal; i += stride) {
    const int j = int(i % budget);
    pos[i] = j < n ? j : -1;
  }
}

}  // namespace lf

// ======================================================================
// host side
// ======================================================================

struct lf_ctx {
  int B, Hq, Hkv, D, G, max_budget;
  cudaStream_t stream;
  int device;
  int sm_count;
  int smem_optin;
  int split_override;
  int* status;  // device status word
  int last_bits;
  unsigned magic;
};

namespace {

constexpr unsigned kMagic = 0x4c46444bu;

bool aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

bool valid_handle(lf_handle h) { return h != nullptr && h->magic == kMagic; }

template <int D, int G>
size_t smem_for(int chunk) {
  return lf::Geometry<D, G>::smem_bytes(chunk);
}

size_t smem_bytes(int D, int G, int chunk) {
#define LF_CASE(DD, GG) \
  if (D == DD && G == GG) return smem_for<DD, GG>(chunk);
  LF_CASE(64, 1) LF_CASE(64, 2) LF_CASE(64, 3) LF_CASE(64, 4)
  LF_CASE(64, 5) LF_CASE(64, 6) LF_CASE(64, 7) LF_CASE(64, 8)
  LF_CASE(128, 1) LF_CASE(128, 2) LF_CASE(128, 3) LF_CASE(128, 4)
  LF_CASE(128, 5) LF_CASE(128, 6) LF_CASE(128, 7) LF_CASE(128, 8)
#undef LF_CASE
  return 0;
}

int tile_slots(int D) { return lf::kTileBytes / (2 * D); }

int chunk_for(int budget, int split, int D) {
  const int T = tile_slots(D);
  const int per = (budget + split - 1) / split;
  return ((per + T - 1) / T) * T;
}

// Split of one row over a cluster: enough CTAs to fill the GPU several
// times over, chunks of at least 256 slots, and shared memory in budget.
int choose_split(const lf_ctx* c, int budget) {
  if (c->split_override > 0) return c->split_override;
  const int rows = c->B * c->Hkv;
  int S = 1;
  while (S < 8 && rows * S < 4 * c->sm_count && chunk_for(budget, 2 * S, c->D) >= 256) S *= 2;
  // long rows: keep each CTA's chunk modest so several CTAs fit per SM
  while (S < 8 && chunk_for(budget, S, c->D) > 512) S *= 2;
  while (S < lf::kMaxSplit &&
         smem_bytes(c->D, c->G, chunk_for(budget, S, c->D)) > size_t(c->smem_optin))
    S *= 2;
  return S;
}

template <int D, int G, bool EVICT>
cudaError_t launch_t(const lf::Params& p, int rows, int S, size_t smem, cudaStream_t st) {
  auto kern = lf::fused_decode_kernel<D, G, EVICT>;
  static std::mutex mu;
  static size_t smem_set = 0;
  static bool nonportable = false;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (smem > smem_set) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           int(smem));
      if (e != cudaSuccess) return e;
      smem_set = smem;
    }
    if (S > 8 && !nonportable) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
      nonportable = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(S), unsigned(rows), 1);
  cfg.blockDim = dim3(lf::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = unsigned(S);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <bool EVICT>
cudaError_t launch(int D, int G, const lf::Params& p, int rows, int S, size_t smem,
                   cudaStream_t st) {
#define LF_CASE(DD, GG) \
  if (D == DD && G == GG) return launch_t<DD, GG, EVICT>(p, rows, S, smem, st);
  LF_CASE(64, 1) LF_CASE(64, 2) LF_CASE(64, 3) LF_CASE(64, 4)
  LF_CASE(64, 5) LF_CASE(64, 6) LF_CASE(64, 7) LF_CASE(64, 8)
  LF_CASE(128, 1) LF_CASE(128, 2) LF_CASE(128, 3) LF_CASE(128, 4)
  LF_CASE(128, 5) LF_CASE(128, 6) LF_CASE(128, 7) LF_CASE(128, 8)
#undef LF_CASE
  return cudaErrorInvalidValue;
}

int run_decode(lf_handle h, const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
               uint16_t* kcache, uint16_t* vcache, int32_t* pos, int budget, int sink,
               int window, float* out, int32_t* evicted, bool evict) {
  if (!valid_handle(h)) return LF_ENOTINIT;
  if (!q || !k_new || !v_new || !kcache || !vcache || !pos || !out) return LF_EINVAL;
  if (evict && !evicted) return LF_EINVAL;
  if (!aligned(q, 16) || !aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(kcache, 16) ||
      !aligned(vcache, 16) || !aligned(out, 16) || !aligned(pos, 4) ||
      (evicted && !aligned(evicted, 4)))
    return LF_EINVAL;
  if (budget < 1 || budget > h->max_budget) return LF_EINVAL;
  if (evict && (sink < 0 || window < 1 || budget <= sink + window)) return LF_EINVAL;

  const int S = choose_split(h, budget);
  const int chunk = chunk_for(budget, S, h->D);
  const size_t smem = smem_bytes(h->D, h->G, chunk);
  if (smem > size_t(h->smem_optin)) return LF_EINVAL;

  lf::Params p;
  p.q = q;
  p.k_new = k_new;
  p.v_new = v_new;
  p.kcache = kcache;
  p.vcache = vcache;
  p.pos = pos;
  p.out = out;
  p.evicted = evicted;
  p.status = h->status;
  p.budget = budget;
  p.chunk = chunk;
  p.sink = evict ? sink : 0;
  p.window = evict ? window : 1;
  p.pos_vec4 = (budget % 4 == 0 && aligned(pos, 16)) ? 1 : 0;
  p.qscale2_64 = 1.4426950408889634 / sqrt(double(h->D));
  p.qscale2 = float(p.qscale2_64);

  const int rows = h->B * h->Hkv;
  cudaError_t e = evict ? launch<true>(h->D, h->G, p, rows, S, smem, h->stream)
                        : launch<false>(h->D, h->G, p, rows, S, smem, h->stream);
  return e == cudaSuccess ? LF_OK : LF_ECUDA;
}

}  // namespace

extern "C" {

int lf_version(void) { return (1 << 16) | 0; }

const char* lf_strerror(int code) {
  switch (code) {
    case LF_OK: return "LF_OK";
    case LF_EINVAL: return "LF_EINVAL: invalid argument";
    case LF_ENOTINIT: return "LF_ENOTINIT: null or destroyed handle";
    case LF_ECUDA: return "LF_ECUDA: CUDA runtime error";
    case LF_EDEVICE: return "LF_EDEVICE: the kernel flagged an error";
    case LF_EUNSUPPORTED: return "LF_EUNSUPPORTED: device is not sm_100";
    default: return "LF_E?: unknown code";
  }
}

int lf_init(lf_handle* out, int B, int Hq, int Hkv, int D, int max_budget, void* cuda_stream) {
  if (!out) return LF_EINVAL;
  *out = nullptr;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return LF_EINVAL;
  const int G = Hq / Hkv;
  if (G > lf::kMaxG || (D != 64 && D != 128)) return LF_EINVAL;
  if (max_budget < 1 || max_budget > (1 << 22)) return LF_EINVAL;
  if (long(B) * Hkv > 65535) return LF_EINVAL;  // grid y holds the rows

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LF_ECUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return LF_ECUDA;
  if (prop.major != 10 || prop.minor != 0) return LF_EUNSUPPORTED;

  lf_ctx* c = static_cast<lf_ctx*>(calloc(1, sizeof(lf_ctx)));
  if (!c) return LF_ECUDA;
  c->B = B;
  c->Hq = Hq;
  c->Hkv = Hkv;
  c->D = D;
  c->G = G;
  c->max_budget = max_budget;
  c->stream = static_cast<cudaStream_t>(cuda_stream);
  c->device = dev;
  c->sm_count = prop.multiProcessorCount;
  c->smem_optin = int(prop.sharedMemPerBlockOptin);
  c->split_override = 0;
  c->magic = kMagic;
  if (cudaMalloc(&c->status, sizeof(int)) != cudaSuccess) {
    free(c);
    return LF_ECUDA;
  }
  if (cudaMemset(c->status, 0, sizeof(int)) != cudaSuccess) {
    cudaFree(c->status);
    free(c);
    return LF_ECUDA;
  }
  *out = c;
  return LF_OK;
}

int lf_set_stream(lf_handle h, void* cuda_stream) {
  if (!valid_handle(h)) return LF_ENOTINIT;
  h->stream = static_cast<cudaStream_t>(cuda_stream);
  return LF_OK;
}

int lf_set_split(lf_handle h, int split) {
  if (!valid_handle(h)) return LF_ENOTINIT;
  if (split < 0 || split > lf::kMaxSplit || (split & (split - 1)) != 0) return LF_EINVAL;
  h->split_override = split;
  return LF_OK;
}

int lf_get_split(lf_handle h, int budget) {
  if (!valid_handle(h)) return LF_ENOTINIT;
  if (budget < 1 || budget > h->max_budget) return LF_EINVAL;
  return choose_split(h, budget);
}

int lf_prefill_cache(lf_handle h, const uint16_t* k, const uint16_t* v, int n, uint16_t* kcache,
                     uint16_t* vcache, int32_t* pos, int budget) {
  if (!valid_handle(h)) return LF_ENOTINIT;
  if (budget < 1 || budget > h->max_budget || n < 0 || n > budget) return LF_EINVAL;
  if (!kcache || !vcache || !pos || (n > 0 && (!k || !v))) return LF_EINVAL;
  if (!aligned(kcache, 16) || !aligned(vcache, 16) || !aligned(pos, 4) ||
      (n > 0 && (!aligned(k, 16) || !aligned(v, 16))))
    return LF_EINVAL;
  const int rows = h->B * h->Hkv;
  const int vec = h->D / 8;
  const size_t work = size_t(rows) * (size_t(n) * vec > size_t(budget) ? size_t(n) * vec : size_t(budget));
  int blocks = int((work + 255) / 256);
  if (blocks > h->sm_count * 8) blocks = h->sm_count * 8;
  if (blocks < 1) blocks = 1;
  lf::prefill_kernel<<<blocks, 256, 0, h->stream>>>(
      reinterpret_cast<const uint4*>(k), reinterpret_cast<const uint4*>(v), n,
      reinterpret_cast<uint4*>(kcache), reinterpret_cast<uint4*>(vcache), pos, budget, rows, vec);
  return cudaGetLastError() == cudaSuccess ? LF_OK : LF_ECUDA;
}

int lf_decode_step(lf_handle h, const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                   uint16_t* kcache, uint16_t* vcache, int32_t* pos, int budget, int sink,
                   int window, float* out, int32_t* evicted_idx) {
  return run_decode(h, q, k_new, v_new, kcache, vcache, pos, budget, sink, window, out,
                    evicted_idx, true);
}

int lf_decode_attention(lf_handle h, const uint16_t* q, const uint16_t* k_new,
                        const uint16_t* v_new, const uint16_t* kcache, const uint16_t* vcache,
                        const int32_t* pos, int budget, float* out) {
  return run_decode(h, q, k_new, v_new, const_cast<uint16_t*>(kcache),
                    const_cast<uint16_t*>(vcache), const_cast<int32_t*>(pos), budget, 0, 1, out,
                    nullptr, false);
}

int lf_get_status(lf_handle h) {
  if (!valid_handle(h)) return LF_ENOTINIT;
  if (cudaStreamSynchronize(h->stream) != cudaSuccess) return LF_ECUDA;
  int bits = 0;
  if (cudaMemcpy(&bits, h->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return LF_ECUDA;
  if (bits != 0 && cudaMemset(h->status, 0, sizeof(int)) != cudaSuccess) return LF_ECUDA;
  h->last_bits = bits;
  return bits ? LF_EDEVICE : LF_OK;
}

int lf_status_bits(lf_handle h) {
  if (!valid_handle(h)) return LF_ENOTINIT;
  return h->last_bits;
}

int lf_destroy(lf_handle h) {
  if (!valid_handle(h)) return LF_ENOTINIT;
  cudaStreamSynchronize(h->stream);
  cudaFree(h->status);
  h->magic = 0;
  free(h);
  return LF_OK;
}

// ----------------------------------------------------------------------
// Allocation-free entry point.  Its scratch (the kernel's status word) is a
// file-scope device array; host code only ever passes the device address
// that cudaGetSymbolAddress returns for it, looked up once per device.
// ----------------------------------------------------------------------

constexpr int kNoAllocScratchBytes = 256;
constexpr int kNoAllocMaxDevices = 64;
static __device__ __align__(256) int g_lf_noalloc_scratch[kNoAllocScratchBytes / sizeof(int)];

namespace {

struct NoAllocDevice {
  bool ready;
  int* scratch;  // device address of g_lf_noalloc_scratch on this device
  int sm_count;
  int smem_optin;
  int major, minor;
};

std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc_dev[kNoAllocMaxDevices];

// Once per device, with that device current.
int noalloc_setup(int dev, NoAllocDevice** out) {
  if (dev < 0 || dev >= kNoAllocMaxDevices) return LF_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocDevice& d = g_noalloc_dev[dev];
  if (!d.ready) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_lf_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return LF_ECUDA;
    int sms = 0, optin = 0, major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return LF_ECUDA;
    d.scratch = static_cast<int*>(ptr);
    d.sm_count = sms;
    d.smem_optin = optin;
    d.major = major;
    d.minor = minor;
    d.ready = true;
  }
  *out = &d;
  return LF_OK;
}

}  // namespace

int lf_decode_step_noalloc(const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                           uint16_t* kcache, uint16_t* vcache, int32_t* pos, int B, int Hq,
                           int Hkv, int D, int budget, int sink, int window, float* out,
                           int32_t* evicted_idx, void* cuda_stream) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return LF_EINVAL;
  const int G = Hq / Hkv;
  if (G > lf::kMaxG || (D != 64 && D != 128)) return LF_EINVAL;
  if (budget < 1 || budget > (1 << 22) || long(B) * Hkv > 65535) return LF_EINVAL;
  // scratch this call needs: one status word
  const size_t scratch_needed = sizeof(int);
  if (scratch_needed > size_t(kNoAllocScratchBytes)) return LF_EINVAL;

  // the argument checks of lf_decode_step, before anything is enqueued
  if (!q || !k_new || !v_new || !kcache || !vcache || !pos || !out || !evicted_idx)
    return LF_EINVAL;
  if (!aligned(q, 16) || !aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(kcache, 16) ||
      !aligned(vcache, 16) || !aligned(out, 16) || !aligned(pos, 4) || !aligned(evicted_idx, 4))
    return LF_EINVAL;
  if (sink < 0 || window < 1 || budget <= sink + window) return LF_EINVAL;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LF_ECUDA;
  NoAllocDevice* d = nullptr;
  const int rc = noalloc_setup(dev, &d);
  if (rc != LF_OK) return rc;
  if (d->major != 10 || d->minor != 0) return LF_EUNSUPPORTED;

  lf_ctx c;  // on the stack: nothing is allocated
  memset(&c, 0, sizeof(c));
  c.B = B;
  c.Hq = Hq;
  c.Hkv = Hkv;
  c.D = D;
  c.G = G;
  c.max_budget = budget;
  c.stream = static_cast<cudaStream_t>(cuda_stream);
  c.device = dev;
  c.sm_count = d->sm_count;
  c.smem_optin = d->smem_optin;
  c.split_override = 0;
  c.status = d->scratch;
  c.magic = kMagic;
  // the status word starts at zero for every call
  if (cudaMemsetAsync(d->scratch, 0, scratch_needed, c.stream) != cudaSuccess) return LF_ECUDA;
  return run_decode(&c, q, k_new, v_new, kcache, vcache, pos, budget, sink, window, out,
                    evicted_idx, true);
}

}  // extern "C"
