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
// Design.  One row = one (batch, KV head) pair; its K and V slabs are each
// [budget, D] of bf16 or E4M3 codes, contiguous.
//   * Persistent thread-block clusters: a cluster of S CTAs owns a row at a
//     time and splits its slots evenly (flash-decoding split); rows come from
//     a static stride, or (ragged batches) from a device counter that rank 0
//     reads and pushes to its peers.  A CTA has 11 consumer warps (8 for
//     groups of more than 4 heads) and 1 producer warp.
//   * The producer streams the chunk's K tiles, then its V tiles, into an
//     mbarrier-guarded ring without a pause between rows: while the
//     consumers finish one row, the next row's position table, query heads
//     and new K/V are loaded and its first tiles are in flight.  Tiles whose
//     slots are all free are never loaded.  No multicast.
//   * K phase, bf16: 128-slot K tiles by TMA tensor copies with 128-byte
//     swizzle; one consumer warp issues tcgen05.mma (M = 128 slots, N = 16
//     heads, K = 16) into a double-buffered TMEM accumulator; a warpgroup
//     reads it back with tcgen05.ld, one slot per thread.  E4M3: 1-D bulk
//     tiles, 8 lanes per slot, packed fp32x2 FMAs against pre-scaled query
//     heads held in a per-lane head order that lets the 8-lane reduce-scatter
//     run without selects.  Logits (log2 domain) stay in shared memory: the
//     exact normalised probabilities need the row-wide max and sum, which
//     only exist once every CTA of the cluster is done.
//   * V phase: p = 2^(s - m_cta), kept for the scores.  8-head groups with
//     bf16 at D = 128: TMA-swizzled V tiles, P as bf16 hi + lo rows of an
//     N = 32 tcgen05 B operand, O^T accumulated in TMEM.  Otherwise: o += p v
//     with 8 elements per lane and packed FMAs (the page-form score also sums
//     |v| there).
//   * Cluster exchange through distributed shared memory by st.async pushes
//     into per-row-parity buffers, completing bytes on the receiver's
//     mbarrier: row max / sum per head, newest position, lowest free slot and
//     the partial outputs; then each CTA scores its own slots (exact
//     normalised probability averaged over the group's heads, optionally
//     times ||v||_1), reduces packed (fp32 score bits << 32 | slot) keys to
//     the two lowest, and combines its share of the output.
//   * Near ties (two lowest scores within a relative 1e-4) are rescored in
//     fp64 from the cache, so the choice follows the exact ranking.
//   * CTA rank 0 writes k_new / v_new / t into the chosen slot (E4M3: the
//     quantised codes) after the key exchange, which every CTA enters only
//     after its last read of the row.
#pragma once
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <limits.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <mutex>

#include "lf_decode.h"
#include "lf_internal.h"
#include "lf_ptx.cuh"

namespace cg = cooperative_groups;

namespace lf {

constexpr int kMaxCW = 11;                  // most consumer warps of any variant
// P.V runs on the tensor cores for groups of at least this many (padded)
// heads.  At 4 heads the CUDA-core V phase measured 1.2% faster over a
// 20,000-step run (236.2 vs 239.1 us at batch 64, budget 4096); at 7 heads the
// tensor cores are 18% faster (69 vs 84 us at batch 16, budget 8192).
#ifndef LF_VMMA_MIN_GP
#define LF_VMMA_MIN_GP 8
#endif
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per barrier wait
constexpr float kTieRel = 1e-4f;                   // near-tie band rescored in fp64
constexpr unsigned long long kNoKey = ~0ull;
constexpr int kBarConsumers = 1;                   // named barrier of the consumer warps

// What the CTAs of a cluster send each other about one row (one copy per
// row parity, in every CTA).  Each CTA writes its own entries [rank] into
// every CTA's copy with st.async; the receiver's mbarrier counts the bytes.
template <int GP>
struct Rx {
  uint32_t sc[kMaxSplit][2 * GP + 4];     // per sender: m[GP], l[GP], maxpos, first_free, err
  unsigned long long key[kMaxSplit][2];   // per sender: two lowest candidate keys
  unsigned long long ref[kMaxSplit][2];   // per sender: fp64 rescoring (score bits, slot)
};

// CTA-local barriers and scalars.
template <int GP>
struct Local {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t row_full[2];  // row metadata (positions, q, k_new, v_new) landed
  uint64_t row_free[2];  // consumers are done with a metadata buffer
  uint64_t xa[2];        // cluster exchange 1 received: max / sum / positions / partial output
  uint64_t xb[2];        // cluster exchange 2 received: candidate keys
  uint64_t xc[2];        // cluster exchange 3 received: fp64 rescoring
  uint64_t grab_bar[2];  // dynamic schedule: the row rank 0 took for this CTA landed
  uint64_t mma_done[2];  // tensor-core K tile: accumulator [tb] written
  uint64_t tmem_free[2]; // tensor-core K tile: accumulator [tb] read back
  uint64_t mma_fin;      // tensor-core: everything issued has completed (exit)
  uint64_t pready[2];    // P.V on the tensor cores: P buffer [pb] written (all consumer warps)
  uint64_t vdone[2];     // P.V on the tensor cores: the MMAs reading P buffer [pb] completed
  uint32_t tmem_base;    // tensor-core: allocated TMEM address
  int grab_val[2];       // dynamic schedule: that row (-1: none left)
  int row_id[2];         // row of a metadata buffer (-1: no more rows)
  int row_nb[2];         // its budget (slots 0 .. nb - 1 exist)
  int row_bad[2];        // its budget was out of range (clamped, nothing written)
  float s_new[GP];
  float Mg[GP], Lg[GP];
  float cf[kMaxSplit][GP];
  float wmax[kMaxCW][GP];
  float wsum[kMaxCW][GP];
  int wpmax[kMaxCW], wpfree[kMaxCW];
  unsigned long long wk1[kMaxCW], wk2[kMaxCW];
  double wref[kMaxCW];
  int wrefs[kMaxCW];
  unsigned long long g_key1;
  int g_t, g_free, g_err, g_refine, g_slot;
  int err;
};

__host__ __device__ constexpr size_t align128(size_t x) { return (x + 127) & ~size_t(127); }
__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }

template <int D, int G, int KVB>
struct Geometry {
  static constexpr int GP = G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8;
  // Consumer warps.  One SM runs one CTA; with 12 warps a scheduler holds 3,
  // which leaves 168 registers per thread: 11 consumers + the producer.  The
  // 8-head variants need more registers per thread and keep 8 consumers.
  static constexpr int CW = GP >= 8 ? 8 : 11;
  static constexpr int kConsumers = CW * 32;
  static constexpr int kThreads = kConsumers + 32;  // + 1 producer warp
  // Bytes per ring stage: large tiles amortise the per-tile work.  A tile
  // holds 16 slots per consumer warp (176 at D = 128) for the small groups,
  // 32 KB for the 8-head variants (which keep twice the probabilities).
  static constexpr int kTile = GP >= 8 ? 32768 : CW * 16 * 2 * 128;
  static constexpr int ROWB = D * KVB;             // bytes of one cached K or V row
  static constexpr int T = kTile / ROWB;           // slots per tile
  // K phase: a slot's 8 lanes each take ROWB / 8 bytes in loads of LDB bytes
  // (EPL elements); load c of lane sub holds elements c*8*EPL + sub*EPL + e
  static constexpr int LB = ROWB / 8;
  static constexpr int LDB = LB < 16 ? LB : 16;
  static constexpr int NLD = LB / LDB;
  static constexpr int EPL = LDB / KVB;
  static constexpr int DPL = D / 8;                // K phase: elements per lane
  static constexpr int GROUPS = T / 4;             // K phase: 4-slot groups per tile
  static constexpr int GPW = GROUPS / CW;          // K phase: groups per warp per tile
  // K phase: groups computed together (more in flight hides latency; the
  // 8-head variants hold twice the query registers, so they take fewer)
  static constexpr int KU = GP >= 8 ? 1 : (GPW < 4 ? GPW : 4);
  static constexpr int VL = D / 8;                 // V phase: lanes per slot (8 dims each)
  static constexpr int SPV = 32 / VL;              // V phase: slots per warp pass
  static constexpr int TPW = T / CW;               // V phase: slots per warp per tile
  static constexpr int VU = TPW / SPV;             // V phase: slot passes per tile
  static constexpr int VUC = VU < VL ? VU : VL;    // V phase: passes per norm reduce-scatter
  // bf16 storage: Q.K on the tensor cores.  K tiles of TK slots arrive by TMA
  // tensor copies (KH boxes of 64 elements x TK slots, 128-byte swizzle); one
  // consumer warp issues tcgen05.mma (NB blocks of M = 128 slots, N = 16
  // heads, K = 16) into one of two TMEM accumulators; EPI_WG warpgroups read
  // them back, one slot per thread.
  static constexpr bool UMMA = KVB == 2;
  static constexpr int TK = UMMA ? 128 : T;        // slots per K tile
  static constexpr int NB = (TK + 127) / 128;      // M = 128 MMA blocks per K tile
  // both warpgroups read every tile, one block each
  static constexpr bool EPI_PAIR = CW >= 9 && NB == 2;
  static constexpr int KH = D / 64;                // 128-byte halves of a K row
  static constexpr int KS = D / 16;                // MMAs (k-steps of 16) per K tile
  static constexpr int kMmaN = 16;
  static constexpr int kQOpBytes = KH * kMmaN * 128;  // the query heads as the MMA's B operand
  static constexpr int EPI_WG = CW >= 9 ? 2 : 1;
  static constexpr int MMA_WARP = CW - 1;
  static constexpr uint32_t kTmemCols = 64;  // two K accumulators (NB x 16 columns each), then O
  static constexpr uint32_t kOCol = 2 * NB * kMmaN;  // P.V on the tensor cores: O^T's columns
  // P.V on the tensor cores (bf16, D = 128, not the page-form score): the
  // V tile is the MN-major A operand (M = 128 dims); the probabilities, split
  // into bf16 hi + lo parts, are the K-major B operand with N = 32 rows (hi
  // of the heads in rows 0-15, lo in rows 16-31): [atom of 64 slots][32 rows
  // x 128 B], double-buffered by V tile.  O^T's hi and lo columns are summed
  // when read back.
  static constexpr int NA = (T + 63) / 64;
  static constexpr int kPBytes = NA * 4096;
  static constexpr int kMmaNV = 32;
  static constexpr int kReaders = 4 * (EPI_PAIR ? 2 : 1);    // warps reading one accumulator
  static_assert(!UMMA || (TK * ROWB <= kTile && kTile % 1024 == 0 && 4 * EPI_WG <= MMA_WARP &&
                          GP <= 8 && KH >= 1 && TK % 8 == 0 && TK <= 256 && NB <= 2 &&
                          (TK * 128) % 1024 == 0),
                "tensor-core K tiles");
  static constexpr int BFLY = GP >= 8 ? 0 : GP == 4 ? 1 : GP == 2 ? 3 : 7;
  static constexpr size_t kMetaStride = align128(size_t(G) * D * 2 + 2 * D * 2);
  // per parity: this CTA's slice of every CTA's partial output, then Rx
  static constexpr size_t kPubStride = align128(size_t(G) * D * 4) + align128(sizeof(Rx<GP>));
  static_assert(GROUPS % CW == 0 && T % CW == 0 && TPW % SPV == 0 && CW <= kMaxCW, "tile split");
  static_assert(NLD * LDB == LB && (LDB == 8 || LDB == 16) && EPL % 8 == 0, "K loads");
  static_assert(VU % VUC == 0 && (VUC & (VUC - 1)) == 0, "V passes");

  struct Layout {
    size_t ring, pl, pos, red, pp, meta, pub, loc, total;
  };
  __host__ __device__ static size_t align1024(size_t x) { return (x + 1023) & ~size_t(1023); }
  __host__ __device__ static size_t roundup(size_t x, size_t m) { return (x + m - 1) / m * m; }
  __host__ __device__ static Layout layout(int chunk, int nst, bool vmma = false) {
    Layout L;
    size_t o = 0;
    L.ring = o; o = align128(o + size_t(nst) * kTile);
    // logits of whole tiles: the last tile of a chunk may be partial
    const size_t plslots = roundup(chunk, T) > roundup(chunk, TK) ? roundup(chunk, T) : roundup(chunk, TK);
    L.pl = o;   o = align128(o + plslots * GP * 4);
    L.pos = o;  o = align128(o + size_t(2) * chunk * 4);
    // the V phase's cross-warp reduction; the K phase's MMA B operand (the
    // query heads, 1024-byte aligned for the swizzle) shares the space
    // (P.V on the tensor cores: the query operand, then the two P buffers,
    // instead of the reduction buffer and the probability pairs)
    o = UMMA ? align1024(o) : o;
    const size_t redb = size_t(CW) * G * D * 4;
    const size_t tcb = size_t(kQOpBytes) + (vmma ? 2 * size_t(kPBytes) : 0);
    L.red = o;  o = align128(o + (vmma ? tcb : (UMMA && tcb > redb ? tcb : redb)));
    L.pp = o;   o = align128(o + (vmma ? 0 : size_t(CW) * TPW * GP * 8));
    L.meta = o; o = align128(o + 2 * kMetaStride);
    L.pub = o;  o = align128(o + 2 * kPubStride);
    L.loc = o;  o = align128(o + sizeof(Local<GP>));
    L.total = o;
    return L;
  }
};

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
// 2^x on the SFU (flushes results below 2^-126 to zero; such probabilities
// change no output, and equal zero scores are settled by the fp64 rescoring)
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ double bf16_to_f64(uint16_t b) {
  return static_cast<double>(__uint_as_float(static_cast<uint32_t>(b) << 16));
}
// two E4M3 codes (low byte first) -> two floats, exactly (through f16)
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xffffu),
                                                   __NV_E4M3);
  return __half22float2(__half2(h));
}
__device__ __forceinline__ double e4m3_to_f64(uint8_t c) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3);
  return static_cast<double>(__half2float(__half(h)));
}
// two floats -> two E4M3 codes (low byte first): round to nearest even,
// finite values beyond +-448 saturate
__device__ __forceinline__ uint32_t float2_to_e4m3x2(float2 f) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3));
}
// a cached element as fp64 (bf16, or the E4M3 code's value without its scale)
template <int KVB>
__device__ __forceinline__ double kv_to_f64(const unsigned char* row, int i) {
  if constexpr (KVB == 2) {
    return bf16_to_f64(reinterpret_cast<const uint16_t*>(row)[i]);
  } else {
    return e4m3_to_f64(row[i]);
  }
}
// Element pairs of a run of cached elements in shared memory: 16 or 8
// bytes at `src` (16-byte / 8-byte aligned) -> NP = bytes / (2 * KVB) pairs.
template <int KVB, int BYTES>
__device__ __forceinline__ void kv_pairs(const unsigned char* src, float2* out) {
  uint32_t w[BYTES / 4];
  if constexpr (BYTES == 16) {
    const uint4 x = *reinterpret_cast<const uint4*>(src);
    w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
  } else {
    static_assert(BYTES == 8, "8 or 16 bytes");
    const uint2 x = *reinterpret_cast<const uint2*>(src);
    w[0] = x.x; w[1] = x.y;
  }
#pragma unroll
  for (int m = 0; m < BYTES / 4; ++m) {
    if constexpr (KVB == 2) {
      out[m] = make_float2(__uint_as_float(w[m] << 16), __uint_as_float(w[m] & 0xffff0000u));
    } else {
      out[2 * m] = e4m3x2_to_float2(w[m]);
      out[2 * m + 1] = e4m3x2_to_float2(w[m] >> 16);
    }
  }
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
__device__ __forceinline__ void top2_warp(unsigned long long& k1, unsigned long long& k2) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) {
    const unsigned long long o1 = __shfl_xor_sync(0xffffffffu, k1, m);
    const unsigned long long o2 = __shfl_xor_sync(0xffffffffu, k2, m);
    top2_merge(k1, k2, o1, o2);
  }
}

// Any slot of tile `tile` (chunk-local) filled / every slot filled?  Warp-uniform.
// (T need not be a multiple of 32: every one of the tile's T slots is checked)
template <int T>
__device__ __forceinline__ bool tile_filled(const int* ps, int tile, int nvalid, int lane) {
  bool any = false;
#pragma unroll
  for (int k = 0; k < (T + 31) / 32; ++k) {
    const int o = k * 32 + lane;
    const int j = tile * T + o;
    any |= (o < T) && (j < nvalid) && (ps[j] >= 0);
  }
  return __any_sync(0xffffffffu, any);
}
template <int T>
__device__ __forceinline__ bool tile_full(const int* ps, int tile, int nvalid, int lane) {
  bool all = true;
#pragma unroll
  for (int k = 0; k < (T + 31) / 32; ++k) {
    const int o = k * 32 + lane;
    const int j = tile * T + o;
    all &= (o >= T) || ((j < nvalid) && (ps[j] >= 0));
  }
  return __all_sync(0xffffffffu, all);
}

// ---- cluster-scope mbarrier signalling (remote arrive, acquire wait)
__device__ __forceinline__ uint32_t map_rank(const void* p, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ uint32_t map_rank_addr(uint32_t smem_address, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_address), "r"(rank));
  return r;
}
__device__ __forceinline__ void arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ void fence_cluster() {
  asm volatile("fence.acq_rel.cluster;" ::: "memory");
}
// Non-blocking poll: a waiter suspended inside try_wait is not woken
// promptly by arrivals from other CTAs, so cluster-level waits poll.
__device__ __forceinline__ bool try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}
__device__ __forceinline__ bool wait_cluster_bounded(uint64_t* bar, uint32_t parity) {
  if (try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (try_wait_cluster(bar, parity)) return true;
    if (global_timer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// Asynchronous stores into the shared memory of a CTA of the cluster (this
// one included), completing `bytes` on that CTA's mbarrier.  No release
// fence is involved: a waiter that sees the mbarrier phase complete sees the
// data.  Addresses are shared::cluster addresses from map_rank().
__device__ __forceinline__ void st_async_b32(uint32_t addr, uint32_t v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(addr),
               "r"(v), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void st_async_b64(uint32_t addr, unsigned long long v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b64 [%0], %1, [%2];" ::"r"(addr),
               "l"(v), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void st_async_v4(uint32_t addr, float4 v, uint32_t bar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(addr),
      "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(bar)
      : "memory");
}

// One reduce-scatter step over the 8 lanes of a slot.  The lane keeps the
// first C/2 partial sums and sends the rest; because every lane holds its
// heads in the order k ^ perm(lane), the partner's second half holds exactly
// the heads of this lane's first half, so no select is needed.  With C == 1
// it is a butterfly step.
template <int C, int MASK, int NA>
__device__ __forceinline__ void rs_step(float (&a)[NA]) {
  if constexpr (C > 1) {
#pragma unroll
    for (int i = 0; i < C / 2; ++i) a[i] += __shfl_xor_sync(0xffffffffu, a[C / 2 + i], MASK);
  } else {
    a[0] += __shfl_xor_sync(0xffffffffu, a[0], MASK);
  }
}

// MODE: kAttendOnly (attention, nothing scored or written), kEvictMeanProb
// (evict the lowest head-averaged probability) or kEvictAlphaL1V (evict the
// lowest head-averaged probability times the L1 norm of the slot's value).
template <int D, int G, int MODE, int KVB>
__global__ void __launch_bounds__(Geometry<D, G, KVB>::kThreads, 1)
    fused_decode_kernel(const __grid_constant__ Params p) {
  using Geo = Geometry<D, G, KVB>;
  constexpr bool EVICT = MODE != kAttendOnly;
  constexpr bool L1V = MODE == kEvictAlphaL1V;
  // P.V on the tensor cores: bf16, D = 128, and not the page-form score
  // (which needs |v| of every slot on the CUDA cores)
  constexpr bool VMMA = Geo::UMMA && !L1V && D == 128 && (Geo::GP >= LF_VMMA_MIN_GP);
  constexpr int CW = Geo::CW, kConsumers = Geo::kConsumers;
  constexpr int T = Geo::T, GP = Geo::GP, DPL = Geo::DPL, ROWB = Geo::ROWB;
  constexpr int NLD = Geo::NLD, LDB = Geo::LDB, EPL = Geo::EPL;
  constexpr int GPW = Geo::GPW, KU = Geo::KU, VU = Geo::VU, VL = Geo::VL, SPV = Geo::SPV,
                TPW = Geo::TPW, VUC = Geo::VUC;
  static_assert(G >= 1 && G <= kMaxG, "group size");
  static_assert(D == 64 || D == 128, "head dim");

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int S = static_cast<int>(cluster.num_blocks());
  const int ncl = static_cast<int>(gridDim.y), cid = static_cast<int>(blockIdx.y);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int N = p.budget, chunk = p.chunk, nst = p.nstages;
  // A row's slots 0 .. nb - 1 are split evenly over the cluster (the shared
  // buffers are sized for nb = N): this CTA owns nvalid slots from slot0.
  struct RowGeo {
    int slot0, nvalid, ntiles;
  };
  auto row_geo = [&](int nb) {
    RowGeo g;
    const int ch = ((nb + S - 1) / S + 3) & ~3;
    g.slot0 = rank * ch;
    g.nvalid = max(0, min(ch, nb - g.slot0));
    g.ntiles = (g.nvalid + T - 1) / T;
    return g;
  };

  extern __shared__ __align__(1024) unsigned char smem[];
  const typename Geo::Layout L = Geo::layout(chunk, nst, VMMA);
  unsigned char* ring = smem + L.ring;
  float* pl = reinterpret_cast<float*>(smem + L.pl);     // [chunk][GP] logits, then p
  int* pos0 = reinterpret_cast<int*>(smem + L.pos);      // [2][chunk]
  float* red = reinterpret_cast<float*>(smem + L.red);   // [CW][G][D]
  float2* pp = reinterpret_cast<float2*>(smem + L.pp);   // [CW][TPW][GP] (p, p) pairs
  unsigned char* meta0 = smem + L.meta;                  // [2] {q[G][D], k_new[D], v_new[D]}
  unsigned char* pub0 = smem + L.pub;                    // [2] {xo[G][D], Pub}
  Local<GP>& loc = *reinterpret_cast<Local<GP>*>(smem + L.loc);

  // Bounded waits.  After a first wait has given up (error flagged), later
  // waits only poll once, so a failed launch ends quickly instead of waiting
  // the full limit at every barrier.
  auto wait_cta = [&](uint64_t* bar, uint32_t par) {
    if (*reinterpret_cast<volatile int*>(&loc.err)) {
      (void)mbar_try_wait(bar, par);
      return;
    }
    if (!mbar_wait_bounded(bar, par, kWaitLimitNs)) flag_error(&loc.err, p.status);
  };
  auto wait_cl = [&](uint64_t* bar, uint32_t par) {
    if (*reinterpret_cast<volatile int*>(&loc.err)) {
      (void)try_wait_cluster(bar, par);
      return;
    }
    if (!wait_cluster_bounded(bar, par)) flag_error(&loc.err, p.status);
  };
  auto pos_buf = [&](int b) { return pos0 + b * chunk; };
  auto q_buf = [&](int b) { return reinterpret_cast<uint16_t*>(meta0 + b * Geo::kMetaStride); };
  auto kn_buf = [&](int b) { return q_buf(b) + G * D; };
  auto vn_buf = [&](int b) { return q_buf(b) + G * D + D; };
  // [S][E / S] partial outputs of every sender for this CTA's output slice
  auto rxo_buf = [&](int b) { return reinterpret_cast<float*>(pub0 + b * Geo::kPubStride); };
  auto rx_buf = [&](int b) {
    return reinterpret_cast<Rx<GP>*>(pub0 + b * Geo::kPubStride + align128(size_t(G) * D * 4));
  };

  if (tid == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(&loc.full[s], 1);
      // a stage is released by every consumer warp, or (P.V on the tensor
      // cores) by the commit of the MMAs that read it
      mbar_init(&loc.empty[s], VMMA ? 1 : CW);
    }
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      mbar_init(&loc.row_full[b], 1);
      mbar_init(&loc.row_free[b], 1);
      mbar_init(&loc.xa[b], 1);  // the receiver's own expect-tx arrival + bytes
      mbar_init(&loc.xb[b], 1);
      mbar_init(&loc.xc[b], 1);
      mbar_init(&loc.grab_bar[b], 1);
      mbar_init(&loc.mma_done[b], 1);   // the MMA issuer's commit
      mbar_init(&loc.tmem_free[b], Geo::kReaders);  // the warps that read an accumulator
      mbar_init(&loc.pready[b], CW - 1);  // every consumer warp but the MMA issuer
      mbar_init(&loc.vdone[b], 1);
    }
    mbar_init(&loc.mma_fin, 1);
    loc.err = 0;
    fence_mbar_init();
  }
  if constexpr (Geo::UMMA) {
    if (warp == 0) tmem_alloc(&loc.tmem_base, Geo::kTmemCols);
    if constexpr (VMMA) {
      // the P operands' rows past the group's heads stay zero
      uint4* pz = reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(red) + Geo::kQOpBytes);
      for (int i = tid; i < 2 * Geo::kPBytes / 16; i += blockDim.x) pz[i] = make_uint4(0, 0, 0, 0);
      fence_proxy_async_smem();
    }
    tc_fence_before();
  }
  __syncthreads();
  if constexpr (Geo::UMMA) tc_fence_after();
  cluster.sync();  // every CTA's barriers exist before the first remote arrival

  // ring position: tiles issued (producer) or consumed (consumers) so far, and
  // the stage / phase parity of the next one; both sides walk the same sequence
  int seq = 0, stg = 0;
  uint32_t sph = 0;

  if (warp == CW) {
    // ================================================================ producer
    // The row of iteration it: a static stride over the rows, or (dynamic
    // schedule) the next row of a global counter, taken by rank 0 and sent
    // to every CTA of the cluster.  Every cluster takes rows until it gets
    // none, so a launch takes exactly rows + clusters values; the one that
    // takes the last value resets the counter for the next launch.
    auto next_row = [&](int it) -> int {
      if (!p.dyn) {
        const int r = cid + it * ncl;
        return r < p.rows ? r : -1;
      }
      const int b = it & 1;
      int r = -1;
      if (lane == 0) {
        if (rank == 0) {
          const unsigned g = atomicAdd(p.grab, 1u);
          const int rr = g < unsigned(p.rows) ? int(g) : -1;
          if (g == unsigned(p.rows + ncl - 1)) atomicExch(p.grab, 0u);
          const uint32_t va = smem_addr(&loc.grab_val[b]), ba = smem_addr(&loc.grab_bar[b]);
          for (int q = 0; q < S; ++q)
            st_async_b32(map_rank_addr(va, q), uint32_t(rr), map_rank_addr(ba, q));
        }
        mbar_arrive_expect_tx(&loc.grab_bar[b], 4u);
        wait_cl(&loc.grab_bar[b], uint32_t((it >> 1) & 1));
        r = loc.grab_val[b];
      }
      return __shfl_sync(0xffffffffu, r, 0);
    };
    // load the metadata of iteration it's row (or mark the end of the rows)
    auto issue_meta = [&](int it, int row) {
      const int b = it & 1;
      if (it >= 2 && lane == 0) wait_cta(&loc.row_free[b], uint32_t((it >> 1) & 1) ^ 1u);
      __syncwarp();
      if (row < 0) {
        if (lane == 0) {
          loc.row_id[b] = -1;
          mbar_arrive(&loc.row_full[b]);
        }
        __syncwarp();
        return;
      }
      int nb = N, bad = 0;
      if (p.seq_budget) {
        nb = p.seq_budget[row / p.hkv];
        bad = (nb < 1 || nb > N) ? 1 : 0;
        nb = min(max(nb, 1), N);
      }
      const RowGeo rg = row_geo(nb);
      const int slot0 = rg.slot0, nvalid = rg.nvalid;
      int* ps = pos_buf(b);
      const int32_t* pg = p.pos + size_t(row) * N + slot0;
      const uint32_t mbytes = uint32_t(G * D * 2 + 2 * D * 2);
      const bool bulk = p.pos_bulk && (nvalid & 3) == 0;
      if (!bulk) {
        for (int j = lane; j < nvalid; j += 32) ps[j] = pg[j];
        __syncwarp();
        __threadfence_block();
      }
      if (lane == 0) {
        loc.row_id[b] = row;
        loc.row_nb[b] = nb;
        loc.row_bad[b] = bad;
        const uint32_t pbytes = bulk ? uint32_t(nvalid) * 4 : 0u;
        mbar_arrive_expect_tx(&loc.row_full[b], mbytes + pbytes);
        if (pbytes) bulk_copy_g2s(ps, pg, pbytes, &loc.row_full[b]);
        bulk_copy_g2s(q_buf(b), p.q + size_t(row) * G * D, G * D * 2, &loc.row_full[b]);
        bulk_copy_g2s(kn_buf(b), p.k_new + size_t(row) * D, D * 2, &loc.row_full[b]);
        bulk_copy_g2s(vn_buf(b), p.v_new + size_t(row) * D, D * 2, &loc.row_full[b]);
      }
      __syncwarp();
    };
    auto issue_tiles = [&](int it, int row, int phase) {
      const int* ps = pos_buf(it & 1);
      const RowGeo rg = row_geo(loc.row_nb[it & 1]);
      const int nvalid = rg.nvalid, ntiles = rg.ntiles;
      if constexpr (Geo::UMMA) {
        if (phase == 0) {  // K tiles: TMA tensor copies with 128-byte swizzle
          constexpr int TK = Geo::TK;
          const int ntk = (nvalid + TK - 1) / TK;
          const int y0 = row * N + rg.slot0;
          for (int tile = 0; tile < ntk; ++tile) {
            if (!tile_filled<TK>(ps, tile, nvalid, lane)) continue;
            const int s = stg;
            const uint32_t par = sph;
            if (lane == 0) {
              if (seq >= nst) wait_cta(&loc.empty[s], par ^ 1u);
              mbar_arrive_expect_tx(&loc.full[s], uint32_t(TK * ROWB));
#pragma unroll
              for (int h = 0; h < Geo::KH; ++h)
                tma_load_2d(ring + size_t(s) * Geo::kTile + h * (TK * 128), &p.kmap, h * 64,
                            y0 + tile * TK, &loc.full[s]);
            }
            __syncwarp();
            ++seq;
            if (++stg == nst) {
              stg = 0;
              sph ^= 1u;
            }
          }
          return;
        }
        if constexpr (VMMA) {  // V tiles: TMA tensor copies with 128-byte swizzle
          const int y0 = row * N + rg.slot0;
          for (int tile = 0; tile < ntiles; ++tile) {
            if (!tile_filled<T>(ps, tile, nvalid, lane)) continue;
            const int s = stg;
            const uint32_t par = sph;
            if (lane == 0) {
              if (seq >= nst) wait_cta(&loc.empty[s], par ^ 1u);
              mbar_arrive_expect_tx(&loc.full[s], uint32_t(T * ROWB));
#pragma unroll
              for (int h = 0; h < Geo::KH; ++h)
                tma_load_2d(ring + size_t(s) * Geo::kTile + h * (T * 128), &p.vmap, h * 64,
                            y0 + tile * T, &loc.full[s]);
            }
            __syncwarp();
            ++seq;
            if (++stg == nst) {
              stg = 0;
              sph ^= 1u;
            }
          }
          return;
        }
      }
      const unsigned char* base = static_cast<const unsigned char*>(phase == 0 ? p.kcache : p.vcache) +
                                  (size_t(row) * N + rg.slot0) * ROWB;
      for (int tile = 0; tile < ntiles; ++tile) {
        if (!tile_filled<T>(ps, tile, nvalid, lane)) continue;
        const int s = stg;
        const uint32_t par = sph;
        if (lane == 0) {
          if (seq >= nst) wait_cta(&loc.empty[s], par ^ 1u);
          const int ns = min(T, nvalid - tile * T);
          const uint32_t bytes = uint32_t(ns) * ROWB;
          mbar_arrive_expect_tx(&loc.full[s], bytes);
          bulk_copy_g2s(ring + size_t(s) * Geo::kTile, base + size_t(tile) * T * ROWB, bytes,
                        &loc.full[s]);
        }
        __syncwarp();
        ++seq;
        if (++stg == nst) {
          stg = 0;
          sph ^= 1u;
        }
      }
    };
    int row = next_row(0);
    issue_meta(0, row);
    for (int it = 0; row >= 0; ++it) {
      wait_cta(&loc.row_full[it & 1], uint32_t((it >> 1) & 1));
      issue_tiles(it, row, 0);
      const int nrow = next_row(it + 1);
      issue_meta(it + 1, nrow);
      issue_tiles(it, row, 1);
      row = nrow;
    }
  } else {
    // ================================================================ consumers
    const int sub = lane & 7;   // lane within the slot's 8 lanes (K phase)
    const int sig = lane >> 3;  // slot within the warp's 4-slot group (K phase)
    const int perm = GP >= 8 ? sub : GP == 4 ? ((sub >> 1) & 3) : GP == 2 ? ((sub >> 2) & 1) : 0;
    const int my_head = perm;   // head whose logit this lane holds after the reduction
    const bool kwriter = ((sub & Geo::BFLY) == 0) && (my_head < G);
    const int vsub = lane % VL, vslot = lane / VL;
    // Page-form score only: in V pass u0 + u (passes go in groups of VUC)
    // this lane takes the warp's slot pair u0 + (u ^ vperm) instead, so that
    // the per-slot L1 norms of a group reduce-scatter over the slot's VL
    // lanes without selects; afterwards the lane holds the norm of pass
    // u0 + vperm's slot.
    const int vperm = L1V ? (vsub >> (ilog2(VL) - ilog2(VUC))) & (VUC - 1) : 0;
    const int eh = lane % GP;   // head of this lane in the probability pass
    uint32_t xc_uses0 = 0, xc_uses1 = 0;
    uint32_t kt_count = 0;  // tensor-core K tiles consumed so far (accumulator kt & 1)
    uint32_t vt_count = 0;  // tensor-core V tiles consumed so far (P buffer vt & 1)

    for (int it = 0;; ++it) {
      const int b = it & 1;
      const uint32_t bpar = uint32_t((it >> 1) & 1);
      const int* ps = pos_buf(b);
      wait_cta(&loc.row_full[b], bpar);
      const int row = loc.row_id[b];
      if (row < 0) break;
      const RowGeo rg = row_geo(loc.row_nb[b]);
      const int slot0 = rg.slot0, nvalid = rg.nvalid, ntiles = rg.ntiles;
      if (tid == 0 && rank == 0 && loc.row_bad[b]) atomicOr(p.status, LF_STATUS_BAD_SEQ_BUDGET);

      // query heads of the group, fp32, pre-scaled, in this lane's head order
      // (tensor-core path: the heads as bf16 rows of the MMA's B operand)
      float2 qp[GP][DPL / 2];
      if constexpr (Geo::UMMA) {
        // 16 rows (heads, zero padded) x D, K-major, 128-byte swizzle: 16-byte
        // chunk c of row r's 128-byte half goes to chunk c ^ (r % 8)
        const uint16_t* qs = q_buf(b);
        unsigned char* qop = reinterpret_cast<unsigned char*>(red);
        for (int i = tid; i < Geo::kMmaN * (D / 8); i += kConsumers) {
          const int r = i / (D / 8), c8 = i % (D / 8);
          uint4 w = make_uint4(0, 0, 0, 0);
          if (r < G) w = *reinterpret_cast<const uint4*>(qs + r * D + c8 * 8);
          const int half = c8 >> 3, c = c8 & 7;
          *reinterpret_cast<uint4*>(qop + half * (Geo::kMmaN * 128) + (r >> 3) * 1024 + (r & 7) * 128 +
                                   ((c ^ (r & 7)) << 4)) = w;
        }
        fence_proxy_async_smem();
      } else {
        const uint16_t* qs = q_buf(b);
#pragma unroll
        for (int k = 0; k < GP; ++k) {
          const int h = k ^ perm;
#pragma unroll
          for (int c = 0; c < NLD; ++c) {
#pragma unroll
            for (int e8 = 0; e8 < EPL / 8; ++e8) {  // 8 query elements per 16-byte load
              uint4 w = make_uint4(0, 0, 0, 0);
              if (h < G)
                w = *reinterpret_cast<const uint4*>(qs + h * D + c * 8 * EPL + sub * EPL + e8 * 8);
              const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int m = 0; m < 4; ++m)
                qp[k][c * (EPL / 2) + e8 * 4 + m] =
                    make_float2(bf16lo(ww[m]) * p.qscale2c, bf16hi(ww[m]) * p.qscale2c);
            }
          }
        }
      }
      if (warp == 0) {  // logit of the new token, per head
        constexpr int DV = D / 32;
        const uint16_t* qs = q_buf(b);
        const uint16_t* kn = kn_buf(b);
#pragma unroll
        for (int i = 0; i < G; ++i) {
          float a = 0.f;
#pragma unroll
          for (int d = 0; d < DV; ++d) {
            const int dd = lane * DV + d;
            a = fmaf(__uint_as_float(uint32_t(qs[i * D + dd]) << 16),
                     __uint_as_float(uint32_t(kn[dd]) << 16), a);
          }
#pragma unroll
          for (int m = 16; m > 0; m >>= 1) a += __shfl_xor_sync(0xffffffffu, a, m);
          if (lane == 0) loc.s_new[i] = a * p.qscale2;
        }
      }
      {  // newest position and lowest free slot of the chunk
        int mx = -1, fr = INT_MAX;
        for (int j = tid; j < nvalid; j += kConsumers) {
          const int v = ps[j];
          if (v >= 0) mx = max(mx, v);
          else fr = min(fr, j);
        }
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) {
          mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, m));
          fr = min(fr, __shfl_xor_sync(0xffffffffu, fr, m));
        }
        if (lane == 0) {
          loc.wpmax[warp] = mx;
          loc.wpfree[warp] = fr == INT_MAX ? INT_MAX : slot0 + fr;
        }
      }
      named_barrier(kBarConsumers, kConsumers);
      bool fastrow = true;  // every slot of the chunk filled: no per-slot masking
#pragma unroll
      for (int w = 0; w < CW; ++w) fastrow &= (loc.wpfree[w] == INT_MAX);

      // ---------------------------------------------------------- K phase
      if constexpr (Geo::UMMA) {
        // One warp issues the tensor-core MMAs of each K tile into accumulator
        // kt & 1; a warpgroup reads it back (one slot per thread), frees the
        // ring stage and the accumulator, and keeps the logits and maxima.
        constexpr int TK = Geo::TK;
        constexpr uint32_t idesc = umma_idesc_bf16(128, Geo::kMmaN);
        constexpr int NB = Geo::NB;
        const int ntk = (nvalid + TK - 1) / TK;
        float hm[GP];
#pragma unroll
        for (int k = 0; k < GP; ++k) hm[k] = -INFINITY;
        const uint32_t qop = smem_addr(red);
        for (int tile = 0; tile < ntk; ++tile) {
          if (!fastrow && !tile_filled<TK>(ps, tile, nvalid, lane)) {
            // a K tile with no filled slot is not loaded; the V phase, whose
            // tiles are larger, may still read its logits: mask them
            for (int i = tid; i < TK * GP; i += kConsumers) pl[size_t(tile) * TK * GP + i] = -INFINITY;
            continue;
          }
          const int s = stg;
          const uint32_t sp = sph;
          ++seq;
          if (++stg == nst) {
            stg = 0;
            sph ^= 1u;
          }
          const int tb = int(kt_count & 1u);
          const uint32_t up = (kt_count >> 1) & 1u;
          ++kt_count;
          const uint32_t tcol = uint32_t(tb * NB * Geo::kMmaN);  // accumulator tb's first column
          // the warps that read this tile's accumulator, and their blocks
          bool mine;
          int bk0, bk1, lead;
          if constexpr (Geo::EPI_PAIR) {
            mine = warp < 8;
            bk0 = warp >> 2;
            bk1 = bk0 + 1;
            lead = 0;
          } else if constexpr (Geo::EPI_WG == 2) {
            mine = (warp >> 2) == tb;
            bk0 = 0;
            bk1 = NB;
            lead = 4 * tb;
          } else {
            mine = warp < 4;
            bk0 = 0;
            bk1 = NB;
            lead = 0;
          }
          if (warp == Geo::MMA_WARP) {
            if (lane == 0) {
              wait_cta(&loc.full[s], sp);
              if (kt_count > 2) wait_cta(&loc.tmem_free[tb], up ^ 1u);
              tc_fence_after();
              const uint32_t a0 = smem_addr(ring + size_t(s) * Geo::kTile);
#pragma unroll
              for (int bk = 0; bk < NB; ++bk) {
#pragma unroll
                for (int kk = 0; kk < Geo::KS; ++kk) {
                  const int h = kk >> 2, k4 = kk & 3;
                  umma_bf16(loc.tmem_base + tcol + uint32_t(bk * Geo::kMmaN),
                            umma_desc_sw128(a0 + h * (TK * 128) + bk * (128 * 128) + k4 * 32),
                            umma_desc_sw128(qop + h * (Geo::kMmaN * 128) + k4 * 32), idesc,
                            kk > 0 ? 1u : 0u);
                }
              }
              umma_commit(&loc.mma_done[tb]);
              if constexpr (VMMA) umma_commit(&loc.empty[s]);  // the tile's keys are consumed
            }
            __syncwarp();
          } else if (mine) {
            wait_cta(&loc.mma_done[tb], up);
            tc_fence_after();
            // the tile's keys are consumed: the ring stage may be refilled
            if constexpr (!VMMA) {
              if (warp == lead && lane == 0) mbar_arrive_count(&loc.empty[s], uint32_t(CW));
            }
            for (int bk = bk0; bk < bk1; ++bk) {
              uint32_t acc[8];
              tmem_ld8(loc.tmem_base + (uint32_t(32 * (warp & 3)) << 16) + tcol +
                           uint32_t(bk * Geo::kMmaN),
                       acc);
              const int o = bk * 128 + 32 * (warp & 3) + lane;  // slot within the tile
              if (o < TK) {
                const int j = tile * TK + o;
                const bool valid = j < nvalid && (fastrow || ps[j] >= 0);
                float v[GP];
#pragma unroll
                for (int k = 0; k < GP; ++k) {
                  v[k] = valid ? __uint_as_float(acc[k]) * p.qscale2c : -INFINITY;
                  hm[k] = fmaxf(hm[k], v[k]);
                }
                if constexpr (GP >= 4) {
#pragma unroll
                  for (int k = 0; k < GP; k += 4)
                    *reinterpret_cast<float4*>(pl + size_t(j) * GP + k) =
                        make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
                } else {
#pragma unroll
                  for (int k = 0; k < GP; ++k) pl[size_t(j) * GP + k] = v[k];
                }
              }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&loc.tmem_free[tb]);
          }
        }
        // the V phase reads whole V tiles: mask the logits past the last K tile
        {
          const int end = (nvalid + T - 1) / T * T;
          for (int i = ntk * TK * GP + tid; i < end * GP; i += kConsumers) pl[i] = -INFINITY;
        }
#pragma unroll
        for (int k = 0; k < GP; ++k) {
#pragma unroll
          for (int m = 16; m > 0; m >>= 1) hm[k] = fmaxf(hm[k], __shfl_xor_sync(0xffffffffu, hm[k], m));
        }
        if (lane == 0) {
#pragma unroll
          for (int k = 0; k < GP; ++k) loc.wmax[warp][k] = hm[k];
        }
      } else {
      float rmax = -INFINITY;
      for (int tile = 0; tile < ntiles; ++tile) {
        bool tfull = fastrow && (tile + 1) * T <= nvalid;
        if (!fastrow) {
          if (!tile_filled<T>(ps, tile, nvalid, lane)) continue;
          tfull = tile_full<T>(ps, tile, nvalid, lane);
        }
        wait_cta(&loc.full[stg], sph);
        const unsigned char* kt = ring + size_t(stg) * Geo::kTile;
#pragma unroll 1
        for (int gb = 0; gb < GPW; gb += KU) {
          float xs[KU];
#pragma unroll
          for (int gu = 0; gu < KU; ++gu) {
            const int si = (warp + (gb + gu) * CW) * 4 + sig;
            float2 acc[GP];
#pragma unroll
            for (int k = 0; k < GP; ++k) acc[k] = make_float2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < NLD; ++c) {
              float2 kv[EPL / 2];
              kv_pairs<KVB, LDB>(kt + si * ROWB + c * 8 * LDB + sub * LDB, kv);
#pragma unroll
              for (int m = 0; m < EPL / 2; ++m) {
#pragma unroll
                for (int k = 0; k < GP; ++k)
                  acc[k] = __ffma2_rn(qp[k][c * (EPL / 2) + m], kv[m], acc[k]);
              }
            }
            float a[kMaxG];
#pragma unroll
            for (int k = 0; k < GP; ++k) a[k] = acc[k].x + acc[k].y;
            rs_step<GP, 4>(a);
            rs_step<(GP > 1 ? GP / 2 : 1), 2>(a);
            rs_step<(GP > 2 ? GP / 4 : 1), 1>(a);
            xs[gu] = a[0];
          }
          if (!tfull) {  // mask free and out-of-range slots
            const int ns = min(T, nvalid - tile * T);
#pragma unroll
            for (int gu = 0; gu < KU; ++gu) {
              const int si = (warp + (gb + gu) * CW) * 4 + sig;
              if (!((si < ns) && (ps[tile * T + si] >= 0))) xs[gu] = -INFINITY;
            }
          }
#pragma unroll
          for (int gu = 0; gu < KU; ++gu) {
            const int j = tile * T + (warp + (gb + gu) * CW) * 4 + sig;
            if (kwriter) pl[j * GP + my_head] = xs[gu];
            rmax = fmaxf(rmax, xs[gu]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&loc.empty[stg]);
        ++seq;
        if (++stg == nst) {
          stg = 0;
          sph ^= 1u;
        }
      }
      rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, 8));
      rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, 16));
      if (sig == 0 && kwriter) loc.wmax[warp][my_head] = rmax;
      }
      named_barrier(kBarConsumers, kConsumers);

      float my_m = -INFINITY;
      if (G == GP || eh < G) {
#pragma unroll
        for (int w = 0; w < CW; ++w) my_m = fmaxf(my_m, loc.wmax[w][eh]);
      }
      // 2^(-inf - m) = 0 on the SFU, so masked slots need no select; only a
      // head with no filled slot in the chunk (m = -inf) needs a finite offset
      if (my_m == -INFINITY) my_m = 0.f;

      // ---------------------------------------------------------- V phase
      float lsum = 0.f;
      float* obuf = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(red) + Geo::kQOpBytes);
      if constexpr (VMMA) {
        // P.V on the tensor cores: the consumer threads (all but the MMA
        // warp) turn their (slot, head) logits into probabilities (kept for
        // the scores) and write them as bf16 hi + lo into the P operand; the
        // MMA warp, which only issues, then adds V^T . P^T of the tile to
        // O^T[dims][heads] in tensor memory.
        constexpr int kWriters = (CW - 1) * 32;
        static_assert(kWriters % GP == 0, "head of a writer thread");
        const bool writer = warp != Geo::MMA_WARP;
        constexpr uint32_t idesc_v = umma_idesc_bf16(128, Geo::kMmaNV, true);
        const bool headok = (G == GP || eh < G);
        unsigned char* Pb = reinterpret_cast<unsigned char*>(obuf);
        bool any_v = false;
        for (int tile = 0; tile < ntiles; ++tile) {
          bool tfull = fastrow && (tile + 1) * T <= nvalid;
          if (!fastrow) {
            if (!tile_filled<T>(ps, tile, nvalid, lane)) continue;
            tfull = tile_full<T>(ps, tile, nvalid, lane);
          }
          const int s = stg;
          const uint32_t sp = sph;
          ++seq;
          if (++stg == nst) {
            stg = 0;
            sph ^= 1u;
          }
          const int pbi = int(vt_count & 1u);
          const uint32_t vpar = (vt_count >> 1) & 1u;
          ++vt_count;
          unsigned char* P = Pb + pbi * Geo::kPBytes;
          if (writer) {
          // P buffer pbi was last read by the MMAs of two tiles ago
          if (vt_count > 2) wait_cta(&loc.vdone[pbi], vpar ^ 1u);
          for (int idx = tid; idx < T * GP; idx += kWriters) {
            const int jl = idx / GP;  // idx % GP == eh: kWriters is a multiple of GP
            const int j = tile * T + jl;
            float pv = 0.f;
            if (headok) {
              pv = ex2_ftz(pl[j * GP + eh] - my_m);
              pl[j * GP + eh] = pv;
            }
            lsum += pv;
            const __nv_bfloat16 hi = __float2bfloat16_rn(pv);
            const __nv_bfloat16 lo = __float2bfloat16_rn(pv - __bfloat162float(hi));
            // row eh (hi) and 16 + eh (lo) of the slot's 64-slot atom
            const int off = (jl >> 6) * 4096 + (eh >> 3) * 1024 + (eh & 7) * 128 +
                            ((((jl & 63) >> 3) ^ (eh & 7)) << 4) + (jl & 7) * 2;
            *reinterpret_cast<__nv_bfloat16*>(P + off) = hi;
            *reinterpret_cast<__nv_bfloat16*>(P + off + 2048) = lo;
          }
          if (!tfull) {
            // a free or out-of-range slot's V row may hold anything, NaN
            // included, and a zero probability does not cancel NaN: zero it
            wait_cta(&loc.full[s], sp);
            unsigned char* vt = ring + size_t(s) * Geo::kTile;
            const int ns = min(T, nvalid - tile * T);
            for (int idx = tid; idx < T * 16; idx += kWriters) {  // 16-byte chunks of the tile
              const int jl = idx % T, hc = idx / T;                  // slot, (half, chunk)
              if (!(jl < ns && ps[tile * T + jl] >= 0))
                *reinterpret_cast<uint4*>(vt + (hc >> 3) * (T * 128) + jl * 128 + (hc & 7) * 16) =
                    make_uint4(0, 0, 0, 0);
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&loc.pready[pbi]);
          } else if (lane == 0) {
            wait_cta(&loc.full[s], sp);
            wait_cta(&loc.pready[pbi], vpar);
            tc_fence_after();
            const uint32_t v0 = smem_addr(ring + size_t(s) * Geo::kTile), p0 = smem_addr(P);
#pragma unroll 1
            for (int kk = 0; kk < T / 16; ++kk)
              umma_bf16(loc.tmem_base + Geo::kOCol, umma_desc_sw128(v0 + kk * 2048, T * 128),
                        umma_desc_sw128(p0 + (kk >> 2) * 4096 + (kk & 3) * 32), idesc_v,
                        (any_v || kk > 0) ? 1u : 0u);
            umma_commit(&loc.vdone[pbi]);
            umma_commit(&loc.empty[s]);  // the tile's values are consumed
          }
          __syncwarp();
          any_v = true;
        }
        // the row's partial output: O^T from tensor memory (one dim per thread)
        if (any_v) {
          wait_cta(&loc.vdone[(vt_count - 1) & 1u], ((vt_count - 1) >> 1) & 1u);
          tc_fence_after();
        }
        if (warp < 4) {
          uint32_t rh[8], rl[8];  // the hi and lo halves of O^T for this dim
          tmem_ld8(loc.tmem_base + (uint32_t(32 * warp) << 16) + Geo::kOCol, rh);
          tmem_ld8(loc.tmem_base + (uint32_t(32 * warp) << 16) + Geo::kOCol + 16, rl);
          const int d = 32 * warp + lane;
#pragma unroll
          for (int i = 0; i < G; ++i)
            obuf[i * D + d] = any_v ? __uint_as_float(rh[i]) + __uint_as_float(rl[i]) : 0.f;
          tc_fence_before();
        }
      } else {
      float2 o[G][4];
#pragma unroll
      for (int i = 0; i < G; ++i)
#pragma unroll
        for (int m = 0; m < 4; ++m) o[i][m] = make_float2(0.f, 0.f);
      float2* ppw = pp + warp * TPW * GP;
      for (int tile = 0; tile < ntiles; ++tile) {
        bool tfull = fastrow && (tile + 1) * T <= nvalid;
        if (!fastrow) {
          if (!tile_filled<T>(ps, tile, nvalid, lane)) continue;
          tfull = tile_full<T>(ps, tile, nvalid, lane);
        }
        wait_cta(&loc.full[stg], sph);
        const unsigned char* vt = ring + size_t(stg) * Geo::kTile;
        // probabilities of this warp's slots, kept for the scores and paired for the FMAs
#pragma unroll
        for (int idx = lane; idx < TPW * GP; idx += 32) {
          const int j = tile * T + warp * TPW + idx / GP;
          float pv = 0.f;
          if (G == GP || eh < G) {
            pv = ex2_ftz(pl[j * GP + eh] - my_m);
            pl[j * GP + eh] = pv;
          }
          lsum += pv;
          ppw[idx] = make_float2(pv, pv);
        }
        __syncwarp();
        const int ns = tfull ? T : min(T, nvalid - tile * T);
#pragma unroll
        for (int u0 = 0; u0 < VU; u0 += VUC) {
        float pn[VUC];  // page-form score: partial L1 norms, by pass
#pragma unroll
        for (int u = 0; u < VUC; ++u) {
          const int ls = (u0 + (u ^ vperm)) * SPV + vslot;
          const int si = warp * TPW + ls;
          float2 v[4];
          kv_pairs<KVB, 8 * KVB>(vt + si * ROWB + vsub * (8 * KVB), v);
          if (!tfull) {  // a free or out-of-range slot may hold anything: keep it out
            const bool valid = (si < ns) && (ps[tile * T + si] >= 0);
            if (!valid) {
#pragma unroll
              for (int m = 0; m < 4; ++m) v[m] = make_float2(0.f, 0.f);
            }
          }
          const float2* pr = ppw + ls * GP;
          float2 pi[GP];
          if constexpr (GP >= 2) {
#pragma unroll
            for (int h2 = 0; h2 < GP; h2 += 2) {
              const float4 f = *reinterpret_cast<const float4*>(pr + h2);
              pi[h2] = make_float2(f.x, f.y);
              pi[h2 + 1] = make_float2(f.z, f.w);
            }
          } else {
            pi[0] = pr[0];
          }
#pragma unroll
          for (int i = 0; i < G; ++i)
#pragma unroll
            for (int m = 0; m < 4; ++m) o[i][m] = __ffma2_rn(pi[i], v[m], o[i][m]);
          if constexpr (L1V) {
            float a = 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m) a += fabsf(v[m].x) + fabsf(v[m].y);
            pn[u] = a;
          }
        }
        if constexpr (L1V) {
          // the page's score: fold ||v_j||_1 (from the tile already in shared
          // memory) into the slot's stored probabilities
          if constexpr (VL == 16) {
            rs_step<VUC, 8>(pn);
            rs_step<(VUC > 1 ? VUC / 2 : 1), 4>(pn);
            rs_step<(VUC > 2 ? VUC / 4 : 1), 2>(pn);
            rs_step<(VUC > 4 ? VUC / 8 : 1), 1>(pn);
          } else {
            static_assert(VL == 8, "lanes per slot");
            rs_step<VUC, 4>(pn);
            rs_step<(VUC > 1 ? VUC / 2 : 1), 2>(pn);
            rs_step<(VUC > 2 ? VUC / 4 : 1), 1>(pn);
          }
          constexpr int DUP = VL / VUC;  // lanes left holding the same slot's norm
          const int j = tile * T + warp * TPW + (u0 + vperm) * SPV + vslot;
          for (int i = vsub & (DUP - 1); i < G; i += DUP) pl[j * GP + i] *= pn[0];
        }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&loc.empty[stg]);
        ++seq;
        if (++stg == nst) {
          stg = 0;
          sph ^= 1u;
        }
      }

#pragma unroll
      for (int msk = VL; msk < 32; msk <<= 1)
#pragma unroll
        for (int i = 0; i < G; ++i)
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            o[i][m].x += __shfl_xor_sync(0xffffffffu, o[i][m].x, msk);
            o[i][m].y += __shfl_xor_sync(0xffffffffu, o[i][m].y, msk);
          }
      if (vslot == 0) {
#pragma unroll
        for (int i = 0; i < G; ++i) {
          float4* dst = reinterpret_cast<float4*>(red + (warp * G + i) * D + vsub * 8);
          dst[0] = make_float4(o[i][0].x, o[i][0].y, o[i][1].x, o[i][1].y);
          dst[1] = make_float4(o[i][2].x, o[i][2].y, o[i][3].x, o[i][3].y);
        }
      }
      }
      // ---------------------------------------------------- chunk results
#pragma unroll
      for (int m = GP; m < 32; m <<= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, m);
      if (lane < G) loc.wsum[warp][lane] = lsum;
      named_barrier(kBarConsumers, kConsumers);

      // ------------------- exchange 1: send this chunk's results to every CTA
      // (the partial output goes by slices: CTA r combines elements
      // [r * E / S, (r + 1) * E / S) of the row's output)
      constexpr int E = G * D;
      const int per = E / S;  // E is a multiple of 16 and S a power of two <= 16
      {
        const uint32_t rxo_l = smem_addr(rxo_buf(b));
        const uint32_t sc_l = smem_addr(&rx_buf(b)->sc[rank][0]);
        const uint32_t bar_l = smem_addr(&loc.xa[b]);
        for (int e4 = tid; e4 < E / 4; e4 += kConsumers) {
          const int e = e4 * 4;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          if constexpr (VMMA) {
            acc = *reinterpret_cast<const float4*>(obuf + e);
          } else {
#pragma unroll
            for (int w = 0; w < CW; ++w) {
              const float4 v = *reinterpret_cast<const float4*>(red + w * E + e);
              acc.x += v.x;
              acc.y += v.y;
              acc.z += v.z;
              acc.w += v.w;
            }
          }
          if constexpr (KVB == 1) {  // E4M3 values were summed without their scale
            acc.x *= p.v_scale;
            acc.y *= p.v_scale;
            acc.z *= p.v_scale;
            acc.w *= p.v_scale;
          }
          const int dst = e / per;
          st_async_v4(map_rank_addr(rxo_l + uint32_t(rank * per + (e - dst * per)) * 4u, dst), acc,
                      map_rank_addr(bar_l, dst));
        }
        if (tid < G) {
          float mm = -INFINITY, ll = 0.f;
#pragma unroll
          for (int w = 0; w < CW; ++w) {
            mm = fmaxf(mm, loc.wmax[w][tid]);
            ll += loc.wsum[w][tid];
          }
          for (int r = 0; r < S; ++r) {
            const uint32_t br = map_rank_addr(bar_l, r);
            st_async_b32(map_rank_addr(sc_l + uint32_t(tid) * 4u, r), __float_as_uint(mm), br);
            st_async_b32(map_rank_addr(sc_l + uint32_t(GP + tid) * 4u, r), __float_as_uint(ll), br);
          }
        }
        if (tid == 32) {
          int mx = -1, fr = INT_MAX;
#pragma unroll
          for (int w = 0; w < CW; ++w) {
            mx = max(mx, loc.wpmax[w]);
            fr = min(fr, loc.wpfree[w]);
          }
          const int er = *reinterpret_cast<volatile int*>(&loc.err);
          for (int r = 0; r < S; ++r) {
            const uint32_t br = map_rank_addr(bar_l, r);
            st_async_b32(map_rank_addr(sc_l + uint32_t(2 * GP) * 4u, r), uint32_t(mx), br);
            st_async_b32(map_rank_addr(sc_l + uint32_t(2 * GP + 1) * 4u, r), uint32_t(fr), br);
            st_async_b32(map_rank_addr(sc_l + uint32_t(2 * GP + 2) * 4u, r), uint32_t(er), br);
          }
        }
      }
      // ----------- receive: every CTA's maxima, sums, positions (warp 0 waits)
      if (warp == 0) {
        if (lane == 0)
          mbar_arrive_expect_tx(&loc.xa[b], uint32_t(S) * uint32_t((2 * G + 3) * 4 + per * 4));
        wait_cl(&loc.xa[b], bpar);
        // all heads at once: lane = (head i, sender r) with S lanes per head
        const int HP = 32 / S;  // heads per pass (S is a power of two <= 16)
        for (int i0 = 0; i0 < G; i0 += HP) {
          const int i = i0 + lane / S, r = lane % S;
          const bool ok = i < G;
          const uint32_t* sc = rx_buf(b)->sc[r];
          const float m = ok ? __uint_as_float(sc[i]) : -INFINITY;
          float M = m;
          for (int o2 = 1; o2 < S; o2 <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o2));
          const float sn = ok ? loc.s_new[i] : 0.f;
          M = fmaxf(M, sn);
          const float cf = ok ? exp2f(m - M) : 0.f;  // 0 for an empty chunk (m = -inf)
          float lv = ok ? __uint_as_float(sc[GP + i]) * cf : 0.f;
          for (int o2 = 1; o2 < S; o2 <<= 1) lv += __shfl_xor_sync(0xffffffffu, lv, o2);
          if (ok) {
            loc.cf[r][i] = cf;
            if (r == 0) {
              loc.Mg[i] = M;
              loc.Lg[i] = lv + exp2f(sn - M);
            }
          }
        }
        const bool has = lane < S;
        const uint32_t* sc = rx_buf(b)->sc[has ? lane : 0];
        int mx = has ? int(sc[2 * GP]) : -1;
        int fr = has ? int(sc[2 * GP + 1]) : INT_MAX;
        int er = has ? int(sc[2 * GP + 2]) : 0;
        for (int o2 = 1; o2 < S; o2 <<= 1) {
          mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
          fr = min(fr, __shfl_xor_sync(0xffffffffu, fr, o2));
          er |= __shfl_xor_sync(0xffffffffu, er, o2);
        }
        if (lane == 0) {
          loc.g_t = mx + 1;
          loc.g_free = fr;
          loc.g_err = er;
        }
      }
      named_barrier(kBarConsumers, kConsumers);
      const bool full_row = (loc.g_free == INT_MAX);

      // ------------------------------------------------ scores of own slots
      if (EVICT) {
        unsigned long long k1 = kNoKey, k2 = kNoKey;
        if (full_row && !loc.g_err) {
          float w[G];
#pragma unroll
          for (int i = 0; i < G; ++i) w[i] = loc.cf[rank][i] / loc.Lg[i] * (1.0f / G);
          const int lim = loc.g_t - p.window;
          for (int j = tid; j < nvalid; j += kConsumers) {
            const int gj = slot0 + j;
            if (gj < p.sink || ps[j] >= lim) continue;
            float sc = 0.f;
#pragma unroll
            for (int i = 0; i < G; ++i) sc = fmaf(pl[j * GP + i], w[i], sc);
            top2_insert(k1, k2, (static_cast<unsigned long long>(__float_as_uint(sc)) << 32) |
                                    static_cast<unsigned int>(gj));
          }
        }
        top2_warp(k1, k2);
        if (lane == 0) {
          loc.wk1[warp] = k1;
          loc.wk2[warp] = k2;
        }
        named_barrier(kBarConsumers, kConsumers);
        // ---------------------------- exchange 2: send the keys to every CTA
        if (warp == 0) {
          k1 = lane < CW ? loc.wk1[lane] : kNoKey;
          k2 = lane < CW ? loc.wk2[lane] : kNoKey;
          top2_warp(k1, k2);
          if (lane < S) {
            const uint32_t ka = map_rank_addr(smem_addr(&rx_buf(b)->key[rank][0]), lane);
            const uint32_t br = map_rank_addr(smem_addr(&loc.xb[b]), lane);
            st_async_b64(ka, k1, br);
            st_async_b64(ka + 8u, k2, br);
          }
        }
      }

      // ------------------------------------------ output: this CTA's slice
      {
        const int e0 = rank * per;
        const uint16_t* vn = vn_buf(b);
        const float* rxo = rxo_buf(b);
        for (int k = tid; k < per; k += kConsumers) {
          const int e = e0 + k;
          const int i = e / D, d = e - i * D;
          float acc = exp2f(loc.s_new[i] - loc.Mg[i]) * __uint_as_float(uint32_t(vn[d]) << 16);
          for (int r = 0; r < S; ++r) acc = fmaf(rxo[r * per + k], loc.cf[r][i], acc);
          p.out[size_t(row) * E + e] = acc / loc.Lg[i];
        }
      }

      if (EVICT) {
        // ----------------------------------- receive: every CTA's keys
        if (warp == 0) {
          if (lane == 0) mbar_arrive_expect_tx(&loc.xb[b], uint32_t(S) * 16u);
          wait_cl(&loc.xb[b], bpar);
          const bool has = lane < S;
          unsigned long long g1 = has ? rx_buf(b)->key[lane][0] : kNoKey;
          unsigned long long g2 = has ? rx_buf(b)->key[lane][1] : kNoKey;
          top2_warp(g1, g2);
          if (lane == 0) {
            int refine = 0;
            if (g1 != kNoKey && g2 != kNoKey) {
              const float s1 = __uint_as_float(uint32_t(g1 >> 32));
              const float s2 = __uint_as_float(uint32_t(g2 >> 32));
              refine = (s2 <= s1 * (1.0f + kTieRel)) ? 1 : 0;
            }
            loc.g_refine = refine;
            loc.g_slot = (g1 == kNoKey) ? -1 : int(uint32_t(g1 & 0xffffffffull));
            loc.g_key1 = g1;
          }
        }
        named_barrier(kBarConsumers, kConsumers);

        if (loc.g_refine) {  // the same decision in every CTA of the cluster
          // fp64 rescoring of the candidates inside the tie band
          const float s1 = __uint_as_float(uint32_t(loc.g_key1 >> 32));
          const float thr = s1 * (1.0f + kTieRel);
          float w[G];
#pragma unroll
          for (int i = 0; i < G; ++i) w[i] = loc.cf[rank][i] / loc.Lg[i] * (1.0f / G);
          const int lim = loc.g_t - p.window;
          const uint16_t* qs = q_buf(b);
          double best = INFINITY;
          int bslot = INT_MAX;
          // candidates inside the band are found 32 at a time per warp; each is
          // then rescored by the whole warp (lane l: dims [l*D/32, (l+1)*D/32))
          constexpr int DL = D / 32;
          for (int base = warp * 32; base < nvalid; base += kConsumers) {
            const int j = base + lane;
            bool in_band = false;
            if (j < nvalid) {
              const int gj = slot0 + j;
              if (gj >= p.sink && ps[j] < lim) {
                float sc = 0.f;
#pragma unroll
                for (int i = 0; i < G; ++i) sc = fmaf(pl[j * GP + i], w[i], sc);
                in_band = sc <= thr;
              }
            }
            unsigned mask = __ballot_sync(0xffffffffu, in_band);
            while (mask) {
              const int src = __ffs(mask) - 1;
              mask &= mask - 1;
              const int gj = slot0 + base + src;
              const unsigned char* krow =
                  static_cast<const unsigned char*>(p.kcache) + (size_t(row) * N + gj) * ROWB;
              double kv[DL];
#pragma unroll
              for (int d = 0; d < DL; ++d) kv[d] = kv_to_f64<KVB>(krow, lane * DL + d);
              double tot = 0.0;
#pragma unroll
              for (int i = 0; i < G; ++i) {
                double dot = 0.0;
#pragma unroll
                for (int d = 0; d < DL; ++d) dot = fma(bf16_to_f64(qs[i * D + lane * DL + d]), kv[d], dot);
#pragma unroll
                for (int m = 16; m > 0; m >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, m);
                tot += exp2(dot * p.qscale2c_64 - double(loc.Mg[i])) / double(loc.Lg[i]);
              }
              tot /= double(G);
              if constexpr (L1V) {
                // (E4M3: without the value scale, a factor common to every slot)
                const unsigned char* vrow =
                    static_cast<const unsigned char*>(p.vcache) + (size_t(row) * N + gj) * ROWB;
                double l1 = 0.0;
#pragma unroll
                for (int d = 0; d < DL; ++d) l1 += fabs(kv_to_f64<KVB>(vrow, lane * DL + d));
#pragma unroll
                for (int m = 16; m > 0; m >>= 1) l1 += __shfl_xor_sync(0xffffffffu, l1, m);
                tot *= l1;
              }
              if (tot < best || (tot == best && gj < bslot)) {
                best = tot;
                bslot = gj;
              }
            }
          }
          if (lane == 0) {
            loc.wref[warp] = best;
            loc.wrefs[warp] = bslot;
          }
          named_barrier(kBarConsumers, kConsumers);
          // -------------------- exchange 3: fp64 rescoring results to every CTA
          const uint32_t xpar = (b ? xc_uses1 : xc_uses0) & 1u;
          if (b) ++xc_uses1;
          else ++xc_uses0;
          if (warp == 0) {
            double bb = lane < CW ? loc.wref[lane] : INFINITY;
            int bs = lane < CW ? loc.wrefs[lane] : INT_MAX;
#pragma unroll
            for (int m = 16; m > 0; m >>= 1) {
              const double ob = __shfl_xor_sync(0xffffffffu, bb, m);
              const int os = __shfl_xor_sync(0xffffffffu, bs, m);
              if (ob < bb || (ob == bb && os < bs)) {
                bb = ob;
                bs = os;
              }
            }
            if (lane < S) {
              const uint32_t ra = map_rank_addr(smem_addr(&rx_buf(b)->ref[rank][0]), lane);
              const uint32_t br = map_rank_addr(smem_addr(&loc.xc[b]), lane);
              st_async_b64(ra, static_cast<unsigned long long>(__double_as_longlong(bb)), br);
              st_async_b64(ra + 8u, static_cast<unsigned long long>(uint32_t(bs)), br);
            }
            if (lane == 0) mbar_arrive_expect_tx(&loc.xc[b], uint32_t(S) * 16u);
            wait_cl(&loc.xc[b], xpar);
            const bool has = lane < S;
            bb = has ? __longlong_as_double(static_cast<long long>(rx_buf(b)->ref[lane][0])) : INFINITY;
            bs = has ? int(uint32_t(rx_buf(b)->ref[lane][1])) : INT_MAX;
#pragma unroll
            for (int m = 16; m > 0; m >>= 1) {
              const double ob = __shfl_xor_sync(0xffffffffu, bb, m);
              const int os = __shfl_xor_sync(0xffffffffu, bs, m);
              if (ob < bb || (ob == bb && os < bs)) {
                bb = ob;
                bs = os;
              }
            }
            if (lane == 0 && bs != INT_MAX) loc.g_slot = bs;
          }
          named_barrier(kBarConsumers, kConsumers);
        }

        // -------------------------------------------- in-place eviction
        if (rank == 0) {
          int e, ev;
          if (loc.g_err || loc.err || loc.row_bad[b]) {
            e = -1;
            ev = -2;
          } else if (!full_row) {
            e = loc.g_free;
            ev = -1;
          } else if (loc.g_slot < 0) {
            e = -1;
            ev = -2;
            if (tid == 0) atomicOr(p.status, LF_STATUS_NO_CANDIDATE);
          } else {
            e = loc.g_slot;
            ev = e;
          }
          if (e >= 0 && e < N) {
            constexpr int V16 = ROWB / 16;  // 16-byte vectors per cached row
            if (tid < 2 * V16) {
              const bool isk = tid < V16;
              const int t16 = isk ? tid : tid - V16;
              unsigned char* dst = static_cast<unsigned char*>(isk ? p.kcache : p.vcache) +
                                   (size_t(row) * N + e) * ROWB;
              const uint16_t* src = isk ? kn_buf(b) : vn_buf(b);
              if constexpr (KVB == 2) {
                reinterpret_cast<uint4*>(dst)[t16] = reinterpret_cast<const uint4*>(src)[t16];
              } else {
                // quantise 16 elements: fp32 quotient by the scale, then E4M3
                const float sc = isk ? p.k_scale : p.v_scale;
                uint32_t w[4];
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                  const uint32_t a = *reinterpret_cast<const uint32_t*>(src + t16 * 16 + 4 * m);
                  const uint32_t c = *reinterpret_cast<const uint32_t*>(src + t16 * 16 + 4 * m + 2);
                  const uint32_t lo = float2_to_e4m3x2(
                      make_float2(__fdiv_rn(bf16lo(a), sc), __fdiv_rn(bf16hi(a), sc)));
                  const uint32_t hi = float2_to_e4m3x2(
                      make_float2(__fdiv_rn(bf16lo(c), sc), __fdiv_rn(bf16hi(c), sc)));
                  w[m] = (lo & 0xffffu) | (hi << 16);
                }
                reinterpret_cast<uint4*>(dst)[t16] = make_uint4(w[0], w[1], w[2], w[3]);
              }
            } else if (tid == 2 * V16) {
              p.pos[size_t(row) * N + e] = loc.g_t;
            }
          }
          if (tid == 0) p.evicted[row] = ev;
        }
      }
      // this row's logits, positions and metadata are no longer needed
      named_barrier(kBarConsumers, kConsumers);
      if (tid == 0) mbar_arrive(&loc.row_free[b]);
    }
  }

  if constexpr (Geo::UMMA) {
    // every MMA this CTA issued has completed before its TMEM is freed
    if (warp == Geo::MMA_WARP && lane == 0) {
      umma_commit(&loc.mma_fin);
      (void)mbar_wait_bounded(&loc.mma_fin, 0u, kWaitLimitNs);
    }
    tc_fence_before();
  }
  __syncthreads();
  // after an error, do not leave with bulk copies still landing in shared memory
  if (loc.err && tid == kConsumers) {
    for (int q = max(0, seq - nst); q < seq; ++q)
      mbar_wait_bounded(&loc.full[q % nst], uint32_t(q / nst) & 1u, kWaitLimitNs);
  }
  if constexpr (Geo::UMMA) {
    tc_fence_after();
    if (warp == 0) tmem_free(loc.tmem_base, Geo::kTmemCols);
  }
  cluster.sync();  // no CTA leaves while a peer may still read its shared memory
}

// ---------------------------------------------------------------- host side
// Per-variant launch planning and launching (instantiated in lf_inst.cu).

constexpr int kRowOverheadSlots = 256;  // per-row cost of the exchange, in slot units

template <int D, int G, int MODE, int KVB>
cudaError_t plan_t(const PlanIn& c, int budget, Plan* out) {
  using Geo = Geometry<D, G, KVB>;
  auto kern = fused_decode_kernel<D, G, MODE, KVB>;
  static std::mutex mu;
  static bool attrs_set = false;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!attrs_set) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           c.smem_optin);
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
      attrs_set = true;
    }
  }
  const int rows = c.rows;
  Plan best = {};
  long long best_cost = -1;
  const int cands[5] = {1, 2, 4, 8, 16};
  for (int ci = 0; ci < 5; ++ci) {
    const int S = cands[ci];
    if (c.split_override > 0 && S != c.split_override) continue;
    const int chunk = chunk_for(budget, S);
    constexpr bool vmma = KVB == 2 && MODE != kEvictAlphaL1V && D == 128 &&
                          (Geo::GP >= LF_VMMA_MIN_GP);
    const size_t fixed = Geo::layout(chunk, 0, vmma).total;
    if (fixed + size_t(kMinStages) * Geo::kTile > size_t(c.smem_optin)) continue;
    int nst = int((size_t(c.smem_optin) - fixed) / Geo::kTile);
    if (nst > kMaxStages) nst = kMaxStages;
    const size_t smem = Geo::layout(chunk, nst, vmma).total;
    if (smem > size_t(c.smem_optin)) continue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(S), unsigned(rows), 1);
    cfg.blockDim = dim3(Geo::kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = unsigned(S);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int ncl = 0;
    if (cudaOccupancyMaxActiveClusters(&ncl, kern, &cfg) != cudaSuccess || ncl < 1) {
      cudaGetLastError();  // clear a refused size
      continue;
    }
    if (ncl > rows) ncl = rows;
    const long long iters = (rows + ncl - 1) / ncl;
    const long long cost = iters * (chunk + kRowOverheadSlots);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best.S = S;
      best.chunk = chunk;
      best.nstages = nst;
      best.nclusters = ncl;
      best.smem = smem;
      best.tk = Geo::TK;
      best.tv = vmma ? Geo::T : 0;
    }
  }
  if (best_cost < 0) return cudaErrorInvalidConfiguration;  // no split fits: budget too large
  best.budget = budget;
  *out = best;
  return cudaSuccess;
}

template <int D, int G, int MODE, int KVB>
cudaError_t launch_t(const Params& p, const Plan& pl, cudaStream_t st) {
  auto kern = fused_decode_kernel<D, G, MODE, KVB>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(pl.S), unsigned(pl.nclusters), 1);
  cfg.blockDim = dim3(Geometry<D, G, KVB>::kThreads, 1, 1);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = unsigned(pl.S);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

#define LF_DISPATCH(D_, G_, CALL)                                                  \
  do {                                                                             \
    switch ((D_) * 16 + (G_)) {                                                    \
      case 64 * 16 + 1: { constexpr int DD = 64, GG = 1; CALL; } break;            \
      case 64 * 16 + 2: { constexpr int DD = 64, GG = 2; CALL; } break;            \
      case 64 * 16 + 3: { constexpr int DD = 64, GG = 3; CALL; } break;            \
      case 64 * 16 + 4: { constexpr int DD = 64, GG = 4; CALL; } break;            \
      case 64 * 16 + 5: { constexpr int DD = 64, GG = 5; CALL; } break;            \
      case 64 * 16 + 6: { constexpr int DD = 64, GG = 6; CALL; } break;            \
      case 64 * 16 + 7: { constexpr int DD = 64, GG = 7; CALL; } break;            \
      case 64 * 16 + 8: { constexpr int DD = 64, GG = 8; CALL; } break;            \
      case 128 * 16 + 1: { constexpr int DD = 128, GG = 1; CALL; } break;          \
      case 128 * 16 + 2: { constexpr int DD = 128, GG = 2; CALL; } break;          \
      case 128 * 16 + 3: { constexpr int DD = 128, GG = 3; CALL; } break;          \
      case 128 * 16 + 4: { constexpr int DD = 128, GG = 4; CALL; } break;          \
      case 128 * 16 + 5: { constexpr int DD = 128, GG = 5; CALL; } break;          \
      case 128 * 16 + 6: { constexpr int DD = 128, GG = 6; CALL; } break;          \
      case 128 * 16 + 7: { constexpr int DD = 128, GG = 7; CALL; } break;          \
      case 128 * 16 + 8: { constexpr int DD = 128, GG = 8; CALL; } break;          \
      default: break;                                                              \
    }                                                                              \
  } while (0)

}  // namespace lf
