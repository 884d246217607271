// Declarations shared by the fused decode kernel's translation units: the
// kernel parameters, the launch plan, and the per-variant plan / launch
// functions.  Each variant (KV storage x kernel mode) is compiled in its own
// translation unit (lf_inst.cu built once per variant) so the variants build
// in parallel; lf_decode.cu holds the C ABI and dispatches to them.
#pragma once
#include <cuda.h>  // CUtensorMap (the type only; no driver library is linked)
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace lf {

constexpr int kMaxStages = 4;
constexpr int kMinStages = 2;
constexpr int kMaxSplit = 16;
constexpr int kMaxG = 8;
// kernel modes
constexpr int kAttendOnly = 0;     // attention only: nothing scored or written
constexpr int kEvictMeanProb = 1;  // evict the lowest head-averaged probability
constexpr int kEvictAlphaL1V = 2;  // ... times the L1 norm of the slot's value
// KV storage: bytes per cached element
constexpr int kKvBf16 = 2;
constexpr int kKvE4m3 = 1;

struct Params {
  // bf16 storage: the key cache as a 2-D tensor [rows * budget, D] for TMA
  // tensor copies with 128-byte swizzle (boxes of 64 elements x Plan::tk slots)
  CUtensorMap kmap;
  CUtensorMap vmap;  // the value cache likewise (boxes of 64 elements x Plan::tv slots)
  const uint16_t* q;      // bf16 [rows * G, D]
  const uint16_t* k_new;  // bf16 [rows, D]
  const uint16_t* v_new;
  void* kcache;           // [rows, budget, D] of bf16 or E4M3 codes
  void* vcache;
  int32_t* pos;
  float* out;
  int32_t* evicted;
  int* status;
  const int32_t* seq_budget;  // [B] per-sequence budgets, or null (every row uses all slots)
  unsigned int* grab;         // row counter of the dynamic schedule (zero between launches)
  int dyn;                    // rows are taken from `grab` instead of a static stride
  int hkv;
  int rows;
  int budget;
  int chunk;
  int sink;
  int window;
  int nstages;
  int pos_bulk;        // position rows may be bulk-copied (16-byte aligned)
  float qscale2;       // log2(e) / sqrt(D): logit of the new token (exact bf16 key)
  float qscale2c;      // the same times the key scale: logits of cached keys
  double qscale2c_64;
  float k_scale, v_scale;  // E4M3 storage: a stored code stands for E4M3(code) * scale
};

// How one call is laid out on the GPU: S CTAs per row (one cluster), the
// slots each CTA owns, the ring depth, and how many persistent clusters run.
struct Plan {
  int budget;  // the budget the plan was made for (0 = none)
  int S, chunk, nstages, nclusters;
  int tk;  // slots per K tile (the key tensor map's box height)
  int tv;  // slots per V tile when P.V runs on the tensor cores (the value map's box height), else 0
  size_t smem;
};

struct PlanIn {
  int rows;            // B * Hkv
  int split_override;  // 0 = automatic
  int smem_optin;      // shared memory a CTA may opt in to
};

// Slots per CTA: an even split, rounded up to 4 slots (16-byte position rows).
inline int chunk_for(int budget, int split) {
  const int per = (budget + split - 1) / split;
  return (per + 3) / 4 * 4;
}

#define LF_VARIANTS(X) X(2, 0) X(2, 1) X(2, 2) X(1, 0) X(1, 1) X(1, 2)
#define LF_DECLARE_VARIANT(KVB, MODE)                                                          \
  cudaError_t plan_kv##KVB##_m##MODE(int D, int G, const PlanIn& in, int budget, Plan* out); \
  cudaError_t launch_kv##KVB##_m##MODE(int D, int G, const Params& p, const Plan& pl,         \
                                       cudaStream_t st);
LF_VARIANTS(LF_DECLARE_VARIANT)
#undef LF_DECLARE_VARIANT

}  // namespace lf
