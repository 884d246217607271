// B200 (sm_100a) LongFlow fused decode step: the C ABI declared in
// include/lf_decode.h (handles, argument checks, launch planning cache,
// dispatch to the compiled kernel variants), the prefill kernels and the
// allocation-free entry point.  The fused kernel itself is in lf_kernel.cuh.
#include "lf_kernel.cuh"

namespace lf {

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

// fp8: quantise the prompt into E4M3 codes (fp32 quotient by the scale,
// round to nearest even, saturate); one thread per 16 elements
__global__ void prefill_fp8_kernel(const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                                   int n, uint4* __restrict__ kc, uint4* __restrict__ vc,
                                   int32_t* __restrict__ pos, int budget, int rows, int vec_per_row,
                                   float k_scale, float v_scale) {
  const size_t stride = size_t(gridDim.x) * blockDim.x;
  const size_t tid = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t per_row = size_t(n) * vec_per_row;
  const size_t total = per_row * rows;
  for (size_t i = tid; i < total; i += stride) {
    const size_t r = i / per_row, rest = i - r * per_row;
    const size_t dst = r * size_t(budget) * vec_per_row + rest;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint16_t* src = (t == 0 ? k : v) + i * 16;
      const float sc = t == 0 ? k_scale : v_scale;
      uint32_t w[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const uint32_t a = *reinterpret_cast<const uint32_t*>(src + 4 * m);
        const uint32_t c = *reinterpret_cast<const uint32_t*>(src + 4 * m + 2);
        const uint32_t lo = float2_to_e4m3x2(make_float2(__fdiv_rn(bf16lo(a), sc), __fdiv_rn(bf16hi(a), sc)));
        const uint32_t hi = float2_to_e4m3x2(make_float2(__fdiv_rn(bf16lo(c), sc), __fdiv_rn(bf16hi(c), sc)));
        w[m] = (lo & 0xffffu) | (hi << 16);
      }
      (t == 0 ? kc : vc)[dst] = make_uint4(w[0], w[1], w[2], w[3]);
    }
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

using lf::Plan;

struct lf_ctx {
  int B, Hq, Hkv, D, G, max_budget;
  cudaStream_t stream;
  int device;
  int sm_count;
  int smem_optin;
  int split_override;
  int* status;          // device status word
  unsigned int* grab;   // device row counter of the dynamic schedule (after the status word)
  int last_bits;
  int score_mode;  // LF_SCORE_* used by lf_decode_step
  Plan plan[2][3];  // [E4M3 storage][kernel mode]
  unsigned magic;
};

namespace {

constexpr unsigned kMagic = 0x4c46444bu;

bool aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

bool valid_handle(lf_handle h) { return h != nullptr && h->magic == kMagic; }

// calls that plan or enqueue work run on the device the handle was made on
bool on_handle_device(const lf_ctx* c) {
  int cur = -1;
  return cudaGetDevice(&cur) == cudaSuccess && cur == c->device;
}

// the compiled variants, by [E4M3 storage][kernel mode]
using PlanFn = cudaError_t (*)(int, int, const lf::PlanIn&, int, Plan*);
using LaunchFn = cudaError_t (*)(int, int, const lf::Params&, const Plan&, cudaStream_t);
const PlanFn kPlanFns[2][3] = {{lf::plan_kv2_m0, lf::plan_kv2_m1, lf::plan_kv2_m2},
                               {lf::plan_kv1_m0, lf::plan_kv1_m1, lf::plan_kv1_m2}};
const LaunchFn kLaunchFns[2][3] = {{lf::launch_kv2_m0, lf::launch_kv2_m1, lf::launch_kv2_m2},
                                   {lf::launch_kv1_m0, lf::launch_kv1_m1, lf::launch_kv1_m2}};

// kernel mode of a call: attention only, or eviction by the handle's score
int kernel_mode(const lf_ctx* c, bool evict) {
  if (!evict) return lf::kAttendOnly;
  return c->score_mode == LF_SCORE_ALPHA_L1V ? lf::kEvictAlphaL1V : lf::kEvictMeanProb;
}

cudaError_t get_plan(lf_ctx* c, int budget, bool fp8, int mode, Plan** out) {
  Plan& pl = c->plan[fp8 ? 1 : 0][mode];
  if (pl.budget != budget) {
    pl.budget = 0;
    lf::PlanIn in;
    in.rows = c->B * c->Hkv;
    in.split_override = c->split_override;
    in.smem_optin = c->smem_optin;
    const cudaError_t e = kPlanFns[fp8 ? 1 : 0][mode](c->D, c->G, in, budget, &pl);
    if (e != cudaSuccess) {
      pl.budget = 0;
      return e;
    }
  }
  *out = &pl;
  return cudaSuccess;
}

bool good_scale(float s) { return s > 0.f && s <= 3.0e38f; }  // positive and finite

// A bf16 cache (keys or values) as a 2-D tensor [rows * budget, D] for TMA
// tensor copies: boxes of 64 elements x (the variant's K or V tile) slots,
// 128-byte swizzle (the layout the tensor-core MMAs read).  The encoder comes from the driver at run time.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}
int encode_kmap(CUtensorMap* map, const void* kcache, int D, long long slots, int box_slots) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return LF_EUNSUPPORTED;
  const cuuint64_t dims[2] = {cuuint64_t(D), cuuint64_t(slots)};
  const cuuint64_t strides[1] = {cuuint64_t(D) * 2};
  const cuuint32_t box[2] = {64, cuuint32_t(box_slots)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(kcache), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LF_OK : LF_ECUDA;
}

// fp8: the cache holds E4M3 codes with scales k_scale / v_scale
int run_decode(lf_handle h, const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
               void* kcache, void* vcache, int32_t* pos, int budget, int sink,
               int window, float* out, int32_t* evicted, bool evict,
               const int32_t* seq_budget = nullptr, bool fp8 = false, float k_scale = 1.f,
               float v_scale = 1.f) {
  if (!valid_handle(h)) return LF_ENOTINIT;
  if (!on_handle_device(h)) return LF_EINVAL;
  if (fp8 && (!good_scale(k_scale) || !good_scale(v_scale))) return LF_EINVAL;
  if (seq_budget && (!aligned(seq_budget, 4) || !h->grab)) return LF_EINVAL;
  if (!q || !k_new || !v_new || !kcache || !vcache || !pos || !out) return LF_EINVAL;
  if (evict && !evicted) return LF_EINVAL;
  if (!aligned(q, 16) || !aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(kcache, 16) ||
      !aligned(vcache, 16) || !aligned(out, 16) || !aligned(pos, 4) ||
      (evicted && !aligned(evicted, 4)))
    return LF_EINVAL;
  if (budget < 1 || budget > h->max_budget) return LF_EINVAL;
  if (evict && (sink < 0 || window < 1 || budget <= sink + window)) return LF_EINVAL;

  const int mode = kernel_mode(h, evict);
  Plan* pl = nullptr;
  {
    const cudaError_t pe = get_plan(h, budget, fp8, mode, &pl);
    if (pe == cudaErrorInvalidConfiguration) return LF_EINVAL;
    if (pe != cudaSuccess) return LF_ECUDA;
  }

  lf::Params p;
  memset(&p, 0, sizeof(p));
  if (!fp8) {
    const long long slots = (long long)h->B * h->Hkv * budget;
    if (slots >= (1LL << 31)) return LF_EINVAL;  // TMA slot coordinates are 32-bit
    int rc = encode_kmap(&p.kmap, kcache, h->D, slots, pl->tk);
    if (rc == LF_OK && pl->tv > 0) rc = encode_kmap(&p.vmap, vcache, h->D, slots, pl->tv);
    if (rc != LF_OK) return rc;
  }
  p.q = q;
  p.k_new = k_new;
  p.v_new = v_new;
  p.kcache = kcache;
  p.vcache = vcache;
  p.pos = pos;
  p.out = out;
  p.evicted = evicted;
  p.status = h->status;
  p.seq_budget = seq_budget;
  p.grab = h->grab;
  p.dyn = seq_budget ? 1 : 0;
  p.hkv = h->Hkv;
  p.rows = h->B * h->Hkv;
  p.budget = budget;
  p.chunk = pl->chunk;
  p.sink = evict ? sink : 0;
  p.window = evict ? window : 1;
  p.nstages = pl->nstages;
  p.pos_bulk = (budget % 4 == 0 && aligned(pos, 16)) ? 1 : 0;
  const double qs2 = 1.4426950408889634 / sqrt(double(h->D));
  p.qscale2 = float(qs2);
  p.k_scale = fp8 ? k_scale : 1.f;
  p.v_scale = fp8 ? v_scale : 1.f;
  p.qscale2c_64 = qs2 * double(p.k_scale);
  p.qscale2c = float(p.qscale2c_64);

  const cudaError_t e = kLaunchFns[fp8 ? 1 : 0][mode](h->D, h->G, p, *pl, h->stream);
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
  c->score_mode = LF_SCORE_MEAN_PROB;
  c->magic = kMagic;
  // the status word, then the row counter of the dynamic schedule
  if (cudaMalloc(&c->status, 2 * sizeof(int)) != cudaSuccess) {
    free(c);
    return LF_ECUDA;
  }
  c->grab = reinterpret_cast<unsigned int*>(c->status + 1);
  if (cudaMemset(c->status, 0, 2 * sizeof(int)) != cudaSuccess) {
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
  for (auto& kv : h->plan)
    for (Plan& pl : kv) pl.budget = 0;
  return LF_OK;
}

int lf_set_score(lf_handle h, int score) {
  if (!valid_handle(h)) return LF_ENOTINIT;
  if (score != LF_SCORE_MEAN_PROB && score != LF_SCORE_ALPHA_L1V) return LF_EINVAL;
  h->score_mode = score;
  return LF_OK;
}

int lf_get_score(lf_handle h) {
  if (!valid_handle(h)) return LF_ENOTINIT;
  return h->score_mode;
}

int lf_get_split(lf_handle h, int budget) {
  if (!valid_handle(h)) return LF_ENOTINIT;
  if (budget < 1 || budget > h->max_budget || !on_handle_device(h)) return LF_EINVAL;
  Plan* pl = nullptr;
  const cudaError_t pe = get_plan(h, budget, false, kernel_mode(h, true), &pl);
  if (pe == cudaErrorInvalidConfiguration) return LF_EINVAL;
  if (pe != cudaSuccess) return LF_ECUDA;
  return pl->S;
}

int lf_prefill_cache(lf_handle h, const uint16_t* k, const uint16_t* v, int n, uint16_t* kcache,
                     uint16_t* vcache, int32_t* pos, int budget) {
  if (!valid_handle(h)) return LF_ENOTINIT;
  if (!on_handle_device(h)) return LF_EINVAL;
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

int lf_prefill_cache_fp8(lf_handle h, const uint16_t* k, const uint16_t* v, int n, uint8_t* kcache,
                         uint8_t* vcache, int32_t* pos, int budget, float k_scale, float v_scale) {
  if (!valid_handle(h)) return LF_ENOTINIT;
  if (!on_handle_device(h)) return LF_EINVAL;
  if (budget < 1 || budget > h->max_budget || n < 0 || n > budget) return LF_EINVAL;
  if (!good_scale(k_scale) || !good_scale(v_scale)) return LF_EINVAL;
  if (!kcache || !vcache || !pos || (n > 0 && (!k || !v))) return LF_EINVAL;
  if (!aligned(kcache, 16) || !aligned(vcache, 16) || !aligned(pos, 4) ||
      (n > 0 && (!aligned(k, 16) || !aligned(v, 16))))
    return LF_EINVAL;
  const int rows = h->B * h->Hkv;
  const int vec = h->D / 16;  // 16-element groups per row
  const size_t work = size_t(rows) * (size_t(n) * vec > size_t(budget) ? size_t(n) * vec : size_t(budget));
  int blocks = int((work + 255) / 256);
  if (blocks > h->sm_count * 8) blocks = h->sm_count * 8;
  if (blocks < 1) blocks = 1;
  lf::prefill_fp8_kernel<<<blocks, 256, 0, h->stream>>>(k, v, n, reinterpret_cast<uint4*>(kcache),
                                                        reinterpret_cast<uint4*>(vcache), pos, budget,
                                                        rows, vec, k_scale, v_scale);
  return cudaGetLastError() == cudaSuccess ? LF_OK : LF_ECUDA;
}

int lf_decode_step_fp8(lf_handle h, const uint16_t* q, const uint16_t* k_new,
                       const uint16_t* v_new, uint8_t* kcache, uint8_t* vcache, int32_t* pos,
                       int budget, const int32_t* seq_budget, int sink, int window,
                       float k_scale, float v_scale, float* out, int32_t* evicted_idx) {
  return run_decode(h, q, k_new, v_new, kcache, vcache, pos, budget, sink, window, out,
                    evicted_idx, true, seq_budget, true, k_scale, v_scale);
}

int lf_decode_attention_fp8(lf_handle h, const uint16_t* q, const uint16_t* k_new,
                            const uint16_t* v_new, const uint8_t* kcache, const uint8_t* vcache,
                            const int32_t* pos, int budget, const int32_t* seq_budget,
                            float k_scale, float v_scale, float* out) {
  return run_decode(h, q, k_new, v_new, const_cast<uint8_t*>(kcache),
                    const_cast<uint8_t*>(vcache), const_cast<int32_t*>(pos), budget, 0, 1, out,
                    nullptr, false, seq_budget, true, k_scale, v_scale);
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

int lf_decode_step_ragged(lf_handle h, const uint16_t* q, const uint16_t* k_new,
                          const uint16_t* v_new, uint16_t* kcache, uint16_t* vcache,
                          int32_t* pos, int budget, const int32_t* seq_budget, int sink,
                          int window, float* out, int32_t* evicted_idx) {
  if (!seq_budget) return LF_EINVAL;
  return run_decode(h, q, k_new, v_new, kcache, vcache, pos, budget, sink, window, out,
                    evicted_idx, true, seq_budget);
}

int lf_decode_attention_ragged(lf_handle h, const uint16_t* q, const uint16_t* k_new,
                               const uint16_t* v_new, const uint16_t* kcache,
                               const uint16_t* vcache, const int32_t* pos, int budget,
                               const int32_t* seq_budget, float* out) {
  if (!seq_budget) return LF_EINVAL;
  return run_decode(h, q, k_new, v_new, const_cast<uint16_t*>(kcache),
                    const_cast<uint16_t*>(vcache), const_cast<int32_t*>(pos), budget, 0, 1, out,
                    nullptr, false, seq_budget);
}

int lf_get_status(lf_handle h) {
  if (!valid_handle(h)) return LF_ENOTINIT;
  if (cudaStreamSynchronize(h->stream) != cudaSuccess) return LF_ECUDA;
  int bits = 0;
  if (cudaMemcpy(&bits, h->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return LF_ECUDA;
  if (bits != 0 && cudaMemset(h->status, 0, sizeof(int)) != cudaSuccess) return LF_ECUDA;
  // a launch whose waits gave up may have left the dynamic schedule's row
  // counter away from zero
  if ((bits & LF_STATUS_WAIT_TIMEOUT) && cudaMemset(h->grab, 0, sizeof(unsigned)) != cudaSuccess)
    return LF_ECUDA;
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
