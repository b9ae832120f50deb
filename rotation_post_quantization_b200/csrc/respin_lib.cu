// Host side of the ReSpinQuant boundary library: the C ABI declared in
// include/respin.h (argument validation, plans, launch configuration, error
// reporting). One translation unit holds every kernel so that the device
// status word is a single symbol without relocatable device code.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <set>
#include <string>
#include <vector>

#include "respin.h"
#include "ptx.cuh"
#include "boundary_kernels.cuh"
#include "boundary_pair.cuh"
#include "boundary_rowtile.cuh"
#include "boundary_tc.cuh"
#include "factor_builder.h"
#include "weight_tool.h"
#include "w4a4_gemm_kernels.cuh"
#include "w4a4_gemm_skinny.cuh"

using namespace respin;

namespace {

thread_local std::string t_last_error;

respin_status_t fail(respin_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return st;
}

respin_status_t ok() {
  return RESPIN_OK;
}

respin_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(RESPIN_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// Host-side fault hook: RESPIN_FAULT=<site> makes the named site fail as if
// the underlying operation had failed, without touching the device. Sites:
// "plan_alloc" (device allocation in plan creation) and "launch" (kernel
// launch in the compute calls).
bool fault_at(const char* site) {
  const char* f = std::getenv("RESPIN_FAULT");
  return f != nullptr && std::strcmp(f, site) == 0;
}

bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

// ------------------------------------------------------------ plans

enum BoundaryKind { kRowTile = 0, kClusterRf = 1, kClusterSmem = 2 };

struct BoundaryConfig {
  BoundaryKind kind = kClusterSmem;  // boundary_rowtile_kernel / cluster kernels
  bool rf = false;          // register-resident factors (boundary_cluster_rf_kernel)
  int T = 0, R = 0, cluster = 0, Dc = 0;
  size_t smem = 0;
  int max_clusters = 0;
  const void* fn = nullptr;
};

}  // namespace

struct respin_plan_s {
  int D = 0, r = 0, r_pad = 0;
  unsigned flags = 0;
  int device = -1;
  __nv_bfloat16* factors = nullptr;  // 2 * D * r_pad bf16: U part then V part (layout of cfg)
  BoundaryConfig cfg;
  // Second configuration for calls with few tokens (row-tile plans only: a
  // cluster splits each tile over several SMs, so a short call is not one
  // SM's whole chain), with its own factor layout.
  bool has_small = false;
  __nv_bfloat16* factors_small = nullptr;
  BoundaryConfig cfg_small;
  // Third configuration for the fewest tokens: 8-CTA instead of 4-CTA
  // clusters (each SM pulls half the factor bytes of a tile from L2).
  bool has_tiny = false;
  __nv_bfloat16* factors_tiny = nullptr;
  BoundaryConfig cfg_tiny;
  // Plans made from the stored subspace form (Q, R_sub): the pair kernel.
  bool subspace = false;
  uint32_t* q_pair = nullptr;    // projection then re-projection fragments of Q (pr_pack_frags)
  float* m_pair = nullptr;       // M = R_sub - I, fp32 [32][32]
  const void* pair_fn = nullptr;
  size_t pair_smem = 0;
  int pair_max = 0;              // co-resident CTA pairs
  // Clusters of 4 (D = 4096: a quarter of the columns per CTA) for short calls.
  const void* quad_fn = nullptr;
  size_t quad_smem = 0;
  int quad_max = 0;              // co-resident 4-CTA clusters
  // Tensor-core passes (boundary_tc.cuh): tensor maps of U^T [tc_rp, D] and
  // V [D, tc_rp], the plan's own factors for padded rank 64 / 128 (the layout
  // of the shared-memory cluster kernel) or a copy padded to 64 (tc_factors)
  // for rank 16 / 32 plans on the register-factor cluster kernel.
  bool has_tc = false;
  int tc_rp = 0;                          // padded rank of the passes (64 or 128)
  int tc_min_tokens = 0;                  // calls from this many tokens on take them
  __nv_bfloat16* tc_factors = nullptr;    // own U^T / V copy when the plan's layout differs
  CUtensorMap tm_ut, tm_v;
  const void* tc_proj_fn = nullptr;
  const void* tc_re_fn = nullptr;
  size_t tc_proj_smem = 0, tc_re_smem = 0;
  int sms = 0;
};

// Calls with at least this many tokens take the tensor-core passes when the
// plan has them: padded rank 64 / 128, and padded rank 16 / 32 on the
// register-factor cluster kernel (D = 8192). Crossovers measured on B200 at
// D = 8192 (passes vs cluster kernel, before the passes became dependent
// launches): r = 64: 33 vs 34 us at 256 tokens; r = 32: 68 vs 62 us at 2048
// tokens and 159 vs 222 us at 8192 (now 140 us).
#ifndef RESPIN_TC_MIN_TOKENS
#define RESPIN_TC_MIN_TOKENS 256
#endif
#ifndef RESPIN_TC_MIN_TOKENS_LOW_RANK
#define RESPIN_TC_MIN_TOKENS_LOW_RANK 4096
#endif

// Calls with at most this many tokens use cfg_small when the plan has one
// (row tiles: one 16-token tile per SM; a 4-CTA cluster tile chain is about a
// third as long, so clusters win until their tile rounds add up).
constexpr int kSmallTokens = 1280;
// Calls with at most this many tokens (and no more tiles than co-resident
// 8-CTA clusters) use cfg_tiny. Measured on B200, D = 4096, r = 32, CUDA-graph
// replay, 4- vs 8-CTA clusters: N = 1: 6.7 vs 5.5 us, 8: 7.2 vs 6.2 us,
// 64: 7.8 vs 6.8 us; at 256 tokens (16 tiles) the 8-CTA clusters take two
// rounds: 7.8 vs 11.6 us.
constexpr int kTinyTokens = 128;

namespace {

std::mutex g_plans_mu;
std::set<respin_plan_s*> g_plans;

bool plan_alive(respin_plan_s* p) {
  std::lock_guard<std::mutex> lk(g_plans_mu);
  return g_plans.count(p) != 0;
}

// cuTensorMapEncodeTiled, fetched once through the runtime's driver entry
// point (no link-time dependency on the driver library).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    cudaGetLastError();
  });
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows, cols] matrix with a box of
// box_rows rows x 64 columns (128 bytes) in the 128-byte swizzle; rows past
// the end read as zeros.
bool make_tmap_bf16_tile(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows = kRtT) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 tensor map over a row-major [rows, cols] array with a
// {box_cols, box_rows} box and the given swizzle.
bool make_tmap_bf16(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_cols,
                    uint32_t box_rows, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int RP>
const void* tc_proj_fn() {
  return reinterpret_cast<const void*>(&boundary_tc_project_kernel<RP>);
}
template <int RP, bool F32>
const void* tc_re_fn() {
  return reinterpret_cast<const void*>(&boundary_tc_reproject_kernel<RP, F32>);
}

// A launch that may begin while the previous kernel of the stream finishes
// (programmatic stream serialization); the kernel waits for that kernel's
// results itself (grid_dep_wait).
cudaError_t launch_dependent(const void* fn, int grid, int block, size_t smem, cudaStream_t s, void** args) {
  cudaLaunchConfig_t lc = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  lc.blockDim = dim3(static_cast<unsigned>(block), 1, 1);
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  lc.attrs = attr;
  lc.numAttrs = 1;
  return cudaLaunchKernelExC(&lc, fn, args);
}

// The tensor-core passes of a plan: padded rank 64 / 128 (factors already
// stored as U^T then V), or padded rank 16 / 32 on the register-factor
// cluster kernel (D = 8192 and other widths the row-tile kernel does not
// take), which gets its own U^T / V copy padded to 64. ub / vb: the bf16 bits
// of U and V, [D][r_pad]. Leaves has_tc false where the passes do not apply.
void configure_tc(respin_plan_s* p, const uint16_t* ub, const uint16_t* vb) {
  const int D = p->D;
  const bool own = p->r_pad <= 32 && p->cfg.kind == kClusterRf;
  if (!own && ((p->r_pad != 64 && p->r_pad != 128) || p->cfg.kind != kClusterSmem || p->cfg.rf ||
               p->factors == nullptr))
    return;
  const int RP = own ? 64 : p->r_pad;
  const bool f32 = (p->flags & RESPIN_H_FP32_DEBUG) != 0;
  const void* pf = RP == 64 ? tc_proj_fn<64>() : tc_proj_fn<128>();
  const void* rf = RP == 64 ? (f32 ? tc_re_fn<64, true>() : tc_re_fn<64, false>())
                            : (f32 ? tc_re_fn<128, true>() : tc_re_fn<128, false>());
  const size_t ps = RP == 64 ? TcProjCfg<64>::kSmem : TcProjCfg<128>::kSmem;
  const size_t rs = RP == 64 ? TcReCfg<64>::kSmem : TcReCfg<128>::kSmem;
  if (cudaFuncSetAttribute(pf, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(ps)) != cudaSuccess ||
      cudaFuncSetAttribute(rf, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(rs)) != cudaSuccess) {
    cudaGetLastError();
    return;
  }
  if (own) {
    std::vector<uint16_t> w(static_cast<size_t>(2) * D * RP, 0);   // U^T [RP][D] then V [D][RP]
    for (int d = 0; d < D; ++d)
      for (int j = 0; j < p->r_pad; ++j) {
        w[static_cast<size_t>(j) * D + d] = ub[static_cast<size_t>(d) * p->r_pad + j];
        w[static_cast<size_t>(RP) * D + static_cast<size_t>(d) * RP + j] = vb[static_cast<size_t>(d) * p->r_pad + j];
      }
    if (cudaMalloc(&p->tc_factors, w.size() * sizeof(uint16_t)) != cudaSuccess) {
      cudaGetLastError();
      p->tc_factors = nullptr;
      return;
    }
    if (cudaMemcpy(p->tc_factors, w.data(), w.size() * sizeof(uint16_t), cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaGetLastError();
      cudaFree(p->tc_factors);
      p->tc_factors = nullptr;
      return;
    }
  }
  const __nv_bfloat16* ut = own ? p->tc_factors : p->factors;
  const __nv_bfloat16* v = ut + static_cast<size_t>(RP) * D;
  if (!make_tmap_bf16(&p->tm_ut, ut, RP, D, 64, RP, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_bf16(&p->tm_v, v, D, RP, 64, kTcBN, CU_TENSOR_MAP_SWIZZLE_128B))
    return;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, p->device) != cudaSuccess || sms <= 0) {
    cudaGetLastError();
    return;
  }
  p->tc_proj_fn = pf;
  p->tc_re_fn = rf;
  p->tc_proj_smem = ps;
  p->tc_re_smem = rs;
  p->sms = sms;
  p->tc_rp = RP;
  p->tc_min_tokens = own ? RESPIN_TC_MIN_TOKENS_LOW_RANK : RESPIN_TC_MIN_TOKENS;
  p->has_tc = true;
}

template <int R, int W, int NB, bool F32>
const void* rowtile_fn() {
  return reinterpret_cast<const void*>(&boundary_rowtile_kernel<R, W, NB, F32>);
}

// Warps per CTA of the row-tile kernel (8: the register budget of the
// prefetched factor fragments; 16 warps with shallower prefetch measured
// slower).
int rowtile_warps(int) { return 8; }

const void* pick_rowtile_fn(int R, int D, bool f32) {
  const int NB = D / (64 * 8);
#define RESPIN_PICK(RR, BB) \
  if (R == RR && NB == BB) return f32 ? rowtile_fn<RR, 8, BB, true>() : rowtile_fn<RR, 8, BB, false>();
  RESPIN_PICK(16, 2) RESPIN_PICK(16, 4) RESPIN_PICK(16, 8)
  RESPIN_PICK(32, 2) RESPIN_PICK(32, 4) RESPIN_PICK(32, 8)
#undef RESPIN_PICK
  return nullptr;
}

size_t rowtile_smem(int R, int D) { return R == 16 ? RtCfg<16, 8>::smem(D) : RtCfg<32, 8>::smem(D); }

template <int T, int R, bool F32, bool VRES>
const void* smem_fn() {
  return reinterpret_cast<const void*>(&boundary_cluster_smem_kernel<T, R, F32, VRES>);
}

// vres = false: the V slice is read from global memory (16-token tiles,
// r = 64 or 128 only).
const void* pick_smem_fn(int T, int R, bool f32, bool vres) {
#define RESPIN_PICK(TT, RR)                                                   \
  if (T == TT && R == RR) return f32 ? smem_fn<TT, RR, true, true>() : smem_fn<TT, RR, false, true>();
  if (vres) {
    RESPIN_PICK(32, 16) RESPIN_PICK(32, 32) RESPIN_PICK(32, 64)
    RESPIN_PICK(16, 16) RESPIN_PICK(16, 32) RESPIN_PICK(16, 64) RESPIN_PICK(16, 128)
    return nullptr;
  }
#undef RESPIN_PICK
  if (T == 16 && R == 64) return f32 ? smem_fn<16, 64, true, false>() : smem_fn<16, 64, false, false>();
  if (T == 16 && R == 128) return f32 ? smem_fn<16, 128, true, false>() : smem_fn<16, 128, false, false>();
  return nullptr;
}

constexpr int kRfT = 16;  // tokens per tile of the register-factor kernel

template <int R, int Dc, bool F32>
const void* rf_fn() {
  return reinterpret_cast<const void*>(&boundary_cluster_rf_kernel<R, kRfT, Dc, F32>);
}

const void* pick_rf_fn(int R, int Dc, bool f32) {
#define RESPIN_PICK(RR, DD)                                                   \
  if (R == RR && Dc == DD) return f32 ? rf_fn<RR, DD, true>() : rf_fn<RR, DD, false>();
  RESPIN_PICK(16, 256) RESPIN_PICK(16, 512) RESPIN_PICK(16, 1024)
  RESPIN_PICK(32, 256) RESPIN_PICK(32, 512) RESPIN_PICK(32, 1024)
#undef RESPIN_PICK
  return nullptr;
}

size_t rf_smem(int R, int Dc) {
#define RESPIN_SMEM(RR, DD) \
  if (R == RR && Dc == DD) return RfCfg<RR, kRfT, DD>::kSmem;
  RESPIN_SMEM(16, 256) RESPIN_SMEM(16, 512) RESPIN_SMEM(16, 1024)
  RESPIN_SMEM(32, 256) RESPIN_SMEM(32, 512) RESPIN_SMEM(32, 1024)
#undef RESPIN_SMEM
  return 0;
}

// Largest number of co-resident clusters of `C` CTAs for kernel `fn`
// (0 if the configuration cannot be launched).
int max_active_clusters(const void* fn, int C, size_t smem, int threads) {
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (C > 8 && cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t lc = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  lc.gridDim = dim3(C, 1, 1);
  lc.blockDim = dim3(threads, 1, 1);
  lc.dynamicSmemBytes = smem;
  lc.attrs = attr;
  lc.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fn, &lc) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

// Choose the boundary kernel. r <= 32: register-resident factors with 512
// (else 256) columns per CTA. Otherwise: shared-memory factors, the smallest
// cluster whose per-CTA slice fits, preferring 32-token tiles.
// only_dc > 0: the register-factor cluster kernel with that column slice, or
// UNSUPPORTED.
respin_status_t configure_boundary(int D, int R, bool f32, BoundaryConfig* out, bool allow_rowtile = true,
                                   int only_dc = 0) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int smem_optin = 0;
  e = cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  // Whole 16-token rows per CTA, factors streamed from L2 (no cluster).
  if (allow_rowtile && R <= 32 && (D == 1024 || D == 2048 || D == 4096)) {
    const size_t smem = rowtile_smem(R, D);
    const void* fn = pick_rowtile_fn(R, D, f32);
    int sms = 0;
    if (fn && smem <= static_cast<size_t>(smem_optin) &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) ==
            cudaSuccess) {
      out->kind = kRowTile; out->rf = false; out->T = kRtT; out->R = R; out->cluster = rowtile_warps(D); out->Dc = D;
      out->smem = smem; out->max_clusters = sms; out->fn = fn;
      return ok();
    }
    cudaGetLastError();
  }
  if (R <= 32) {
    for (int Dc : {1024, 512, 256}) {
      if (D % Dc || D / Dc > 16 || (only_dc > 0 && Dc != only_dc)) continue;
      const int C = D / Dc;
      const size_t smem = rf_smem(R, Dc);
      if (smem == 0 || smem > static_cast<size_t>(smem_optin)) continue;
      const void* fn = pick_rf_fn(R, Dc, f32);
      const int n = max_active_clusters(fn, C, smem, kRfThreads);
      if (n <= 0) continue;
      out->kind = kClusterRf; out->rf = true; out->T = kRfT; out->R = R; out->cluster = C; out->Dc = Dc;
      out->smem = smem; out->max_clusters = n; out->fn = fn;
      return ok();
    }
  }
  if (only_dc > 0) return fail(RESPIN_ERR_UNSUPPORTED, "no register-factor configuration with Dc=%d", only_dc);
  // Shared-memory factor slices (both, else U^T only with V read from L2).
  for (bool vres : {true, false}) {
    for (int C : {1, 2, 4, 8, 16}) {
      if (D % C) continue;
      const int Dc = D / C;
      if (Dc % 64) continue;
      for (int T : {32, 16}) {
        if (T * R > 2048) continue;
        const void* fn = pick_smem_fn(T, R, f32, vres);
        if (!fn) continue;
        const size_t smem = boundary_smem_layout(T, R, Dc, vres).total;
        if (smem > static_cast<size_t>(smem_optin)) continue;
        const int n = max_active_clusters(fn, C, smem, kBoundaryThreads);
        if (n <= 0) continue;
        out->kind = kClusterSmem; out->rf = false; out->T = T; out->R = R; out->cluster = C; out->Dc = Dc;
        out->smem = smem; out->max_clusters = n; out->fn = fn;
        return ok();
      }
    }
  }
  return fail(RESPIN_ERR_UNSUPPORTED,
              "no cluster configuration holds the factor slices for D=%d, padded r=%d", D, R);
}

template <int DC, bool F32, int CS = 2>
const void* pair_fn() {
  return reinterpret_cast<const void*>(&boundary_pair_kernel<DC, F32, CS>);
}

// The pair kernel for D columns (D / 2 per CTA) and its co-resident pairs.
respin_status_t configure_pair(int D, bool f32, respin_plan_s* p) {
  const int DC = D / 2;
  const void* fn = nullptr;
  size_t smem = 0;
  if (DC == 1024) { fn = f32 ? pair_fn<1024, true>() : pair_fn<1024, false>(); smem = PrCfg<1024>::kSmem; }
  if (DC == 2048) { fn = f32 ? pair_fn<2048, true>() : pair_fn<2048, false>(); smem = PrCfg<2048>::kSmem; }
  if (fn == nullptr)
    return fail(RESPIN_ERR_UNSUPPORTED, "subspace plans need D in {2048, 4096} (got D=%d)", D);
  const int n = max_active_clusters(fn, 2, smem, kPrThreads);
  if (n <= 0) return fail(RESPIN_ERR_UNSUPPORTED, "the pair kernel (%zu bytes of shared memory) cannot be launched", smem);
  p->pair_fn = fn;
  p->pair_smem = smem;
  p->pair_max = n;
  if (D == 4096) {   // clusters of 4 for short calls (optional)
    const void* qf = f32 ? pair_fn<1024, true, 4>() : pair_fn<1024, false, 4>();
    const size_t qs = PrCfg<1024, 4>::kSmem;
    const int nq = max_active_clusters(qf, 4, qs, kPrThreads);
    if (nq > 0) {
      p->quad_fn = qf;
      p->quad_smem = qs;
      p->quad_max = nq;
    }
    cudaGetLastError();
  }
  return ok();
}

respin_status_t check_device(int want) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != want)
    return fail(RESPIN_ERR_INVALID_ARG, "plan was created on device %d but device %d is current",
                want, dev);
  return ok();
}

}  // namespace

// Up to 128 tokens the weight stream is the bound and w4a4_gemm_skinny_kernel
// spreads it over O / 16 CTAs. Measured on B200 (K = O = 4096, CUDA-graph
// replay, weights larger than L2), skinny vs the tensor-memory kernel:
// N = 1: 4.1 vs 11.6 us, 64: 8.6 vs 16.9 us, 128: 14.3 vs 21.4 us; from 160
// tokens on the CTA-pair tiles win (19.4 us, flat up to 512 tokens; a
// 256-token skinny variant took 22-27 us and single CTAs with K split over a
// cluster 22-24 us there).
#ifndef RESPIN_GEMM_SKINNY_MAX_TOKENS
#define RESPIN_GEMM_SKINNY_MAX_TOKENS 128
#endif
static_assert(RESPIN_GEMM_SKINNY_MAX_TOKENS <= 128, "the skinny GEMM holds at most 128 tokens per CTA");

template <int NT, int TG>
static cudaError_t launch_skinny(const uint8_t* qa, const float* sa, const uint8_t* qw, const float* sw, int N,
                                 int K, int O, void* out, cudaStream_t s, bool i32) {
  const dim3 grid(static_cast<unsigned>(O / kSkRows)), block(kSkThreads);
  if (i32)
    w4a4_gemm_skinny_kernel<NT, TG, true><<<grid, block, 0, s>>>(qa, sa, qw, sw, N, K, O, out);
  else
    w4a4_gemm_skinny_kernel<NT, TG, false><<<grid, block, 0, s>>>(qa, sa, qw, sw, N, K, O, out);
  return cudaGetLastError();
}

static respin_status_t gemm_skinny(const uint8_t* qa, const float* sa, const uint8_t* qw, const float* sw, int N,
                                   int K, int O, void* out, cudaStream_t s, bool i32) {
  cudaError_t e;
  if (N <= 8) e = launch_skinny<1, 1>(qa, sa, qw, sw, N, K, O, out, s, i32);
  else if (N <= 16) e = launch_skinny<2, 1>(qa, sa, qw, sw, N, K, O, out, s, i32);
  else if (N <= 32) e = launch_skinny<4, 1>(qa, sa, qw, sw, N, K, O, out, s, i32);
  else if (N <= 64) e = launch_skinny<4, 2>(qa, sa, qw, sw, N, K, O, out, s, i32);
  else e = launch_skinny<4, 4>(qa, sa, qw, sw, N, K, O, out, s, i32);
  if (e != cudaSuccess) return cuda_fail(e, "w4a4_gemm_skinny_kernel launch");
  return ok();
}

extern "C" {

const char* respin_last_error(void) { return t_last_error.c_str(); }

const char* respin_version(void) { return "respin-b200 0.1 (sm_100a)"; }

respin_status_t respin_plan_create(respin_plan_t* out, int D, int r, const float* U_r,
                                   const float* V_r, unsigned flags) {
  t_last_error.clear();
  if (out == nullptr) return fail(RESPIN_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (D < 128 || D > 65536 || D % 128)
    return fail(RESPIN_ERR_UNSUPPORTED, "D=%d: need 128 <= D <= 65536 and D %% 128 == 0", D);
  if (r < 0 || r > 128 || r % 8)
    return fail(RESPIN_ERR_UNSUPPORTED, "r=%d: need 0 <= r <= 128 and r %% 8 == 0", r);
  if (r > 0 && (U_r == nullptr || V_r == nullptr))
    return fail(RESPIN_ERR_INVALID_ARG, "U_r and V_r must be non-NULL when r > 0");
  if (flags & ~(RESPIN_H_FP32_DEBUG | RESPIN_ACT_INT3))
    return fail(RESPIN_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  const int r_pad = r == 0 ? 0 : (r <= 16 ? 16 : r <= 32 ? 32 : r <= 64 ? 64 : 128);
  if (fault_at("plan_alloc")) return fail(RESPIN_ERR_OOM, "injected fault at plan_alloc");

  respin_plan_s* p = new respin_plan_s();
  p->D = D; p->r = r; p->r_pad = r_pad; p->flags = flags;
  cudaError_t e = cudaGetDevice(&p->device);
  if (e != cudaSuccess) { delete p; return cuda_fail(e, "cudaGetDevice"); }
  if (r > 0) {
    respin_status_t st = configure_boundary(D, r_pad, (flags & RESPIN_H_FP32_DEBUG) != 0, &p->cfg);
    if (st != RESPIN_OK) { delete p; return st; }
    // Factors as bf16 (round to nearest even), zero padded to r_pad columns.
    std::vector<uint16_t> ub(static_cast<size_t>(D) * r_pad, 0), vb(static_cast<size_t>(D) * r_pad, 0);
    for (int d = 0; d < D; ++d)
      for (int j = 0; j < r; ++j) {
        const __nv_bfloat16 u = __float2bfloat16_rn(U_r[static_cast<size_t>(d) * r + j]);
        const __nv_bfloat16 v = __float2bfloat16_rn(V_r[static_cast<size_t>(d) * r + j]);
        ub[static_cast<size_t>(d) * r_pad + j] = *reinterpret_cast<const uint16_t*>(&u);
        vb[static_cast<size_t>(d) * r_pad + j] = *reinterpret_cast<const uint16_t*>(&v);
      }
    // Device layouts: fragment order for the row-tile and the register-factor
    // kernels, else U^T [r_pad, D] followed by V [D, r_pad].
    auto layout = [&](const BoundaryConfig& c) {
      std::vector<uint32_t> w(static_cast<size_t>(D) * r_pad, 0);  // 2 * D * r_pad bf16
      const size_t half = static_cast<size_t>(D) * r_pad / 2;
      if (c.kind == kRowTile) {
        rt_pack_factors(ub.data(), vb.data(), D, r_pad, w.data(), w.data() + half);
      } else if (c.rf) {
        rf_pack_factors(ub.data(), vb.data(), D, r_pad, c.T, c.Dc, w.data(), w.data() + half);
      } else {
        uint16_t* h16 = reinterpret_cast<uint16_t*>(w.data());
        for (int d = 0; d < D; ++d)
          for (int j = 0; j < r_pad; ++j) {
            h16[static_cast<size_t>(j) * D + d] = ub[static_cast<size_t>(d) * r_pad + j];
            h16[static_cast<size_t>(r_pad) * D + static_cast<size_t>(d) * r_pad + j] =
                vb[static_cast<size_t>(d) * r_pad + j];
          }
      }
      return w;
    };
    auto upload = [&](const BoundaryConfig& c, __nv_bfloat16** dst) -> respin_status_t {
      const std::vector<uint32_t> w = layout(c);
      cudaError_t e2 = cudaMalloc(dst, w.size() * sizeof(uint32_t));
      if (e2 != cudaSuccess) {
        cudaGetLastError();
        *dst = nullptr;
        return fail(RESPIN_ERR_OOM, "cudaMalloc factors: %s", cudaGetErrorString(e2));
      }
      e2 = cudaMemcpy(*dst, w.data(), w.size() * sizeof(uint32_t), cudaMemcpyHostToDevice);
      if (e2 != cudaSuccess) return cuda_fail(e2, "cudaMemcpy factors");
      return ok();
    };
    respin_status_t st2 = upload(p->cfg, &p->factors);
    if (st2 == RESPIN_OK && p->cfg.kind == kRowTile &&
        configure_boundary(D, r_pad, (flags & RESPIN_H_FP32_DEBUG) != 0, &p->cfg_small, false) == RESPIN_OK) {
      st2 = upload(p->cfg_small, &p->factors_small);
      p->has_small = st2 == RESPIN_OK;
    }
    if (st2 == RESPIN_OK && p->has_small && p->cfg_small.rf && p->cfg_small.cluster == 4 &&
        configure_boundary(D, r_pad, (flags & RESPIN_H_FP32_DEBUG) != 0, &p->cfg_tiny, false, 512) == RESPIN_OK &&
        p->cfg_tiny.cluster == 8) {
      st2 = upload(p->cfg_tiny, &p->factors_tiny);
      p->has_tiny = st2 == RESPIN_OK;
    }
    t_last_error.clear();
    if (st2 != RESPIN_OK || p->factors == nullptr) {
      if (p->factors) cudaFree(p->factors);
      if (p->factors_small) cudaFree(p->factors_small);
      if (p->factors_tiny) cudaFree(p->factors_tiny);
      delete p;
      return st2 != RESPIN_OK ? st2 : fail(RESPIN_ERR_OOM, "factor upload failed");
    }
    configure_tc(p, ub.data(), vb.data());
    t_last_error.clear();
  }
  {
    std::lock_guard<std::mutex> lk(g_plans_mu);
    g_plans.insert(p);
  }
  *out = p;
  return ok();
}

respin_status_t respin_plan_create_subspace(respin_plan_t* out, int D, int r, const float* Q,
                                            const float* R_sub, unsigned flags) {
  t_last_error.clear();
  if (out == nullptr) return fail(RESPIN_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (D < 128 || D > 65536 || D % 128)
    return fail(RESPIN_ERR_UNSUPPORTED, "D=%d: need 128 <= D <= 65536 and D %% 128 == 0", D);
  if (r < 1 || r > kPrR) return fail(RESPIN_ERR_UNSUPPORTED, "r=%d: subspace plans need 1 <= r <= %d", r, kPrR);
  if (Q == nullptr || R_sub == nullptr) return fail(RESPIN_ERR_INVALID_ARG, "Q and R_sub must be non-NULL");
  if (flags & ~(RESPIN_H_FP32_DEBUG | RESPIN_ACT_INT3))
    return fail(RESPIN_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if (fault_at("plan_alloc")) return fail(RESPIN_ERR_OOM, "injected fault at plan_alloc");
  respin_plan_s* p = new respin_plan_s();
  p->D = D; p->r = r; p->r_pad = kPrR; p->flags = flags; p->subspace = true;
  cudaError_t e = cudaGetDevice(&p->device);
  if (e != cudaSuccess) { delete p; return cuda_fail(e, "cudaGetDevice"); }
  respin_status_t st = configure_pair(D, (flags & RESPIN_H_FP32_DEBUG) != 0, p);
  if (st != RESPIN_OK) { delete p; return st; }
  // Q as bf16 (round to nearest even), as the kernel's two fragment streams;
  // M = R_sub - I formed exactly in double and rounded once to float, zero
  // padded.
  std::vector<uint16_t> qb(static_cast<size_t>(D) * r);
  std::vector<uint32_t> qpk(static_cast<size_t>(D) * kPrR);   // 2 streams of D * 32 bf16
  for (size_t i = 0; i < qb.size(); ++i) {
    const __nv_bfloat16 v = __float2bfloat16_rn(Q[i]);
    qb[i] = *reinterpret_cast<const uint16_t*>(&v);
  }
  pr_pack_frags(qb.data(), D, r, qpk.data(), qpk.data() + qpk.size() / 2);
  std::vector<float> m(kPrR * kPrR, 0.0f);
  for (int i = 0; i < r; ++i)
    for (int j = 0; j < r; ++j)
      m[i * kPrR + j] = static_cast<float>(static_cast<double>(R_sub[static_cast<size_t>(i) * r + j]) - (i == j ? 1.0 : 0.0));
  e = cudaMalloc(&p->q_pair, qpk.size() * sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMalloc(&p->m_pair, m.size() * sizeof(float));
  if (e != cudaSuccess) {
    cudaGetLastError();
    if (p->q_pair) cudaFree(p->q_pair);
    delete p;
    return fail(RESPIN_ERR_OOM, "cudaMalloc subspace factors: %s", cudaGetErrorString(e));
  }
  e = cudaMemcpy(p->q_pair, qpk.data(), qpk.size() * sizeof(uint32_t), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(p->m_pair, m.data(), m.size() * sizeof(float), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(p->q_pair);
    cudaFree(p->m_pair);
    delete p;
    return cuda_fail(e, "cudaMemcpy subspace factors");
  }
  {
    std::lock_guard<std::mutex> lk(g_plans_mu);
    g_plans.insert(p);
  }
  *out = p;
  return ok();
}

respin_status_t respin_plan_destroy(respin_plan_t plan) {
  t_last_error.clear();
  if (plan == nullptr) return ok();
  {
    std::lock_guard<std::mutex> lk(g_plans_mu);
    if (!g_plans.erase(plan)) return fail(RESPIN_ERR_INVALID_ARG, "unknown or destroyed plan");
  }
  respin_status_t st = RESPIN_OK;
  if (plan->factors || plan->q_pair) {
    int cur = -1;
    cudaGetDevice(&cur);
    cudaSetDevice(plan->device);
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess && plan->factors) e = cudaFree(plan->factors);
    if (e == cudaSuccess && plan->q_pair) e = cudaFree(plan->q_pair);
    if (e == cudaSuccess && plan->m_pair) e = cudaFree(plan->m_pair);
    if (e == cudaSuccess && plan->factors_small) e = cudaFree(plan->factors_small);
    if (e == cudaSuccess && plan->factors_tiny) e = cudaFree(plan->factors_tiny);
    if (e == cudaSuccess && plan->tc_factors) e = cudaFree(plan->tc_factors);
    if (e != cudaSuccess) st = cuda_fail(e, "releasing plan factors");
    cudaSetDevice(cur);
  }
  delete plan;
  return st;
}

respin_status_t respin_boundary_forward(respin_plan_t plan, const void* x, const void* residual,
                                        int N, void* h_out, uint8_t* q_packed, float* scale,
                                        void* stream) {
  t_last_error.clear();
  if (plan == nullptr || !plan_alive(plan)) return fail(RESPIN_ERR_INVALID_ARG, "unknown or destroyed plan");
  if (N < 0) return fail(RESPIN_ERR_INVALID_ARG, "N=%d is negative", N);
  if (N == 0) return ok();
  if (x == nullptr || q_packed == nullptr || scale == nullptr)
    return fail(RESPIN_ERR_INVALID_ARG, "x, q_packed and scale must be non-NULL");
  if (!aligned(x, 16) || !aligned(residual, 16) || !aligned(h_out, 16) || !aligned(q_packed, 16))
    return fail(RESPIN_ERR_ALIGNMENT, "x, residual, h_out and q_packed must be 16-byte aligned");
  if (!aligned(scale, 4)) return fail(RESPIN_ERR_ALIGNMENT, "scale must be 4-byte aligned");
  if (fault_at("launch")) return fail(RESPIN_ERR_CUDA, "injected fault at launch");
  respin_status_t st = check_device(plan->device);
  if (st != RESPIN_OK) return st;

  const int D = plan->D;
  const bool f32 = (plan->flags & RESPIN_H_FP32_DEBUG) != 0;
  float qmax = (plan->flags & RESPIN_ACT_INT3) != 0 ? 3.0f : 7.0f;   // largest code magnitude
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bf16* xb = static_cast<const bf16*>(x);
  const bf16* rb = static_cast<const bf16*>(residual);

  if (plan->r == 0 || residual == nullptr) {
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, plan->device);
    const int grid = N < sms * 16 ? N : sms * 16;
#define RESPIN_ROWWISE(TH, VP)                                                                           \
  {                                                                                                     \
    if (f32) boundary_rowwise_kernel<TH, VP, true><<<grid, TH, 0, s>>>(xb, rb, N, D, h_out, q_packed, scale, qmax); \
    else boundary_rowwise_kernel<TH, VP, false><<<grid, TH, 0, s>>>(xb, rb, N, D, h_out, q_packed, scale, qmax);   \
  }
    if (D <= 256 * 8 * 2) RESPIN_ROWWISE(256, 2)
    else if (D <= 256 * 8 * 4) RESPIN_ROWWISE(256, 4)
    else if (D <= 256 * 8 * 8) RESPIN_ROWWISE(256, 8)
    else RESPIN_ROWWISE(1024, 8)
#undef RESPIN_ROWWISE
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "boundary_rowwise_kernel launch");
    return ok();
  }

  if (plan->subspace) {
    // T <= 16 tokens per tile. While full tiles need at most half of the
    // co-resident pairs (one CTA per SM), tiles are full; beyond that T is
    // chosen so that every pair gets the same number of tiles (two CTAs per
    // SM share the work evenly).
    const long long tiles16 = (static_cast<long long>(N) + kPrT - 1) / kPrT;
    if (plan->quad_fn != nullptr && tiles16 <= plan->quad_max / 2) {
      // short call: clusters of 4, full 16-token tiles, at most one CTA per SM
      CUtensorMap tmR, tmX;
      if (!make_tmap_bf16_tile(&tmR, residual, N, D, kPrT) || !make_tmap_bf16_tile(&tmX, x, N, D, kPrT))
        return fail(RESPIN_ERR_CUDA, "cuTensorMapEncodeTiled failed for the residual / x tiles");
      const uint4* pf = reinterpret_cast<const uint4*>(plan->q_pair);
      const uint4* rf = reinterpret_cast<const uint4*>(plan->q_pair + static_cast<size_t>(D) * kPrR / 2);
      const float* mg = plan->m_pair;
      int Dv = D, Tq = kPrT;
      void* args[] = {&tmR, &tmX, &pf, &rf, &mg, &N, &Dv, &Tq, &h_out, &q_packed, &scale, &qmax};
      cudaLaunchConfig_t lc = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 4;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      lc.gridDim = dim3(static_cast<unsigned>(4 * tiles16), 1, 1);
      lc.blockDim = dim3(kPrThreads, 1, 1);
      lc.dynamicSmemBytes = plan->quad_smem;
      lc.stream = s;
      lc.attrs = attr;
      lc.numAttrs = 1;
      cudaError_t e = cudaLaunchKernelExC(&lc, plan->quad_fn, args);
      if (e != cudaSuccess) return cuda_fail(e, "boundary_pair_kernel (clusters of 4) launch");
      return ok();
    }
    int T = kPrT;
    if (tiles16 > plan->pair_max / 2) {
      const long long per = static_cast<long long>(plan->pair_max) * kPrT;
      const int k = static_cast<int>((N + per - 1) / per);
      const long long slots = static_cast<long long>(plan->pair_max) * k;
      T = static_cast<int>((N + slots - 1) / slots);
    }
    if (T < 1) T = 1;
    const int ntiles = (N + T - 1) / T;
    const int pairs = ntiles < plan->pair_max ? ntiles : plan->pair_max;
    CUtensorMap tmR, tmX;
    if (!make_tmap_bf16_tile(&tmR, residual, N, D, kPrT) || !make_tmap_bf16_tile(&tmX, x, N, D, kPrT))
      return fail(RESPIN_ERR_CUDA, "cuTensorMapEncodeTiled failed for the residual / x tiles");
    const uint4* pf = reinterpret_cast<const uint4*>(plan->q_pair);
    const uint4* rf = reinterpret_cast<const uint4*>(plan->q_pair + static_cast<size_t>(D) * kPrR / 2);
    const float* mg = plan->m_pair;
    int Dv = D;
    void* args[] = {&tmR, &tmX, &pf, &rf, &mg, &N, &Dv, &T, &h_out, &q_packed, &scale, &qmax};
    cudaLaunchConfig_t lc = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    lc.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
    lc.blockDim = dim3(kPrThreads, 1, 1);
    lc.dynamicSmemBytes = plan->pair_smem;
    lc.stream = s;
    lc.attrs = attr;
    lc.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelExC(&lc, plan->pair_fn, args);
    if (e != cudaSuccess) return cuda_fail(e, "boundary_pair_kernel launch");
    return ok();
  }

  if (plan->has_tc && N >= plan->tc_min_tokens && h_out != nullptr) {
    // Three launches: y partials (into the code buffer's rows), h' with the
    // per-token amax (into the scale buffer), codes and scales.
    const int RP = plan->tc_rp;
    int KB = D / 64;
    const int mtiles = (N + kTcBM - 1) / kTcBM;
    int S = plan->sms / mtiles;   // one CTA per SM, all in one wave
    const int smax = D / (8 * RP);   // partials of a token fit in its D / 2 code bytes
    if (S > smax) S = smax;
    if (S > KB) S = KB;
    if (S > 8) S = 8;
    if (S < 1) S = 1;
    CUtensorMap tmR, tmRc, tmXc, tmH;
    if (!make_tmap_bf16(&tmR, residual, N, D, 64, kTcBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_bf16(&tmRc, residual, N, D, kTcChunk, kTcBM, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_tmap_bf16(&tmXc, x, N, D, kTcChunk, kTcBM, CU_TENSOR_MAP_SWIZZLE_64B) ||
        (!f32 && !make_tmap_bf16(&tmH, h_out, N, D, kTcChunk, 32, CU_TENSOR_MAP_SWIZZLE_64B)))
      return fail(RESPIN_ERR_CUDA, "cuTensorMapEncodeTiled failed for the tensor-core boundary tiles");
    if (f32) tmH = tmRc;   // not used by the fp32-h variant
    cudaError_t e;
    uint8_t* ypart = static_cast<uint8_t*>(q_packed);
    int ypitch = D / 2, Nv = N, Dv = D;
    {
      void* args[] = {&tmR, &plan->tm_ut, &Nv, &KB, &S, &ypart, &ypitch, &scale};
      e = cudaLaunchKernel(plan->tc_proj_fn, dim3(static_cast<unsigned>(mtiles * S)), dim3(128), args,
                           plan->tc_proj_smem, s);
      if (e != cudaSuccess) return cuda_fail(e, "boundary_tc_project_kernel launch");
    }
    {
      const long long tiles = static_cast<long long>(mtiles) * (D / kTcBN);
      const int grid = tiles < plan->sms ? static_cast<int>(tiles) : plan->sms;
      const uint8_t* yp = ypart;
      void* args[] = {&tmRc, &tmXc, &tmH, &plan->tm_v, &Nv, &Dv, &S, &yp, &ypitch, &h_out, &scale};
      e = launch_dependent(plan->tc_re_fn, grid, 320, plan->tc_re_smem, s, args);
      if (e != cudaSuccess) return cuda_fail(e, "boundary_tc_reproject_kernel launch");
    }
    {
      const int grid = N < plan->sms * 8 ? N : plan->sms * 8;
      const void* hq = h_out;
      uint8_t* qp = q_packed;
      float* sp = scale;
      void* args[] = {&hq, &Nv, &Dv, &qp, &sp, &qmax};
      e = launch_dependent(f32 ? reinterpret_cast<const void*>(&boundary_quant_rows_kernel<true>)
                               : reinterpret_cast<const void*>(&boundary_quant_rows_kernel<false>),
                           grid, 256, 0, s, args);
      if (e != cudaSuccess) return cuda_fail(e, "boundary_quant_rows_kernel launch");
    }
    return ok();
  }

  const bool tiny = plan->has_tiny && N <= kTinyTokens && (N + kRfT - 1) / kRfT <= plan->cfg_tiny.max_clusters;
  const bool small = !tiny && plan->has_small && N <= kSmallTokens;
  const BoundaryConfig& c = tiny ? plan->cfg_tiny : small ? plan->cfg_small : plan->cfg;
  const bf16* fac = tiny ? plan->factors_tiny : small ? plan->factors_small : plan->factors;
  const int ntiles = (N + c.T - 1) / c.T;
  if (c.kind == kRowTile) {
    CUtensorMap tmR, tmX;
    if (!make_tmap_bf16_tile(&tmR, residual, N, D) || !make_tmap_bf16_tile(&tmX, x, N, D))
      return fail(RESPIN_ERR_CUDA, "cuTensorMapEncodeTiled failed for the boundary tiles");
    const uint4* ut = reinterpret_cast<const uint4*>(fac);
    const uint4* vt = reinterpret_cast<const uint4*>(fac + static_cast<size_t>(plan->r_pad) * D);
    const int grid = ntiles < c.max_clusters ? ntiles : c.max_clusters;
    void* args[] = {&tmR, &tmX, &ut, &vt, &N, &h_out, &q_packed, &scale, &qmax};
    cudaError_t e = launch_dependent(c.fn, grid, 32 * c.cluster, c.smem, s, args);
    if (e != cudaSuccess) return cuda_fail(e, "boundary_rowtile_kernel launch");
    return ok();
  }
  const int nclusters = ntiles < c.max_clusters ? ntiles : c.max_clusters;
  cudaLaunchConfig_t lc = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = c.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  lc.gridDim = dim3(nclusters * c.cluster, 1, 1);
  lc.blockDim = dim3(c.rf ? kRfThreads : kBoundaryThreads, 1, 1);
  lc.dynamicSmemBytes = c.smem;
  lc.stream = s;
  lc.attrs = attr;
  lc.numAttrs = 1;
  cudaError_t e;
  if (c.rf) {
    const uint4* uf = reinterpret_cast<const uint4*>(fac);
    const uint4* vf = reinterpret_cast<const uint4*>(fac + static_cast<size_t>(plan->r_pad) * D);
    void* args[] = {&xb, &rb, &uf, &vf, &N, const_cast<int*>(&D), &h_out, &q_packed, &scale, &qmax};
    e = cudaLaunchKernelExC(&lc, c.fn, args);
  } else {
    const bf16* ut = fac;
    const bf16* v = fac + static_cast<size_t>(plan->r_pad) * D;
    int Dc = c.Dc;
    void* args[] = {&xb, &rb, &ut, &v, &N, const_cast<int*>(&D), &Dc, &h_out, &q_packed, &scale, &qmax};
    e = cudaLaunchKernelExC(&lc, c.fn, args);
  }
  if (e != cudaSuccess) return cuda_fail(e, "boundary_cluster_kernel launch");
  return ok();
}

extern "C++" {
template <int CG, bool I32, bool RM = false>
const void* gemm_fn() {
  return reinterpret_cast<const void*>(&w4a4_gemm_kernel<CG, I32, RM>);
}
template <bool I32, bool RM = false>
const void* gemm_ta_fn() {
  return reinterpret_cast<const void*>(&w4a4_gemm_ta_kernel<I32, RM>);
}
}

// CTA pairs read the activation operand from tensor memory
// (w4a4_gemm_ta_kernel); RESPIN_GEMM_PAIR_SMEM_A=1 builds the pair path on
// w4a4_gemm_kernel<2, ...> (both operands through shared memory) instead.
#ifndef RESPIN_GEMM_PAIR_SMEM_A
#define RESPIN_GEMM_PAIR_SMEM_A 0
#endif
static const void* gemm_pair_fn(bool i32, bool rm) {
#if RESPIN_GEMM_PAIR_SMEM_A
  return rm ? gemm_fn<2, false, true>() : i32 ? gemm_fn<2, true>() : gemm_fn<2, false>();
#else
  return rm ? gemm_ta_fn<false, true>() : i32 ? gemm_ta_fn<true>() : gemm_ta_fn<false>();
#endif
}
static constexpr int kGemmPairThreads = RESPIN_GEMM_PAIR_SMEM_A ? kGemmThreads : kTaThreads;
static constexpr int kGemmPairSmem = RESPIN_GEMM_PAIR_SMEM_A ? GemmCfg<2>::Smem : GemmTaCfg::Smem;

// The GEMM kernels need the large dynamic shared-memory carve-out; set it
// once per device and record how many CTA pairs can be co-resident.
struct GemmDeviceInfo {
  bool ready = false;
  int sms = 0;
  int max_pairs = 0;
};

static cudaError_t gemm_prepare(int dev, GemmDeviceInfo* info) {
  static std::mutex mu;
  static GemmDeviceInfo infos[256];
  if (dev < 0 || dev >= 256) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  GemmDeviceInfo& d = infos[dev];
  if (!d.ready) {
    cudaError_t e = cudaSuccess;
    const void* fns[6] = {gemm_fn<1, false>(), gemm_fn<1, true>(),   gemm_pair_fn(false, false),
                          gemm_pair_fn(true, false), gemm_fn<1, false, true>(), gemm_pair_fn(false, true)};
    const int smem[6] = {GemmCfg<1>::Smem, GemmCfg<1>::Smem, kGemmPairSmem,
                         kGemmPairSmem,    GemmCfg<1>::Smem, kGemmPairSmem};
    for (int i = 0; i < 6 && e == cudaSuccess; ++i)
      e = cudaFuncSetAttribute(fns[i], cudaFuncAttributeMaxDynamicSharedMemorySize, smem[i]);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t lc = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    lc.gridDim = dim3(2, 1, 1);
    lc.blockDim = dim3(kGemmPairThreads, 1, 1);
    lc.dynamicSmemBytes = kGemmPairSmem;
    lc.attrs = attr;
    lc.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&d.max_pairs, fns[2], &lc) != cudaSuccess) {
      cudaGetLastError();
      d.max_pairs = 0;
    }
    d.ready = true;
  }
  *info = d;
  return cudaSuccess;
}

// 2-D uint8 tensor map over a row-major [rows, cols] byte matrix with a box
// of [box_rows, box_cols] (out-of-range reads return zeros).
static bool make_tmap_u8(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols,
                         uint32_t box_rows, uint32_t box_cols,
                         CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D tensor map over the GEMM output [rows, cols] (bf16 or int32) for the
// epilogue's tensor stores: box of 64 bytes x 32 rows, 64-byte swizzle.
static bool make_tmap_out(CUtensorMap* m, void* ptr, uint64_t rows, uint64_t cols, bool i32) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const uint32_t es = i32 ? 4u : 2u;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * es};
  const cuuint32_t box[2] = {64u / es, 32u};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, i32 ? CU_TENSOR_MAP_DATA_TYPE_INT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static respin_status_t gemm_common(const uint8_t* q_act, const float* scale_act, const uint8_t* q_w,
                                   const float* scale_w, int N, int K, int O, void* out,
                                   void* stream, bool i32, float* rowmax = nullptr) {
  t_last_error.clear();
  if (N < 0) return fail(RESPIN_ERR_INVALID_ARG, "N=%d is negative", N);
  if (K < 128 || K > 65536 || K % 128)
    return fail(RESPIN_ERR_UNSUPPORTED, "K=%d: need 128 <= K <= 65536 and K %% 128 == 0", K);
  if (O < 16 || O % 16) return fail(RESPIN_ERR_UNSUPPORTED, "O=%d: need O >= 16 and O %% 16 == 0", O);
  if (N == 0) return ok();
  if (q_act == nullptr || q_w == nullptr || out == nullptr || (!i32 && (scale_act == nullptr || scale_w == nullptr)))
    return fail(RESPIN_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(q_act, 16) || !aligned(q_w, 16) || !aligned(out, 16))
    return fail(RESPIN_ERR_ALIGNMENT, "q_act, q_w and out must be 16-byte aligned");
  if (!aligned(scale_act, 4) || !aligned(scale_w, 16))
    return fail(RESPIN_ERR_ALIGNMENT, "scale_act must be 4-byte and scale_w 16-byte aligned");
  if (fault_at("launch")) return fail(RESPIN_ERR_CUDA, "injected fault at launch");

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (rowmax != nullptr && N <= RESPIN_GEMM_SKINNY_MAX_TOKENS)
    return fail(RESPIN_ERR_UNSUPPORTED, "row maxima need N > %d (the tensor-memory GEMM)", RESPIN_GEMM_SKINNY_MAX_TOKENS);
  if (rowmax != nullptr && !aligned(rowmax, 4)) return fail(RESPIN_ERR_ALIGNMENT, "rowmax must be 4-byte aligned");
  if (N <= RESPIN_GEMM_SKINNY_MAX_TOKENS) return gemm_skinny(q_act, scale_act, q_w, scale_w, N, K, O, out, s, i32);

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  GemmDeviceInfo info;
  e = gemm_prepare(dev, &info);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemm smem)");
  // CTA pairs (256-token tiles) from this many tokens on.
#ifndef RESPIN_GEMM_PAIR_MIN_TOKENS
#define RESPIN_GEMM_PAIR_MIN_TOKENS (kGemmBM + 1)
#endif
  const int CG = (N >= RESPIN_GEMM_PAIR_MIN_TOKENS && info.max_pairs > 0) ? 2 : 1;
  const long long tiles = static_cast<long long>((O + kGemmBN - 1) / kGemmBN) *
                          ((N + kGemmBM * CG - 1) / (kGemmBM * CG));
  CUtensorMap tmA, tmB, tmO;
  // the tensor-memory A path reads packed A rows one per lane: 64-byte swizzle
  const CUtensorMapSwizzle a_swizzle =
      (CG == 2 && !RESPIN_GEMM_PAIR_SMEM_A) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE;
  if (!make_tmap_u8(&tmA, q_act, N, K / 2, kGemmBM, kGemmBK / 2, a_swizzle) ||
      !make_tmap_u8(&tmB, q_w, O, K / 2, kGemmBN / CG, kGemmBK / 2) ||
      !make_tmap_out(&tmO, out, N, O, i32))
    return fail(RESPIN_ERR_CUDA, "cuTensorMapEncodeTiled failed for the GEMM operands or output");
  const void* fn = CG == 2             ? gemm_pair_fn(i32, rowmax != nullptr)
                   : rowmax != nullptr ? gemm_fn<1, false, true>()
                                       : (i32 ? gemm_fn<1, true>() : gemm_fn<1, false>());
  const long long groups = CG == 2 ? (tiles < info.max_pairs ? tiles : info.max_pairs)
                                   : (tiles < info.sms ? tiles : info.sms);
  cudaLaunchConfig_t lc = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CG;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent: set-up overlaps the previous kernel's tail; the
  // kernel waits for it before its first global access
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  lc.gridDim = dim3(static_cast<unsigned>(groups * CG), 1, 1);
  lc.blockDim = dim3(CG == 2 ? kGemmPairThreads : kGemmThreads, 1, 1);
  lc.dynamicSmemBytes = CG == 2 ? kGemmPairSmem : GemmCfg<1>::Smem;
  lc.stream = s;
  lc.attrs = attr;
  lc.numAttrs = 2;
  void* args[] = {&tmA, &tmB, &tmO, const_cast<float**>(&scale_act), const_cast<float**>(&scale_w), &N, &K, &O, &rowmax};
  e = cudaLaunchKernelExC(&lc, fn, args);
  if (e != cudaSuccess) return cuda_fail(e, "w4a4_gemm_kernel launch");
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "w4a4_gemm_kernel launch");
  return ok();
}

respin_status_t w4a4_gemm(const uint8_t* q_act, const float* scale_act, const uint8_t* q_w,
                          const float* scale_w, int N, int K, int O, void* out, void* stream) {
  return gemm_common(q_act, scale_act, q_w, scale_w, N, K, O, out, stream, false);
}

respin_status_t w4a4_gemm_i32(const uint8_t* q_act, const uint8_t* q_w, int N, int K, int O,
                              int32_t* acc_out, void* stream) {
  return gemm_common(q_act, nullptr, q_w, nullptr, N, K, O, acc_out, stream, true);
}

respin_status_t w4a4_gemm_rowmax(const uint8_t* q_act, const float* scale_act, const uint8_t* q_w,
                                 const float* scale_w, int N, int K, int O, void* out, float* rowmax,
                                 void* stream) {
  if (rowmax == nullptr) {
    t_last_error.clear();
    return fail(RESPIN_ERR_INVALID_ARG, "rowmax is NULL");
  }
  return gemm_common(q_act, scale_act, q_w, scale_w, N, K, O, out, stream, false, rowmax);
}

respin_status_t respin_quantize_rowmax(const void* u, const float* rowmax, int N, int D, uint8_t* q_packed,
                                       float* scale, unsigned flags, void* stream) {
  t_last_error.clear();
  if (N < 0) return fail(RESPIN_ERR_INVALID_ARG, "N=%d is negative", N);
  if (D < 256 || D > 65536 || D % 256)
    return fail(RESPIN_ERR_UNSUPPORTED, "D=%d: need 256 <= D <= 65536 and D %% 256 == 0", D);
  if (flags & ~RESPIN_ACT_INT3) return fail(RESPIN_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if (N == 0) return ok();
  if (u == nullptr || rowmax == nullptr || q_packed == nullptr || scale == nullptr)
    return fail(RESPIN_ERR_INVALID_ARG, "u, rowmax, q_packed and scale must be non-NULL");
  if (!aligned(u, 16) || !aligned(q_packed, 16)) return fail(RESPIN_ERR_ALIGNMENT, "u and q_packed must be 16-byte aligned");
  if (!aligned(rowmax, 4) || !aligned(scale, 4)) return fail(RESPIN_ERR_ALIGNMENT, "rowmax and scale must be 4-byte aligned");
  if (fault_at("launch")) return fail(RESPIN_ERR_CUDA, "injected fault at launch");
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  float qmax = (flags & RESPIN_ACT_INT3) != 0 ? 3.0f : 7.0f;
  int parts = D / kGemmBN;
  const int grid = N < sms * 8 ? N : sms * 8;
  void* args[] = {const_cast<void**>(&u), const_cast<float**>(&rowmax), &N, &D, &parts, &q_packed, &scale, &qmax};
  e = launch_dependent(reinterpret_cast<const void*>(&quant_rowmax_kernel), grid, 256, 0,
                       static_cast<cudaStream_t>(stream), args);
  if (e != cudaSuccess) return cuda_fail(e, "quant_rowmax_kernel launch");
  return ok();
}

respin_status_t respin_factors_from_subspace(int D, int r, const float* Q, const float* R_sub, float* U_r,
                                            float* V_r) {
  t_last_error.clear();
  if (host::factors_from_subspace(D, r, Q, R_sub, U_r, V_r) != host::BuildResult::kOk)
    return fail(RESPIN_ERR_INVALID_ARG, "need 0 < r <= D and non-NULL Q, R_sub, U_r, V_r");
  return ok();
}

respin_status_t respin_factors_from_transition(int D, int r, const float* T, double gap_tol, float* U_r,
                                               float* V_r, double* sigma) {
  t_last_error.clear();
  if (!(gap_tol >= 0.0)) return fail(RESPIN_ERR_INVALID_ARG, "gap_tol must be >= 0");
  double s[129] = {0.0};
  if (r > 128) return fail(RESPIN_ERR_INVALID_ARG, "r=%d: at most 128", r);
  host::BuildResult res;
  try {   // float64 copies of T (D x D) and of the iteration blocks
    res = host::factors_from_transition(D, r, T, gap_tol, U_r, V_r, s);
  } catch (const std::bad_alloc&) {
    return fail(RESPIN_ERR_OOM, "host memory for the %d x %d float64 transition", D, D);
  }
  switch (res) {
    case host::BuildResult::kOk:
      break;
    case host::BuildResult::kBadArg:
      return fail(RESPIN_ERR_INVALID_ARG, "need 0 < r < D and non-NULL T, U_r, V_r");
    case host::BuildResult::kNoGap:
      if (sigma != nullptr) std::memcpy(sigma, s, sizeof(double) * (r + 1));
      return fail(RESPIN_ERR_UNSUPPORTED,
                  "s_r - s_(r+1) = %.3e - %.3e is not above gap_tol * s_1 = %.3e: the top-%d truncation is not unique",
                  s[r - 1], s[r], gap_tol * s[0], r);
    default:
      return fail(RESPIN_ERR_UNSUPPORTED, "the subspace iteration did not converge");
  }
  if (sigma != nullptr) std::memcpy(sigma, s, sizeof(double) * (r + 1));
  return ok();
}

}  // extern "C"

namespace {

// One thread waits on an mbarrier that nothing arrives on, with the given
// limit: the wait gives up and records kSiteSelfTest. Nothing is copied, so
// nothing is in flight when the kernel returns.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  fence_mbarrier_init();
  mbar_wait(b, 0, kSiteSelfTest, limit_ns);
}

}  // namespace

extern "C" {

respin_status_t respin_selftest_wait_limit(unsigned limit_us, void* stream) {
  t_last_error.clear();
  if (limit_us == 0 || limit_us > 2000000u)
    return fail(RESPIN_ERR_INVALID_ARG, "limit_us=%u: need 1 <= limit_us <= 2000000", limit_us);
  selftest_wait_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint64_t>(limit_us) * 1000u);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "selftest_wait_kernel launch");
  return ok();
}

respin_status_t respin_fuse_weight(int O, int K, const float* W, const float* R_in, const float* R_out,
                                   float* W_fused) {
  t_last_error.clear();
  bool ok_ = false;
  try {
    ok_ = host::fuse_weight(O, K, W, R_in, R_out, W_fused);
  } catch (const std::bad_alloc&) {
    return fail(RESPIN_ERR_OOM, "host memory for the float64 copies of W and the rotations");
  }
  if (!ok_) return fail(RESPIN_ERR_INVALID_ARG, "need O > 0, K > 0 and non-NULL W, R_in, W_fused");
  return ok();
}

respin_status_t respin_quantize_weight(int O, int K, const float* W, int qmax, uint8_t* q_w, float* scale_w) {
  t_last_error.clear();
  if (!host::quantize_weight_rows(O, K, W, qmax, q_w, scale_w))
    return fail(RESPIN_ERR_INVALID_ARG, "need O > 0, even K > 0, qmax 7 or 3 and non-NULL pointers");
  return ok();
}

respin_status_t respin_device_status(int* code) {
  t_last_error.clear();
  if (code == nullptr) return fail(RESPIN_ERR_INVALID_ARG, "code is NULL");
  *code = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device status word");
    *code = v;
    return fail(RESPIN_ERR_DEVICE_CHECK, "a kernel gave up on a bounded wait (site %d)", v);
  }
  return ok();
}

}  // extern "C"
