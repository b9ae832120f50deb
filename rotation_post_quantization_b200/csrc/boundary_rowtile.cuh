// Row-tile block-boundary kernel: the rank-r basis fix and per-token INT4
// quantization for 16 whole tokens per CTA (r <= 32, D = 1024 / 2048 / 4096).
//
// Same arithmetic as the cluster kernels (subspace residual rotation of the
// ReSpinQuant explainers, zh §2.2 steps 1-3, row convention, then W4A4
// activation quantization, zh §3-§4):
//   y = residual U ;  h = (residual + x) + y V^T  (fp32) ;  h' = bf16(h)
//   amax = max|h'| ; inv = qmax/amax ; q = rint(h' inv)   (qmax = 7 or 3)
//
// Design (one CTA per SM, persistent over 16-token tiles, no cluster):
//  * the residual tile (16 x D bf16) is brought into shared memory by 2-D
//    tensor copies of 64-column blocks (16 rows x 128 bytes, 128-byte
//    swizzle: conflict-free ldmatrix and fragment accesses) and is turned into
//    h' in place;
//  * warp w owns columns [w D/8, (w+1) D/8). Phase 1 (projection y = res U)
//    runs on tensor cores (mma.sync m16n8k16 bf16, fp32 accumulate) with U
//    fragments read straight from global memory (L2-resident, shared by every
//    CTA, fragment-ordered by the plan so each load is a coalesced 16-byte
//    vector), two blocks ahead in registers. The eight partial y are summed in
//    warp order in shared memory (deterministic);
//  * phase 2 (re-projection): y split into bf16 hi + lo parts; V fragments
//    stream like U; x arrives per warp through a ring of 64-column blocks
//    (tensor copies), so the accumulators are finished as
//    h = (res + x) + y V^T, rounded to bf16 and written over the residual;
//  * the row amax is reduced across the warps, then all threads read the h'
//    tile once more in 16-byte chunks and write h' (128-byte row segments per
//    8 lanes) and the packed codes (32-byte row segments per 8 lanes). A
//    tensor store would hold its issuing thread for about 2 us on B200, longer
//    than these plain stores take.
// Each tensor copy is issued by its own lane: bulk copies from one thread
// complete one after the other, copies from different threads overlap.
// No wait is unbounded; a wait that gives up records a status code.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "boundary_kernels.cuh"
#include "ptx.cuh"

namespace respin {

constexpr int kRtT = 16;                 // tokens per tile
constexpr int kRtBlockBytes = 2048;      // one 64-column block: 16 rows x 128 bytes

// W warps per CTA; warp w owns D / W columns (NB 64-column blocks).
template <int R, int W>
struct RtCfg {
  static_assert(R == 16 || R == 32, "row-tile kernel: r <= 32");
  static_assert(W == 8 || W == 16, "8 or 16 warps");
  static constexpr int kWarps = W;
  static constexpr int kThreads = 32 * W;
  static constexpr int XS = W == 8 ? 4 : 2;      // x ring slots per warp
  static constexpr int RING = W == 8 ? 3 : 2;    // factor fragments of RING blocks in registers
  static constexpr int KK = R / 16;        // k16 steps of the re-projection
  static constexpr int NT = R / 8;         // n8 tiles of y
  static constexpr int UQ = R / 16;        // uint4 of U fragments per lane per k16 step
  static constexpr int UB = 4 * UQ;        // ... per 64-column block (4 k16 steps)
  static constexpr int VB = R / 4;         // uint4 of V fragments per lane per 64-column block
  static constexpr int YP = R + 4;         // padded fp32 row of y
  // shared-memory layout (offsets from a 1024-byte aligned base)
  __host__ __device__ static constexpr uint32_t x_ring(int D) { return static_cast<uint32_t>(D) * 32; }
  __host__ __device__ static constexpr uint32_t ypart(int D) { return x_ring(D) + W * XS * kRtBlockBytes; }
  __host__ __device__ static constexpr uint32_t ysum(int D) { return ypart(D) + W * kRtT * YP * 4; }
  __host__ __device__ static constexpr uint32_t wamax(int D) { return ysum(D) + kRtT * YP * 4; }
  __host__ __device__ static constexpr uint32_t rowinv(int D) { return wamax(D) + W * kRtT * 4; }
  __host__ __device__ static constexpr uint32_t bars(int D) { return rowinv(D) + kRtT * 4; }
  __host__ __device__ static constexpr uint32_t smem(int D) { return bars(D) + (W + W * XS) * 8 + 1024; }
};

// Byte offset of (row, 16-byte chunk c) inside a 64-column block in the
// tensor-map 128-byte swizzle (chunk index XOR row mod 8).
__device__ __forceinline__ uint32_t sw128(int row, int c) {
  return static_cast<uint32_t>(row * 128 + ((c ^ (row & 7)) << 4));
}

// Component c (compile-time after unrolling) of a uint4.
__device__ __forceinline__ uint32_t u4c(const uint4& v, int c) {
  return c == 0 ? v.x : c == 1 ? v.y : c == 2 ? v.z : v.w;
}

// Paired binary32 arithmetic (sm_100 f32x2): each lane rounds exactly as the
// scalar operation would, so results equal the scalar sequence.
__device__ __forceinline__ float2 add_f32x2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 a, b, r;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "add.rn.f32x2 r, a, b;\n\tmov.b64 {%0, %1}, r;\n\t}"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
__device__ __forceinline__ float2 mul_f32x2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 a, b, r;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mul.rn.f32x2 r, a, b;\n\tmov.b64 {%0, %1}, r;\n\t}"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
// Running maximum of |v| over both bf16 halves (bf16 values are compared
// exactly; a NaN operand is ignored like fmaxf does).
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t m, uint32_t v) {
  uint32_t r;
  asm("{\n\t.reg .b32 t;\n\tabs.bf16x2 t, %2;\n\tmax.bf16x2 %0, %1, t;\n\t}" : "=r"(r) : "r"(m), "r"(v));
  return r;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}
__device__ __forceinline__ float2 bf16x2_to_f32x2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// 8 bf16 values -> 8 packed INT4 codes (as quantize8_fast): u = fl(fl(g inv)
// + 1.5 2^23) keeps rint(g inv) in its low byte (two's complement, since
// |g inv| < 8); the low bytes are gathered with byte permutes and their low
// nibbles packed, element e at bits 4e..4e+3. The products are paired; the
// additions are scalar __fadd_rn, because a paired add after a paired
// multiply may be contracted into a fused multiply-add, which skips the
// binary32 rounding of g inv (measured: 7 codes in 2^20 differ).
__device__ __forceinline__ uint32_t quantize8_x2(const uint4 hv, float inv) {
  const float2 iv = make_float2(inv, inv);
  const float2 p0 = mul_f32x2(bf16x2_to_f32x2(hv.x), iv), p1 = mul_f32x2(bf16x2_to_f32x2(hv.y), iv);
  const float2 p2 = mul_f32x2(bf16x2_to_f32x2(hv.z), iv), p3 = mul_f32x2(bf16x2_to_f32x2(hv.w), iv);
  auto u = [](float v) { return __float_as_uint(__fadd_rn(v, 12582912.0f)); };
  // bytes [c0 c1 c2 c3] and [c4 c5 c6 c7]
  const uint32_t w0 = prmt(prmt(u(p0.x), u(p0.y), 0x0040u), prmt(u(p1.x), u(p1.y), 0x0040u), 0x5410u);
  const uint32_t w1 = prmt(prmt(u(p2.x), u(p2.y), 0x0040u), prmt(u(p3.x), u(p3.y), 0x0040u), 0x5410u);
  // byte 0 <- c0 | c1 << 4, byte 2 <- c2 | c3 << 4 (bytes 1, 3 unused)
  const uint32_t y0 = (w0 & 0x000F000Fu) | ((w0 >> 4) & 0x00F000F0u);
  const uint32_t y1 = (w1 & 0x000F000Fu) | ((w1 >> 4) & 0x00F000F0u);
  return prmt(y0, y1, 0x6420u);
}

// tmR / tmX: bf16 [N, D] tensor maps (residual, x), box {64, 16}, 128-byte
// swizzle. Ut / Vt: U and V fragments in the order rt_pack_factors
// writes. NB = D / 512 (64-column blocks per warp).
template <int R, int W, int NB, bool F32OUT>
__global__ void __launch_bounds__(32 * W, 1)
boundary_rowtile_kernel(const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmX,
                        const uint4* __restrict__ Ut,
                        const uint4* __restrict__ Vt, int N, void* __restrict__ h_out,
                        uint8_t* __restrict__ q_out, float* __restrict__ scale_out, float qmax) {
  using C = RtCfg<R, W>;
  constexpr int XS = C::XS, RING = C::RING, D = NB * 64 * W;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q4 = lane & 3;
  const int ntiles = (N + kRtT - 1) / kRtT;
  const uint32_t tileA = base;                       // block b at tileA + b * 2048
  const uint32_t xring = base + C::x_ring(D);        // warp w, slot s at xring + (w XS + s) * 2048
  float* ypart = reinterpret_cast<float*>(smem + C::ypart(D));
  float* ysum = reinterpret_cast<float*>(smem + C::ysum(D));
  float* wamax = reinterpret_cast<float*>(smem + C::wamax(D));
  float* rowinv = reinterpret_cast<float*>(smem + C::rowinv(D));
  const uint32_t res_bar = base + C::bars(D) + 8 * warp;                  // this warp's residual blocks
  const uint32_t xbar0 = base + C::bars(D) + 8 * W + 8 * warp * XS;  // this warp's x slots

  // Each warp initialises its own barriers and starts its copies at once (no
  // CTA-wide barrier before the first tensor copy).
  if (lane == 0) {
    mbar_init(res_bar, NB);
    for (int i = 0; i < XS; ++i) mbar_init(xbar0 + 8 * i, 1);
    fence_mbarrier_init();
    if (warp == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(&tmR) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(&tmX) : "memory");
    }
  }
  __syncwarp();
  // launched as a programmatic dependent: residual and x may come from the
  // previous kernel of the stream, so every global access waits for it; the
  // next kernel (the GEMM on these codes) may be scheduled from here on
  grid_dep_wait();
  grid_dep_launch();

  // x block stream of this warp: use u is block u % NB of the warp's slice in
  // its tile iteration u / NB, staged in slot u % XS by lane u % XS.
  // residual and x are read once and h' is not read again by this launch:
  // their L2 lines go first, so the codes (read next by the GEMM) and the
  // GEMM's weights stay (bench step: boundary 26.0 -> 25.0 us, steady step
  // 88.8 -> 87.3 us)
  const uint64_t pol_ef = l2_policy_evict_first();
  auto issue_x = [&](int u) {
    const int tile = static_cast<int>(blockIdx.x) + (u / NB) * static_cast<int>(gridDim.x);
    if (tile >= ntiles) return;
    const int slot = u % XS;
    mbar_arrive_expect_tx(xbar0 + 8 * slot, kRtBlockBytes);
    tma_load_2d_hint(xring + (warp * XS + slot) * kRtBlockBytes, &tmX, (warp * NB + u % NB) * 64, tile * kRtT,
                xbar0 + 8 * slot, pol_ef);
  };
  if (lane < XS) issue_x(lane);
  // ok: false once a wait gave up (warp-uniform after each wait, CTA-uniform
  // at the CTA barriers). From then on no copy is issued and nothing is
  // stored; waits still run for copies already issued (uses u < x_issued of
  // the x stream, tiles with res_issued), so none is in flight at exit.
  int x_issued = XS;
  bool res_issued = false;

  auto load_u = [&](uint4 (&dst)[C::UB], int j) {
    const uint4* src = Ut + static_cast<size_t>(warp * NB + j) * C::UB * 32 + lane;
#pragma unroll
    for (int i = 0; i < C::UB; ++i) dst[i] = __ldg(src + i * 32);
  };
  auto load_v = [&](uint4 (&dst)[C::VB], int j) {
    const uint4* src = Vt + static_cast<size_t>(warp * NB + j) * C::VB * 32 + lane;
#pragma unroll
    for (int i = 0; i < C::VB; ++i) dst[i] = __ldg(src + i * 32);
  };

  bool ok = true;
  int it = 0;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int row0 = tile * kRtT;
    // ---- residual tile: lane j < NB loads block warp * NB + j (after its
    // own h' store of the previous tile has finished reading the block)
    res_issued = ok;
    if (ok && lane < NB) {
      const int b = warp * NB + lane;
      mbar_arrive_expect_tx(res_bar, kRtBlockBytes);
      tma_load_2d_hint(tileA + b * kRtBlockBytes, &tmR, b * 64, row0, res_bar, pol_ef);
    }

    // ---- phase 1: partial y over this warp's columns
    uint4 ub[RING][C::UB];
#pragma unroll
    for (int j = 0; j < RING - 1; ++j)
      if (j < NB) load_u(ub[j], j);
    float acc1[C::NT][4];
#pragma unroll
    for (int p = 0; p < C::NT; ++p) acc1[p][0] = acc1[p][1] = acc1[p][2] = acc1[p][3] = 0.f;
    if (res_issued) ok = mbar_wait(res_bar, it & 1, kSiteBoundaryLoad) && ok;
    ok = __all_sync(0xffffffffu, ok);
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      if (j + RING - 1 < NB) load_u(ub[(j + RING - 1) % RING], j + RING - 1);
      const uint32_t blk = tileA + (warp * NB + j) * kRtBlockBytes;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
        uint32_t a[4];
        ldmatrix_x4(blk + sw128(row, 2 * kk + (lane >> 4)), a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int p = 0; p < C::NT; ++p) {
          const uint4& v = ub[j % RING][kk * C::UQ + p / 2];
          mma_bf16_16816(acc1[p], a, u4c(v, 2 * (p & 1)), u4c(v, 2 * (p & 1) + 1));
        }
      }
    }
    // V fragments of the first blocks load while y is reduced
    uint4 vb[RING][C::VB];
#pragma unroll
    for (int j = 0; j < RING - 1; ++j)
      if (j < NB) load_v(vb[j], j);
    {
      float* yp = ypart + warp * kRtT * C::YP;
#pragma unroll
      for (int p = 0; p < C::NT; ++p) {
        *reinterpret_cast<float2*>(yp + g * C::YP + 8 * p + 2 * q4) = make_float2(acc1[p][0], acc1[p][1]);
        *reinterpret_cast<float2*>(yp + (g + 8) * C::YP + 8 * p + 2 * q4) = make_float2(acc1[p][2], acc1[p][3]);
      }
    }
    ok = __syncthreads_and(ok) != 0;
    if (tid < kRtT * R / 2) {
      const int row = tid / (R / 2), c2 = 2 * (tid % (R / 2));
      float2 s = make_float2(0.f, 0.f);
#pragma unroll
      for (int w = 0; w < W; ++w) {
        const float2 v = *reinterpret_cast<const float2*>(ypart + (w * kRtT + row) * C::YP + c2);
        s.x += v.x;
        s.y += v.y;
      }
      *reinterpret_cast<float2*>(ysum + row * C::YP + c2) = s;
    }
    __syncthreads();

    // ---- phase 2: h = (res + x) + y V^T over this warp's columns
    uint32_t ahi[C::KK][4], alo[C::KK][4];
#pragma unroll
    for (int kk = 0; kk < C::KK; ++kk) {
      const float2 y0 = *reinterpret_cast<const float2*>(ysum + g * C::YP + 16 * kk + 2 * q4);
      const float2 y1 = *reinterpret_cast<const float2*>(ysum + (g + 8) * C::YP + 16 * kk + 2 * q4);
      const float2 y2 = *reinterpret_cast<const float2*>(ysum + g * C::YP + 16 * kk + 2 * q4 + 8);
      const float2 y3 = *reinterpret_cast<const float2*>(ysum + (g + 8) * C::YP + 16 * kk + 2 * q4 + 8);
      split_bf16x2(y0, ahi[kk][0], alo[kk][0]);
      split_bf16x2(y1, ahi[kk][1], alo[kk][1]);
      split_bf16x2(y2, ahi[kk][2], alo[kk][2]);
      split_bf16x2(y3, ahi[kk][3], alo[kk][3]);
    }
    uint32_t amax2[2] = {0u, 0u};   // running max |h'| (bf16x2) of rows g and g + 8
    // The plan orders V so that n8 tile t of a block holds columns
    // 16 (n / 2) + 2 t + n % 2 (n = 0..7 the tile's column index): this lane's
    // accumulators are then columns 16 q4 .. 16 q4 + 15, i.e. the 16-byte
    // chunks 2 q4 (tiles 0-3) and 2 q4 + 1 (tiles 4-7) of rows g and g + 8,
    // at row * 128 + ((chunk ^ row % 8) << 4) (row % 8 = g for both rows).
    uint32_t cb[2][2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
      for (int half = 0; half < 2; ++half)
        cb[hh][half] = static_cast<uint32_t>((g + 8 * hh) * 128 + (((2 * q4 + half) ^ g) << 4));
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      if (j + RING - 1 < NB) load_v(vb[(j + RING - 1) % RING], j + RING - 1);
      const int u = it * NB + j;
      const int slot = u % XS;
      if (u < x_issued) ok = mbar_wait(xbar0 + 8 * slot, (u / XS) & 1, kSiteBoundaryLoad) && ok;
      ok = __all_sync(0xffffffffu, ok);
      uint8_t* blk = smem + (warp * NB + j) * kRtBlockBytes;
      const uint8_t* xblk = smem + C::x_ring(D) + (warp * XS + slot) * kRtBlockBytes;
      const int colb = (warp * NB + j) * 64;
      // all MMAs of the block first (8 independent accumulators), then the
      // epilogue; per accumulator the order is hi, lo per k16 step
      float acc[8][4];
#pragma unroll
      for (int t = 0; t < 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < C::KK; ++kk) {
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int ri = (t * C::KK + kk) * 2;
          const uint4& v = vb[j % RING][ri / 4];
          mma_bf16_16816(acc[t], ahi[kk], u4c(v, ri % 4), u4c(v, ri % 4 + 1));
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int ri = (t * C::KK + kk) * 2;
          const uint4& v = vb[j % RING][ri / 4];
          mma_bf16_16816(acc[t], alo[kk], u4c(v, ri % 4), u4c(v, ri % 4 + 1));
        }
      }
      // All loads of the block first (four 16-byte chunks of residual and
      // of x), then the arithmetic, then the in-place h' stores.
      uint32_t rw[2][2][4], xw[2][2][4];   // [hh][half][word]: word i = tile 4 half + i
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint4 rv = *reinterpret_cast<const uint4*>(blk + cb[hh][half]);
          const uint4 xv = *reinterpret_cast<const uint4*>(xblk + cb[hh][half]);
          rw[hh][half][0] = rv.x; rw[hh][half][1] = rv.y; rw[hh][half][2] = rv.z; rw[hh][half][3] = rv.w;
          xw[hh][half][0] = xv.x; xw[hh][half][1] = xv.y; xw[hh][half][2] = xv.z; xw[hh][half][3] = xv.w;
        }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int half = 0; half < 2; ++half)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int t = 4 * half + i;
            const float2 sum = add_f32x2(bf16x2_to_f32x2(rw[hh][half][i]), bf16x2_to_f32x2(xw[hh][half][i]));
            const float2 h = add_f32x2(sum, make_float2(acc[t][2 * hh], acc[t][2 * hh + 1]));
            const uint32_t hb = pack_bf16x2(h.x, h.y);
            rw[hh][half][i] = hb;
            amax2[hh] = absmax_bf16x2(amax2[hh], hb);
            if constexpr (F32OUT) {
              const int row = g + 8 * hh;
              if (ok && h_out != nullptr && row0 + row < N)
                *reinterpret_cast<float2*>(static_cast<float*>(h_out) + static_cast<size_t>(row0 + row) * D +
                                           colb + 16 * q4 + 2 * t) = h;
            }
          }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int half = 0; half < 2; ++half)
          *reinterpret_cast<uint4*>(blk + cb[hh][half]) =
              make_uint4(rw[hh][half][0], rw[hh][half][1], rw[hh][half][2], rw[hh][half][3]);
      // the slot's bytes were read (generic proxy) before its next tensor copy
      fence_proxy_async_smem();
      __syncwarp();
      if (ok) {
        if (lane == slot) issue_x(u + XS);
        x_issued = u + XS + 1;
      }
    }
    float rmax[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) rmax[hh] = fmaxf(bf16_lo_f32(amax2[hh]), bf16_hi_f32(amax2[hh]));

    // ---- row amax over the 8 warps, scales
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float m = rmax[hh];
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      if (q4 == 0) wamax[warp * kRtT + g + 8 * hh] = m;
    }
    ok = __syncthreads_and(ok) != 0;
    if (tid < kRtT) {
      float m = 0.f;
#pragma unroll
      for (int w = 0; w < W; ++w) m = fmaxf(m, wamax[w * kRtT + tid]);
      float inv, sc;
      inv_and_scale(m, qmax, inv, sc);
      rowinv[tid] = inv;
      if (ok && row0 + tid < N) scale_out[row0 + tid] = sc;
    }
    __syncthreads();

    // ---- h' out and codes: chunk i = (block, row, 16-byte chunk); 8 lanes
    // write one 128-byte h' row segment and one 32-byte code segment
    constexpr int kChunks = kRtT * D / 8;
#pragma unroll 4
    for (int i = tid; i < kChunks; i += C::kThreads) {
      const int b = i >> 7, row = (i >> 3) & 15, c = i & 7;
      const uint4 hv = *reinterpret_cast<const uint4*>(smem + b * kRtBlockBytes + sw128(row, c));
      const uint32_t code = quantize8_x2(hv, rowinv[row]);
      if (ok && row0 + row < N) {
        const size_t grow = static_cast<size_t>(row0 + row);
        reinterpret_cast<uint32_t*>(q_out)[grow * (D / 8) + b * 8 + c] = code;
        if constexpr (!F32OUT) {
          if (h_out != nullptr)
            st_global_v4_hint(static_cast<bf16*>(h_out) + grow * D + b * 64 + c * 8, hv, pol_ef);
        }
      }
    }
    fence_proxy_async_smem();   // these reads before the next residual copy into the tile
    __syncthreads();
  }
}

// Host side: U and V (bf16 bits, [D][R] row-major) in the fragment order of
// boundary_rowtile_kernel. Ut: for 64-column block b, k16 step kk, lane
// (g = lane / 4, q = lane % 4), register i = 2p + e of n8 tile p holds
// (U[d][n], U[d+1][n]) with d = 64 b + 16 kk + 2q + 8e, n = 8p + g, stored at
// uint4 ((b 4 + kk) R/16 + i/4) * 32 + lane, component i % 4. Vt: for block b,
// register i = 2 (t R/16 + kk) + e holds (V[d][m], V[d][m+1]) with
// d = 64 b + 16 (g / 2) + 2 t + g % 2 (the column order that gives each lane
// 16 contiguous output columns), m = 16 kk + 2q + 8e, stored at uint4
// (b R/4 + i/4) * 32 + lane, component i % 4.
inline void rt_pack_factors(const uint16_t* Ub, const uint16_t* Vb, int D, int R, uint32_t* Ut, uint32_t* Vt) {
  auto pair = [](uint16_t lo, uint16_t hi) { return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16); };
  const int UQ = R / 16, KK = R / 16, VB = R / 4;
  for (int b = 0; b < D / 64; ++b)
    for (int lane = 0; lane < 32; ++lane) {
      const int g = lane >> 2, q = lane & 3;
      for (int kk = 0; kk < 4; ++kk)
        for (int i = 0; i < 4 * UQ; ++i) {
          const int p = i / 2, e = i % 2;
          const int d = 64 * b + 16 * kk + 2 * q + 8 * e, n = 8 * p + g;
          const size_t idx = ((static_cast<size_t>(b * 4 + kk) * UQ + i / 4) * 32 + lane) * 4 + i % 4;
          Ut[idx] = pair(Ub[static_cast<size_t>(d) * R + n], Ub[static_cast<size_t>(d + 1) * R + n]);
        }
      for (int i = 0; i < 4 * VB; ++i) {
        const int e = i % 2, tk = i / 2, kk = tk % KK, t = tk / KK;
        const int d = 64 * b + 16 * (g >> 1) + 2 * t + (g & 1), m = 16 * kk + 2 * q + 8 * e;
        const size_t idx = ((static_cast<size_t>(b) * VB + i / 4) * 32 + lane) * 4 + i % 4;
        Vt[idx] = pair(Vb[static_cast<size_t>(d) * R + m], Vb[static_cast<size_t>(d) * R + m + 1]);
      }
    }
}

}  // namespace respin
