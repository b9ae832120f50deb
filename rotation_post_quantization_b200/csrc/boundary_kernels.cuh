// Fused block-boundary kernels: rank-r basis fix + per-token INT4 quantization.
//
// Per token (row) n, with the plan's bfloat16 factors U (D x r) and V (D x r):
//   y = residual[n] U ;  h = (residual[n] + x[n]) + y V^T  (fp32)
//   h' = bf16(h) ; amax = max|h'| ; inv = qmax/amax ; q = rint(h' inv)
// This is the subspace residual rotation of the ReSpinQuant explainers (zh page
// §2.2 steps 1-3: projection, transform inside the subspace, re-projection and
// residual) in the row convention, followed by 4-bit (qmax = 7, W4A4) or
// 3-bit (qmax = 3, W3A3) activation quantization (zh §3-§4, fr §4). Since
// |h'| <= amax, |fl(h' * fl(qmax/amax))| <= qmax (1+2^-24)^2 < qmax + 0.5, so
// the code is always in [-qmax, qmax] and no clamp is needed.
//
// Cluster design (B200): a tile of T tokens is split along D over a
// thread-block cluster of C CTAs (one per SM); CTA c owns the columns
// [c*Dc, (c+1)*Dc) of every token in the tile and works through the tiles of
// its cluster in a persistent loop. Residual and x tiles arrive by 1-D bulk
// copies (one per row) into a shared-memory ring, so later tiles are in
// flight while one is computed. The two whole-row dependencies - y needs the
// full row before the re-projection, amax needs the full row before
// quantization - are resolved with a cluster barrier each and
// distributed-shared-memory reads (all remote loads of a value in flight at
// once, summed in rank order so every CTA gets the identical y). Both skinny
// products run on tensor cores (mma.sync m16n8k16 bf16, fp32 accumulate); y is
// split into bf16 hi + lo parts for the re-projection, keeping ~16 mantissa
// bits. HBM sees each input byte once and each output byte once.
//
// Two variants:
//  * boundary_cluster_rf_kernel (r <= 32): each CTA keeps its slices of U and V
//    in REGISTERS for the whole launch, loaded once from a fragment-ordered
//    copy that the plan prepares (coalesced 16-byte loads), which leaves the
//    shared memory to a 3-stage tile ring.
//  * boundary_cluster_smem_kernel (r = 64, 128): the factor slices live in
//    shared memory (U^T with padded rows, V with 16-byte chunks swizzled),
//    2-stage tile ring.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace respin {

using bf16 = __nv_bfloat16;

constexpr int kBoundaryThreads = 256;
constexpr float kZeroTokenAmax = 2.3509887e-38f;  // 2^-125

__device__ __forceinline__ float bf16_lo_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 8 consecutive bf16 values (one 16-byte vector) -> 8 packed INT4 codes.
__device__ __forceinline__ uint32_t quantize8(const uint4 hv, float inv) {
  const uint32_t w[4] = {hv.x, hv.y, hv.z, hv.w};
  uint32_t packed = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const uint32_t word = w[e >> 1];
    const float f = (e & 1) ? bf16_hi_f32(word) : bf16_lo_f32(word);
    const int q = __float2int_rn(__fmul_rn(f, inv));
    packed |= (static_cast<uint32_t>(q) & 0xFu) << (4 * e);
  }
  return packed;
}

// qmax = 7 (INT4 codes) or 3 (INT3 codes, W3A3).
__device__ __forceinline__ void inv_and_scale(float amax, float qmax, float& inv, float& scale) {
  if (amax >= kZeroTokenAmax) {
    inv = __fdiv_rn(qmax, amax);
    scale = __fdiv_rn(amax, qmax);
  } else {
    inv = 0.0f;
    scale = 0.0f;
  }
}

// y in fp32 (two floats) -> bf16x2 hi and lo parts with hi + lo ~ y.
__device__ __forceinline__ void split_bf16x2(float2 v, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(v.x - hf.x, v.y - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Stage the residual and x rows of one tile with 1-D bulk copies (warp 0;
// lane i copies row i). Rows past N are not copied.
__device__ __forceinline__ void stage_tile(const bf16* __restrict__ x, const bf16* __restrict__ res,
                                           int row0, int N, int D, int col0, int Dc, int T,
                                           uint32_t rdst, uint32_t xdst, uint32_t pitch,
                                           uint32_t bar_r, uint32_t bar_x, int lane) {
  const int rows = min(T, N - row0);
  const uint32_t bytes = static_cast<uint32_t>(Dc) * 2;
  if (lane == 0) {
    mbar_arrive_expect_tx(bar_r, rows * bytes);
    mbar_arrive_expect_tx(bar_x, rows * bytes);
  }
  __syncwarp();
  if (lane < rows) {
    const size_t gofs = static_cast<size_t>(row0 + lane) * D + col0;
    bulk_g2s(rdst + lane * pitch, res + gofs, bytes, bar_r);
    bulk_g2s(xdst + lane * pitch, x + gofs, bytes, bar_x);
  }
}

// Residual and x words (bf16 pairs at column `colc`) of rows g and g + 8 of
// every m16 tile, read before the previous n8 block's in-place stores so the
// loads need not wait behind them.
template <int MT>
__device__ __forceinline__ void load_n8(uint32_t (&w)[MT][2][2], const uint8_t* rs_ptr,
                                        const uint8_t* xs_ptr, uint32_t pitch, int g, int colc) {
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const uint32_t off = (mt * 16 + g + 8 * hh) * pitch + colc * 2;
      w[mt][hh][0] = *reinterpret_cast<const uint32_t*>(rs_ptr + off);
      w[mt][hh][1] = *reinterpret_cast<const uint32_t*>(xs_ptr + off);
    }
}

// Epilogue of one n8 column block of the re-projection for the rows of one
// m16 tile: h = (res + x) + corr from the preloaded words, bf16 round in place
// (into the x slot), row amax, optional fp32 store.
template <bool F32OUT>
__device__ __forceinline__ void finish_n8(const float (&acc)[4], const uint32_t (&w)[2][2], uint8_t* xs_ptr,
                                          uint32_t pitch, int rowA, int colc, float (&rmax)[2],
                                          void* h_out, int row0, int N, int D, int col0, bool ok) {
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int row = rowA + 8 * hh;
    const uint32_t off = row * pitch + colc * 2;
    const uint32_t rw = w[hh][0], xw = w[hh][1];
    const float h0 = (bf16_lo_f32(rw) + bf16_lo_f32(xw)) + acc[2 * hh];
    const float h1 = (bf16_hi_f32(rw) + bf16_hi_f32(xw)) + acc[2 * hh + 1];
    const uint32_t hb = pack_bf16x2(h0, h1);
    *reinterpret_cast<uint32_t*>(xs_ptr + off) = hb;
    rmax[hh] = fmaxf(rmax[hh], fmaxf(fabsf(bf16_lo_f32(hb)), fabsf(bf16_hi_f32(hb))));
    if constexpr (F32OUT) {
      if (ok && h_out != nullptr && row0 + row < N) {
        float* hf = static_cast<float*>(h_out) + static_cast<size_t>(row0 + row) * D + col0 + colc;
        *reinterpret_cast<float2*>(hf) = make_float2(h0, h1);
      }
    }
  }
}

// Row amax: per-thread row maxima -> warp maxima in `wamax` [8][T] -> after a
// CTA barrier the T row maxima of this CTA's slice in `amaxbuf`. Returns `ok`
// ANDed over the CTA (taken at that barrier).
template <int MT, int T>
__device__ __forceinline__ bool publish_amax(float (&rmax)[MT][2], float* wamax, float* amaxbuf,
                                             int warp, int lane, int tid, bool ok) {
  const int g = lane >> 2, q4 = lane & 3;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float m = rmax[mt][hh];
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      if (q4 == 0) wamax[warp * T + mt * 16 + g + 8 * hh] = m;
    }
  ok = __syncthreads_and(ok) != 0;
  if (tid < T) {
    float m = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) m = fmaxf(m, wamax[w * T + tid]);
    amaxbuf[tid] = m;
  }
  return ok;
}

// After the amax cluster barrier: gather every CTA's row maxima in parallel
// (one remote load per thread), reduce, and set the rows' 1/scale factors.
template <int T>
__device__ __forceinline__ void gather_amax(uint32_t amaxbuf_addr, float* am2, float* rowinv,
                                            float* scale_out, uint32_t csize, uint32_t crank,
                                            int row0, int N, int tid, float qmax, bool ok) {
  for (int i = tid; i < static_cast<int>(csize) * T; i += kBoundaryThreads) {
    const uint32_t c = static_cast<uint32_t>(i / T);
    am2[i] = ld_dsmem_f32(map_to_rank(amaxbuf_addr + 4u * (i % T), c));
  }
  __syncthreads();
  if (tid < T) {
    float m = 0.f;
    for (uint32_t c = 0; c < csize; ++c) m = fmaxf(m, am2[c * T + tid]);
    float inv, sc;
    inv_and_scale(m, qmax, inv, sc);
    rowinv[tid] = inv;
    if (ok && crank == 0 && row0 + tid < N) scale_out[row0 + tid] = sc;
  }
  __syncthreads();
}

// Store h' (bf16) and the packed codes of this CTA's slice of the tile.
template <bool F32OUT>
__device__ __forceinline__ void store_tile(const uint8_t* xs_ptr, uint32_t pitch, const float* rowinv,
                                           int T, int Dc, int row0, int N, int D, int col0,
                                           void* h_out, uint8_t* q_out, int tid, bool ok) {
  const int vpr = Dc / 8;
  for (int i = tid; ok && i < T * vpr; i += kBoundaryThreads) {
    const int row = i / vpr, v = i % vpr;
    if (row0 + row >= N) continue;
    const uint4 hv = *reinterpret_cast<const uint4*>(xs_ptr + row * pitch + v * 16);
    const size_t gi = static_cast<size_t>(row0 + row) * D + col0 + v * 8;
    if constexpr (!F32OUT) {
      if (h_out != nullptr) *reinterpret_cast<uint4*>(static_cast<bf16*>(h_out) + gi) = hv;
    }
    *reinterpret_cast<uint32_t*>(q_out + gi / 2) = quantize8(hv, rowinv[row]);
  }
}

// ============================================================================
// Register-resident factors (r <= 32): T tokens per tile, Dc columns per CTA,
// 3-stage tile ring. Warp 0 stages the tile two ahead while it waits at the
// tile's two cluster barriers (residual rows at the first, x rows at the
// second), so the copy issue overlaps the barrier latency. 8 warps keep the
// 255-register budget that the resident fragments need.
// ============================================================================

constexpr int kRfThreads = 256;

template <int R, int T, int Dc>
struct RfCfg {
  static constexpr int S = 3;
  static constexpr int MT = T / 16;            // m16 tiles per token tile
  static constexpr int WK = 8 / MT;            // warps along Dc in phase 1
  static constexpr int KS = Dc / 16;           // k16 steps of phase 1
  static constexpr int KPW = KS / WK;          // k16 steps per warp in phase 1
  static constexpr int NPW = R / 8;            // n8 tiles of y per warp (all of r)
  static constexpr int KS2 = R / 16;           // k16 steps of the re-projection
  static constexpr int NTW = Dc / 64;          // n8 column tiles per warp (phase 2)
  static constexpr int UREG = KPW * NPW * 2;   // 32-bit U fragment registers per lane
  static constexpr int VREG = NTW * KS2 * 2;   // 32-bit V fragment registers per lane
  static constexpr int RP = R + 8;             // padded fp32 row (conflict-free float2)
  static constexpr uint32_t pitch = Dc * 2 + 16;
  static constexpr uint32_t kStage = 2 * T * pitch;           // residual rows, then x rows
  static constexpr uint32_t oPart = S * kStage;               // [WK][T][RP]; y aliases [0]
  static constexpr uint32_t oYbuf = oPart + WK * T * RP * 4;  // [T][R] this CTA's partial y
  static constexpr uint32_t oWamax = oYbuf + T * R * 4;       // [8][T]
  static constexpr uint32_t oAm2 = oWamax + 8 * T * 4;        // [16][T]
  static constexpr uint32_t oAmax = oAm2 + 16 * T * 4;        // [T]
  static constexpr uint32_t oRinv = oAmax + T * 4;            // [T]
  static constexpr uint32_t oBars = oRinv + T * 4;            // full_res[S], full_x[S]
  static constexpr uint32_t kSmem = oBars + 2 * S * 8;
  static_assert(R == 16 || R == 32, "register-resident factors need r <= 32");
  static_assert(T == 16 || T == 32, "token tile");
  static_assert(KS % WK == 0 && Dc % 64 == 0, "column slice");
  static_assert(UREG % 4 == 0 && VREG % 4 == 0, "fragment chunks");
  static_assert(T * R / 4 <= kRfThreads, "one float4 of y per thread");
};

// 8 bf16 values -> 8 packed INT4 codes using round-to-nearest-even by
// addition: for |t| < 2^22, fl(t + 1.5*2^23) = 1.5*2^23 + rint(t) (ties to
// even), and its low 4 bits are rint(t) mod 16, the two's-complement nibble.
// t = fl(g * inv) exactly as in the definition (separate multiply and add).
__device__ __forceinline__ uint32_t quantize8_fast(const uint4 hv, float inv) {
  const uint32_t w[4] = {hv.x, hv.y, hv.z, hv.w};
  uint32_t packed = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const uint32_t word = w[e >> 1];
    const float f = (e & 1) ? bf16_hi_f32(word) : bf16_lo_f32(word);
    const float u = __fadd_rn(__fmul_rn(f, inv), 12582912.0f);
    packed |= (__float_as_uint(u) & 0xFu) << (4 * e);
  }
  return packed;
}

template <int R, int T, int Dc, bool F32OUT>
__global__ void __launch_bounds__(kRfThreads, 1)
boundary_cluster_rf_kernel(const bf16* __restrict__ x, const bf16* __restrict__ res,
                           const uint4* __restrict__ Uf, const uint4* __restrict__ Vf, int N,
                           int D, void* __restrict__ h_out, uint8_t* __restrict__ q_out,
                           float* __restrict__ scale_out, float qmax) {
  using C = RfCfg<R, T, Dc>;
  constexpr int S = C::S, RP = C::RP;
  constexpr uint32_t pitch = C::pitch;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q4 = lane & 3;
  const uint32_t crank = cluster_ctarank();
  const uint32_t csize = static_cast<uint32_t>(D / Dc);
  const int col0 = static_cast<int>(crank) * Dc;
  const uint32_t cid = cluster_id_x(), ncl = ncluster_x();
  const int ntiles = (N + T - 1) / T;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + C::oBars;   // full_res[s] = bars + 8s, full_x[s] = bars + 8(S+s)

  if (tid == 0) {
    for (int i = 0; i < 2 * S; ++i) mbar_init(bars + 8 * i, 1);
    fence_mbarrier_init();
  }
  __syncthreads();

  // ok: false once a wait of this CTA gave up (CTA-uniform at the CTA
  // barriers). From then on no copy is issued and nothing is stored; waits
  // still run for copies already issued, so none is in flight at exit.
  bool ok = true;
  int issued[2] = {0, 0};   // loop iterations whose residual / x copies were issued
  // Warp 0: bulk-copy the residual (which = 0) or x (which = 1) rows of loop
  // iteration `it` into stage it % S.
  auto issue = [&](int it, int which) {
    const int tile = static_cast<int>(cid) + it * static_cast<int>(ncl);
    if (!ok || tile >= ntiles) return;
    issued[which] = it + 1;
    if (warp != 0) return;
    const int s = it % S;
    const int row0 = tile * T;
    const int rows = min(T, N - row0);
    constexpr uint32_t bytes = Dc * 2;
    const uint32_t bar = bars + 8 * (which * S + s);
    const uint32_t dst = sbase + s * C::kStage + which * T * pitch;
    const bf16* src = which ? x : res;
    if (lane == 0) mbar_arrive_expect_tx(bar, rows * bytes);
    __syncwarp();
    if (lane < rows)
      bulk_g2s(dst + lane * pitch, src + static_cast<size_t>(row0 + lane) * D + col0, bytes, bar);
    __syncwarp();
  };
  issue(0, 0);
  issue(0, 1);
  issue(1, 0);
  issue(1, 1);

  // Factor fragments, resident for the whole launch.
  const int wm = warp % C::MT, wk = warp / C::MT;
  uint32_t ub[C::UREG], vb[C::VREG];
  {
    const uint4* up = Uf + (static_cast<size_t>(crank) * C::WK + wk) * (C::UREG / 4) * 32 + lane;
#pragma unroll
    for (int ch = 0; ch < C::UREG / 4; ++ch) {
      const uint4 v = __ldg(up + ch * 32);
      ub[4 * ch] = v.x; ub[4 * ch + 1] = v.y; ub[4 * ch + 2] = v.z; ub[4 * ch + 3] = v.w;
    }
    const uint4* vp = Vf + (static_cast<size_t>(crank) * 8 + warp) * (C::VREG / 4) * 32 + lane;
#pragma unroll
    for (int ch = 0; ch < C::VREG / 4; ++ch) {
      const uint4 v = __ldg(vp + ch * 32);
      vb[4 * ch] = v.x; vb[4 * ch + 1] = v.y; vb[4 * ch + 2] = v.z; vb[4 * ch + 3] = v.w;
    }
  }

  float* part = reinterpret_cast<float*>(smem + C::oPart);
  float* yfull = part;  // the partials are dead once reduced into ybuf
  float* ybuf = reinterpret_cast<float*>(smem + C::oYbuf);
  float* wamax = reinterpret_cast<float*>(smem + C::oWamax);
  float* am2 = reinterpret_cast<float*>(smem + C::oAm2);
  float* amaxbuf = reinterpret_cast<float*>(smem + C::oAmax);
  float* rowinv = reinterpret_cast<float*>(smem + C::oRinv);

  for (int it = 0;; ++it) {
    const int tile = static_cast<int>(cid) + it * static_cast<int>(ncl);
    if (tile >= ntiles) break;
    const int s = it % S;
    const uint32_t par = static_cast<uint32_t>(it / S) & 1u;
    const int row0 = tile * T;
    const uint32_t rs = sbase + s * C::kStage;
    const uint8_t* rs_ptr = smem + s * C::kStage;
    uint8_t* xs_ptr = smem + s * C::kStage + T * pitch;

    // ---- phase 1: this CTA's partial y = residual[:, slice] U_slice
    if (it < issued[0]) ok = mbar_wait(bars + 8 * s, par, kSiteBoundaryLoad) && ok;
    {
      float acc[C::NPW][4];
#pragma unroll
      for (int p = 0; p < C::NPW; ++p) acc[p][0] = acc[p][1] = acc[p][2] = acc[p][3] = 0.f;
      const uint32_t a_base = rs + (wm * 16 + (lane & 15)) * pitch + (lane >> 4) * 16;
#pragma unroll
      for (int j = 0; j < C::KPW; ++j) {
        uint32_t a[4];
        ldmatrix_x4(a_base + (wk * C::KPW + j) * 32, a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int p = 0; p < C::NPW; ++p)
          mma_bf16_16816(acc[p], a, ub[(j * C::NPW + p) * 2], ub[(j * C::NPW + p) * 2 + 1]);
      }
      float* pw = part + wk * T * RP;
#pragma unroll
      for (int p = 0; p < C::NPW; ++p) {
        const int col = p * 8 + 2 * q4, row = wm * 16 + g;
        *reinterpret_cast<float2*>(&pw[row * RP + col]) = make_float2(acc[p][0], acc[p][1]);
        *reinterpret_cast<float2*>(&pw[(row + 8) * RP + col]) = make_float2(acc[p][2], acc[p][3]);
      }
    }
    ok = __syncthreads_and(ok) != 0;
    if (tid < T * R / 4) {
      const int e = 4 * tid, row = e / R, col = e % R;
      float4 sum = *reinterpret_cast<const float4*>(&part[row * RP + col]);
#pragma unroll
      for (int w = 1; w < C::WK; ++w) {
        const float4 v = *reinterpret_cast<const float4*>(&part[(w * T + row) * RP + col]);
        sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
      }
      *reinterpret_cast<float4*>(&ybuf[e]) = sum;
    }

    // ---- y over the cluster; warp 0 stages the residual rows of iteration
    // it+2 meanwhile (its stage was released at the end of iteration it-1)
    cluster_arrive();
    issue(it + 2, 0);
    cluster_wait();
    if (tid < T * R / 4) {
      const int e = 4 * tid, row = e / R, col = e % R;
      *reinterpret_cast<float4*>(&yfull[row * RP + col]) =
          cluster_sum_f32x4(sbase + C::oYbuf + 16u * tid, csize);
    }
    __syncthreads();

    // ---- phase 2: h = (res + x) + y V_slice^T, bf16 round, row amax
    if (it < issued[1]) ok = mbar_wait(bars + 8 * (S + s), par, kSiteBoundaryLoad) && ok;
    {
      uint32_t ahi[C::MT][C::KS2][4], alo[C::MT][C::KS2][4];
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
        for (int ks = 0; ks < C::KS2; ++ks) {
          const int r0 = mt * 16 + g, c0 = ks * 16 + 2 * q4;
          split_bf16x2(*reinterpret_cast<const float2*>(&yfull[r0 * RP + c0]), ahi[mt][ks][0], alo[mt][ks][0]);
          split_bf16x2(*reinterpret_cast<const float2*>(&yfull[(r0 + 8) * RP + c0]), ahi[mt][ks][1], alo[mt][ks][1]);
          split_bf16x2(*reinterpret_cast<const float2*>(&yfull[r0 * RP + c0 + 8]), ahi[mt][ks][2], alo[mt][ks][2]);
          split_bf16x2(*reinterpret_cast<const float2*>(&yfull[(r0 + 8) * RP + c0 + 8]), ahi[mt][ks][3], alo[mt][ks][3]);
        }
      __nv_bfloat162 rmax2[C::MT];   // .x: row mt*16+g, .y: row mt*16+g+8
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt) rmax2[mt] = __float2bfloat162_rn(0.f);
      // The residual/x words of the next n8 tile are loaded before this
      // tile's h' is stored in place: the compiler cannot tell the
      // computed offsets apart, so loads after a store would wait for it.
      auto load_rx = [&](int t, int mt, uint32_t (&w)[4]) {
        const uint32_t offA = (mt * 16 + g) * pitch + ((warp * C::NTW + t) * 8 + 2 * q4) * 2;
        w[0] = *reinterpret_cast<const uint32_t*>(rs_ptr + offA);
        w[1] = *reinterpret_cast<const uint32_t*>(xs_ptr + offA);
        w[2] = *reinterpret_cast<const uint32_t*>(rs_ptr + offA + 8 * pitch);
        w[3] = *reinterpret_cast<const uint32_t*>(xs_ptr + offA + 8 * pitch);
      };
      uint32_t rx[2][C::MT][4];
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt) load_rx(0, mt, rx[0][mt]);
#pragma unroll
      for (int t = 0; t < C::NTW; ++t) {
        const int d0 = (warp * C::NTW + t) * 8;
        if (t + 1 < C::NTW) {
#pragma unroll
          for (int mt = 0; mt < C::MT; ++mt) load_rx(t + 1, mt, rx[(t + 1) & 1][mt]);
        }
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) {
          const int rowA = mt * 16 + g;
          const uint32_t offA = rowA * pitch + (d0 + 2 * q4) * 2;
          const uint32_t offB = offA + 8 * pitch;
          const uint32_t rA = rx[t & 1][mt][0], xA = rx[t & 1][mt][1];
          const uint32_t rB = rx[t & 1][mt][2], xB = rx[t & 1][mt][3];
          // accumulators start at residual + x; the tensor cores add y V^T
          float acc[4] = {bf16_lo_f32(rA) + bf16_lo_f32(xA), bf16_hi_f32(rA) + bf16_hi_f32(xA),
                          bf16_lo_f32(rB) + bf16_lo_f32(xB), bf16_hi_f32(rB) + bf16_hi_f32(xB)};
#pragma unroll
          for (int ks = 0; ks < C::KS2; ++ks) {
            const uint32_t b0 = vb[(t * C::KS2 + ks) * 2], b1 = vb[(t * C::KS2 + ks) * 2 + 1];
            mma_bf16_16816(acc, ahi[mt][ks], b0, b1);
            mma_bf16_16816(acc, alo[mt][ks], b0, b1);
          }
          const __nv_bfloat162 hA = __floats2bfloat162_rn(acc[0], acc[1]);
          const __nv_bfloat162 hB = __floats2bfloat162_rn(acc[2], acc[3]);
          *reinterpret_cast<__nv_bfloat162*>(xs_ptr + offA) = hA;
          *reinterpret_cast<__nv_bfloat162*>(xs_ptr + offB) = hB;
          const __nv_bfloat162 mA = __habs2(hA), mB = __habs2(hB);
          rmax2[mt] = __hmax2(rmax2[mt],
                              __halves2bfloat162(__hmax(__low2bfloat16(mA), __high2bfloat16(mA)),
                                                 __hmax(__low2bfloat16(mB), __high2bfloat16(mB))));
          if constexpr (F32OUT) {
            if (h_out != nullptr && ok) {
              float* hf = static_cast<float*>(h_out) + col0 + d0 + 2 * q4;
              if (row0 + rowA < N)
                *reinterpret_cast<float2*>(hf + static_cast<size_t>(row0 + rowA) * D) = make_float2(acc[0], acc[1]);
              if (row0 + rowA + 8 < N)
                *reinterpret_cast<float2*>(hf + static_cast<size_t>(row0 + rowA + 8) * D) = make_float2(acc[2], acc[3]);
            }
          }
        }
      }
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt) {
        float mA = __bfloat162float(__low2bfloat16(rmax2[mt]));
        float mB = __bfloat162float(__high2bfloat16(rmax2[mt]));
        mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 1));
        mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 2));
        mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, 1));
        mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, 2));
        if (q4 == 0) {
          wamax[warp * T + mt * 16 + g] = mA;
          wamax[warp * T + mt * 16 + g + 8] = mB;
        }
      }
      ok = __syncthreads_and(ok) != 0;
      if (tid < T) {
        float m = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) m = fmaxf(m, wamax[w * T + tid]);
        amaxbuf[tid] = m;
      }
    }

    // ---- amax over the cluster (warp 0 stages the x rows of iteration it+2)
    cluster_arrive();
    issue(it + 2, 1);
    cluster_wait();
    for (int i = tid; i < static_cast<int>(csize) * T; i += kRfThreads)
      am2[i] = ld_dsmem_f32(map_to_rank(sbase + C::oAmax + 4u * (i % T), static_cast<uint32_t>(i / T)));
    __syncthreads();
    if (tid < T) {
      float m = 0.f;
      for (uint32_t c = 0; c < csize; ++c) m = fmaxf(m, am2[c * T + tid]);
      float inv, sc;
      inv_and_scale(m, qmax, inv, sc);
      rowinv[tid] = inv;
      if (ok && crank == 0 && row0 + tid < N) scale_out[row0 + tid] = sc;
    }
    __syncthreads();

    // ---- h' (bf16) and packed codes of this CTA's slice
    {
      constexpr int vpr = Dc / 8;
#pragma unroll 4
      for (int i = tid; i < T * vpr; i += kRfThreads) {
        const int row = i / vpr, v = i % vpr;
        if (!ok || row0 + row >= N) continue;
        const uint4 hv = *reinterpret_cast<const uint4*>(xs_ptr + row * pitch + v * 16);
        const size_t gi = static_cast<size_t>(row0 + row) * D + col0 + v * 8;
        if constexpr (!F32OUT) {
          if (h_out != nullptr) *reinterpret_cast<uint4*>(static_cast<bf16*>(h_out) + gi) = hv;
        }
        *reinterpret_cast<uint32_t*>(q_out + gi / 2) = quantize8_fast(hv, rowinv[row]);
      }
    }
    // This stage is refilled by bulk copies during the next iteration: order
    // the generic-proxy accesses above before those async-proxy writes (the
    // first CTA barrier of the next iteration completes the hand-off).
    fence_proxy_async_smem();
  }
  // No CTA may leave while a peer can still read its shared memory.
  cluster_sync();
}

// ============================================================================
// Shared-memory-resident factors (r = 64, 128), 2-stage tile ring.
// ============================================================================

template <int T, int R>
struct SmemCfg {
  static constexpr int kWarps = kBoundaryThreads / 32;
  static constexpr int MT = T / 16;                       // m16 tiles per token tile
  static constexpr int NT1 = R / 8;                       // n8 tiles of y
  static constexpr int WN = (NT1 / 4) > 1 ? NT1 / 4 : 1;  // warps along r (phase 1)
  static constexpr int WK = kWarps / (MT * WN);           // warps along Dc (phase 1)
  static constexpr int NPW = NT1 / WN;                    // n8 tiles per warp (2 or 4)
  static constexpr int KS2 = R / 16;                      // k16 steps of phase 2
  static constexpr int CPR = R / 8;                       // 16-byte chunks per V row
  static constexpr int VL = (8 / CPR) > 1 ? 8 / CPR : 1;  // V rows per 128-byte line
  static constexpr int VXM = (CPR < 8 ? CPR : 8) - 1;     // chunk swizzle mask
  static constexpr int RP = R + 8;                        // padded fp32 row
  static_assert(T == 16 || T == 32, "token tile");
  static_assert(R == 16 || R == 32 || R == 64 || R == 128, "padded rank");
  static_assert(MT * WN * WK == kWarps, "warp split");
  static_assert(NPW == 2 || NPW == 4, "phase-1 n tiles per warp");
};

// Shared-memory carve-up of the shared-memory-factor kernel (host and device).
struct BoundarySmem {
  uint32_t us, vs, stage0, stage_bytes, partial, ybuf, wamax, am2, amaxbuf, rowinv, bars, total;
};

// vres: V slice resident in shared memory (else read from global memory in
// the re-projection).
__host__ __device__ inline BoundarySmem boundary_smem_layout(int T, int R, int Dc, bool vres = true) {
  const int MT = T / 16, NT1 = R / 8;
  const int WN = (NT1 / 4) > 1 ? NT1 / 4 : 1;
  const int WK = 8 / (MT * WN);
  const int RP = R + 8;
  const uint32_t pitch = static_cast<uint32_t>(Dc) * 2 + 16;
  BoundarySmem L;
  uint32_t off = 0;
  L.us = off;          off += R * pitch;                          // U^T slice, padded rows
  L.vs = off;          off += vres ? static_cast<uint32_t>(Dc) * R * 2 : 0u;  // V slice, swizzled
  L.stage0 = off;      L.stage_bytes = 2 * T * pitch;  off += 2 * L.stage_bytes;
  L.partial = off;     off += WK * T * RP * 4;                    // y (padded) aliases [0]
  L.ybuf = off;        off += T * R * 4;
  L.wamax = off;       off += 8 * T * 4;
  L.am2 = off;         off += 16 * T * 4;
  L.amaxbuf = off;     off += T * 4;
  L.rowinv = off;      off += T * 4;
  off = (off + 15u) & ~15u;
  L.bars = off;        off += 4 * 8;
  L.total = off;
  return L;
}

// VRES = false: only the U^T slice is resident; the re-projection reads its V
// fragments from global memory (L2), for shapes whose two slices do not fit.
template <int T, int R, bool F32OUT, bool VRES = true>
__global__ void __launch_bounds__(kBoundaryThreads, 1)
boundary_cluster_smem_kernel(const bf16* __restrict__ x, const bf16* __restrict__ res,
                             const bf16* __restrict__ Ut,   // [R, D]  (U transposed, zero padded)
                             const bf16* __restrict__ V,    // [D, R]  (zero padded)
                             int N, int D, int Dc, void* __restrict__ h_out,
                             uint8_t* __restrict__ q_out, float* __restrict__ scale_out, float qmax) {
  using C = SmemCfg<T, R>;
  constexpr int RP = C::RP;
  extern __shared__ __align__(128) uint8_t smem[];
  const BoundarySmem L = boundary_smem_layout(T, R, Dc, VRES);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q4 = lane & 3;
  const uint32_t crank = cluster_ctarank();
  const uint32_t csize = static_cast<uint32_t>(D / Dc);
  const int col0 = static_cast<int>(crank) * Dc;
  const uint32_t cid = cluster_id_x(), ncl = ncluster_x();
  const int ntiles = (N + T - 1) / T;
  const uint32_t pitch = static_cast<uint32_t>(Dc) * 2 + 16;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + L.bars;

  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(bars + 8 * i, 1);
    fence_mbarrier_init();
  }
  __syncthreads();

  // ok: false once a wait of this CTA gave up (CTA-uniform at the CTA
  // barriers). From then on no copy is issued and nothing is stored; waits
  // still run for copies already issued, so none is in flight at exit.
  bool ok = true;
  int issued = 0;   // loop iterations whose copies were issued
  auto issue = [&](int it) {
    const int tile = static_cast<int>(cid) + it * static_cast<int>(ncl);
    if (!ok || tile >= ntiles) return;
    issued = it + 1;
    if (warp != 0) return;
    const int s = it & 1;
    const uint32_t st = sbase + L.stage0 + s * L.stage_bytes;
    stage_tile(x, res, tile * T, N, D, col0, Dc, T, st, st + T * pitch, pitch, bars + 16 * s,
               bars + 16 * s + 8, lane);
  };
  issue(0);
  issue(1);

  // Resident factor slices: U^T rows [R x Dc] (padded pitch), V rows [Dc x R] (swizzled).
  {
    const int vpr = Dc / 8;
    for (int i = tid; i < R * vpr; i += kBoundaryThreads) {
      const int n = i / vpr, v = i % vpr;
      const uint4 val = __ldg(reinterpret_cast<const uint4*>(Ut + static_cast<size_t>(n) * D + col0) + v);
      *reinterpret_cast<uint4*>(smem + L.us + n * pitch + v * 16) = val;
    }
    for (int i = tid; VRES && i < Dc * C::CPR; i += kBoundaryThreads) {
      const int d = i / C::CPR, j = i % C::CPR;
      const uint4 val = __ldg(reinterpret_cast<const uint4*>(V + static_cast<size_t>(col0 + d) * R) + j);
      const int js = j ^ ((d / C::VL) & C::VXM);
      *reinterpret_cast<uint4*>(smem + L.vs + d * (R * 2) + js * 16) = val;
    }
  }
  __syncthreads();

  float* part = reinterpret_cast<float*>(smem + L.partial);
  float* yfull = part;
  float* ybuf = reinterpret_cast<float*>(smem + L.ybuf);
  float* wamax = reinterpret_cast<float*>(smem + L.wamax);
  float* am2 = reinterpret_cast<float*>(smem + L.am2);
  float* amaxbuf = reinterpret_cast<float*>(smem + L.amaxbuf);
  float* rowinv = reinterpret_cast<float*>(smem + L.rowinv);

  for (int it = 0;; ++it) {
    const int tile = static_cast<int>(cid) + it * static_cast<int>(ncl);
    if (tile >= ntiles) break;
    const int s = it & 1;
    const uint32_t par = static_cast<uint32_t>(it >> 1) & 1u;
    const int row0 = tile * T;
    const uint32_t rs = sbase + L.stage0 + s * L.stage_bytes;
    const uint8_t* rs_ptr = smem + L.stage0 + s * L.stage_bytes;
    uint8_t* xs_ptr = smem + L.stage0 + s * L.stage_bytes + T * pitch;

    // ---- phase 1: partial y = residual_tile[:, slice] * U_slice (tensor cores)
    if (it < issued) ok = mbar_wait(bars + 16 * s, par, kSiteBoundaryLoad) && ok;
    {
      const int wm = warp % C::MT;
      const int wn = (warp / C::MT) % C::WN;
      const int wk = warp / (C::MT * C::WN);
      float acc[C::NPW][4];
#pragma unroll
      for (int j = 0; j < C::NPW; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
      const uint32_t a_base = rs + (wm * 16 + (lane & 15)) * pitch + (lane >> 4) * 16;
      const uint32_t b_base = sbase + L.us +
                              (wn * C::NPW * 8 + (lane & 7) + (lane >> 4) * 8) * pitch +
                              ((lane >> 3) & 1) * 16;
      const int KS = Dc / 16;
#pragma unroll 4
      for (int ks = wk; ks < KS; ks += C::WK) {
        uint32_t a[4];
        ldmatrix_x4(a_base + ks * 32, a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int p = 0; p < C::NPW / 2; ++p) {
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4(b_base + p * 16 * pitch + ks * 32, b0, b1, b2, b3);
          mma_bf16_16816(acc[2 * p], a, b0, b1);
          mma_bf16_16816(acc[2 * p + 1], a, b2, b3);
        }
      }
      float* pw = part + wk * T * RP;
#pragma unroll
      for (int j = 0; j < C::NPW; ++j) {
        const int col = (wn * C::NPW + j) * 8 + 2 * q4;
        const int row = wm * 16 + g;
        *reinterpret_cast<float2*>(&pw[row * RP + col]) = make_float2(acc[j][0], acc[j][1]);
        *reinterpret_cast<float2*>(&pw[(row + 8) * RP + col]) = make_float2(acc[j][2], acc[j][3]);
      }
    }
    ok = __syncthreads_and(ok) != 0;
    for (int e = tid * 4; e < T * R; e += kBoundaryThreads * 4) {
      const int row = e / R, col = e % R;
      float4 sum = *reinterpret_cast<const float4*>(&part[row * RP + col]);
#pragma unroll
      for (int w = 1; w < C::WK; ++w) {
        const float4 v = *reinterpret_cast<const float4*>(&part[(w * T + row) * RP + col]);
        sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
      }
      *reinterpret_cast<float4*>(&ybuf[e]) = sum;
    }

    // ---- y over the cluster
    cluster_sync();
    for (int e = tid * 4; e < T * R; e += kBoundaryThreads * 4) {
      const int row = e / R, col = e % R;
      *reinterpret_cast<float4*>(&yfull[row * RP + col]) =
          cluster_sum_f32x4(sbase + L.ybuf + 4u * e, csize);
    }
    __syncthreads();

    // ---- phase 2: h = (res + x) + y V_slice^T, bf16 round, row amax
    if (it < issued) ok = mbar_wait(bars + 16 * s + 8, par, kSiteBoundaryLoad) && ok;
    {
      uint32_t ahi[C::MT][C::KS2][4], alo[C::MT][C::KS2][4];
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
        for (int ks = 0; ks < C::KS2; ++ks) {
          const int r0 = mt * 16 + g, c0 = ks * 16 + 2 * q4;
          split_bf16x2(*reinterpret_cast<const float2*>(&yfull[r0 * RP + c0]), ahi[mt][ks][0], alo[mt][ks][0]);
          split_bf16x2(*reinterpret_cast<const float2*>(&yfull[(r0 + 8) * RP + c0]), ahi[mt][ks][1], alo[mt][ks][1]);
          split_bf16x2(*reinterpret_cast<const float2*>(&yfull[r0 * RP + c0 + 8]), ahi[mt][ks][2], alo[mt][ks][2]);
          split_bf16x2(*reinterpret_cast<const float2*>(&yfull[(r0 + 8) * RP + c0 + 8]), ahi[mt][ks][3], alo[mt][ks][3]);
        }
      float rmax[C::MT][2];
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt) rmax[mt][0] = rmax[mt][1] = 0.f;

      const int ntw = Dc / 64;  // n8 tiles per warp
      uint32_t wcur[C::MT][2][2];
      load_n8<C::MT>(wcur, rs_ptr, xs_ptr, pitch, g, warp * ntw * 8 + 2 * q4);
      for (int t8 = 0; t8 < ntw; ++t8) {
        const int d0 = (warp * ntw + t8) * 8;
        uint32_t b[C::KS2][2];
        if constexpr (!VRES) {
          // B fragment of column d0 + g: (V[d][16ks + 2q], +1) and (+8, +9)
          const uint32_t* vr = reinterpret_cast<const uint32_t*>(V + static_cast<size_t>(col0 + d0 + g) * R) + q4;
#pragma unroll
          for (int ks = 0; ks < C::KS2; ++ks) {
            b[ks][0] = __ldg(vr + 8 * ks);
            b[ks][1] = __ldg(vr + 8 * ks + 4);
          }
        } else {
          const int d = d0 + (lane & 7);
          const uint32_t vrow = sbase + L.vs + d * (R * 2);
          const int sw = (d / C::VL) & C::VXM;
          if constexpr (C::KS2 == 1) {
            ldmatrix_x2(vrow + ((((lane >> 3) & 1) ^ sw) << 4), b[0][0], b[0][1]);
          } else {
#pragma unroll
            for (int p = 0; p < C::KS2 / 2; ++p)
              ldmatrix_x4(vrow + (((p * 4 + (lane >> 3)) ^ sw) << 4), b[2 * p][0], b[2 * p][1],
                          b[2 * p + 1][0], b[2 * p + 1][1]);
          }
        }
        float acc[C::MT][4];
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) {
          acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
#pragma unroll
          for (int ks = 0; ks < C::KS2; ++ks) {
            mma_bf16_16816(acc[mt], ahi[mt][ks], b[ks][0], b[ks][1]);
            mma_bf16_16816(acc[mt], alo[mt][ks], b[ks][0], b[ks][1]);
          }
        }
        // next block's words (the last block re-reads its own) before this block's stores
        uint32_t wnext[C::MT][2][2];
        load_n8<C::MT>(wnext, rs_ptr, xs_ptr, pitch, g, (t8 + 1 < ntw ? d0 + 8 : d0) + 2 * q4);
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt)
          finish_n8<F32OUT>(acc[mt], wcur[mt], xs_ptr, pitch, mt * 16 + g, d0 + 2 * q4, rmax[mt], h_out, row0,
                            N, D, col0, ok);
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            wcur[mt][hh][0] = wnext[mt][hh][0];
            wcur[mt][hh][1] = wnext[mt][hh][1];
          }
      }
      ok = publish_amax<C::MT, T>(rmax, wamax, amaxbuf, warp, lane, tid, ok);
    }

    // ---- amax over the cluster, then codes
    cluster_sync();
    gather_amax<T>(sbase + L.amaxbuf, am2, rowinv, scale_out, csize, crank, row0, N, tid, qmax, ok);
    store_tile<F32OUT>(xs_ptr, pitch, rowinv, T, Dc, row0, N, D, col0, h_out, q_out, tid, ok);
    fence_proxy_async_smem();
    __syncthreads();
    issue(it + 2);
  }
  cluster_sync();
}

// One CTA per token row (grid-stride): r == 0 or no residual. h = residual + x.
// VPT: 16-byte vectors per thread (D <= THREADS * 8 * VPT); the host picks
// the smallest that covers D, so registers (and the CTAs an SM holds) follow
// the row length.
template <int THREADS, int VPT, bool F32OUT>
__global__ void __launch_bounds__(THREADS)
boundary_rowwise_kernel(const bf16* __restrict__ x, const bf16* __restrict__ res, int N, int D,
                        void* __restrict__ h_out, uint8_t* __restrict__ q_out,
                        float* __restrict__ scale_out, float qmax) {
  __shared__ float red[THREADS / 32];
  __shared__ float s_inv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nv = D / 8;
  for (int row = blockIdx.x; row < N; row += gridDim.x) {
    const size_t base = static_cast<size_t>(row) * D;
    uint4 hv[VPT], xin[VPT], rin[VPT];
    float amax = 0.f;
    // all loads of the row first (predicated, so they are in flight together)
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = tid + j * THREADS;
      xin[j] = rin[j] = make_uint4(0u, 0u, 0u, 0u);
      if (v < nv) {
        xin[j] = __ldg(reinterpret_cast<const uint4*>(x + base) + v);
        if (res != nullptr) rin[j] = __ldg(reinterpret_cast<const uint4*>(res + base) + v);
      }
    }
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = tid + j * THREADS;
      if (v >= nv) break;
      const uint4 xv = xin[j], rv = rin[j];
      const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
      const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
      uint32_t hw[4];
      float hf[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        hf[2 * k] = bf16_lo_f32(rw[k]) + bf16_lo_f32(xw[k]);
        hf[2 * k + 1] = bf16_hi_f32(rw[k]) + bf16_hi_f32(xw[k]);
        hw[k] = pack_bf16x2(hf[2 * k], hf[2 * k + 1]);
        amax = fmaxf(amax, fmaxf(fabsf(bf16_lo_f32(hw[k])), fabsf(bf16_hi_f32(hw[k]))));
      }
      hv[j] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      if constexpr (F32OUT) {
        if (h_out != nullptr) {
          float4* hp = reinterpret_cast<float4*>(static_cast<float*>(h_out) + base) + 2 * v;
          hp[0] = make_float4(hf[0], hf[1], hf[2], hf[3]);
          hp[1] = make_float4(hf[4], hf[5], hf[6], hf[7]);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    if (tid == 0) {
      float m = 0.f;
      for (int w = 0; w < THREADS / 32; ++w) m = fmaxf(m, red[w]);
      float inv, sc;
      inv_and_scale(m, qmax, inv, sc);
      s_inv = inv;
      scale_out[row] = sc;
    }
    __syncthreads();
    const float inv = s_inv;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = tid + j * THREADS;
      if (v >= nv) break;
      if constexpr (!F32OUT) {
        if (h_out != nullptr) reinterpret_cast<uint4*>(static_cast<bf16*>(h_out) + base)[v] = hv[j];
      }
      reinterpret_cast<uint32_t*>(q_out + base / 2)[v] = quantize8(hv[j], inv);
    }
    __syncthreads();
  }
}

// Fragment-ordered factor copies for boundary_cluster_rf_kernel<R, T, Dc>,
// built on the host by the plan. `Ub`/`Vb` are the bf16 bit patterns of U and
// V, [D, R] row-major (R = padded rank). Output: arrays of 32-bit words in the
// order the kernel loads them: for CTA c and phase-1 warp group wk, register
// i = (j*NPW + p)*2 + e of lane (g, q) holds (U[d][n], U[d+1][n]) with
// d = c*Dc + (wk*KPW + j)*16 + 2q + 8e and n = 8p + g; for compute warp w,
// register i = (t*KS2 + k)*2 + e holds (V[d][m], V[d][m+1]) with
// d = c*Dc + (w*NTW + t)*8 + g and m = 16k + 2q + 8e.
inline void rf_pack_factors(const uint16_t* Ub, const uint16_t* Vb, int D, int R, int T, int Dc,
                            uint32_t* Uf, uint32_t* Vf) {
  const int MT = T / 16, WK = 8 / MT, KPW = Dc / 16 / WK, NPW = R / 8, KS2 = R / 16, NTW = Dc / 64;
  const int UREG = KPW * NPW * 2, VREG = NTW * KS2 * 2;
  const int C = D / Dc;
  auto pair = [](uint16_t lo, uint16_t hi) { return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16); };
  for (int c = 0; c < C; ++c)
    for (int wk = 0; wk < WK; ++wk)
      for (int lane = 0; lane < 32; ++lane) {
        const int g = lane >> 2, q = lane & 3;
        for (int i = 0; i < UREG; ++i) {
          const int e = i & 1, p = (i >> 1) % NPW, j = (i >> 1) / NPW;
          const int d = c * Dc + (wk * KPW + j) * 16 + 2 * q + 8 * e;
          const int n = p * 8 + g;
          const size_t idx = ((static_cast<size_t>(c * WK + wk) * (UREG / 4) + i / 4) * 32 + lane) * 4 + i % 4;
          Uf[idx] = pair(Ub[static_cast<size_t>(d) * R + n], Ub[static_cast<size_t>(d + 1) * R + n]);
        }
      }
  for (int c = 0; c < C; ++c)
    for (int w = 0; w < 8; ++w)
      for (int lane = 0; lane < 32; ++lane) {
        const int g = lane >> 2, q = lane & 3;
        for (int i = 0; i < VREG; ++i) {
          const int e = i & 1, k = (i >> 1) % KS2, t = (i >> 1) / KS2;
          const int d = c * Dc + (w * NTW + t) * 8 + g;
          const int m = k * 16 + 2 * q + 8 * e;
          const size_t idx = ((static_cast<size_t>(c * 8 + w) * (VREG / 4) + i / 4) * 32 + lane) * 4 + i % 4;
          Vf[idx] = pair(Vb[static_cast<size_t>(d) * R + m], Vb[static_cast<size_t>(d) * R + m + 1]);
        }
      }
}

}  // namespace respin
