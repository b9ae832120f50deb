// Fused block-boundary kernels: rank-r basis fix + per-token INT4 quantization.
//
// Per token (row) n, with the plan's bfloat16 factors U (D x r) and V (D x r):
//   y = residual[n] U ;  h = (residual[n] + x[n]) + y V^T  (fp32)
//   h' = bf16(h) ; amax = max|h'| ; inv = 7/amax ; q = clamp(rint(h' inv), -8, 7)
// This is the subspace residual rotation of the ReSpinQuant explainers (zh page
// §2.2 steps 1-3: projection, transform inside the subspace, re-projection and
// residual) in the row convention, followed by 4-bit activation quantization
// (zh §3-§4, W4A4).
//
// Cluster kernel design (B200): a token tile of T rows is split along D over a
// thread-block cluster of C CTAs (one per SM). CTA c owns columns
// [c*Dc, (c+1)*Dc) and keeps its slices of U^T and V resident in shared memory
// for the whole (persistent) launch, so the factors are read from L2 once per
// CTA, not once per tile. Residual and x tiles arrive by 1-D bulk copies into
// a two-stage shared-memory ring (next tile in flight while this one is
// computed). The two whole-row dependencies - y needs the full row before the
// re-projection, amax needs the full row before quantization - are resolved
// with two cluster barriers per tile and distributed-shared-memory reads. Both
// skinny products run on tensor cores (mma.sync m16n8k16 bf16, fp32
// accumulate); y is split into bf16 hi + lo parts for the second product so
// that it keeps ~16 mantissa bits. HBM sees each input byte once and each
// output byte once.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace respin {

using bf16 = __nv_bfloat16;

constexpr int kBoundaryThreads = 256;
constexpr float kZeroTokenAmax = 2.3509887e-38f;  // 2^-125

template <int T, int R>
struct BoundaryCfg {
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
  static_assert(T == 16 || T == 32, "token tile");
  static_assert(R == 16 || R == 32 || R == 64 || R == 128, "padded rank");
  static_assert(MT * WN * WK == kWarps, "warp split");
  static_assert(NPW == 2 || NPW == 4, "phase-1 n tiles per warp");
};

// Shared-memory carve-up of the cluster kernel (identical on host and device).
struct BoundarySmem {
  uint32_t us, vs, stage[2][2], partial, ybuf, yfull, wamax, amaxbuf, rowinv, bars, total;
};

__host__ __device__ inline BoundarySmem boundary_smem_layout(int T, int R, int Dc) {
  const int MT = T / 16, NT1 = R / 8;
  const int WN = (NT1 / 4) > 1 ? NT1 / 4 : 1;
  const int WK = 8 / (MT * WN);
  const uint32_t pitch = static_cast<uint32_t>(Dc) * 2 + 16;
  BoundarySmem L;
  uint32_t off = 0;
  L.us = off;       off += R * pitch;                       // U^T slice, padded rows
  L.vs = off;       off += static_cast<uint32_t>(Dc) * R * 2;  // V slice, swizzled
  for (int s = 0; s < 2; ++s)
    for (int t = 0; t < 2; ++t) { L.stage[s][t] = off; off += T * pitch; }
  L.partial = off;  off += WK * T * R * 4;
  L.ybuf = off;     off += T * R * 4;
  L.yfull = off;    off += T * R * 4;
  L.wamax = off;    off += 8 * T * 4;
  L.amaxbuf = off;  off += T * 4;
  L.rowinv = off;   off += T * 4;
  off = (off + 15u) & ~15u;
  L.bars = off;     off += 4 * 8;
  L.total = off;
  return L;
}

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
    int q = __float2int_rn(__fmul_rn(f, inv));
    q = min(max(q, -8), 7);
    packed |= (static_cast<uint32_t>(q) & 0xFu) << (4 * e);
  }
  return packed;
}

__device__ __forceinline__ void inv_and_scale(float amax, float& inv, float& scale) {
  if (amax >= kZeroTokenAmax) {
    inv = __fdiv_rn(7.0f, amax);
    scale = __fdiv_rn(amax, 7.0f);
  } else {
    inv = 0.0f;
    scale = 0.0f;
  }
}

template <int T, int R, bool F32OUT>
__global__ void __launch_bounds__(kBoundaryThreads, 1)
boundary_cluster_kernel(const bf16* __restrict__ x, const bf16* __restrict__ res,
                        const bf16* __restrict__ Ut,   // [R, D]  (U transposed, zero padded)
                        const bf16* __restrict__ V,    // [D, R]  (zero padded)
                        int N, int D, int Dc, void* __restrict__ h_out,
                        uint8_t* __restrict__ q_out, float* __restrict__ scale_out) {
  using C = BoundaryCfg<T, R>;
  extern __shared__ __align__(128) uint8_t smem[];
  const BoundarySmem L = boundary_smem_layout(T, R, Dc);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q4 = lane & 3;
  const uint32_t crank = cluster_ctarank();
  const uint32_t csize = static_cast<uint32_t>(D / Dc);
  const int col0 = static_cast<int>(crank) * Dc;
  const uint32_t cid = cluster_id_x(), ncl = ncluster_x();
  const int ntiles = (N + T - 1) / T;
  const uint32_t pitch = static_cast<uint32_t>(Dc) * 2 + 16;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_res0 = sbase + L.bars, bar_x0 = sbase + L.bars + 16;

  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(sbase + L.bars + 8 * i, 1);
    fence_mbarrier_init();
  }
  __syncthreads();

  // Stage the residual and x tiles of loop iteration `it` (warp 0 only).
  auto issue = [&](int it) {
    const int tile = static_cast<int>(cid) + it * static_cast<int>(ncl);
    if (tile >= ntiles || warp != 0) return;
    const int row0 = tile * T;
    const int rows = min(T, N - row0);
    const int s = it & 1;
    const uint32_t bytes = static_cast<uint32_t>(Dc) * 2;
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_res0 + 8 * s, rows * bytes);
      mbar_arrive_expect_tx(bar_x0 + 8 * s, rows * bytes);
    }
    __syncwarp();
    if (lane < rows) {
      const size_t gofs = static_cast<size_t>(row0 + lane) * D + col0;
      const uint32_t rdst = sbase + (s ? L.stage[1][0] : L.stage[0][0]) + lane * pitch;
      const uint32_t xdst = sbase + (s ? L.stage[1][1] : L.stage[0][1]) + lane * pitch;
      bulk_g2s(rdst, res + gofs, bytes, bar_res0 + 8 * s);
      bulk_g2s(xdst, x + gofs, bytes, bar_x0 + 8 * s);
    }
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
    for (int i = tid; i < Dc * C::CPR; i += kBoundaryThreads) {
      const int d = i / C::CPR, j = i % C::CPR;
      const uint4 val = __ldg(reinterpret_cast<const uint4*>(V + static_cast<size_t>(col0 + d) * R) + j);
      const int js = j ^ ((d / C::VL) & C::VXM);
      *reinterpret_cast<uint4*>(smem + L.vs + d * (R * 2) + js * 16) = val;
    }
  }
  __syncthreads();

  float* part = reinterpret_cast<float*>(smem + L.partial);
  float* ybuf = reinterpret_cast<float*>(smem + L.ybuf);
  float* yfull = reinterpret_cast<float*>(smem + L.yfull);
  float* wamax = reinterpret_cast<float*>(smem + L.wamax);
  float* amaxbuf = reinterpret_cast<float*>(smem + L.amaxbuf);
  float* rowinv = reinterpret_cast<float*>(smem + L.rowinv);

  for (int it = 0;; ++it) {
    const int tile = static_cast<int>(cid) + it * static_cast<int>(ncl);
    if (tile >= ntiles) break;
    const int s = it & 1;
    const uint32_t par = static_cast<uint32_t>(it >> 1) & 1u;
    const int row0 = tile * T;
    const uint32_t rs_off = s ? L.stage[1][0] : L.stage[0][0];
    const uint32_t xs_off = s ? L.stage[1][1] : L.stage[0][1];
    const uint32_t rs = sbase + rs_off;
    uint8_t* xs_ptr = smem + xs_off;
    const uint8_t* rs_ptr = smem + rs_off;

    // ---- phase 1: partial y = residual_tile[:, slice] * U_slice (tensor cores)
    mbar_wait(bar_res0 + 8 * s, par, kSiteBoundaryLoad);
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
      float* pw = part + wk * T * R;
#pragma unroll
      for (int j = 0; j < C::NPW; ++j) {
        const int col = (wn * C::NPW + j) * 8 + 2 * q4;
        const int row = wm * 16 + g;
        *reinterpret_cast<float2*>(&pw[row * R + col]) = make_float2(acc[j][0], acc[j][1]);
        *reinterpret_cast<float2*>(&pw[(row + 8) * R + col]) = make_float2(acc[j][2], acc[j][3]);
      }
    }
    __syncthreads();
    for (int i = tid * 4; i < T * R; i += kBoundaryThreads * 4) {
      float4 sum = *reinterpret_cast<const float4*>(&part[i]);
#pragma unroll
      for (int w = 1; w < C::WK; ++w) {
        const float4 v = *reinterpret_cast<const float4*>(&part[w * T * R + i]);
        sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
      }
      *reinterpret_cast<float4*>(&ybuf[i]) = sum;
    }

    // ---- cluster reduction of y (same order in every CTA -> identical y)
    cluster_sync();
    {
      const uint32_t yb = sbase + L.ybuf;
      for (int i = tid; i < T * R; i += kBoundaryThreads) {
        float sum = 0.f;
        for (uint32_t c = 0; c < csize; ++c) sum += ld_dsmem_f32(map_to_rank(yb, c) + 4u * i);
        yfull[i] = sum;
      }
    }
    __syncthreads();

    // ---- phase 2: h = (res + x) + y V_slice^T, bf16 round, row amax
    mbar_wait(bar_x0 + 8 * s, par, kSiteBoundaryLoad);
    {
      uint32_t ahi[C::MT][C::KS2][4], alo[C::MT][C::KS2][4];
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
        for (int ks = 0; ks < C::KS2; ++ks) {
          const int r0 = mt * 16 + g, c0 = ks * 16 + 2 * q4;
          const float2 v[4] = {*reinterpret_cast<const float2*>(&yfull[r0 * R + c0]),
                               *reinterpret_cast<const float2*>(&yfull[(r0 + 8) * R + c0]),
                               *reinterpret_cast<const float2*>(&yfull[r0 * R + c0 + 8]),
                               *reinterpret_cast<const float2*>(&yfull[(r0 + 8) * R + c0 + 8])};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 hi = __floats2bfloat162_rn(v[e].x, v[e].y);
            const float2 hf = __bfloat1622float2(hi);
            const __nv_bfloat162 lo = __floats2bfloat162_rn(v[e].x - hf.x, v[e].y - hf.y);
            ahi[mt][ks][e] = *reinterpret_cast<const uint32_t*>(&hi);
            alo[mt][ks][e] = *reinterpret_cast<const uint32_t*>(&lo);
          }
        }
      float rmax[C::MT][2];
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt) rmax[mt][0] = rmax[mt][1] = 0.f;

      const int ntw = Dc / 64;  // n8 tiles per warp
      for (int t8 = 0; t8 < ntw; ++t8) {
        const int d0 = (warp * ntw + t8) * 8;
        uint32_t b[C::KS2][2];
        {
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
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) {
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ks = 0; ks < C::KS2; ++ks) {
            mma_bf16_16816(acc, ahi[mt][ks], b[ks][0], b[ks][1]);
            mma_bf16_16816(acc, alo[mt][ks], b[ks][0], b[ks][1]);
          }
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int row = mt * 16 + g + 8 * hh;
            const uint32_t off = row * pitch + (d0 + 2 * q4) * 2;
            const uint32_t rw = *reinterpret_cast<const uint32_t*>(rs_ptr + off);
            const uint32_t xw = *reinterpret_cast<const uint32_t*>(xs_ptr + off);
            const float h0 = (bf16_lo_f32(rw) + bf16_lo_f32(xw)) + acc[2 * hh];
            const float h1 = (bf16_hi_f32(rw) + bf16_hi_f32(xw)) + acc[2 * hh + 1];
            const uint32_t hb = pack_bf16x2(h0, h1);
            *reinterpret_cast<uint32_t*>(xs_ptr + off) = hb;
            rmax[mt][hh] = fmaxf(rmax[mt][hh], fmaxf(fabsf(bf16_lo_f32(hb)), fabsf(bf16_hi_f32(hb))));
            if constexpr (F32OUT) {
              if (h_out != nullptr && row0 + row < N) {
                float* hf = static_cast<float*>(h_out) +
                            static_cast<size_t>(row0 + row) * D + col0 + d0 + 2 * q4;
                *reinterpret_cast<float2*>(hf) = make_float2(h0, h1);
              }
            }
          }
        }
      }
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float m = rmax[mt][hh];
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
          if (q4 == 0) wamax[warp * T + mt * 16 + g + 8 * hh] = m;
        }
    }
    __syncthreads();
    if (tid < T) {
      float m = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) m = fmaxf(m, wamax[w * T + tid]);
      amaxbuf[tid] = m;
    }

    // ---- cluster reduction of the row amax
    cluster_sync();
    if (tid < T) {
      const uint32_t ab = sbase + L.amaxbuf + 4u * tid;
      float m = 0.f;
      for (uint32_t c = 0; c < csize; ++c) m = fmaxf(m, ld_dsmem_f32(map_to_rank(ab, c)));
      float inv, sc;
      inv_and_scale(m, inv, sc);
      rowinv[tid] = inv;
      if (crank == 0 && row0 + tid < N) scale_out[row0 + tid] = sc;
    }
    __syncthreads();

    // ---- store h' (bf16) and the packed codes of this CTA's slice
    {
      const int vpr = Dc / 8;
      for (int i = tid; i < T * vpr; i += kBoundaryThreads) {
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
    // This stage is refilled by bulk copies next: order the generic-proxy
    // writes above before those async-proxy writes.
    fence_proxy_async_smem();
    __syncthreads();
    issue(it + 2);
  }
  // No CTA may leave while a peer can still read its shared memory.
  cluster_sync();
}

// One CTA per token row (grid-stride): r == 0 or no residual. h = residual + x.
template <int THREADS, bool F32OUT>
__global__ void __launch_bounds__(THREADS)
boundary_rowwise_kernel(const bf16* __restrict__ x, const bf16* __restrict__ res, int N, int D,
                        void* __restrict__ h_out, uint8_t* __restrict__ q_out,
                        float* __restrict__ scale_out) {
  constexpr int VPT = 8;  // 16-byte vectors per thread (D <= THREADS * 64)
  __shared__ float red[THREADS / 32];
  __shared__ float s_inv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nv = D / 8;
  for (int row = blockIdx.x; row < N; row += gridDim.x) {
    const size_t base = static_cast<size_t>(row) * D;
    uint4 hv[VPT];
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = tid + j * THREADS;
      if (v >= nv) break;
      const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + base) + v);
      uint4 rv = make_uint4(0u, 0u, 0u, 0u);
      if (res != nullptr) rv = __ldg(reinterpret_cast<const uint4*>(res + base) + v);
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
      inv_and_scale(m, inv, sc);
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

}  // namespace respin
