// Tensor-core boundary passes for large ranks (r = 33 .. 128, padded to
// RP = 64 or 128): the same fix and quantizer as the fused boundary kernels
//   y = residual U ; h = (residual + x) + y V^T (fp32) ; h' = bf16(h)
//   amax = max|h'| ; inv = qmax/amax ; q = rint(h' inv)
// (ReSpinQuant explainers, zh page §2.2 steps 1-3 in the row convention, and
// the activation quantization of zh §3-§4), as three launches:
//
//  1. boundary_tc_project_kernel: y = residual U on tcgen05 (M = 128 tokens,
//     N = RP, K = a share of D; bf16 operands by tensor copies in the 128-byte
//     swizzled K-major layout, fp32 accumulators in TMEM). The K range of a
//     token tile is split over S CTAs so that about one CTA per SM streams
//     the residual; each writes its fp32 partial y into the row of the code
//     buffer that the token's codes later overwrite (the caller's memory, so
//     nothing is allocated).
//  2. boundary_tc_reproject_kernel: per tile of 128 tokens x 128 columns,
//     A = [y_hi | y_lo] (the S partials summed in split order, then split into
//     bf16 hi + lo parts, built in shared memory once per token tile) and
//     B = the tile's rows of V: two tcgen05 MMA chains into one TMEM
//     accumulator give y V^T. The epilogue adds residual + x (32-column
//     chunks by tensor copies, 64-byte swizzle), rounds to bf16, writes h'
//     over the chunk's residual rows and out by tensor stores, and folds the
//     tile's row maxima of |h'| into the scale buffer with an atomic max
//     (non-negative floats order like their bit patterns).
//  3. boundary_quant_rows_kernel: codes and scales of every token from h' and
//     its amax.
// Passes 2 and 3 are launched as programmatic dependents: a pass starts while
// the previous one finishes (pass 2 streams residual, x and V at once) and
// waits for the previous pass's results only where it reads them. Pass 1
// clears the amax accumulators.
//
// HBM traffic per token: residual twice, x once, h' written and read back,
// codes and scale: 10 D + 4 bytes (8.5 D + 4 for h' in fp32 aside), against
// 6.5 D + 4 for the fused kernels, which cannot hold r = 64 / 128 slices and
// a token's whole row at once. Waits are bounded; after one gives up the CTA
// stops issuing copies and MMAs, stores nothing more, waits (bounded) for the
// copies and MMAs already issued, and leaves.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "boundary_kernels.cuh"
#include "ptx.cuh"

namespace respin {

constexpr int kTcBM = 128;                  // tokens per tile (MMA M)
constexpr uint32_t kTcKBlock = kTcBM * 128; // one 128-row x 64-element bf16 K block (16 KB)
constexpr int kTcBN = 128;                  // columns per re-projection tile (MMA N)
constexpr int kTcChunk = 32;                // columns per epilogue chunk

// 16-byte chunk j (0..3) of row r in a 64-byte-row tile with the tensor-map
// 64-byte swizzle (chunk index XOR bits 7-8 of the offset).
__device__ __forceinline__ uint32_t tc_sw64(int r, int j) {
  return static_cast<uint32_t>(r * 64 + ((j ^ ((r >> 1) & 3)) << 4));
}

// ---------------------------------------------------------------- pass 1

template <int RP>
struct TcProjCfg {
  static_assert(RP == 64 || RP == 128, "padded rank");
  static constexpr int STG = RP == 64 ? 8 : 6;        // K-block stages (192 KB either way)
  static constexpr uint32_t ABytes = kTcKBlock;       // 128 tokens x 64
  static constexpr uint32_t BBytes = RP * 128;        // RP rows of U^T x 64
  static constexpr uint32_t Stage = ABytes + BBytes;
  static constexpr uint32_t oBars = STG * Stage;      // full[STG], empty[STG], done
  static constexpr uint32_t oMisc = oBars + (2 * STG + 1) * 8;   // tmem slot, counters, abort
  static constexpr uint32_t kSmem = oMisc + 32 + 1024;
  static constexpr int kThreads = 128;
};

// tmR: residual bf16 [N, D], box {64, 128}, 128-byte swizzle. tmU: U^T bf16
// [RP, D], box {64, RP}, 128-byte swizzle. CTA b: token tile b / S, K blocks
// [kb0, kb1) of split b % S. Partial y of token n, split s: RP floats at byte
// n * ypitch + s * RP * 4 of ypart.
template <int RP>
__global__ void __launch_bounds__(128, 1)
boundary_tc_project_kernel(const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmU,
                           int N, int KB, int S, uint8_t* __restrict__ ypart, int ypitch,
                           float* __restrict__ amax) {
  using C = TcProjCfg<RP>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mt = static_cast<int>(blockIdx.x) / S, split = static_cast<int>(blockIdx.x) % S;
  const int kb0 = (split * KB) / S, kb1 = ((split + 1) * KB) / S, nk = kb1 - kb0;
  const int m0 = mt * kTcBM;
  const uint32_t bars = base + C::oBars;
  auto full = [&](int s) { return bars + 8 * s; };
  auto empty = [&](int s) { return bars + 8 * (C::STG + s); };
  const uint32_t done = bars + 16 * C::STG;
  volatile int* misc = reinterpret_cast<volatile int*>(smem + C::oMisc + 16);   // [1] consumed [2] abort
  const uint32_t tslot = base + C::oMisc;

  if (tid == 0) {
    for (int s = 0; s < C::STG; ++s) { mbar_init(full(s), 2); mbar_init(empty(s), 1); }   // full: A and B copies
    mbar_init(done, 1);
    misc[1] = 0; misc[2] = 0;
    fence_mbarrier_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmR) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmU) : "memory");
  }
  if (warp == 0) { tmem_alloc(tslot, RP); tmem_relinquish(); }
  // the re-projection pass may start its independent work now
  grid_dep_launch();
  // the amax accumulator of this token tile starts at zero (bit pattern 0)
  if (split == 0 && m0 + tid < N) amax[m0 + tid] = 0.0f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + C::oMisc);

  if (warp == 0 && lane < 2 * C::STG) {
    // ---- producer lanes: lane 2s copies the residual K blocks of stage s,
    // lane 2s + 1 the U^T K blocks (copies issued by one thread complete one
    // after the other, so every stream of copies has its own thread)
    const int s = lane >> 1;
    const bool is_u = (lane & 1) != 0;
    int last = -1;
    for (int i = s; i < nk; i += C::STG) {
      if (misc[2]) break;
      const int u = i / C::STG;
      if (!mbar_wait(empty(s), (u & 1) ^ 1, kSiteTcFree)) { misc[2] = 1; break; }
      const uint32_t dst = base + s * C::Stage;
      if (is_u) {
        mbar_arrive_expect_tx(full(s), C::BBytes);
        tma_load_2d(dst + C::ABytes, &tmU, (kb0 + i) * 64, 0, full(s));
      } else {
        mbar_arrive_expect_tx(full(s), C::ABytes);
        tma_load_2d(dst, &tmR, (kb0 + i) * 64, m0, full(s));
      }
      last = u;
    }
    // after a give-up: the copies this lane issued have landed before the
    // shared memory is released
    if (last >= 0) mbar_wait(full(s), last & 1, kSiteTcLoad);
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer
    constexpr uint32_t idesc = umma_idesc_bf16(kTcBM, RP);
    for (int i = 0; i < nk; ++i) {
      if (misc[2]) break;
      const int s = i % C::STG;
      if (!mbar_wait(full(s), (i / C::STG) & 1, kSiteTcLoad)) { misc[2] = 1; break; }
      tc_fence_after();
      const uint32_t a = base + s * C::Stage, b = a + C::ABytes;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        tc_mma_bf16(tmem, umma_desc_sw128(a + 32 * k), umma_desc_sw128(b + 32 * k), idesc, (i | k) != 0 ? 1u : 0u);
      tc_commit(empty(s));
      misc[1] = i + 1;
    }
    tc_commit(done);   // also after a give-up: completes once the issued MMAs have
  }
  __syncthreads();
  bool ok = mbar_wait(done, 0, kSiteTcAccum);
  ok = ok && misc[2] == 0 && misc[1] == nk;
  tc_fence_after();
  const int row = m0 + 32 * warp + lane;
#pragma unroll 1
  for (int c = 0; c < RP / 32; ++c) {
    uint32_t v[32];
    tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 32 * c, v);
    tmem_wait_ld();
    if (ok && row < N) {
      float4* dst = reinterpret_cast<float4*>(ypart + static_cast<size_t>(row) * ypitch) + (split * RP + 32 * c) / 4;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]), __uint_as_float(v[4 * j + 2]),
                             __uint_as_float(v[4 * j + 3]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, RP);
  }
}

// ---------------------------------------------------------------- pass 2

template <int RP>
struct TcReCfg {
  static_assert(RP == 64 || RP == 128, "padded rank");
  static constexpr int KBR = RP / 64;                          // K blocks of y (hi or lo)
  static constexpr uint32_t ABytes = 2 * KBR * kTcKBlock;      // [y_hi | y_lo], 128 rows
  static constexpr int BST = 2;                                // V tile stages
  static constexpr uint32_t BBytes = KBR * kTcBN * 128;        // 128 rows of V x RP
  static constexpr int CST = RP == 128 ? 6 : 8;                // residual + x chunk stages
  static constexpr int HST = CST / 2;                          // stages of each half's ring
  static constexpr uint32_t CHalf = kTcBM * kTcChunk * 2;      // 128 rows x 32 columns bf16 (8 KB)
  static constexpr uint32_t CBytes = 2 * CHalf;                // residual then x
  static constexpr uint32_t oA = 0;
  static constexpr uint32_t oB = ABytes;
  static constexpr uint32_t oC = oB + BST * BBytes;
  static constexpr uint32_t oBars = oC + CST * CBytes;
  // bfull[BST] bempty[BST] cfull[CST] cempty[CST] afull[2] aempty[2] opa_full opa_empty fin
  static constexpr int kBars = 2 * BST + 2 * CST + 4 + 3;
  static constexpr uint32_t oMisc = oBars + kBars * 8;        // tmem slot, abort flag
  static constexpr uint32_t kSmem = oMisc + 16 + 1024;
  static constexpr int kThreads = 320;                         // producer, MMA, 8 epilogue warps
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

// tmRc / tmXc: residual / x bf16 [N, D], box {32, 128}, 64-byte swizzle.
// tmH: h_out bf16 [N, D], box {32, 32}, 64-byte swizzle (unused for fp32 h).
// tmV: V bf16 [D, RP], box {64, 128}, 128-byte swizzle. Tiles t = m * (D /
// 128) + n (token tile m, column tile n); CTA b takes the contiguous range
// [b T / G, (b+1) T / G). amax: the scale buffer, zero on entry, receives
// the bit pattern of max |h'| per token.
template <int RP, bool F32OUT>
__global__ void __launch_bounds__(320, 1)
boundary_tc_reproject_kernel(const __grid_constant__ CUtensorMap tmRc, const __grid_constant__ CUtensorMap tmXc,
                             const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmV,
                             int N, int D, int S,
                             const uint8_t* __restrict__ ypart, int ypitch, void* __restrict__ h_out,
                             float* __restrict__ amax) {
  using C = TcReCfg<RP>;
  constexpr int KBR = C::KBR;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntn = D / kTcBN;
  const int mtiles = (N + kTcBM - 1) / kTcBM;
  const int T = mtiles * ntn, G = static_cast<int>(gridDim.x), b = static_cast<int>(blockIdx.x);
  const int t0 = static_cast<int>((static_cast<long long>(b) * T) / G);
  const int t1 = static_cast<int>((static_cast<long long>(b + 1) * T) / G);
  const int nloc = t1 - t0;
  const uint32_t bars = base + C::oBars;
  auto bfull = [&](int s) { return bars + 8 * s; };
  auto bempty = [&](int s) { return bars + 8 * (C::BST + s); };
  auto cfull = [&](int s) { return bars + 8 * (2 * C::BST + s); };
  auto cempty = [&](int s) { return bars + 8 * (2 * C::BST + C::CST + s); };
  auto afull = [&](int a) { return bars + 8 * (2 * C::BST + 2 * C::CST + a); };
  auto aempty = [&](int a) { return bars + 8 * (2 * C::BST + 2 * C::CST + 2 + a); };
  const uint32_t opa_full = bars + 8 * (2 * C::BST + 2 * C::CST + 4);
  const uint32_t opa_empty = opa_full + 8;
  const uint32_t fin = opa_full + 16;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::oMisc + 8);
  const uint32_t tslot = base + C::oMisc;

  if (tid == 0) {
    for (int s = 0; s < C::BST; ++s) { mbar_init(bfull(s), 1); mbar_init(bempty(s), 1); }
    for (int s = 0; s < C::CST; ++s) { mbar_init(cfull(s), 2); mbar_init(cempty(s), 4); }   // residual + x copies
    for (int a = 0; a < 2; ++a) { mbar_init(afull(a), 1); mbar_init(aempty(a), 8); }
    mbar_init(opa_full, 8);
    mbar_init(opa_empty, 1);
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmRc) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmXc) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmV) : "memory");
  }
  if (warp == 0) { tmem_alloc(tslot, 2 * kTcBN); tmem_relinquish(); }
  grid_dep_launch();   // the code pass may be scheduled (it waits for this grid)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + C::oMisc);
  auto tile_m = [&](int i) { return (t0 + i) / ntn; };
  auto tile_n = [&](int i) { return (t0 + i) % ntn; };
  auto new_m = [&](int i) { return i == 0 || tile_m(i) != tile_m(i - 1); };

  if (warp == 0) {
    // ---- producer lanes: lane c < CST copies the residual chunks of stage
    // c and lane 8 + c its x chunks (copies issued by one thread complete one
    // after the other), lane 16 + s owns V stage s; each stage has at most
    // one fill in flight. The chunk stages form two rings, one per epilogue
    // half (stages h HST .. h HST + HST - 1 carry half h's chunks 2h, 2h + 1
    // of every tile, in order), so every stage is consumed by the same four
    // warps in order and no consumer can run two phases ahead of a stage.
    static_assert(C::CST <= 8, "chunk producer lanes");
    int last = -1;   // this lane's last issued use (for the final drain)
    if (lane < 16 && (lane & 7) < C::CST) {
      const int st = lane & 7;
      const bool is_x = lane >= 8;
      const int h = st / C::HST, j = st % C::HST;
      const int np = 2 * nloc;   // chunks of half h
      for (int pidx = j; pidx < np; pidx += C::HST) {
        if (*abort_flag) break;
        const int u = pidx / C::HST;
        if (!mbar_wait(cempty(st), (u & 1) ^ 1, kSiteTcFree)) { *abort_flag = 1; break; }
        const int i = pidx >> 1, c = 2 * h + (pidx & 1);
        const int x0 = tile_n(i) * kTcBN + c * kTcChunk, y0 = tile_m(i) * kTcBM;
        const uint32_t dst = base + C::oC + st * C::CBytes;
        mbar_arrive_expect_tx(cfull(st), C::CHalf);
        if (is_x) tma_load_2d(dst + C::CHalf, &tmXc, x0, y0, cfull(st));
        else tma_load_2d(dst, &tmRc, x0, y0, cfull(st));
        last = u;
      }
      if (last >= 0) mbar_wait(cfull(st), last & 1, kSiteTcLoad);
    } else if (lane >= 16 && lane < 16 + C::BST) {
      const int s = lane - 16;
      for (int i = s; i < nloc; i += C::BST) {
        if (*abort_flag) break;
        const int u = i / C::BST;
        if (!mbar_wait(bempty(s), (u & 1) ^ 1, kSiteTcFree)) { *abort_flag = 1; break; }
        const uint32_t dst = base + C::oB + s * C::BBytes;
        mbar_arrive_expect_tx(bfull(s), C::BBytes);
#pragma unroll
        for (int kb = 0; kb < KBR; ++kb) tma_load_2d(dst + kb * kTcKBlock, &tmV, kb * 64, tile_n(i) * kTcBN, bfull(s));
        last = u;
      }
      if (last >= 0) mbar_wait(bfull(s), last & 1, kSiteTcLoad);
    }
  } else if (warp == 1) {
    // ---- MMA issuer: acc = y_hi V^T + y_lo V^T
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(kTcBM, kTcBN);
      int seg = 0;
      for (int i = 0; i < nloc; ++i) {
        if (*abort_flag) break;
        if (new_m(i)) {
          if (!mbar_wait(opa_full, seg & 1, kSiteTcAccum)) { *abort_flag = 1; break; }
          ++seg;
        }
        const int ab = i & 1, bs = i % C::BST;
        if (!mbar_wait(aempty(ab), ((i >> 1) & 1) ^ 1, kSiteTcAccum)) { *abort_flag = 1; break; }
        if (!mbar_wait(bfull(bs), (i / C::BST) & 1, kSiteTcLoad)) { *abort_flag = 1; break; }
        tc_fence_after();
        const uint32_t d = tmem + ab * kTcBN;
        const uint32_t a = base + C::oA, bb = base + C::oB + bs * C::BBytes;
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int kb = 0; kb < KBR; ++kb)
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc_mma_bf16(d, umma_desc_sw128(a + (part * KBR + kb) * kTcKBlock + 32 * k),
                          umma_desc_sw128(bb + kb * kTcKBlock + 32 * k), idesc, (part | kb | k) != 0 ? 1u : 0u);
        tc_commit(bempty(bs));
        tc_commit(afull(ab));
        if (i + 1 == nloc || new_m(i + 1)) tc_commit(opa_empty);
      }
    }
    if (lane == 0) tc_commit(fin);   // completes once every issued MMA has
  } else {
    // ---- epilogue warps 2..9: TMEM lane quarter qd = warp % 4 holds tile
    // rows 32 qd .. 32 qd + 31 (thread = one token row); warps 2-5 take the
    // 32-column chunks 0 and 1 of a tile, warps 6-9 chunks 2 and 3.
    const int qd = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = 32 * qd + lane;
    // the partial y and the zeroed amax come from the projection pass, which
    // may still be running (the tensor copies of residual, x and V need not
    // wait for it)
    grid_dep_wait();
    int seg = 0;
    bool ok = true;
    for (int i = 0; i < nloc && ok; ++i) {
      const int m = tile_m(i), n = tile_n(i);
      const int tok = m * kTcBM + r;
      if (new_m(i)) {
        // the previous token tile's MMAs are done with operand A
        if (seg > 0) ok = mbar_wait(opa_empty, (seg - 1) & 1, kSiteTcAccum) && ok;
        ok = __all_sync(0xffffffffu, ok && *abort_flag == 0);   // warp-uniform
        if (!ok) break;
        // A = [y_hi | y_lo] of the tile's rows: the S partials summed in split
        // order, then split into bf16 hi and lo parts
        uint8_t* arow = smem + C::oA + (r >> 3) * 1024 + (r & 7) * 128;
        const float* yp = reinterpret_cast<const float*>(ypart + static_cast<size_t>(tok < N ? tok : 0) * ypitch);
#pragma unroll 1
        for (int c8 = half * (RP / 16); c8 < (half + 1) * (RP / 16); ++c8) {
          float y[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) y[e] = 0.f;
          if (tok < N) {
            for (int s = 0; s < S; ++s) {
              const float4 p0 = *reinterpret_cast<const float4*>(yp + s * RP + 8 * c8);
              const float4 p1 = *reinterpret_cast<const float4*>(yp + s * RP + 8 * c8 + 4);
              y[0] += p0.x; y[1] += p0.y; y[2] += p0.z; y[3] += p0.w;
              y[4] += p1.x; y[5] += p1.y; y[6] += p1.z; y[7] += p1.w;
            }
          }
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) split_bf16x2(make_float2(y[2 * e], y[2 * e + 1]), hi[e], lo[e]);
          const int kb = c8 >> 3, j = c8 & 7;
          const uint32_t off = static_cast<uint32_t>(((j ^ (r & 7)) << 4));
          *reinterpret_cast<uint4*>(arow + kb * kTcKBlock + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(arow + (KBR + kb) * kTcKBlock + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(opa_full);
        ++seg;
      }
      const int ab = i & 1;
      if (ok) ok = mbar_wait(afull(ab), (i >> 1) & 1, kSiteTcAccum);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      // both chunks' accumulators at once, then the buffer goes back to the
      // MMA issuer
      uint32_t v[2][32];
      const uint32_t tb = tmem + (static_cast<uint32_t>(32 * qd) << 16) + ab * kTcBN + kTcChunk * 2 * half;
      tmem_ld_32x32b_x32(tb, v[0]);
      tmem_ld_32x32b_x32(tb + kTcChunk, v[1]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(aempty(ab));
      float rmax = 0.f;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * half + cc;
        const int pidx = 2 * i + cc;   // position in this half's chunk ring
        const int cs = half * C::HST + pidx % C::HST;
        if (ok) ok = mbar_wait(cfull(cs), (pidx / C::HST) & 1, kSiteTcLoad);
        ok = __all_sync(0xffffffffu, ok);
        uint8_t* rs = smem + C::oC + cs * C::CBytes;
        const uint8_t* xs = rs + C::CHalf;
        uint4 rv[4], xv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          rv[j] = *reinterpret_cast<const uint4*>(rs + tc_sw64(r, j));
          xv[j] = *reinterpret_cast<const uint4*>(xs + tc_sw64(r, j));
        }
        const size_t gcol = static_cast<size_t>(n) * kTcBN + kTcChunk * c;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t rw[4] = {rv[j].x, rv[j].y, rv[j].z, rv[j].w}, xw[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
          uint32_t hw[4];
          float2 hf[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 sum = add_f32x2(bf16x2_to_f32x2(rw[e]), bf16x2_to_f32x2(xw[e]));
            const float2 acc =
                make_float2(__uint_as_float(v[cc][8 * j + 2 * e]), __uint_as_float(v[cc][8 * j + 2 * e + 1]));
            hf[e] = add_f32x2(sum, acc);
            hw[e] = pack_bf16x2(hf[e].x, hf[e].y);
            rmax = fmaxf(rmax, fmaxf(fabsf(bf16_lo_f32(hw[e])), fabsf(bf16_hi_f32(hw[e]))));
          }
          if constexpr (F32OUT) {
            if (ok && tok < N) {
              float4* hp =
                  reinterpret_cast<float4*>(static_cast<float*>(h_out) + static_cast<size_t>(tok) * D + gcol + 8 * j);
              hp[0] = make_float4(hf[0].x, hf[0].y, hf[1].x, hf[1].y);
              hp[1] = make_float4(hf[2].x, hf[2].y, hf[3].x, hf[3].y);
            }
          } else {
            // h' over this thread's own residual row of the stage
            *reinterpret_cast<uint4*>(rs + tc_sw64(r, j)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          }
        }
        // generic-proxy accesses of the stage before the tensor store reads
        // it and before its next copy
        fence_proxy_async_smem();
        __syncwarp();
        if constexpr (!F32OUT) {
          // this warp's 32 rows of h' go out as one tensor store (rows past N
          // are clipped); the stage is released once the store has read them
          const int y0 = tile_m(i) * kTcBM + 32 * qd;
          if (lane == 0 && ok && y0 < N) {
            tma_store_2d(&tmH, static_cast<int>(gcol), y0, base + C::oC + cs * C::CBytes + 32 * qd * 64);
            bulk_commit_group();
            bulk_wait_group_read<0>();
          }
          __syncwarp();
        }
        if (lane == 0) mbar_arrive(cempty(cs));
      }
      if (ok && tok < N) atomicMax(reinterpret_cast<unsigned int*>(amax) + tok, __float_as_uint(rmax));
    }
    // every h' tensor store of this warp has completed before the launch ends
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
    if (!ok) *abort_flag = 1;
  }
  __syncthreads();
  // every MMA issued has completed (the issuer's last commit) before TMEM goes
  if (tid == 0) mbar_wait(fin, 0, kSiteTcAccum);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kTcBN);
  }
}

// ---------------------------------------------------------------- pass 3

// Codes and scale of every token from h' (bf16, or fp32 rounded to bf16) and
// amax (the bit pattern left in the scale buffer by pass 2), which is then
// overwritten by the scale. One CTA per token row at a time.
template <bool F32IN>
__global__ void __launch_bounds__(256)
boundary_quant_rows_kernel(const void* __restrict__ h, int N, int D, uint8_t* __restrict__ q_out,
                           float* __restrict__ scale_io, float qmax) {
  constexpr int VPT = 8;   // 16-byte vectors of h' per thread per pass (D <= 16384 in one pass)
  const int tid = threadIdx.x;
  const int nv = D / 8;
  grid_dep_wait();   // h' and amax come from the re-projection pass
  for (int row = blockIdx.x; row < N; row += gridDim.x) {
    const float amax = scale_io[row];
    float inv, sc;
    inv_and_scale(amax, qmax, inv, sc);
    for (int v0 = 0; v0 < nv; v0 += 256 * VPT) {
      uint4 hv[VPT];
      // all loads first (predicated, in flight together), then the codes
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        const int v = v0 + tid + 256 * j;
        hv[j] = make_uint4(0u, 0u, 0u, 0u);
        if (v < nv) {
          if constexpr (F32IN) {
            const float4* hp =
                reinterpret_cast<const float4*>(static_cast<const float*>(h) + static_cast<size_t>(row) * D) + 2 * v;
            const float4 a = hp[0], b = hp[1];
            hv[j] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                               pack_bf16x2(b.z, b.w));
          } else {
            hv[j] = reinterpret_cast<const uint4*>(static_cast<const bf16*>(h) + static_cast<size_t>(row) * D)[v];
          }
        }
      }
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        const int v = v0 + tid + 256 * j;
        if (v < nv) reinterpret_cast<uint32_t*>(q_out + static_cast<size_t>(row) * (D / 2))[v] = quantize8(hv[j], inv);
      }
    }
    __syncthreads();   // every thread has read amax before it is replaced
    if (tid == 0) scale_io[row] = sc;
  }
}

// Codes and scales of rows of a bf16 matrix u [N, D] whose per-row maxima of
// |u| come in `parts` partial maxima per row (rowmax [N, parts], e.g. one per
// 256-column tile from the GEMM that wrote u). Rows are taken from the last
// to the first, so the rows written last (still in L2) are read first.
__global__ void __launch_bounds__(256)
quant_rowmax_kernel(const void* __restrict__ u, const float* __restrict__ rowmax, int N, int D, int parts,
                    uint8_t* __restrict__ q_out, float* __restrict__ scale_out, float qmax) {
  constexpr int VPT = 8;
  const int tid = threadIdx.x;
  const int nv = D / 8;
  grid_dep_wait();   // u and its row maxima come from the previous kernel
  for (int k = blockIdx.x; k < N; k += gridDim.x) {
    const int row = N - 1 - k;
    float amax = 0.f;
    for (int p = 0; p < parts; ++p) amax = fmaxf(amax, rowmax[static_cast<size_t>(row) * parts + p]);
    float inv, sc;
    inv_and_scale(amax, qmax, inv, sc);
    for (int v0 = 0; v0 < nv; v0 += 256 * VPT) {
      uint4 hv[VPT];
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        const int v = v0 + tid + 256 * j;
        hv[j] = make_uint4(0u, 0u, 0u, 0u);
        if (v < nv) hv[j] = reinterpret_cast<const uint4*>(static_cast<const bf16*>(u) + static_cast<size_t>(row) * D)[v];
      }
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        const int v = v0 + tid + 256 * j;
        if (v < nv) reinterpret_cast<uint32_t*>(q_out + static_cast<size_t>(row) * (D / 2))[v] = quantize8(hv[j], inv);
      }
    }
    if (tid == 0) scale_out[row] = sc;
  }
}

}  // namespace respin
