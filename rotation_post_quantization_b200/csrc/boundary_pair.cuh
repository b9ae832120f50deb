// Pair boundary kernel: the stored subspace form of the basis fix (one D x r
// basis Q and one r x r transform M = R_sub - I per boundary, the ReSpinQuant
// explainers' zh page §2.2 steps 1-3, row convention) fused with per-token
// INT4 / INT3 quantization (zh §3-§4):
//   y = residual Q ; z = y M^T ; h = (residual + x) + z Q^T   (fp32)
//   h' = bf16(h) ; amax = max|h'| ; inv = qmax/amax ; q = rint(h' inv)
//
// Design (B200; clusters of CS = 2 CTAs (pairs) or 4, 8 warps, two CTAs per
// SM):
//  * The CTAs of a cluster split the D columns: CTA c owns the DC = D/CS
//    columns [c DC, (c+1) DC) of every token; warp w owns DC/8 of them
//    (NB blocks of 64) in every phase, so each shared-memory block is private
//    to one warp, which refills it as soon as it is done with it. Pairs serve
//    most calls; clusters of 4 halve each CTA's chain for short calls.
//  * A round is one tile of T <= 16 tokens (one m16 tile; the host picks T so
//    that every pair gets the same number of rounds). Each CTA keeps about
//    110 KB of shared memory and at most 128 registers per thread, so two
//    CTAs (of two different pairs) share an SM: 148 pairs run at once, 2048
//    tokens are one round, and the phases of one CTA (tensor-core work, the
//    peer exchanges, waits on copies) overlap those of the other.
//  * The residual tile (16 rows x DC, 2-D tensor copies of 64-column x
//    16-row boxes, 128-byte swizzle) has one buffer; h' is written back over
//    it. The next round's residual is fetched into L2 ahead of time (tensor
//    prefetch) and copied into the buffer once this round's codes are
//    written. x goes through two slots of one 64-column block per warp:
//    slot 0 receives the first block of a round during the previous round,
//    slot 1 (whose bytes hold the partial sums of y between the two
//    products) the second block once y is reduced.
//  * Both products run on mma.sync m16n8k16 (bf16, fp32 accumulate), tokens
//    on the M side. Q is read from global memory (L2-resident, shared by all
//    CTAs) as pre-arranged fragments, one 16-byte load per lane per fragment
//    group, one step ahead in registers: the projection's B fragments (pairs
//    along the column) and the re-projection's (pairs along r, output columns
//    permuted so that in each half-block step a lane's outputs are one
//    16-byte chunk of a row and the chunks of a quarter-warp fall in distinct
//    bank groups). z is split into bf16 hi + lo parts.
//  * The two whole-row dependencies (y needs every column, amax needs every
//    column) are exchanged by pushing this CTA's partials into every other
//    CTA's shared memory with st.async (completion counted on the receiver's
//    mbarrier, polled with a non-blocking test). Partial sums are combined in
//    rank order, so every CTA of the cluster uses the identical y and z.
//  * Every wait is bounded; after a wait gave up the CTA stores nothing more
//    and requests no further tensor copies (those in flight are waited for).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "boundary_kernels.cuh"
#include "boundary_rowtile.cuh"
#include "ptx.cuh"

namespace respin {

constexpr int kPrR = 32;          // padded rank of the pair kernel
constexpr int kPrT = 16;          // token slots per round (one m16 tile)
constexpr int kPrThreads = 256;   // 8 warps
constexpr int kPrBlockBytes = kPrT * 128;   // one 64-column block of a 16-row tile
constexpr int kPrXSlots = 2;      // x slots per warp

// Column (within a 64-column block) of output column n of re-projection n8
// tile t: lane (g, q) then owns columns 16q + 8(t/4) .. + 7 of its rows in
// tiles 4(t/4) .. 4(t/4) + 3, i.e. one 16-byte chunk per row and half block.
__host__ __device__ constexpr int pr_channel(int t, int n) {
  return 16 * (n >> 1) + 8 * (t >> 2) + 2 * (t & 3) + (n & 1);
}

template <int DC, int CS = 2>
struct PrCfg {
  static_assert(DC == 1024 || DC == 2048, "columns per CTA");
  static_assert(CS == 2 || CS == 4, "CTAs per cluster");
  static constexpr int NB = DC / 512;                          // 64-column blocks per warp
  static constexpr uint32_t kTileBytes = kPrT * DC * 2;        // one 16-row tile
  static constexpr uint32_t kXBytes = 8 * kPrXSlots * kPrBlockBytes;   // x slots of all warps
  static constexpr int YP = 40;                                // z row pitch (floats)
  static constexpr int BP = 33;                                // y / M row pitch (floats)
  static constexpr uint32_t oRes = 0;                          // residual tile (h' in place)
  static constexpr uint32_t oX = kTileBytes;                   // x slots [2][8 warps]; partial y [8][16][32] in slot 1
  // partials from the other CS - 1 CTAs: slot (src - rank - 1) mod CS
  static constexpr uint32_t oYpeer = oX + kXBytes;             // [2][CS-1][16][32] partial y
  static constexpr uint32_t oY = oYpeer + 2 * (CS - 1) * kPrT * kPrR * 4;   // [16][BP] full y
  static constexpr uint32_t oZ = oY + kPrT * BP * 4;           // [16][YP] z
  static constexpr uint32_t oM = oZ + kPrT * YP * 4;           // [32][BP] M
  static constexpr uint32_t oWamax = oM + kPrR * BP * 4;       // [8][16]
  static constexpr uint32_t oApeer = oWamax + 8 * kPrT * 4;    // [2][CS-1][16] row maxima
  static constexpr uint32_t oRinv = oApeer + 2 * (CS - 1) * kPrT * 4;   // [16]
  static constexpr uint32_t oBars = oRinv + kPrT * 4;  // rbar[8], xbar[8][2], ybar[2], abar[2]
  static constexpr uint32_t kSmem = oBars + 28 * 8 + 1024;     // + alignment slack
  static_assert(8 * kPrT * kPrR * 4 <= kXBytes / 2, "the partial y fits in the slot-1 blocks");
  static_assert(oBars % 8 == 0 && oX % 1024 == 0 && kTileBytes % 1024 == 0, "alignment");
  static_assert(2 * (kSmem + 1024) <= 228 * 1024, "two CTAs per SM");
};

// Asynchronous 8- / 4-byte stores into a peer CTA's shared memory; their bytes
// complete a transaction count on the peer's mbarrier (both addresses are
// shared::cluster addresses).
__device__ __forceinline__ void st_async_f32x2(uint32_t raddr, float a, float b, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(raddr),
               "f"(a), "f"(b), "r"(rbar)
               : "memory");
}
__device__ __forceinline__ void st_async_f32(uint32_t raddr, float a, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(raddr),
               "r"(__float_as_uint(a)), "r"(rbar)
               : "memory");
}

// tmR / tmX: bf16 [N, D] residual / x, box {64 columns, 16 rows}, 128-byte
// swizzle. Pf / Rf: the plan's projection / re-projection fragments of both
// column halves (pr_pack_frags), 8 uint4 per lane per 64-column block.
// Mg: M = R_sub - I, fp32 [32][32] row-major (zero padded).
template <int DC, bool F32OUT, int CS = 2>
__global__ void __launch_bounds__(kPrThreads, 2)
boundary_pair_kernel(const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmX,
                     const uint4* __restrict__ Pf, const uint4* __restrict__ Rf, const float* __restrict__ Mg,
                     int N, int D, int T, void* __restrict__ h_out, uint8_t* __restrict__ q_out,
                     float* __restrict__ scale_out, float qmax) {
  using C = PrCfg<DC, CS>;
  constexpr int NB = C::NB, YP = C::YP, BP = C::BP;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q4 = lane & 3;
  const uint32_t rank = cluster_ctarank();
  const int cid = static_cast<int>(cluster_id_x()), ncl = static_cast<int>(ncluster_x());
  const int ntiles = (N + T - 1) / T;
  const int rounds = cid < ntiles ? (ntiles - cid + ncl - 1) / ncl : 0;
  const int col0 = static_cast<int>(rank) * DC;
  const int b0 = warp * NB;                         // this warp's first block

  uint8_t* resp = smem + C::oRes;
  const uint32_t sRes = base + C::oRes;
  // slot s of warp w at oX + (8 s + w) * kPrBlockBytes
  uint8_t* xslots = smem + C::oX + warp * kPrBlockBytes;
  const uint32_t sX = base + C::oX + warp * kPrBlockBytes;
  float* ypart = reinterpret_cast<float*>(smem + C::oX + 8 * kPrBlockBytes);
  const float* ypeer = reinterpret_cast<const float*>(smem + C::oYpeer);
  float* ybuf = reinterpret_cast<float*>(smem + C::oY);
  float* zbuf = reinterpret_cast<float*>(smem + C::oZ);
  float* msm = reinterpret_cast<float*>(smem + C::oM);
  float* wamax = reinterpret_cast<float*>(smem + C::oWamax);
  const float* apeer = reinterpret_cast<const float*>(smem + C::oApeer);
  float* rowinv = reinterpret_cast<float*>(smem + C::oRinv);
  const uint32_t bars = base + C::oBars;
  const uint32_t rbar = bars + 8 * warp;
  auto xbar = [&](int s) { return bars + 64 + 16 * warp + 8 * s; };
  auto ybar = [&](int p) { return bars + 192 + 8 * p; };
  auto abar = [&](int p) { return bars + 208 + 8 * p; };
  const uint4* pf = Pf + static_cast<size_t>(rank) * (DC / 64) * 8 * 32 + lane;   // this half's fragments
  const uint4* rf = Rf + static_cast<size_t>(rank) * (DC / 64) * 8 * 32 + lane;

  if (lane == 0) {
    mbar_init(rbar, 1);
    mbar_init(xbar(0), 1);
    mbar_init(xbar(1), 1);
    if (warp == 0)
      for (int p = 0; p < 2; ++p) { mbar_init(ybar(p), 1); mbar_init(abar(p), 1); }
    fence_mbarrier_init();
    if (warp == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(&tmR) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(&tmX) : "memory");
    }
  }
  __syncthreads();
  // the peer may push into this CTA only after its barriers exist; the
  // matching wait precedes this CTA's first push
  cluster_arrive();

  // Tensor copies of this warp's blocks. Lane j < NB copies residual block
  // j; lane s < 2 copies the x block of ring slot s. Completed phases are
  // counted per barrier for the parity of the next wait.
  bool res_pend = false, x_pend0 = false, x_pend1 = false;
  uint32_t res_done = 0, x_done0 = 0, x_done1 = 0;
  // residual and x are read once and h' is not read again by this launch:
  // their L2 lines go first, so the codes and the next GEMM's weights stay
  const uint64_t pol_ef = l2_policy_evict_first();
  auto issue_res = [&](int r) {
    if (lane == 0) mbar_arrive_expect_tx(rbar, NB * kPrBlockBytes);
    __syncwarp();
    if (lane < NB)
      tma_load_2d_hint(sRes + (b0 + lane) * kPrBlockBytes, &tmR, col0 + (b0 + lane) * 64, (cid + r * ncl) * T, rbar,
                       pol_ef);
    res_pend = true;
  };
  auto issue_x = [&](int r, int j) {   // block j of round r into slot j & 1
    const int s = j & 1;
    if (lane == s) {
      mbar_arrive_expect_tx(xbar(s), kPrBlockBytes);
      tma_load_2d_hint(sX + s * 8 * kPrBlockBytes, &tmX, col0 + (b0 + j) * 64, (cid + r * ncl) * T, xbar(s), pol_ef);
    }
    if (s) x_pend1 = true; else x_pend0 = true;
  };
  auto prefetch = [&](const CUtensorMap* tm, int r) {   // round r's blocks of this warp into L2
    if (lane < NB) tma_prefetch_2d(tm, col0 + (b0 + lane) * 64, (cid + r * ncl) * T);
  };
  if (rounds > 0) { issue_res(0); issue_x(0, 0); }
  for (int i = tid; i < kPrR * kPrR; i += kPrThreads) msm[(i >> 5) * BP + (i & 31)] = __ldg(Mg + i);

  const int arow = (lane & 7) + 8 * ((lane >> 3) & 1);   // ldmatrix A row
  bool ok = true;
  bool cluster_waited = false;
  for (int r = 0; r < rounds; ++r) {
    const int tile = cid + r * ncl, row0 = tile * T;
    const int par = r & 1;
    const uint32_t upar = static_cast<uint32_t>(r >> 1) & 1u;
    if (tid == 0) {
      mbar_arrive_expect_tx(ybar(par), (CS - 1) * kPrT * kPrR * 4);
      mbar_arrive_expect_tx(abar(par), (CS - 1) * kPrT * 4);
    }

    // ---- projection: this warp's partial y over its NB blocks
    {
      uint4 fr[2][8];
#pragma unroll
      for (int i = 0; i < 8; ++i) fr[0][i] = __ldg(pf + (b0 * 8 + i) * 32);
      if (res_pend) {
        ok = mbar_wait(rbar, res_done & 1u, kSitePairLoad) && ok;
        ++res_done;
        res_pend = false;
      }
      ok = __all_sync(0xffffffffu, ok);
      if (ok) prefetch(&tmX, r);   // the rest of this round's x, behind the residual
      float acc1[4][4];
#pragma unroll
      for (int p = 0; p < 4; ++p) acc1[p][0] = acc1[p][1] = acc1[p][2] = acc1[p][3] = 0.f;
#pragma unroll
      for (int j = 0; j < NB; ++j) {
        if (j + 1 < NB) {
#pragma unroll
          for (int i = 0; i < 8; ++i) fr[(j + 1) & 1][i] = __ldg(pf + ((b0 + j + 1) * 8 + i) * 32);
        }
        const uint32_t blk = sRes + (b0 + j) * kPrBlockBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t a[4];
          ldmatrix_x4(blk + sw128(arow, 2 * kk + (lane >> 4)), a[0], a[1], a[2], a[3]);
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const uint4& v = fr[j & 1][kk * 2 + (p >> 1)];
            mma_bf16_16816(acc1[p], a, u4c(v, 2 * (p & 1)), u4c(v, 2 * (p & 1) + 1));
          }
        }
      }
      // partial y of this warp (into the slot-1 blocks, idle between the
      // rounds' x): element (tok, r) at tok * 32 + (r ^ 8 (tok & 3))
      float* yp = ypart + warp * kPrT * kPrR;
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const int c = 8 * (p ^ (g & 3)) + 2 * q4;
        *reinterpret_cast<float2*>(yp + g * kPrR + c) = make_float2(acc1[p][0], acc1[p][1]);
        *reinterpret_cast<float2*>(yp + (g + 8) * kPrR + c) = make_float2(acc1[p][2], acc1[p][3]);
      }
    }
    // first re-projection fragments load while y is exchanged
    uint4 fnext[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) fnext[i] = __ldg(rf + (b0 * 8 + i) * 32);
    ok = __syncthreads_and(ok) != 0;
    if (ok && r + 1 < rounds) prefetch(&tmR, r + 1);

    // ---- y over the cluster: thread t owns token t/16, r = 2 (t%16), +1;
    // its partial (warps summed in order) goes to every other CTA
    const int yt = tid >> 4, yc = 2 * (tid & 15);
    {
      float2 ys = make_float2(0.f, 0.f);
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float2 v =
            *reinterpret_cast<const float2*>(ypart + (w * kPrT + yt) * kPrR + (yc ^ (8 * (yt & 3))));
        ys.x += v.x;
        ys.y += v.y;
      }
      // the ring is refilled by tensor copies once every thread is past here
      fence_proxy_async_smem();
      if (!cluster_waited) { cluster_wait(); cluster_waited = true; }
#pragma unroll
      for (int p = 1; p < CS; ++p) {   // to CTA rank + p, into its slot CS - 1 - p
        const uint32_t dst = (rank + p) % CS;
        const uint32_t yslot = base + C::oYpeer + (((par * (CS - 1) + (CS - 1 - p)) * kPrT + yt) * kPrR + yc) * 4;
        st_async_f32x2(map_to_rank(yslot, dst), ys.x, ys.y, map_to_rank(ybar(par), dst));
      }
      ok = mbar_spin_cluster(ybar(par), upar, kSitePairPeer) && ok;
      // y = sum of the CS partials in rank order
      float2 y = make_float2(0.f, 0.f);
#pragma unroll
      for (int src = 0; src < CS; ++src) {
        const int sl = (src - static_cast<int>(rank) - 1 + CS) % CS;   // sender's slot here
        const float2 v = src == static_cast<int>(rank)
                             ? ys
                             : *reinterpret_cast<const float2*>(ypeer + ((par * (CS - 1) + sl) * kPrT + yt) * kPrR + yc);
        if (src == 0) y = v; else { y.x += v.x; y.y += v.y; }
      }
      ybuf[yt * BP + yc] = y.x;
      ybuf[yt * BP + yc + 1] = y.y;
    }
    __syncwarp();   // the 16 threads of a token share a warp
    {
      // z[t][i] = sum_j y[t][j] M[i][j] (j in order), i = yc, yc + 1
      float z0 = 0.f, z1 = 0.f;
      const float* yrow = ybuf + yt * BP;
#pragma unroll
      for (int jj = 0; jj < kPrR; ++jj) {
        const float yv = yrow[jj];
        z0 = __fmaf_rn(yv, msm[yc * BP + jj], z0);
        z1 = __fmaf_rn(yv, msm[(yc + 1) * BP + jj], z1);
      }
      *reinterpret_cast<float2*>(zbuf + yt * YP + yc) = make_float2(z0, z1);
    }
    ok = __syncthreads_and(ok) != 0;
    if (ok) issue_x(r, 1);   // slot 1 held the partial y

    // ---- re-projection: h = (residual + x) + z Q^T over this warp's blocks,
    // in half blocks (n8 tiles 4c .. 4c + 3, lane chunk 2 q + c of each row)
    uint32_t ahi[2][4], alo[2][4];
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      const float* z0 = zbuf + g * YP + 16 * kk + 2 * q4;
      split_bf16x2(*reinterpret_cast<const float2*>(z0), ahi[kk][0], alo[kk][0]);
      split_bf16x2(*reinterpret_cast<const float2*>(z0 + 8 * YP), ahi[kk][1], alo[kk][1]);
      split_bf16x2(*reinterpret_cast<const float2*>(z0 + 8), ahi[kk][2], alo[kk][2]);
      split_bf16x2(*reinterpret_cast<const float2*>(z0 + 8 * YP + 8), ahi[kk][3], alo[kk][3]);
    }
    uint32_t amax2[2] = {0u, 0u};   // running max |h'| (bf16x2) of rows g and g + 8
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const int b = b0 + j, s = j & 1;
      if (s ? x_pend1 : x_pend0) {
        uint32_t& done = s ? x_done1 : x_done0;
        ok = mbar_wait(xbar(s), done & 1u, kSitePairLoad) && ok;
        ++done;
        if (s) x_pend1 = false; else x_pend0 = false;
      }
      ok = __all_sync(0xffffffffu, ok);
      uint8_t* rblk = resp + b * kPrBlockBytes;
      const uint8_t* xblk = xslots + s * 8 * kPrBlockBytes;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint4 fcur[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) fcur[i] = fnext[i];
        if (c == 0 || j + 1 < NB) {   // next half's fragments
          const int nb = c == 0 ? b : b + 1, nc = c ^ 1;
#pragma unroll
          for (int i = 0; i < 4; ++i) fnext[i] = __ldg(rf + (nb * 8 + 4 * nc + i) * 32);
        }
        float acc[4][4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const uint32_t bb0 = u4c(fcur[t], 2 * kk), bb1 = u4c(fcur[t], 2 * kk + 1);
            mma_bf16_16816(acc[t], ahi[kk], bb0, bb1);
            mma_bf16_16816(acc[t], alo[kk], bb0, bb1);
          }
        }
        // epilogue: rows g and g + 8, columns 16 q + 8 c .. + 7 (word i from
        // tile 4 c + i)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int row = g + 8 * hh;
          const bool store = ok && row < T && row0 + row < N;
          const uint32_t so = sw128(row, 2 * q4 + c);
          const uint4 rv = *reinterpret_cast<const uint4*>(rblk + so);
          const uint4 xv = *reinterpret_cast<const uint4*>(xblk + so);
          const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w}, xw[4] = {xv.x, xv.y, xv.z, xv.w};
          uint32_t hw[4];
          float2 hf[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 sum = add_f32x2(bf16x2_to_f32x2(rw[i]), bf16x2_to_f32x2(xw[i]));
            hf[i] = add_f32x2(sum, make_float2(acc[i][2 * hh], acc[i][2 * hh + 1]));
            hw[i] = pack_bf16x2(hf[i].x, hf[i].y);
            amax2[hh] = absmax_bf16x2(amax2[hh], hw[i]);
          }
          const uint4 hv = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(rblk + so) = hv;
          if (store && h_out != nullptr) {
            const size_t gi = static_cast<size_t>(row0 + row) * D + col0 + b * 64 + 16 * q4 + 8 * c;
            if constexpr (F32OUT) {
              float4* hp = reinterpret_cast<float4*>(static_cast<float*>(h_out) + gi);
              hp[0] = make_float4(hf[0].x, hf[0].y, hf[1].x, hf[1].y);
              hp[1] = make_float4(hf[2].x, hf[2].y, hf[3].x, hf[3].y);
            } else {
              st_global_v4_hint(static_cast<bf16*>(h_out) + gi, hv, pol_ef);
            }
          }
        }
      }
      // slot s is read: block j + 2's x, or after the round's last use of
      // slot 0 the first block of the next round
      fence_proxy_async_smem();
      __syncwarp();
      if (ok && j + 2 < NB) issue_x(r, j + 2);
      else if (ok && s == 0 && r + 1 < rounds) issue_x(r + 1, 0);
    }

    // ---- row amax over the warps, then over the cluster
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float m = fmaxf(bf16_lo_f32(amax2[hh]), bf16_hi_f32(amax2[hh]));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      if (q4 == 0) wamax[warp * kPrT + g + 8 * hh] = m;
    }
    ok = __syncthreads_and(ok) != 0;
    if (tid < kPrT) {
      float m = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) m = fmaxf(m, wamax[w * kPrT + tid]);
#pragma unroll
      for (int p = 1; p < CS; ++p) {
        const uint32_t dst = (rank + p) % CS;
        const uint32_t aslot = base + C::oApeer + ((par * (CS - 1) + (CS - 1 - p)) * kPrT + tid) * 4;
        st_async_f32(map_to_rank(aslot, dst), m, map_to_rank(abar(par), dst));
      }
      ok = mbar_spin_cluster(abar(par), upar, kSitePairPeer) && ok;
#pragma unroll
      for (int sl = 0; sl < CS - 1; ++sl) m = fmaxf(m, apeer[(par * (CS - 1) + sl) * kPrT + tid]);
      float inv, sc;
      inv_and_scale(m, qmax, inv, sc);
      rowinv[tid] = inv;
      if (ok && rank == 0 && tid < T && row0 + tid < N) scale_out[row0 + tid] = sc;
    }
    ok = __syncthreads_and(ok) != 0;

    // ---- codes of this warp's columns from h' in shared memory: lane l of
    // step s takes chunk (32 s + l) of the warp's 16 rows x 8 NB chunks
    constexpr int kRowChunks = 8 * NB;
#pragma unroll 4
    for (int s = 0; s < kPrT * kRowChunks / 32; ++s) {
      const int k = 32 * s + lane;
      const int tok = k / kRowChunks, cc = k % kRowChunks;
      const int b = b0 + (cc >> 3);
      const uint4 hv = *reinterpret_cast<const uint4*>(resp + b * kPrBlockBytes + sw128(tok, cc & 7));
      const uint32_t code = quantize8_x2(hv, rowinv[tok]);
      if (ok && tok < T && row0 + tok < N)
        reinterpret_cast<uint32_t*>(q_out)[(static_cast<size_t>(row0 + tok) * D + col0 + 64 * b + 8 * (cc & 7)) / 8] =
            code;
    }
    // this warp's residual blocks are read: the next round's residual (from L2)
    fence_proxy_async_smem();
    __syncwarp();
    if (ok && r + 1 < rounds) issue_res(r + 1);
  }
  if (!cluster_waited) cluster_wait();   // no round: close the set-up barrier phase
  // no CTA may leave while another can still push into it
  cluster_sync();
}

// Host side: the plan's Q fragments for boundary_pair_kernel<D/2>. Qb: bf16
// bits of Q, [D][rr] row-major (rr <= 32, zero padded to 32 here). For column
// half c and its 64-column block b (columns d0 = c D/2 + 64 b ..), lane
// (g, q) gets 8 uint4 per block:
//   projection (Pf): register i = 2 (4 kk + p) + e holds (Q[d][n], Q[d+1][n])
//     with d = d0 + 16 kk + 2q + 8e, n = 8p + g;
//   re-projection (Rf): register i = 2 (2 t + kk) + e holds (Q[d][m], Q[d][m+1])
//     with d = d0 + pr_channel(t, g), m = 16 kk + 2q + 8e (uint4 t is tile t);
// stored at uint4 ((c D/128 + b) 8 + i/4) 32 + lane, component i % 4.
inline void pr_pack_frags(const uint16_t* Qb, int D, int rr, uint32_t* Pf, uint32_t* Rf) {
  auto q = [&](int d, int r) -> uint32_t {
    return r < rr ? Qb[static_cast<size_t>(d) * rr + r] : 0u;
  };
  const int nblk = D / 64;   // blocks of both halves, in order
  for (int bb = 0; bb < nblk; ++bb)
    for (int lane = 0; lane < 32; ++lane) {
      const int g = lane >> 2, qq = lane & 3;
      const int d0 = 64 * bb;
      for (int i = 0; i < 32; ++i) {
        const size_t idx = ((static_cast<size_t>(bb) * 8 + i / 4) * 32 + lane) * 4 + i % 4;
        {
          const int e = i & 1, p = (i >> 1) & 3, kk = i >> 3;
          const int d = d0 + 16 * kk + 2 * qq + 8 * e, n = 8 * p + g;
          Pf[idx] = q(d, n) | (q(d + 1, n) << 16);
        }
        {
          const int e = i & 1, kk = (i >> 1) & 1, t = i >> 2;
          const int d = d0 + pr_channel(t, g), m = 16 * kk + 2 * qq + 8 * e;
          Rf[idx] = q(d, m) | (q(d, m + 1) << 16);
        }
      }
    }
}

}  // namespace respin
