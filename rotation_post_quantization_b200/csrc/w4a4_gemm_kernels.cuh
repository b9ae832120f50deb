// W4A4 GEMM on the 5th-generation tensor cores (tcgen05, kind::i8).
//
//   acc[n, o] = sum_k a[n, k] w[o, k]            (exact, int32 in TMEM)
//   out[n, o] = bf16((float(acc) * sa[n]) * sw[o])
//
// W4A4 linear layers of the ReSpinQuant explainers (zh §3-§4, fr §4): the
// rotations are fused into the weights offline, so at inference every linear
// is a plain low-bit GEMM.
//
// tcgen05 has no plain signed-int4 operand kind, so INT4 is widened to INT8 in
// shared memory by producer warps. Two choices keep that cheap:
//  * nibble-high widening: a byte holding code c in its high nibble and zero in
//    its low nibble is the int8 value 16 c, so widening is one AND (high
//    nibbles) or one SHIFT + AND (low nibbles) per 4 bytes, with no sign
//    extension. Both operands are widened this way; the MMA computes 256 acc
//    exactly (|256 acc| <= 256 * 64 * K < 2^31 for K <= 65536) and the
//    epilogue shifts it back.
//  * K permutation: the even-indexed codes of a 16-byte packed chunk go to one
//    16-byte K slot and the odd-indexed codes to the next. A and B use the same
//    permutation, so the dot product over K is unchanged and no byte
//    interleaving is needed.
//
// Structure (persistent, warp-specialised, one CTA per SM):
//  * 1 TMA warp brings each packed K block (A: 128 rows x 64 bytes, B: 256 rows
//    x 64 bytes) into a 3-stage packed ring with two 2-D tensor copies (rows
//    past N or O arrive as zeros). Loading through TMA keeps the packed bytes
//    off the LSU data pipe, where sector-granular global loads cost 4x the
//    wavefronts of the shared-memory reads that replace them;
//  * 8 producer warps read the packed chunks (conflict-free 16-byte loads),
//    widen them and store them into a 3-stage shared-memory ring in the
//    128-byte-swizzled K-major canonical layout (128 tokens x 256 channels x
//    128 K per stage, 48 KB);
//  * 1 MMA warp: one thread issues 4 MMAs (M=128, N=256, K=32) per stage and
//    commits to the stage's empty barrier; accumulators alternate between two
//    256-column TMEM buffers;
//  * 4 epilogue warps drain the other TMEM buffer (tcgen05.ld), apply the two
//    scales and store bf16, overlapping the next tile's main loop.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace respin {

constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 128;                 // int8 K per stage (64 packed bytes per row)
constexpr int kGemmStages = 3;               // widened (int8) stages
constexpr int kGemmPStages = 3;              // packed (int4) stages
constexpr int kGemmProducerWarps = 8;
constexpr int kGemmEpilogueWarps = 4;
constexpr int kGemmMmaWarp = kGemmProducerWarps;                 // warp 8
constexpr int kGemmEpiWarp0 = kGemmProducerWarps + 1;            // warps 9..12
constexpr int kGemmTmaWarp = kGemmEpiWarp0 + kGemmEpilogueWarps;  // warp 13
constexpr int kGemmThreads = (kGemmTmaWarp + 1) * 32;
constexpr int kGemmAStage = kGemmBM * kGemmBK;  // 16 KB
constexpr int kGemmBStage = kGemmBN * kGemmBK;  // 32 KB
constexpr int kGemmStageBytes = kGemmAStage + kGemmBStage;
constexpr int kGemmPAStage = kGemmBM * kGemmBK / 2;   // 8 KB packed A
constexpr int kGemmPStageBytes = (kGemmBM + kGemmBN) * kGemmBK / 2;  // 24 KB
constexpr int kGemmChunks = (kGemmBM + kGemmBN) * (kGemmBK / 32);  // 16-byte packed chunks
constexpr int kGemmChunksPerThread = kGemmChunks / (kGemmProducerWarps * 32);
constexpr int kGemmSmemBytes =
    kGemmStages * kGemmStageBytes + kGemmPStages * kGemmPStageBytes + 1024 + 256;
static_assert(kGemmChunks % (kGemmProducerWarps * 32) == 0, "chunk split");

// tmA: uint8 [N, K/2] box {64, 128}; tmB: uint8 [O, K/2] box {64, 256}
// (inner dimension first), no swizzle, out-of-range elements zero filled.
template <bool I32OUT>
__global__ void __launch_bounds__(kGemmThreads, 1)
w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const float* __restrict__ sa, const float* __restrict__ sw, int N, int K,
                 int O, void* __restrict__ out) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t pbase = base + kGemmStages * kGemmStageBytes;   // packed ring
  const uint32_t bars = pbase + kGemmPStages * kGemmPStageBytes;
  const uint32_t full0 = bars, empty0 = bars + 8 * kGemmStages;
  const uint32_t pfull0 = bars + 16 * kGemmStages;
  const uint32_t pempty0 = pfull0 + 8 * kGemmPStages;
  const uint32_t afull0 = pempty0 + 8 * kGemmPStages;     // accumulator buffer b full: afull0 + 8b
  const uint32_t aempty0 = afull0 + 16;                    // accumulator buffer b drained
  const uint32_t tslot = aempty0 + 16;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KB = K / kGemmBK;
  const int mtiles = (N + kGemmBM - 1) / kGemmBM;
  const int ntiles = (O + kGemmBN - 1) / kGemmBN;
  const int tiles = mtiles * ntiles;

  if (tid == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(full0 + 8 * s, kGemmProducerWarps * 32);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int s = 0; s < kGemmPStages; ++s) {
      mbar_init(pfull0 + 8 * s, 1);
      mbar_init(pempty0 + 8 * s, kGemmProducerWarps * 32);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(afull0 + 8 * b, 1);
      mbar_init(aempty0 + 8 * b, kGemmEpilogueWarps * 32);
    }
    fence_mbarrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + (tslot - base));

  if (warp < kGemmProducerWarps) {
    // ------------------------------------------------ producers: widen packed -> int8
    bool ok = true;
    int kstep = 0;  // running k-block counter over all tiles (selects the stages)
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      for (int kb = 0; kb < KB; ++kb, ++kstep) {
        const int ps = kstep % kGemmPStages, s = kstep % kGemmStages;
        if (ok) ok = mbar_wait(pfull0 + 8 * ps, (kstep / kGemmPStages) & 1, kSiteGemmPackedFull);
        const uint8_t* pk = smem + (pbase - base) + ps * kGemmPStageBytes;
        uint4 b[kGemmChunksPerThread];
#pragma unroll
        for (int j = 0; j < kGemmChunksPerThread; ++j)   // chunk q = row*4 + c, 16 bytes each
          b[j] = *reinterpret_cast<const uint4*>(pk + (tid + j * kGemmProducerWarps * 32) * 16);
        if (ok) ok = mbar_wait(empty0 + 8 * s, ((kstep / kGemmStages) & 1) ^ 1, kSiteGemmEmpty);
        uint8_t* sA = smem + s * kGemmStageBytes;
#pragma unroll
        for (int j = 0; j < kGemmChunksPerThread; ++j) {
          const int q = tid + j * kGemmProducerWarps * 32;
          const bool is_a = q < kGemmBM * 4;
          const int qq = is_a ? q : q - kGemmBM * 4;
          const int row = qq >> 2, c = qq & 3;
          uint8_t* rowp = sA + (is_a ? 0 : kGemmAStage) + (row >> 3) * 1024 + (row & 7) * 128;
          const uint4 p = b[j];
          const uint4 lo = make_uint4((p.x << 4) & 0xF0F0F0F0u, (p.y << 4) & 0xF0F0F0F0u,
                                      (p.z << 4) & 0xF0F0F0F0u, (p.w << 4) & 0xF0F0F0F0u);
          const uint4 hi = make_uint4(p.x & 0xF0F0F0F0u, p.y & 0xF0F0F0F0u, p.z & 0xF0F0F0F0u,
                                      p.w & 0xF0F0F0F0u);
          *reinterpret_cast<uint4*>(rowp + (((2 * c) ^ (row & 7)) << 4)) = lo;
          *reinterpret_cast<uint4*>(rowp + (((2 * c + 1) ^ (row & 7)) << 4)) = hi;
        }
        // Widened stage -> MMA (async proxy reads): proxy fence, then signal.
        // The packed stage is released only now, after its bytes were
        // consumed, so the next TMA refill (async-proxy write) cannot land
        // before these shared-memory reads retired.
        fence_proxy_async_smem();
        mbar_arrive(full0 + 8 * s);
        mbar_arrive(pempty0 + 8 * ps);
      }
    }
  } else if (warp == kGemmTmaWarp) {
    // ------------------------------------------------ TMA warp: packed K blocks
    bool ok = true;
    int kstep = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      const int m0 = (t / ntiles) * kGemmBM, n0 = (t % ntiles) * kGemmBN;
      for (int kb = 0; kb < KB; ++kb, ++kstep) {
        const int ps = kstep % kGemmPStages;
        if (ok) ok = mbar_wait(pempty0 + 8 * ps, ((kstep / kGemmPStages) & 1) ^ 1, kSiteGemmPackedEmpty);
        if (lane == 0) {
          const uint32_t dst = pbase + ps * kGemmPStageBytes;
          mbar_arrive_expect_tx(pfull0 + 8 * ps, kGemmPStageBytes);
          tma_load_2d(dst, &tmA, kb * (kGemmBK / 2), m0, pfull0 + 8 * ps);
          tma_load_2d(dst + kGemmPAStage, &tmB, kb * (kGemmBK / 2), n0, pfull0 + 8 * ps);
        }
        __syncwarp();
      }
    }
  } else if (warp == kGemmMmaWarp) {
    // ------------------------------------------------ MMA issuer (one warp)
    constexpr uint32_t idesc = umma_idesc_s8(kGemmBM, kGemmBN);
    bool ok = true;
    int kstep = 0, local = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++local) {
      const int ab = local & 1;
      // wait until the epilogue drained this accumulator buffer (two tiles ago)
      if (ok) ok = mbar_wait(aempty0 + 8 * ab, ((local >> 1) & 1) ^ 1, kSiteGemmAccum);
      tc_fence_after();
      const uint32_t dtm = tmem + ab * kGemmBN;
      for (int kb = 0; kb < KB; ++kb, ++kstep) {
        const int s = kstep % kGemmStages;
        if (ok) ok = mbar_wait(full0 + 8 * s, (kstep / kGemmStages) & 1, kSiteGemmFull);
        tc_fence_after();
        if (lane == 0 && ok) {
          const uint32_t a_addr = base + s * kGemmStageBytes;
          const uint32_t b_addr = a_addr + kGemmAStage;
#pragma unroll
          for (int k = 0; k < kGemmBK / 32; ++k)
            tc_mma_i8(dtm, umma_desc_sw128(a_addr + 32 * k), umma_desc_sw128(b_addr + 32 * k), idesc,
                      (kb | k) != 0 ? 1u : 0u);
          tc_commit(empty0 + 8 * s);
        }
        __syncwarp();
      }
      if (lane == 0) tc_commit(afull0 + 8 * ab);
      __syncwarp();
    }
  } else {
    // ------------------------------------------------ epilogue warps
    const int ew = warp - kGemmEpiWarp0;   // TMEM lane quadrant of this warp
    const int quad = warp & 3;             // hardware rule: warp w reads lanes 32*(w%4)..
    (void)ew;
    bool ok = true;
    int local = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++local) {
      const int ab = local & 1;
      const int m0 = (t / ntiles) * kGemmBM, n0 = (t % ntiles) * kGemmBN;
      if (ok) ok = mbar_wait(afull0 + 8 * ab, (local >> 1) & 1, kSiteGemmAccum);
      tc_fence_after();
      const int row = m0 + quad * 32 + lane;
      const float sa_r = (row < N && !I32OUT) ? __ldg(sa + row) : 0.f;
#pragma unroll 1
      for (int cc = 0; cc < kGemmBN / 32; ++cc) {
        const int colb = n0 + cc * 32;
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + ab * kGemmBN + cc * 32, v);
        tmem_wait_ld();
        if (!ok || row >= N) continue;
        if constexpr (I32OUT) {
          int32_t* op = static_cast<int32_t*>(out) + static_cast<size_t>(row) * O + colb;
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            if (colb + e >= O) break;
            *reinterpret_cast<int4*>(op + e) =
                make_int4(static_cast<int32_t>(v[e]) >> 8, static_cast<int32_t>(v[e + 1]) >> 8,
                          static_cast<int32_t>(v[e + 2]) >> 8, static_cast<int32_t>(v[e + 3]) >> 8);
          }
        } else {
          __nv_bfloat16* op = static_cast<__nv_bfloat16*>(out) + static_cast<size_t>(row) * O + colb;
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            if (colb + e >= O) break;
            const float4 w0 = __ldg(reinterpret_cast<const float4*>(sw + colb + e));
            const float4 w1 = __ldg(reinterpret_cast<const float4*>(sw + colb + e + 4));
            const float ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            uint32_t w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int e0 = e + 2 * u;
              const float f0 = __fmul_rn(
                  __fmul_rn(static_cast<float>(static_cast<int32_t>(v[e0]) >> 8), sa_r), ws[2 * u]);
              const float f1 = __fmul_rn(
                  __fmul_rn(static_cast<float>(static_cast<int32_t>(v[e0 + 1]) >> 8), sa_r), ws[2 * u + 1]);
              w[u] = pack_bf16x2(f0, f1);
            }
            *reinterpret_cast<uint4*>(op + e) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      // hand the accumulator buffer back to the MMA warp
      tc_fence_before();
      mbar_arrive(aempty0 + 8 * ab);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace respin
