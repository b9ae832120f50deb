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
// Tiles: 128 tokens x 256 channels x 128 K per stage, 4-stage shared-memory
// ring (48 KB per stage) in the 128-byte-swizzled K-major canonical layout,
// mbarrier full/empty handshake, one thread issues 4 MMAs (K = 32 each) per
// stage and commits to the stage's empty barrier.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace respin {

constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 128;                 // int8 K per stage (64 packed bytes per row)
constexpr int kGemmStages = 4;
constexpr int kGemmProducerWarps = 8;
constexpr int kGemmThreads = (kGemmProducerWarps + 1) * 32;
constexpr int kGemmAStage = kGemmBM * kGemmBK;  // 16 KB
constexpr int kGemmBStage = kGemmBN * kGemmBK;  // 32 KB
constexpr int kGemmStageBytes = kGemmAStage + kGemmBStage;
constexpr int kGemmChunks = (kGemmBM + kGemmBN) * (kGemmBK / 32);  // 16-byte packed chunks
constexpr int kGemmChunksPerThread = kGemmChunks / (kGemmProducerWarps * 32);
constexpr int kGemmSmemBytes = kGemmStages * kGemmStageBytes + 1024 + 128;
static_assert(kGemmChunks % (kGemmProducerWarps * 32) == 0, "chunk split");

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <bool I32OUT>
__global__ void __launch_bounds__(kGemmThreads, 1)
w4a4_gemm_kernel(const uint8_t* __restrict__ qa, const float* __restrict__ sa,
                 const uint8_t* __restrict__ qw, const float* __restrict__ sw, int N, int K,
                 int O, void* __restrict__ out) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t bars = base + kGemmStages * kGemmStageBytes;
  const uint32_t full0 = bars, empty0 = bars + 8 * kGemmStages;
  const uint32_t accum = bars + 16 * kGemmStages;
  const uint32_t tslot = accum + 8;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.y * kGemmBM, n0 = blockIdx.x * kGemmBN;
  const int KB = K / kGemmBK;
  const size_t krow = static_cast<size_t>(K) / 2;

  if (tid == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(full0 + 8 * s, kGemmProducerWarps * 32);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(accum, 1);
    fence_mbarrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + (tslot - base));

  if (warp < kGemmProducerWarps) {
    // ------------------------------------------------ producers
    // Packed chunks of the next k-block are loaded into registers while the
    // current one is widened and stored (two register buffers, K loop
    // unrolled by two so that both stay in registers).
    uint4 buf0[kGemmChunksPerThread], buf1[kGemmChunksPerThread];
    auto load = [&](uint4 (&b)[kGemmChunksPerThread], int kb) {
#pragma unroll
      for (int j = 0; j < kGemmChunksPerThread; ++j) {
        const int q = tid + j * kGemmProducerWarps * 32;
        const bool is_a = q < kGemmBM * 4;
        const int qq = is_a ? q : q - kGemmBM * 4;
        const int row = qq >> 2, c = qq & 3;
        const int grow = (is_a ? m0 : n0) + row;
        const bool valid = grow < (is_a ? N : O);
        const uint8_t* src = (is_a ? qa : qw) + static_cast<size_t>(grow) * krow + kb * 64 + c * 16;
        b[j] = valid ? ldg_nc_v4(src) : make_uint4(0u, 0u, 0u, 0u);
      }
    };
    bool ok = true;
    auto produce = [&](const uint4 (&b)[kGemmChunksPerThread], int kb) {
      const int s = kb % kGemmStages;
      if (ok) ok = mbar_wait(empty0 + 8 * s, ((kb / kGemmStages) & 1) ^ 1, kSiteGemmEmpty);
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
      fence_proxy_async_smem();
      mbar_arrive(full0 + 8 * s);
    };
    load(buf0, 0);
    for (int kb = 0; kb < KB; kb += 2) {
      if (kb + 1 < KB) load(buf1, kb + 1);
      produce(buf0, kb);
      if (kb + 1 >= KB) break;
      if (kb + 2 < KB) load(buf0, kb + 2);
      produce(buf1, kb + 1);
    }
  } else {
    // ------------------------------------------------ MMA issuer (one warp)
    constexpr uint32_t idesc = umma_idesc_s8(kGemmBM, kGemmBN);
    bool ok = true;
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % kGemmStages;
      if (ok) ok = mbar_wait(full0 + 8 * s, (kb / kGemmStages) & 1, kSiteGemmFull);
      tc_fence_after();
      if (lane == 0 && ok) {
        const uint32_t a_addr = base + s * kGemmStageBytes;
        const uint32_t b_addr = a_addr + kGemmAStage;
#pragma unroll
        for (int k = 0; k < kGemmBK / 32; ++k)
          tc_mma_i8(tmem, umma_desc_sw128(a_addr + 32 * k), umma_desc_sw128(b_addr + 32 * k), idesc,
                    (kb | k) != 0 ? 1u : 0u);
        tc_commit(empty0 + 8 * s);
      }
      __syncwarp();
    }
    if (lane == 0) tc_commit(accum);
    __syncwarp();
  }

  if (warp < kGemmProducerWarps) {
    // ------------------------------------------------ epilogue
    const bool ok = mbar_wait(accum, 0, kSiteGemmAccum);
    tc_fence_after();
    const int quad = warp & 3, half = warp >> 2;
    const int row = m0 + quad * 32 + lane;
    const float sa_r = (row < N) ? __ldg(sa + row) : 0.f;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      const int colb = n0 + half * 128 + cc * 32;
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + half * 128 + cc * 32, v);
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
          uint32_t w[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int e0 = e + 2 * u;
            const float f0 = __fmul_rn(
                __fmul_rn(static_cast<float>(static_cast<int32_t>(v[e0]) >> 8), sa_r),
                __ldg(sw + colb + e0));
            const float f1 = __fmul_rn(
                __fmul_rn(static_cast<float>(static_cast<int32_t>(v[e0 + 1]) >> 8), sa_r),
                __ldg(sw + colb + e0 + 1));
            w[u] = pack_bf16x2(f0, f1);
          }
          *reinterpret_cast<uint4*>(op + e) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace respin
