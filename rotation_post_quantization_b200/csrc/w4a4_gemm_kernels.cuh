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
// Structure (persistent, warp-specialised, one CTA per SM; CG = 1, or a pair
// of CTAs with CG = 2):
//  * 1 TMA warp brings each packed K block (this CTA's 128 token rows and its
//    share of the channel rows, 64 bytes each) into a packed ring with two 2-D
//    tensor copies (rows past N or O arrive as zeros). Loading through TMA
//    keeps the packed bytes off the LSU data pipe, where sector-granular
//    global loads cost 4x the wavefronts of the shared-memory reads that
//    replace them. Bulk copies issued by one thread complete one after the
//    other (about 0.3 us each on B200, whatever their size), while copies
//    from different threads overlap, so 2 * PS lanes issue: lane 2p + o
//    copies operand o (A or B) of every K block that lands in packed stage
//    p. One lane pair per stage keeps each stage's waits in order (a lane
//    serving two stages could run two phases ahead of a barrier, where the
//    parity test no longer tells the phases apart);
//  * 8 producer warps read the packed chunks (conflict-free 16-byte loads),
//    widen them and store them into a ring in the 128-byte-swizzled K-major
//    canonical layout;
//  * 1 MMA warp: one thread issues 4 MMAs (K = 32 each) per stage; the
//    accumulators alternate between two 256-column TMEM buffers.
//    CG = 1: M = 128, N = 256 per CTA. CG = 2: the leader CTA of the pair
//    issues M = 256, N = 256 MMAs that read A rows and B channels from both
//    CTAs (each CTA stages 128 token rows and 128 of the 256 channels), so
//    every SM widens and stores half the weight bytes it would alone;
//  * 4 epilogue warps drain the other TMEM buffer (tcgen05.ld), apply the two
//    scales and store bf16, overlapping the next tile's main loop.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace respin {

constexpr int kGemmBK = 128;                 // int8 K per stage (64 packed bytes per row)
constexpr int kGemmBM = 128;                 // token rows per CTA
constexpr int kGemmBN = 256;                 // channels per tile
constexpr int kGemmProducerWarps = 8;
constexpr int kGemmEpilogueWarps = 4;
constexpr int kGemmMmaWarp = kGemmProducerWarps;                 // warp 8
constexpr int kGemmEpiWarp0 = kGemmProducerWarps + 1;            // warps 9..12
constexpr int kGemmTmaWarp = kGemmEpiWarp0 + kGemmEpilogueWarps;  // warp 13
constexpr int kGemmThreads = (kGemmTmaWarp + 1) * 32;

#ifndef RESPIN_GEMM_US1
#define RESPIN_GEMM_US1 2
#endif
#ifndef RESPIN_GEMM_PS1
#define RESPIN_GEMM_PS1 4
#endif
#ifndef RESPIN_GEMM_EB
#define RESPIN_GEMM_EB 2
#endif
#ifndef RESPIN_GEMM_US2
#define RESPIN_GEMM_US2 4
#endif
#ifndef RESPIN_GEMM_PS2
#define RESPIN_GEMM_PS2 4
#endif

template <int CG>
struct GemmCfg {
  static constexpr int BNC = kGemmBN / CG;              // channel rows staged by this CTA
  static constexpr int US = CG == 1 ? RESPIN_GEMM_US1 : RESPIN_GEMM_US2;  // widened stages
  static constexpr int PS = CG == 1 ? RESPIN_GEMM_PS1 : RESPIN_GEMM_PS2;  // packed stages
  static constexpr int AStage = kGemmBM * kGemmBK;      // widened A bytes
  static constexpr int BStage = BNC * kGemmBK;          // widened B bytes
  static constexpr int Stage = AStage + BStage;
  static constexpr int PAStage = kGemmBM * kGemmBK / 2; // packed A bytes
  static constexpr int PStage = (kGemmBM + BNC) * kGemmBK / 2;
  static constexpr int Chunks = (kGemmBM + BNC) * (kGemmBK / 32);  // 16-byte packed chunks
  static constexpr int ChunksPerThread = Chunks / (kGemmProducerWarps * 32);
  static constexpr int TileM = kGemmBM * CG;            // token rows per tile
  static constexpr int EB = RESPIN_GEMM_EB;             // output staging units per epilogue warp
  static constexpr int Unit = 32 * 64;                  // one unit: 32 rows x 64 bytes
  static constexpr int SwBytes = kGemmBN * 4;          // one tile's channel scales, per epilogue warp
  static constexpr int Smem =
      US * Stage + PS * PStage + kGemmEpilogueWarps * (EB * Unit + SwBytes) + 1024 + 256;
  static_assert(Chunks % (kGemmProducerWarps * 32) == 0, "chunk split");
  static_assert(2 * PS <= 32, "one issuing lane pair per packed stage");
};

// Exact int32 -> binary32 for |a| <= 2^22: adding a to the bit pattern of
// 1.5 * 2^23 gives the float 1.5 * 2^23 + a (the sum stays within
// [2^23, 2^24], where consecutive floats are the integers), and subtracting
// 1.5 * 2^23 is exact. Two full-rate ALU operations instead of a conversion.
__device__ __forceinline__ float exact_i22_to_f32(int32_t a) {
  return __int_as_float(a + 0x4B400000) - 12582912.0f;
}

// Byte offset of 16-byte piece j (0..3) of row r (0..31) in a 32 x 64-byte
// staging unit in the tensor-map 64-byte swizzle (piece index XOR bits 7-8 of
// the offset). The unit starts on a 1024-byte boundary. Rows written by the
// eight lanes of one quarter-warp land in eight distinct bank groups.
__device__ __forceinline__ uint32_t sw64_offset(int r, int j) {
  return static_cast<uint32_t>(r * 64 + ((j ^ ((r >> 1) & 3)) << 4));
}

// Output path of one epilogue warp: a 32-column chunk of accumulators (lane =
// one token row; 256 acc each) is scaled to bf16 (or shifted back to int32),
// written into one of EB 32 x 64-byte staging units in shared memory
// (tensor-map 64-byte swizzle, conflict-free row-per-lane writes), and lane 0
// sends the unit to global memory with one 2-D tensor store, so every output
// row segment reaches L2 as whole sectors. int32 output takes two units
// (16 columns each) per chunk.
template <bool I32OUT, bool ROWMAX, int EB>
struct GemmOut {
  static constexpr int Unit = 32 * 64;
  const CUtensorMap* tmO;
  uint8_t* smem;     // generic pointer to shared address `base`
  uint32_t base;
  uint32_t ubase;    // this warp's first staging unit (shared address)
  int lane, O;
  int unit;
  uint64_t policy;   // the output is not read again by this kernel: its lines go first from L2

  __device__ __forceinline__ GemmOut(const CUtensorMap* tm, uint8_t* sm, uint32_t b, uint32_t ub, int ln, int o)
      : tmO(tm), smem(sm), base(b), ubase(ub), lane(ln), O(o), unit(0), policy(l2_policy_evict_first()) {}

  // Staging of one unit: begin() waits until the unit's previous tensor store
  // has read it and returns its generic address; the caller writes the
  // lane's four 16-byte pieces (put), then end() sends the unit.
  __device__ __forceinline__ uint8_t* begin() {
    if (lane == 0) bulk_wait_group_read<EB - 1>();   // this unit's previous store read it
    __syncwarp();
    return smem + (ubase + static_cast<uint32_t>((unit % EB) * Unit) - base);
  }
  __device__ __forceinline__ void put(uint8_t* up, int j, uint4 piece) {
    *reinterpret_cast<uint4*>(up + sw64_offset(lane, j)) = piece;
  }
  __device__ __forceinline__ void end(int x, int y) {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d_hint(tmO, x, y, ubase + static_cast<uint32_t>((unit % EB) * Unit), policy);
      bulk_commit_group();
    }
    ++unit;
  }

  // chunk v (columns colb..colb+31 of row y + lane) with row scale sa_r and
  // the chunk's 32 channel scales at swp; rmax takes the max |bf16 output|.
  // Each 16-byte piece goes to shared memory as soon as it is formed.
  __device__ __forceinline__ void chunk(const uint32_t (&v)[32], int colb, int y, float sa_r, const float* swp,
                                        float& rmax) {
    if constexpr (I32OUT) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        if (colb + 16 * half >= O) break;
        uint8_t* up = begin();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int e = 16 * half + 4 * j;
          put(up, j,
              make_uint4(static_cast<uint32_t>(static_cast<int32_t>(v[e]) >> 8),
                         static_cast<uint32_t>(static_cast<int32_t>(v[e + 1]) >> 8),
                         static_cast<uint32_t>(static_cast<int32_t>(v[e + 2]) >> 8),
                         static_cast<uint32_t>(static_cast<int32_t>(v[e + 3]) >> 8)));
        }
        end(colb + 16 * half, y);
      }
    } else {
      uint8_t* up = begin();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (colb + 8 * j >= O) {   // O % 16 == 0: a chunk is full or half full
          put(up, j, make_uint4(0u, 0u, 0u, 0u));
          continue;
        }
        const float4 w0 = reinterpret_cast<const float4*>(swp)[2 * j];
        const float4 w1 = reinterpret_cast<const float4*>(swp)[2 * j + 1];
        const float ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        uint32_t w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = 8 * j + 2 * u;
          const float f0 = __fmul_rn(__fmul_rn(exact_i22_to_f32(static_cast<int32_t>(v[e]) >> 8), sa_r), ws[2 * u]);
          const float f1 =
              __fmul_rn(__fmul_rn(exact_i22_to_f32(static_cast<int32_t>(v[e + 1]) >> 8), sa_r), ws[2 * u + 1]);
          w[u] = pack_bf16x2(f0, f1);
          if constexpr (ROWMAX)
            rmax = fmaxf(rmax, fmaxf(fabsf(__uint_as_float(w[u] << 16)), fabsf(__uint_as_float(w[u] & 0xFFFF0000u))));
        }
        put(up, j, make_uint4(w[0], w[1], w[2], w[3]));
      }
      end(colb, y);
    }
  }
};

// tmA: uint8 [N, K/2] box {64, 128}; tmB: uint8 [O, K/2] box {64, 256/CG}
// (inner dimension first), no swizzle, out-of-range elements zero filled.
// tmO: the output [N, O] (bf16, or int32 for I32OUT), box {64 bytes, 32 rows},
// 64-byte swizzle; the store clips rows >= N and columns >= O.
template <int CG, bool I32OUT, bool ROWMAX = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmO, const float* __restrict__ sa,
                 const float* __restrict__ sw, int N, int K, int O, float* __restrict__ rowmax) {
  using G = GemmCfg<CG>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t pbase = base + G::US * G::Stage;   // packed ring
  const uint32_t ebase = pbase + G::PS * G::PStage;  // output staging units
  const uint32_t swbase = ebase + kGemmEpilogueWarps * G::EB * G::Unit;  // channel scales
  const uint32_t bars = swbase + kGemmEpilogueWarps * G::SwBytes;
  const uint32_t full0 = bars;                       // [US] widened stage ready (leader counts both CTAs)
  const uint32_t empty0 = full0 + 8 * G::US;         // [US] widened stage consumed (MMA commit)
  const uint32_t pfull0 = empty0 + 8 * G::US;        // [PS] packed stage landed (TMA)
  const uint32_t pempty0 = pfull0 + 8 * G::PS;       // [PS] packed stage consumed
  const uint32_t afull0 = pempty0 + 8 * G::PS;       // [2] accumulator buffer full (MMA commit)
  const uint32_t aempty0 = afull0 + 16;              // [2] accumulator buffer drained (leader)
  const uint32_t tslot = aempty0 + 16;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
  const int group = static_cast<int>(blockIdx.x) / CG;
  const int ngroups = static_cast<int>(gridDim.x) / CG;
  const int KB = K / kGemmBK;   // K blocks
  const int mtiles = (N + G::TileM - 1) / G::TileM;
  const int ntiles = (O + kGemmBN - 1) / kGemmBN;
  const int tiles = mtiles * ntiles;

  if (tid == 0) {
    for (int s = 0; s < G::US; ++s) {
      mbar_init(full0 + 8 * s, CG * kGemmProducerWarps);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int s = 0; s < G::PS; ++s) {
      mbar_init(pfull0 + 8 * s, 2);   // the A and the B copy each arrive with their bytes
      mbar_init(pempty0 + 8 * s, kGemmProducerWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(afull0 + 8 * b, 1);
      mbar_init(aempty0 + 8 * b, CG * kGemmEpilogueWarps);
    }
    fence_mbarrier_init();
  }
  if (warp == 0) {
    if constexpr (CG == 2) {
      tmem_alloc_pair(tslot, 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tslot, 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (CG == 2) cluster_sync(); else __syncthreads();
  tc_fence_after();
  grid_dep_launch();   // the next kernel of the stream may be scheduled
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + (tslot - base));
  // barriers signalled in the leader CTA by both CTAs of the pair
  const uint32_t full_leader0 = CG == 2 ? map_to_rank(full0, 0) : full0;
  const uint32_t aempty_leader0 = CG == 2 ? map_to_rank(aempty0, 0) : aempty0;

  // Epilogue output staging (epilogue warps): EB 32 x 64-byte units per warp,
  // each written to global memory by one tensor store.
  const int quad = warp & 3;   // hardware rule: warp w reads TMEM lanes 32*(w%4)..
  GemmOut<I32OUT, ROWMAX, G::EB> out(&tmO, smem, base, ebase + static_cast<uint32_t>(quad * G::EB * G::Unit),
                                     lane, O);

  if (warp < kGemmProducerWarps) {
    // ------------------------------------------------ producers: widen packed -> int8
    bool ok = true;
    int kstep = 0;  // running k-block counter over all tiles (selects the stages)
    for (int t = group; t < tiles; t += ngroups) {
      const int m_base = (t / ntiles) * G::TileM + static_cast<int>(rank) * kGemmBM;
      for (int kb = 0; kb < KB; ++kb, ++kstep) {
        const int ps = kstep % G::PS, s = kstep % G::US;
        if (ok) ok = mbar_wait(pfull0 + 8 * ps, (kstep / G::PS) & 1, kSiteGemmPackedFull);
        const uint8_t* pk = smem + (pbase - base) + ps * G::PStage;
        uint4 b[G::ChunksPerThread];
#pragma unroll
        for (int j = 0; j < G::ChunksPerThread; ++j)   // chunk q = row*4 + c, 16 bytes each
          b[j] = *reinterpret_cast<const uint4*>(pk + (tid + j * kGemmProducerWarps * 32) * 16);
        if (ok) ok = mbar_wait(empty0 + 8 * s, ((kstep / G::US) & 1) ^ 1, kSiteGemmEmpty);
        uint8_t* sA = smem + s * G::Stage;
#pragma unroll
        for (int j = 0; j < G::ChunksPerThread; ++j) {
          const int q = tid + j * kGemmProducerWarps * 32;
          const bool is_a = q < kGemmBM * 4;
          const int qq = is_a ? q : q - kGemmBM * 4;
          const int row = qq >> 2, c = qq & 3;
          // A rows past N: the accumulator rows they feed are never stored,
          // so whatever the stage holds there is fine (saves the widening of
          // mostly empty A tiles at small N, which runs on single CTAs; the
          // test costs the CTA-pair kernel 5 %, so it has none)
          if constexpr (CG == 1) {
            if (is_a && m_base + row >= N) continue;
          }
          uint8_t* rowp = sA + (is_a ? 0 : G::AStage) + (row >> 3) * 1024 + (row & 7) * 128;
          const uint4 p = b[j];
          const uint4 lo = make_uint4((p.x << 4) & 0xF0F0F0F0u, (p.y << 4) & 0xF0F0F0F0u,
                                      (p.z << 4) & 0xF0F0F0F0u, (p.w << 4) & 0xF0F0F0F0u);
          const uint4 hi = make_uint4(p.x & 0xF0F0F0F0u, p.y & 0xF0F0F0F0u, p.z & 0xF0F0F0F0u,
                                      p.w & 0xF0F0F0F0u);
          *reinterpret_cast<uint4*>(rowp + (((2 * c) ^ (row & 7)) << 4)) = lo;
          *reinterpret_cast<uint4*>(rowp + (((2 * c + 1) ^ (row & 7)) << 4)) = hi;
        }
        // Widened stage -> MMA (async-proxy reads): every thread fences its
        // own writes, then one lane per warp signals. The packed stage is
        // released only now: the same proxy fence orders the reads of its
        // bytes (generic proxy) before the next tensor copy into it (async
        // proxy). A separate fence right after the reads costs more than the
        // earlier release gains.
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if constexpr (CG == 2) mbar_arrive_cluster(full_leader0 + 8 * s);
          else mbar_arrive(full0 + 8 * s);
          mbar_arrive(pempty0 + 8 * ps);
        }
      }
    }
  } else if (warp == kGemmTmaWarp) {
    // ------------------------------------------------ TMA warp: packed K blocks
    // launched as a programmatic dependent: the codes (and possibly the
    // weights) come from earlier kernels of the stream
    grid_dep_wait();
    if (lane < 2 * G::PS) {
      const int stage = lane >> 1;
      const bool is_b = (lane & 1) != 0;
      const uint32_t bytes = is_b ? G::PStage - G::PAStage : G::PAStage;
      bool ok = true;
      int kstep = 0;
      for (int t = group; t < tiles; t += ngroups) {
        const int arow = (t / ntiles) * G::TileM + static_cast<int>(rank) * kGemmBM;
        const int brow = (t % ntiles) * kGemmBN + static_cast<int>(rank) * G::BNC;
        for (int kb = 0; kb < KB; ++kb, ++kstep) {
          const int ps = kstep % G::PS;
          if (ps != stage) continue;
          if (ok) ok = mbar_wait(pempty0 + 8 * ps, ((kstep / G::PS) & 1) ^ 1, kSiteGemmPackedEmpty);
          if (!ok) continue;
          const uint32_t dst = pbase + ps * G::PStage;
          mbar_arrive_expect_tx(pfull0 + 8 * ps, bytes);
          if (is_b) tma_load_2d(dst + G::PAStage, &tmB, kb * (kGemmBK / 2), brow, pfull0 + 8 * ps);
          else tma_load_2d(dst, &tmA, kb * (kGemmBK / 2), arow, pfull0 + 8 * ps);
        }
      }
    }
  } else if (warp == kGemmMmaWarp) {
    // ------------------------------------------------ MMA issuer (leader CTA)
    if (CG == 1 || rank == 0) {
      constexpr uint32_t idesc = umma_idesc_s8(kGemmBM * CG, kGemmBN);
      bool ok = true;
      int kstep = 0, local = 0;
      for (int t = group; t < tiles; t += ngroups, ++local) {
        const int ab = local & 1;
        // wait until both epilogues drained this accumulator buffer (two tiles ago)
        if (ok) ok = mbar_wait_cluster(aempty0 + 8 * ab, ((local >> 1) & 1) ^ 1, kSiteGemmAccum);
        tc_fence_after();
        const uint32_t dtm = tmem + ab * kGemmBN;
        for (int kb = 0; kb < KB; ++kb, ++kstep) {
          const int s = kstep % G::US;
          if (ok) ok = mbar_wait_cluster(full0 + 8 * s, (kstep / G::US) & 1, kSiteGemmFull);
          tc_fence_after();
          if (lane == 0 && ok) {
            const uint32_t a_addr = base + s * G::Stage;
            const uint32_t b_addr = a_addr + G::AStage;
#pragma unroll
            for (int k = 0; k < kGemmBK / 32; ++k) {
              const uint64_t ad = umma_desc_sw128(a_addr + 32 * k), bd = umma_desc_sw128(b_addr + 32 * k);
              const uint32_t acc = (kb | k) != 0 ? 1u : 0u;
              if constexpr (CG == 2) tc_mma_i8_pair(dtm, ad, bd, idesc, acc);
              else tc_mma_i8(dtm, ad, bd, idesc, acc);
            }
            if constexpr (CG == 2) tc_commit_pair_multicast(empty0 + 8 * s, 0x3);
            else tc_commit(empty0 + 8 * s);
          }
          __syncwarp();
        }
        if (lane == 0) {
          if constexpr (CG == 2) tc_commit_pair_multicast(afull0 + 8 * ab, 0x3);
          else tc_commit(afull0 + 8 * ab);
        }
        __syncwarp();
      }
    }
  } else {
    // ------------------------------------------------ epilogue warps
    // Each warp owns 32 accumulator rows (TMEM lanes) and EB staging units.
    // Per 32-column chunk: tcgen05.ld (lane = row, registers = columns),
    // scale, write the row's 64 bytes (bf16) into a swizzled unit, and one
    // lane issues a TMA tensor store of the 32 x 32 block, so every output
    // row segment reaches L2 as whole sectors. int32 output takes two units
    // (16 columns each) per chunk.
    float* sws = reinterpret_cast<float*>(smem + (swbase - base) + quad * G::SwBytes);
    grid_dep_wait();   // the activation scales and the output buffer
    bool ok = true;
    int local = 0;
    for (int t = group; t < tiles; t += ngroups, ++local) {
      const int ab = local & 1;
      const int m0 = (t / ntiles) * G::TileM + static_cast<int>(rank) * kGemmBM;
      const int n0 = (t % ntiles) * kGemmBN;
      const int y = m0 + quad * 32;           // first row of this warp's blocks
      const int row = y + lane;
      // Fetch the tile's scales while its accumulators are still being
      // computed: sa for this lane's row, 8 channel scales per lane.
      float sa_r = 0.f;
      float4 sw0 = make_float4(0.f, 0.f, 0.f, 0.f), sw1 = sw0;
      if constexpr (!I32OUT) {
        if (row < N) sa_r = __ldg(sa + row);
        if (n0 + 8 * lane < O) {   // O % 16 == 0: then all 8 channels are in range
          sw0 = __ldg(reinterpret_cast<const float4*>(sw + n0 + 8 * lane));
          sw1 = __ldg(reinterpret_cast<const float4*>(sw + n0 + 8 * lane + 4));
        }
      }
      if (ok) ok = mbar_wait(afull0 + 8 * ab, (local >> 1) & 1, kSiteGemmAccum);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      if constexpr (!I32OUT) {
        reinterpret_cast<float4*>(sws)[2 * lane] = sw0;
        reinterpret_cast<float4*>(sws)[2 * lane + 1] = sw1;
        __syncwarp();
      }
      const uint32_t tbase = tmem + (static_cast<uint32_t>(quad * 32) << 16) + ab * kGemmBN;
      float rmax = 0.f;   // this row's max |bf16 output| over the tile
#pragma unroll 1
      for (int cc = 0; cc < kGemmBN / 32; cc += 2) {
        uint32_t v[2][32];
        tmem_ld_32x32b_x32(tbase + cc * 32, v[0]);
        tmem_ld_32x32b_x32(tbase + cc * 32 + 32, v[1]);
        tmem_wait_ld();
        if (!ok || y >= N) continue;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int colb = n0 + (cc + h) * 32;
          if (colb >= O) break;
          out.chunk(v[h], colb, y, sa_r, sws + (colb - n0), rmax);
        }
      }
      // optional per-(row, channel tile) maxima of |out| for a later per-token
      // quantization of this output (one writer per entry)
      if constexpr (ROWMAX && !I32OUT) {
        if (ok && row < N) rowmax[static_cast<size_t>(row) * ((O + kGemmBN - 1) / kGemmBN) + n0 / kGemmBN] = rmax;
      }
      // hand the accumulator buffer back to the MMA warp (of the leader CTA)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (CG == 2) mbar_arrive_cluster(aempty_leader0 + 8 * ab);
        else mbar_arrive(aempty0 + 8 * ab);
      }
    }
    // the staging units must not be released while a store still reads them
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }
  tc_fence_before();
  // Neither CTA of a pair may release its TMEM or shared memory while the
  // other can still reach it.
  if constexpr (CG == 2) cluster_sync(); else __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    if constexpr (CG == 2) tmem_dealloc_pair(tmem, 512);
    else tmem_dealloc(tmem, 512);
  }
}


// ---------------------------------------------------------------------------
// CTA-pair GEMM with the activation operand in tensor memory.
//
// In the kernel above both widened operands pass through shared memory. Here
// the producers widen A straight into tensor memory (tcgen05.st, one token
// row per lane) and the MMA reads A from there (tcgen05.mma with A in TMEM):
// a stage's shared memory holds only the widened B (16 KB instead of 32 KB),
// the A write and read leave the shared-memory pipe, and the space freed
// buys a deeper packed ring (7 stages): under load a packed copy takes
// 1-2.5 us from issue to arrival (per-K-block timestamps), which 4 stages did
// not cover (8192 x 8192 -> 28672: 1514 us with both operands in shared
// memory and 4 packed stages, 1209 us here).
//
// Tensor memory (512 columns): the int32 accumulator of the current tile in
// columns [0, 256) (one buffer), then US A stages of 32 columns (128 int8 K
// values per row, four per 32-bit column). With one accumulator the next
// tile's first MMA waits until the epilogues have read the accumulator, so
// 16 epilogue warps (four per TMEM lane quarter, 64 columns each) read their
// whole share in one round and hand it back before converting anything
// (measured with 8 warps that converted half their columns first: the
// tensor pipe idled ~1.4 us at every tile switch). Splitting the hand-over
// by column halves instead needs N = 128 MMAs, which measured 40 % slower
// than N = 256.
//
// Warps: 0-3 producers (warp w widens the A rows of TMEM lane quarter w and
// four 16-byte B chunks per thread), 4 MMA (leader CTA, one thread), 5-20
// epilogue, 21 TMA.
constexpr int kTaProducerWarps = 4;
constexpr int kTaMmaWarp = 4;
constexpr int kTaEpiWarp0 = 5;
constexpr int kTaEpilogueWarps = 16;
constexpr int kTaTmaWarp = kTaEpiWarp0 + kTaEpilogueWarps;   // 21
constexpr int kTaThreads = (kTaTmaWarp + 1) * 32;            // 704

#ifndef RESPIN_GEMM_TA_US
#define RESPIN_GEMM_TA_US 4
#endif
#ifndef RESPIN_GEMM_TA_PS
#define RESPIN_GEMM_TA_PS 7
#endif
#ifndef RESPIN_GEMM_TA_EB
#define RESPIN_GEMM_TA_EB 1
#endif

struct GemmTaCfg {
  static constexpr int BNC = kGemmBN / 2;                       // channel rows staged by this CTA
  static constexpr int US = RESPIN_GEMM_TA_US;                  // widened stages (B in smem, A in TMEM)
  static constexpr int PS = RESPIN_GEMM_TA_PS;                  // packed stages
  static constexpr int AC = kGemmBK / 32;                       // packed 16-byte A pieces per row
  static constexpr int BStage = BNC * kGemmBK;                  // widened B bytes
  static constexpr int PAStage = kGemmBM * kGemmBK / 2;         // packed A bytes
  static constexpr int PStage = (kGemmBM + BNC) * kGemmBK / 2;  // packed A + B bytes
  static constexpr int BChunksPerThread = BNC * (kGemmBK / 32) / (kTaProducerWarps * 32);
  static constexpr int TileM = 2 * kGemmBM;
  static constexpr int EB = RESPIN_GEMM_TA_EB;                  // output staging units per epilogue warp
  static constexpr int Unit = 32 * 64;
  static constexpr int EpiCols = kGemmBN / 4;                   // accumulator columns per epilogue warp
  static constexpr int SwBytes = EpiCols * 4;
  static constexpr int AccCols = kGemmBN;                       // TMEM columns of the accumulator
  static constexpr int ACols = kGemmBK / 4;                     // TMEM columns per A stage
  static constexpr int RmaxBytes = 2 * 4 * 4 * 32 * 4;          // [2][quarter][part][row] partial row maxima
  static constexpr int Smem = US * BStage + PS * PStage + kTaEpilogueWarps * (EB * Unit + SwBytes) +
                              RmaxBytes + 1024 + 256;
  static_assert(AccCols + US * ACols <= 512, "TMEM: accumulator and A stages");
  static_assert(2 * PS <= 32, "one issuing lane pair per packed stage");
  static_assert(BChunksPerThread * kTaProducerWarps * 32 == BNC * (kGemmBK / 32), "chunk split");
  static_assert(kTaProducerWarps == 4, "producer warp w widens the A rows of TMEM lane quarter w");
  static_assert(8 * (2 * US + 2 * PS + 2) + 4 <= 256, "barrier area");
  static_assert(Smem <= 227 * 1024, "shared memory of one CTA");
};

// tmA: uint8 [N, K/2] box {64, 128}, 64-byte swizzle (row r's 16-byte piece j
// lands at r*64 + ((j ^ ((r >> 1) & 3)) << 4): the eight rows a quarter-warp
// reads fall in eight distinct bank groups); tmB: uint8 [O, K/2] box
// {64, 128}, no swizzle; tmO as above. Launched as clusters of 2.
template <bool I32OUT, bool ROWMAX = false>
__global__ void __launch_bounds__(kTaThreads, 1)
w4a4_gemm_ta_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmO, const float* __restrict__ sa,
                    const float* __restrict__ sw, int N, int K, int O, float* __restrict__ rowmax) {
  using G = GemmTaCfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t pbase = base + G::US * G::BStage;    // packed ring
  const uint32_t ebase = pbase + G::PS * G::PStage;   // output staging units
  const uint32_t swbase = ebase + kTaEpilogueWarps * G::EB * G::Unit;   // channel scales
  const uint32_t rmbase = swbase + kTaEpilogueWarps * G::SwBytes;       // partial row maxima
  const uint32_t bars = rmbase + G::RmaxBytes;
  const uint32_t full0 = bars;                      // [US] widened stage ready (leader counts both CTAs)
  const uint32_t empty0 = full0 + 8 * G::US;        // [US] widened stage consumed (MMA commit)
  const uint32_t pfull0 = empty0 + 8 * G::US;       // [PS] packed stage landed (TMA)
  const uint32_t pempty0 = pfull0 + 8 * G::PS;      // [PS] packed stage consumed
  const uint32_t afull = pempty0 + 8 * G::PS;       // accumulator complete (MMA commit)
  const uint32_t aempty = afull + 8;                // accumulator read out (leader)
  const uint32_t tslot = aempty + 8;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int group = static_cast<int>(blockIdx.x) / 2;
  const int ngroups = static_cast<int>(gridDim.x) / 2;
  const int KB = K / kGemmBK;
  const int mtiles = (N + G::TileM - 1) / G::TileM;
  const int ntiles = (O + kGemmBN - 1) / kGemmBN;
  const int tiles = mtiles * ntiles;

  if (tid == 0) {
    for (int s = 0; s < G::US; ++s) {
      mbar_init(full0 + 8 * s, 2 * kTaProducerWarps);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int s = 0; s < G::PS; ++s) {
      mbar_init(pfull0 + 8 * s, 2);   // the A and the B copy each arrive with their bytes
      mbar_init(pempty0 + 8 * s, kTaProducerWarps);
    }
    mbar_init(afull, 1);
    mbar_init(aempty, 2 * kTaEpilogueWarps);
    fence_mbarrier_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(tslot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  grid_dep_launch();   // the next kernel of the stream may be scheduled
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + (tslot - base));
  const uint32_t full_leader0 = map_to_rank(full0, 0);
  const uint32_t aempty_leader = map_to_rank(aempty, 0);

  if (warp < kTaProducerWarps) {
    // ------------------------------------------------ producers: widen packed -> int8
    const int quad = warp;       // TMEM lanes 32*quad.. (hardware rule: warp w, lanes 32*(w%4)..)
    const int arow = quad * 32 + lane;
    const uint32_t a_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16) + G::AccCols;
    bool ok = true;
    int kstep = 0;
    for (int t = group; t < tiles; t += ngroups) {
      for (int kb = 0; kb < KB; ++kb, ++kstep) {
        const int ps = kstep % G::PS, s = kstep % G::US;
        if (ok) ok = mbar_wait(pfull0 + 8 * ps, (kstep / G::PS) & 1, kSiteGemmPackedFull);
        const uint8_t* pk = smem + (pbase - base) + ps * G::PStage;
        uint4 a[G::AC], b[G::BChunksPerThread];
#pragma unroll
        for (int j = 0; j < G::AC; ++j)
          a[j] = *reinterpret_cast<const uint4*>(pk + arow * 64 + ((j ^ ((arow >> 1) & 3)) << 4));
#pragma unroll
        for (int j = 0; j < G::BChunksPerThread; ++j)   // chunk q = row*4 + c, 16 bytes each
          b[j] = *reinterpret_cast<const uint4*>(pk + G::PAStage + (tid + j * kTaProducerWarps * 32) * 16);
        if (ok) ok = mbar_wait(empty0 + 8 * s, ((kstep / G::US) & 1) ^ 1, kSiteGemmEmpty);
        tc_fence_after();   // the MMAs that read this stage's A columns are complete
        // B: widened into the 128-byte-swizzled K-major layout
        uint8_t* sB = smem + s * G::BStage;
#pragma unroll
        for (int j = 0; j < G::BChunksPerThread; ++j) {
          const int q = tid + j * kTaProducerWarps * 32;
          const int row = q >> 2, c = q & 3;
          uint8_t* rowp = sB + (row >> 3) * 1024 + (row & 7) * 128;
          const uint4 p = b[j];
          const uint4 lo = make_uint4((p.x << 4) & 0xF0F0F0F0u, (p.y << 4) & 0xF0F0F0F0u,
                                      (p.z << 4) & 0xF0F0F0F0u, (p.w << 4) & 0xF0F0F0F0u);
          const uint4 hi = make_uint4(p.x & 0xF0F0F0F0u, p.y & 0xF0F0F0F0u, p.z & 0xF0F0F0F0u,
                                      p.w & 0xF0F0F0F0u);
          *reinterpret_cast<uint4*>(rowp + (((2 * c) ^ (row & 7)) << 4)) = lo;
          *reinterpret_cast<uint4*>(rowp + (((2 * c + 1) ^ (row & 7)) << 4)) = hi;
        }
        // A: the same K permutation (even codes of a 16-byte piece, then its
        // odd codes), as 32-bit TMEM columns of this lane's row
#pragma unroll
        for (int h = 0; h < G::AC / 2; ++h) {
          uint32_t w[16];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const uint4 p = a[2 * h + j];
            w[8 * j + 0] = (p.x << 4) & 0xF0F0F0F0u;
            w[8 * j + 1] = (p.y << 4) & 0xF0F0F0F0u;
            w[8 * j + 2] = (p.z << 4) & 0xF0F0F0F0u;
            w[8 * j + 3] = (p.w << 4) & 0xF0F0F0F0u;
            w[8 * j + 4] = p.x & 0xF0F0F0F0u;
            w[8 * j + 5] = p.y & 0xF0F0F0F0u;
            w[8 * j + 6] = p.z & 0xF0F0F0F0u;
            w[8 * j + 7] = p.w & 0xF0F0F0F0u;
          }
          tmem_st_32x32b_x16(a_lane + static_cast<uint32_t>(s * G::ACols + 16 * h), w);
        }
        tmem_wait_st();
        // Stage -> MMA: the TMEM stores are complete and ordered before the
        // arrival (tcgen05 fence), the shared-memory stores are made visible
        // to the async proxy; the packed stage is released by the same
        // proxy fence (its generic reads before the next tensor copy).
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_cluster(full_leader0 + 8 * s);
          mbar_arrive(pempty0 + 8 * ps);
        }
      }
    }
  } else if (warp == kTaTmaWarp) {
    // ------------------------------------------------ TMA warp: packed K blocks
    grid_dep_wait();   // the codes (and possibly the weights) come from earlier kernels
    if (lane < 2 * G::PS) {
      const int stage = lane >> 1;
      const bool is_b = (lane & 1) != 0;
      const uint32_t bytes = is_b ? G::PStage - G::PAStage : G::PAStage;
      bool ok = true;
      int kstep = 0;
      for (int t = group; t < tiles; t += ngroups) {
        const int arow = (t / ntiles) * G::TileM + static_cast<int>(rank) * kGemmBM;
        const int brow = (t % ntiles) * kGemmBN + static_cast<int>(rank) * G::BNC;
        for (int kb = 0; kb < KB; ++kb, ++kstep) {
          const int ps = kstep % G::PS;
          if (ps != stage) continue;
          if (ok) ok = mbar_wait(pempty0 + 8 * ps, ((kstep / G::PS) & 1) ^ 1, kSiteGemmPackedEmpty);
          if (!ok) continue;
          const uint32_t dst = pbase + ps * G::PStage;
          mbar_arrive_expect_tx(pfull0 + 8 * ps, bytes);
          if (is_b) tma_load_2d(dst + G::PAStage, &tmB, kb * (kGemmBK / 2), brow, pfull0 + 8 * ps);
          else tma_load_2d(dst, &tmA, kb * (kGemmBK / 2), arow, pfull0 + 8 * ps);
        }
      }
    }
  } else if (warp == kTaMmaWarp) {
    // ------------------------------------------------ MMA issuer (leader CTA)
    if (rank == 0) {
      constexpr uint32_t idesc = umma_idesc_s8(G::TileM, kGemmBN);
      bool ok = true;
      int kstep = 0, local = 0;
      for (int t = group; t < tiles; t += ngroups, ++local) {
        // both CTAs' epilogues have read the previous tile's accumulator
        if (ok) ok = mbar_wait_cluster(aempty, (local & 1) ^ 1, kSiteGemmAccum);
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb, ++kstep) {
          const int s = kstep % G::US;
          if (ok) ok = mbar_wait_cluster(full0 + 8 * s, (kstep / G::US) & 1, kSiteGemmFull);
          tc_fence_after();
          if (lane == 0 && ok) {
            const uint32_t b_addr = base + s * G::BStage;
            const uint32_t a_tm = tmem + G::AccCols + static_cast<uint32_t>(s * G::ACols);
#pragma unroll
            for (int k = 0; k < kGemmBK / 32; ++k) {
              const uint64_t bd = umma_desc_sw128(b_addr + 32 * k);
              tc_mma_i8_pair_ta(tmem, a_tm + 8 * k, bd, idesc, (kb | k) != 0 ? 1u : 0u);
            }
            tc_commit_pair_multicast(empty0 + 8 * s, 0x3);
          }
          __syncwarp();
        }
        if (lane == 0) tc_commit_pair_multicast(afull, 0x3);
        __syncwarp();
      }
    }
  } else {
    // ------------------------------------------------ epilogue warps
    // Four warps per TMEM lane quarter, 64 accumulator columns each: a warp
    // holds its whole share in registers after one round of tcgen05.ld, so
    // the accumulator goes back to the MMA warp before any conversion.
    const int e = warp - kTaEpiWarp0;
    const int quad = warp & 3;   // TMEM lanes 32*quad.. = token rows of this warp
    const int part = e >> 2;     // accumulator columns [64 part, 64 part + 64)
    GemmOut<I32OUT, ROWMAX, G::EB> out(&tmO, smem, base, ebase + static_cast<uint32_t>(e * G::EB * G::Unit), lane, O);
    float* sws = reinterpret_cast<float*>(smem + (swbase - base) + e * G::SwBytes);
    float* rmx = reinterpret_cast<float*>(smem + (rmbase - base));
    grid_dep_wait();   // the activation scales and the output buffer
    bool ok = true;
    int local = 0;
    for (int t = group; t < tiles; t += ngroups, ++local) {
      const int m0 = (t / ntiles) * G::TileM + static_cast<int>(rank) * kGemmBM;
      const int n0 = (t % ntiles) * kGemmBN;
      const int c0 = n0 + part * G::EpiCols;   // first output column of this warp
      const int y = m0 + quad * 32;            // first row of this warp's blocks
      const int row = y + lane;
      float sa_r = 0.f;
      float2 sw2 = make_float2(0.f, 0.f);
      if constexpr (!I32OUT) {
        if (row < N) sa_r = __ldg(sa + row);
        if (c0 + 2 * lane < O) sw2 = __ldg(reinterpret_cast<const float2*>(sw + c0 + 2 * lane));   // O % 16 == 0
      }
      if (ok) ok = mbar_wait(afull, local & 1, kSiteGemmAccum);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      const uint32_t tb = tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(part * G::EpiCols);
      uint32_t v[2][32];
      tmem_ld_32x32b_x32(tb, v[0]);
      tmem_ld_32x32b_x32(tb + 32, v[1]);
      tmem_wait_ld();
      // the accumulator is read out: hand it back to the MMA warp of the leader
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(aempty_leader);
      if constexpr (!I32OUT) {
        reinterpret_cast<float2*>(sws)[lane] = sw2;
        __syncwarp();
      }
      float rmax = 0.f;
      if (ok && y < N) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
          if (c0 + 32 * h < O) out.chunk(v[h], c0 + 32 * h, y, sa_r, sws + 32 * h, rmax);
      }
      // optional per-(row, 256-channel tile) maxima of |out|: the four warps
      // of a lane quarter each hold a quarter of the tile's columns
      if constexpr (ROWMAX && !I32OUT) {
        float* slot = rmx + ((local & 1) * 4 + quad) * 4 * 32;
        slot[part * 32 + lane] = rmax;
        named_bar_sync(1 + quad, 128);
        if (part == 0 && ok && row < N)
          rowmax[static_cast<size_t>(row) * ntiles + n0 / kGemmBN] =
              fmaxf(fmaxf(slot[lane], slot[32 + lane]), fmaxf(slot[64 + lane], slot[96 + lane]));
      }
    }
    // the staging units must not be released while a store still reads them
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }
  tc_fence_before();
  // Neither CTA of the pair may release its TMEM or shared memory while the
  // other can still reach it.
  cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace respin
