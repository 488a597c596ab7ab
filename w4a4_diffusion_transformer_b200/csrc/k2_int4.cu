// K2 for the INT4 variant: W4A4 GEMM with symmetric INT4 codes in groups of
// 64 and BF16 scales (SOTA-314 practice page, "Do this": "group size 64 with
// 16-bit scales for INT4"), with the low-rank up projection and the bias fused
// into the same accumulator as in the NVFP4 kernel.
//
// sm_100a has no 4-bit integer tensor-core MMA and no block-scaled MMA whose
// scales can carry an arbitrary BF16 value, so each 64-element group is
// dequantized on chip into FP16, where it is EXACT: a code c in [-7, 7] needs
// 3 bits and a BF16 scale 8 significant bits, so c * s fits FP16's 11.  The
// products of two such values are exact in the FP32 accumulator of a
// tcgen05.mma kind::f16, so the GEMM evaluates
//     acc = sum_g sum_{k in g} (c_x s_x 2^-ex) (c_w s_w 2^-ew)
// with no rounding beyond FP32 accumulation.  ex and ew are power-of-two
// exponents fixed when the layer is prepared (ew from the weights, ex from the
// calibration batch) that keep the FP16 values in range;
// alpha = 2^(ex + ew) is applied in the epilogue, and the branch operand is
// L2b / alpha (exact in BF16), exactly as in the NVFP4 kernel:
//     acc  = XL (L2b / alpha) + sum (...)          Y = bf16([gelu](alpha acc + b)).
// Exactness holds for every scale s with 2^-17 <= s 2^-e <= 8192: at the top
// a group whose scaled activation scale exceeds 8192 is clamped there (its
// products stay finite, and the group contributes less than it should); ex puts
// that limit at about 220x the largest activation of the calibration batch.  At
// the bottom FP16 subnormals keep every BF16 scale down to 2^-17 (2^-24 of the
// calibration maximum, 2^-30 of the largest weight residual) exactly; smaller
// ones are rounded to multiples of 2^-24 (operand units).
//
// Structure (one CTA per SM, persistent over 128 x 256 output tiles, k-step =
// one group of 64):
//   warp 0      producer: TMA loads of the packed codes (A 128 x 32 B, B 256 x
//               32 B) and bulk copies of the group's scales (A BF16 from the
//               first kernel, B FP16 prepared) into a 3-deep staging ring; per
//               tile the XL and L2b/alpha tiles into a branch buffer.
//   warp 1      TMEM (two 256-column accumulators) and the MMA issuer: 2 BF16
//               MMAs for the branch, then 4 FP16 MMAs (K = 16) per group.
//   warps 2-3   idle (they complete the first warpgroup).
//   warps 4-7   epilogue, one per TMEM lane quarter, 32 columns at a time
//               (tcgen05.ld of the next chunk overlaps the current chunk's math),
//               BF16 out through swizzled shared memory and TMA stores.  The
//               accumulator is double-buffered, so the epilogue of tile t runs
//               under the mainloop of tile t+1.
//   warps 8-23  converters: staging -> FP16 operand tiles (128-byte swizzle,
//               K-major) in a 3-deep operand ring.
// Within each 8-element chunk the k order in shared memory is (0,4,1,5,2,6,3,7)
// of the packed codes -- the order in which nibble pairs come out of a 32-bit
// word with one mask -- for both operands alike, so the sum over k is unchanged.
// Every wait is bounded (sm100.cuh).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100.cuh"

namespace svdq {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kPStages = 3;                          // staging ring (packed codes + scales)
constexpr int kOStages = 3;                          // operand ring (FP16 tiles)
constexpr int kEpiWarps = 4;
// Warp roles by warpgroup: 0 producer, 1 MMA issuer, 2-3 idle; 4-7 epilogue
// (one per TMEM lane quarter); 8 .. 8 + kConvWarps - 1 converters.  The
// converters are latency-bound (a load, a short dependent chain, a store per
// group), so there are four per scheduler; the register budget is moved to the
// epilogue with setmaxnreg.
constexpr int kConvWarps = 16;
constexpr int kEpiWarp0 = 4;
constexpr int kConvWarp0 = 8;
constexpr int kThreads = (kConvWarp0 + kConvWarps) * 32;
constexpr int kLaunchRegs = 80;                      // per thread: 65536 / 768, rounded down to 8
constexpr int kRegsCtl = 40, kRegsEpi = 160, kRegsConv = 64;
static_assert(128 * kRegsCtl + 128 * kRegsEpi + kConvWarps * 32 * kRegsConv <= kThreads * kLaunchRegs,
              "register split");
constexpr int kConvThreads = kConvWarps * 32;
// conversion units of a group: 16 codes (a quarter row) of A's 128 and B's 256 rows
constexpr int kUnits = (kBM + kBN) * 4;
constexpr int kUnitsPerThread = kUnits / kConvThreads;
static_assert(kUnits % kConvThreads == 0 && (kBM * 4) % 32 == 0, "converter work split");

// staging stage: A codes, B codes, A scales, B scales
constexpr int kPA = 0;
constexpr int kPB = kPA + kBM * 32;                  // 4096
constexpr int kPSA = kPB + kBN * 32;                 // 12288
constexpr int kPSB = kPSA + kBM * 2;                 // 12544
constexpr int kPStageBytes = 13 * 1024;
static_assert(kPSB + kBN * 2 <= kPStageBytes, "staging stage");
// operand stage: A 128 x 64 FP16, B 256 x 64 FP16 (128-byte rows)
constexpr int kOABytes = kBM * 128;
constexpr int kOBBytes = kBN * 128;
constexpr int kOStageBytes = kOABytes + kOBBytes;    // 48 KiB
// branch buffer: XL 128 x 32 BF16 and (L2b / alpha)^T 256 x 32 BF16 (64-byte rows)
constexpr int kBrABytes = kBM * 64;
constexpr int kBrBytes = kBrABytes + kBN * 64;       // 24 KiB
constexpr int kEpiBufBytes = 32 * 64;                // one 32 x 32 BF16 output chunk
constexpr int kEpiWarpBytes = 2 * kEpiBufBytes;
constexpr int kSmemBytes =
    kOStages * kOStageBytes + kBrBytes + kPStages * kPStageBytes + kEpiWarps * kEpiWarpBytes + 256 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory per block");
constexpr int kTmemCols = 512;

__device__ __forceinline__ void record_error(int* err, volatile int* abort_flag, int code) {
  atomicCAS(err, 0, code);
  *abort_flag = 1;
}

// Instruction descriptor: FP16 x FP16 -> FP32, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Packed 4-bit two's-complement codes of one 32-bit word, scaled: out[j] =
// (c_j s, c_{j+4} s) as FP16 pairs.  (w >> 4j) & 0x000F000F puts nibbles j and
// j+4 in the low bits of the two halves; XOR 0x6408 makes each half the FP16
// 1024 + (n ^ 8) = 1032 + c (exact), minus 1032 is c, times s is c s (exact).
__device__ __forceinline__ void dequant_word(uint32_t w, __half2 s2, uint32_t (&out)[4]) {
  const __half2 bias = __half2half2(__ushort_as_half((unsigned short)0x6408u));
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t h = ((w >> (4 * j)) & 0x000F000Fu) ^ 0x64086408u;
    const __half2 c = __hsub2(*reinterpret_cast<const __half2*>(&h), bias);
    const __half2 v = __hmul2(c, s2);
    out[j] = *reinterpret_cast<const uint32_t*>(&v);
  }
}

// A LoRA adapter (p.lora) reuses the branch buffer within each tile: the
// producer reloads it with XL_lora and (s B / alpha)^T once the tile's branch
// MMAs have read it (after issuing group kLoraLoadG), and the MMA warp adds the
// adapter after group kLoraMmaG, so the reload overlaps the group stream.  The
// buffer's barriers then complete twice per tile; both sides count the phases.
constexpr int kLoraLoadG = 2, kLoraMmaG = 5;

__global__ void __launch_bounds__(kThreads, 1)
    k2_int4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_xl, const __grid_constant__ CUtensorMap tm_l2,
                   const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_xla,
                   const __grid_constant__ CUtensorMap tm_l2a, K2Int4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* oring = smem;                                          // operand ring (1 KiB aligned)
  uint8_t* brbuf = oring + kOStages * kOStageBytes;               // branch buffer
  uint8_t* pring = brbuf + kBrBytes;                              // staging ring
  uint8_t* epi_buf = pring + kPStages * kPStageBytes;
  uint64_t* pfull = reinterpret_cast<uint64_t*>(epi_buf + kEpiWarps * kEpiWarpBytes);
  uint64_t* pempty = pfull + kPStages;
  uint64_t* ofull = pempty + kPStages;
  uint64_t* oempty = ofull + kOStages;
  uint64_t* bfull = oempty + kOStages;
  uint64_t* bempty = bfull + 1;
  uint64_t* acc_full = bempty + 1;                                // [2]
  uint64_t* acc_empty = acc_full + 2;                             // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int M = p.M, N = p.N, K = p.K;
  const int tiles_m = (M + kBM - 1) / kBM;
  const int tiles_n = (N + kBN - 1) / kBN;
  const int num_tiles = tiles_m * tiles_n;
  const int G = K >> 6;

  if (threadIdx.x == 0) {
    // the next kernel on the stream may launch now; it waits for this grid's
    // completion before it touches anything this grid reads or writes
    dev::griddep_launch_dependents();
    for (int s = 0; s < kPStages; ++s) {
      dev::mbar_init(&pfull[s], 1);
      dev::mbar_init(&pempty[s], kConvWarps);
    }
    for (int s = 0; s < kOStages; ++s) {
      dev::mbar_init(&ofull[s], kConvWarps);
      dev::mbar_init(&oempty[s], 1);
    }
    dev::mbar_init(bfull, 1);
    dev::mbar_init(bempty, 1);
    for (int b = 0; b < 2; ++b) {
      dev::mbar_init(&acc_full[b], 1);
      dev::mbar_init(&acc_empty[b], kEpiWarps);
    }
    dev::mbar_init(drain, 1);
    *abort_flag = 0;
    dev::fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    dev::tmem_alloc(tmem_slot, kTmemCols);
    dev::tmem_relinquish();
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    dev::setmaxnreg_dec<kRegsCtl>();
    if (lane == 0) {
      dev::tma_prefetch_desc(&tm_a);
      dev::tma_prefetch_desc(&tm_b);
      if (p.branch) {
        dev::tma_prefetch_desc(&tm_xl);
        dev::tma_prefetch_desc(&tm_l2);
      }
      if (p.lora) {
        dev::tma_prefetch_desc(&tm_xla);
        dev::tma_prefetch_desc(&tm_l2a);
      }
      const int lora_g = min(kLoraLoadG, G - 1);
      int it = 0, bc = 0;                           // bc: branch-buffer loads so far
      bool ok = true, deps_ready = false;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m0 = (tile % tiles_m) * kBM;
        const int n0 = (tile / tiles_m) * kBN;
        if (p.branch) {
          if (!dev::mbar_wait(bempty, ((uint32_t)bc & 1u) ^ 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x301);
            break;
          }
          dev::mbar_arrive_expect_tx(bfull, kBrBytes);
          dev::tma_load_2d(brbuf + kBrABytes, &tm_l2, bfull, 0, n0);
          if (!deps_ready) {
            dev::griddep_wait();
            deps_ready = true;
          }
          dev::tma_load_2d(brbuf, &tm_xl, bfull, 0, m0);
          ++bc;
        }
        for (int g = 0; g < G; ++g, ++it) {
          const int s = it % kPStages;
          if (!dev::mbar_wait(&pempty[s], ((uint32_t)(it / kPStages) & 1u) ^ 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x302);
            ok = false;
            break;
          }
          uint8_t* st = pring + s * kPStageBytes;
          dev::mbar_arrive_expect_tx(&pfull[s], kBM * 32 + kBN * 32 + kBM * 2 + kBN * 2);
          // weights first: they do not depend on the preceding kernel
          dev::tma_load_2d(st + kPB, &tm_b, &pfull[s], g * 32, n0);
          dev::bulk_load(st + kPSB, p.sb + (size_t)g * p.npad + n0, kBN * 2, &pfull[s]);
          if (!deps_ready) {
            dev::griddep_wait();
            deps_ready = true;
          }
          dev::tma_load_2d(st + kPA, &tm_a, &pfull[s], g * 32, m0);
          dev::bulk_load(st + kPSA, p.sa + (size_t)g * p.mpad + m0, kBM * 2, &pfull[s]);
          if (p.lora && g == lora_g) {
            // the adapter's tiles, once the tile's branch MMAs have read the buffer
            if (!dev::mbar_wait(bempty, ((uint32_t)bc & 1u) ^ 1u, abort_flag, p.budget_ns)) {
              record_error(p.err, abort_flag, 0x306);
              ok = false;
              break;
            }
            dev::mbar_arrive_expect_tx(bfull, kBrBytes);
            dev::tma_load_2d(brbuf + kBrABytes, &tm_l2a, bfull, 0, n0);
            dev::tma_load_2d(brbuf, &tm_xla, bfull, 0, m0);
            ++bc;
          }
        }
      }
      // every exit path waits for the preceding grid, so that this grid never
      // completes before it (the next launch on the stream waits only for this one)
      if (!deps_ready) dev::griddep_wait();
      for (int j = max(0, it - kPStages); j < it; ++j)
        if (!dev::mbar_wait(&pfull[j % kPStages], (uint32_t)(j / kPStages) & 1u, abort_flag, p.budget_ns)) break;
      if (bc > 0) dev::mbar_wait(bfull, (uint32_t)(bc - 1) & 1u, abort_flag, p.budget_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    dev::setmaxnreg_dec<kRegsCtl>();
    if (lane == 0) {
      const uint32_t id16 = idesc_f16(kBM, kBN);
      const uint32_t idbf = dev::idesc_bf16(kBM, kBN);
      const int lora_g = min(kLoraMmaG, G - 1);
      int it = 0, tcount = 0, bc = 0;               // bc: branch-buffer phases consumed
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tcount) {
        const int ab = tcount & 1;
        const uint32_t dacc = tmem + (uint32_t)(ab * 256);
        if (!dev::mbar_wait(&acc_empty[ab], ((uint32_t)(tcount >> 1) & 1u) ^ 1u, abort_flag, p.budget_ns)) {
          record_error(p.err, abort_flag, 0x303);
          break;
        }
        dev::tc_fence_after();
        uint32_t accumulate = 0;
        if (p.branch) {
          if (!dev::mbar_wait(bfull, (uint32_t)bc & 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x304);
            break;
          }
          ++bc;
          dev::tc_fence_after();
          const uint32_t a0 = dev::smem_u32(brbuf);
          const uint32_t b0 = a0 + kBrABytes;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            dev::mma_bf16(dacc, dev::smem_desc(a0 + 32 * j, 16, 512, 4), dev::smem_desc(b0 + 32 * j, 16, 512, 4),
                          idbf, accumulate);
            accumulate = 1;
          }
          dev::tc_commit(bempty);
        }
        for (int g = 0; g < G; ++g, ++it) {
          const int s = it % kOStages;
          if (!dev::mbar_wait(&ofull[s], (uint32_t)(it / kOStages) & 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x305);
            ok = false;
            break;
          }
          dev::tc_fence_after();
          const uint32_t a0 = dev::smem_u32(oring + s * kOStageBytes);
          const uint32_t b0 = a0 + kOABytes;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            dev::mma_bf16(dacc, dev::smem_desc(a0 + 32 * j, 16, 1024, 2), dev::smem_desc(b0 + 32 * j, 16, 1024, 2),
                          id16, accumulate);
            accumulate = 1;
          }
          dev::tc_commit(&oempty[s]);
          if (p.lora && g == lora_g) {
            if (!dev::mbar_wait(bfull, (uint32_t)bc & 1u, abort_flag, p.budget_ns)) {
              record_error(p.err, abort_flag, 0x307);
              ok = false;
              break;
            }
            ++bc;
            dev::tc_fence_after();
            const uint32_t la = dev::smem_u32(brbuf);
            const uint32_t lb = la + kBrABytes;
#pragma unroll
            for (int j = 0; j < 2; ++j)
              dev::mma_bf16(dacc, dev::smem_desc(la + 32 * j, 16, 512, 4), dev::smem_desc(lb + 32 * j, 16, 512, 4),
                            idbf, 1u);
            dev::tc_commit(bempty);
          }
        }
        if (!ok) break;
        dev::tc_commit(&acc_full[ab]);
      }
      // Wait until every MMA this thread issued has completed.
      dev::tc_commit(drain);
      dev::mbar_wait(drain, 0, abort_flag, p.budget_ns);
    }
  } else if (warp >= kConvWarp0) {
    // ------------------------------------------------------------ converters
    dev::setmaxnreg_dec<kRegsConv>();
    const int ct = threadIdx.x - kConvWarp0 * 32;   // 0 .. kConvThreads - 1
    const float xs = p.xscale;                      // 2^-ex
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      for (int g = 0; g < G; ++g, ++it) {
        const int ps = it % kPStages, os = it % kOStages;
        const bool got =
            dev::mbar_wait(&pfull[ps], (uint32_t)(it / kPStages) & 1u, abort_flag, p.budget_ns) &&
            dev::mbar_wait(&oempty[os], ((uint32_t)(it / kOStages) & 1u) ^ 1u, abort_flag, p.budget_ns);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) record_error(p.err, abort_flag, 0x306);
          ok = false;
          break;
        }
        const uint8_t* st = pring + ps * kPStageBytes;
        // unit u = ct + kConvThreads i: operand row u / 4 (rows 0-127 of A, then
        // B's 256), 16 codes (8 bytes) at quarter u % 4 of the row (a warp's
        // units are all of A or all of B)
        uint2 w[kUnitsPerThread];
        __half2 s2[kUnitsPerThread];
#pragma unroll
        for (int i = 0; i < kUnitsPerThread; ++i) {
          const int u = ct + kConvThreads * i;
          const int row = u >> 2, q = u & 3;
          if (row < kBM) {
            w[i] = *reinterpret_cast<const uint2*>(st + kPA + row * 32 + q * 8);
            const uint16_t sb = *reinterpret_cast<const uint16_t*>(st + kPSA + row * 2);
            const float sf = fminf(__uint_as_float((uint32_t)sb << 16) * xs, 8192.0f);
            s2[i] = __float2half2_rn(sf);
          } else {
            const int r = row - kBM;
            w[i] = *reinterpret_cast<const uint2*>(st + kPB + r * 32 + q * 8);
            const __half h = *reinterpret_cast<const __half*>(st + kPSB + r * 2);
            s2[i] = __half2half2(h);
          }
        }
        // the staging slot has been read
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(&pempty[ps]);
        uint8_t* ob = oring + os * kOStageBytes;
#pragma unroll
        for (int i = 0; i < kUnitsPerThread; ++i) {
          const int u = ct + kConvThreads * i;
          const int row = u >> 2, q = u & 3;
          const bool is_a = row < kBM;
          const int r = is_a ? row : row - kBM;
          uint8_t* base = ob + (is_a ? 0 : kOABytes) + r * 128;
          uint32_t v0[4], v1[4];
          dequant_word(w[i].x, s2[i], v0);
          dequant_word(w[i].y, s2[i], v1);
          // 128-byte swizzle: 16-byte chunk c of row r sits at c ^ (r & 7)
          *reinterpret_cast<uint4*>(base + (((2 * q) ^ (r & 7)) << 4)) = make_uint4(v0[0], v0[1], v0[2], v0[3]);
          *reinterpret_cast<uint4*>(base + (((2 * q + 1) ^ (r & 7)) << 4)) = make_uint4(v1[0], v1[1], v1[2], v1[3]);
        }
        dev::fence_async_shared();                    // the tensor core reads these tiles
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(&ofull[os]);
      }
    }
  } else if (warp < kEpiWarp0) {
    dev::setmaxnreg_dec<kRegsCtl>();                 // idle warps of the first warpgroup
  } else {
    // ------------------------------------------------------------ epilogue
    dev::setmaxnreg_inc<kRegsEpi>();
    const int q = warp & 3;                          // TMEM lane quarter of this warp
    uint8_t* wbuf = epi_buf + (warp - kEpiWarp0) * kEpiWarpBytes;
    if (lane == 0) dev::tma_prefetch_desc(&tm_y);
    int tcount = 0, chunk = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tcount) {
      const int m0 = (tile % tiles_m) * kBM;
      const int n0 = (tile / tiles_m) * kBN;
      const int ab = tcount & 1;
      const bool got = dev::mbar_wait(&acc_full[ab], (uint32_t)(tcount >> 1) & 1u, abort_flag, p.budget_ns);
      if (!__all_sync(0xffffffffu, got)) {          // warp-uniform exit (tcgen05.ld is warp-collective)
        if (lane == 0) record_error(p.err, abort_flag, 0x307);
        break;
      }
      __syncwarp();
      dev::tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(ab * 256);
      uint32_t va[32], vb[32];
      dev::tmem_load_32cols(taddr, va);
      dev::tmem_load_wait(va);
#pragma unroll
      for (int c = 0; c < 8; ++c, ++chunk) {
        uint32_t (&cur)[32] = (c & 1) ? vb : va;
        uint32_t (&nxt)[32] = (c & 1) ? va : vb;
        if (c + 1 < 8) dev::tmem_load_32cols(taddr + (uint32_t)((c + 1) * 32), nxt);
        // this chunk's 32 bias values (uniform addresses: broadcast loads)
        float bias[32];
#pragma unroll
        for (int f = 0; f < 8; ++f) {
          const int col = n0 + c * 32 + 4 * f;
          const float4 b4 = col < N ? __ldg(reinterpret_cast<const float4*>(p.bias + col))
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
          bias[4 * f] = b4.x;
          bias[4 * f + 1] = b4.y;
          bias[4 * f + 2] = b4.z;
          bias[4 * f + 3] = b4.w;
        }
        // the buffer of this chunk was last read by the store issued two chunks ago
        if (lane == 0) dev::bulk_wait_group_read<1>();
        __syncwarp();
        uint8_t* buf = wbuf + (chunk & 1) * kEpiBufBytes;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t packed[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i0 = j * 8 + 2 * e;
            float y0 = p.alpha * __uint_as_float(cur[i0]) + bias[i0];
            float y1 = p.alpha * __uint_as_float(cur[i0 + 1]) + bias[i0 + 1];
            if (p.gelu) {
              y0 = dev::gelu_tanh(y0);
              y1 = dev::gelu_tanh(y1);
            }
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
            packed[e] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          // 64-byte swizzle: 16-byte chunk j of row `lane` sits at j ^ ((lane >> 1) & 3)
          *reinterpret_cast<uint4*>(buf + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
              make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
        dev::fence_async_shared();                    // make the writes visible to the TMA engine
        __syncwarp();
        if (lane == 0) {
          dev::tma_store_2d(&tm_y, buf, n0 + c * 32, m0 + q * 32);
          dev::bulk_commit_group();
        }
        if (c + 1 < 8) dev::tmem_load_wait(nxt);
        if (c == 6) {
          // the last chunk is in registers: hand the accumulator back to the MMA warp
          dev::tc_fence_before();
          __syncwarp();
          if (lane == 0) dev::mbar_arrive(&acc_empty[ab]);
        }
      }
      __syncwarp();
    }
    if (lane == 0) dev::bulk_wait_group_all();
  }

  __syncwarp();                                      // single-lane roles rejoin their warps first
  dev::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    dev::tc_fence_after();
    dev::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_k2_int4(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const CUtensorMap& tm_xl,
                           const CUtensorMap& tm_l2, const CUtensorMap& tm_y, const CUtensorMap& tm_xla,
                           const CUtensorMap& tm_l2a, const K2Int4Params& p, int num_sms, cudaStream_t stream) {
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(k2_int4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    // the warpgroups' register budgets fit the launch allocation
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, k2_int4_kernel);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    configured_device = dev;
  }
  const int tiles = ((p.M + kBM - 1) / kBM) * ((p.N + kBN - 1) / kBN);
  const int grid = tiles < num_sms ? tiles : num_sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k2_int4_kernel, tm_a, tm_b, tm_xl, tm_l2, tm_y, tm_xla, tm_l2a, p);
}

}  // namespace svdq
