// K2 for the INT4 variant on CTA pairs: the group-64 INT4 GEMM with exact FP16
// dequantization of the single-CTA kernel (same arithmetic, same results),
// computed by two CTAs (one cluster) per 256 x 256 output tile with the
// fifth-generation tensor core's pair mode (tcgen05 cta_group::2).
//
// Why pairs: the single-CTA kernel is bound by its converter warps, which turn
// every (A tile, B tile) pair's packed codes into FP16 operand tiles.  In pair
// mode each CTA holds its own 128 rows of A and only half (128 rows) of the
// 256-row B tile; the two SMs' tensor cores share the B halves.  A CTA then
// converts 256 rows per group instead of 384 for the same flops.  On this part
// it measures slower than the single-CTA kernel all the same (pair MMAs deliver
// less per SM than single-CTA ones), so it runs only when selected.
//
// Layout of the work (CTA rank r of the pair):
//   both CTAs   warp 0 producer: packed A codes of rows m0 + 128 r, packed B
//               codes of rows n0 + 128 r and their scales into the staging
//               ring; per tile the XL rows and the (L2b / alpha)^T rows of this
//               CTA into the branch buffer.  Warps 8-23 converters: staging ->
//               FP16 operand tiles in this CTA's shared memory; rank 1's
//               converters report to rank 0's barrier (remote arrives).
//               Warps 4-7 epilogue of this CTA's 128 accumulator rows.
//   rank 0      warp 1: MMA issuer (pair MMAs, M = 256, N = 256).
//   rank 1      warp 1: forwards "branch operands landed" to rank 0.
// Rank 0's commits arrive on both CTAs' barriers (multicast commit).  Every wait
// is bounded (sm100.cuh).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100.cuh"

namespace svdq {

namespace {

constexpr int kBM = 128;                             // rows of A per CTA
constexpr int kPM = 256;                             // rows per pair tile
constexpr int kBN = 256;                             // columns per tile
constexpr int kBNh = 128;                            // rows of B per CTA
constexpr int kPStages = 3;                          // staging ring (packed codes + scales)
constexpr int kOStages = 4;                          // operand ring (FP16 tiles)
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
// conversion units of a group: 16 codes (a quarter row) of this CTA's 128 rows
// of A and 128 rows of B
constexpr int kUnits = (kBM + kBNh) * 4;
constexpr int kUnitsPerThread = kUnits / kConvThreads;
static_assert(kUnits % kConvThreads == 0 && (kBM * 4) % 32 == 0, "converter work split");

// staging stage: A codes, B codes, A scales, B scales
constexpr int kPA = 0;
constexpr int kPB = kPA + kBM * 32;                  // 4096
constexpr int kPSA = kPB + kBNh * 32;                // 8192
constexpr int kPSB = kPSA + kBM * 2;                 // 8448
constexpr int kPStageBytes = 9 * 1024;
static_assert(kPSB + kBNh * 2 <= kPStageBytes, "staging stage");
// operand stage: A 128 x 64 FP16, B 128 x 64 FP16 (128-byte rows)
constexpr int kOABytes = kBM * 128;
constexpr int kOBBytes = kBNh * 128;
constexpr int kOStageBytes = kOABytes + kOBBytes;    // 32 KiB
// branch buffer: XL 128 x 32 BF16 and (L2b / alpha)^T 128 x 32 BF16 (64-byte rows)
constexpr int kBrABytes = kBM * 64;
constexpr int kBrBytes = kBrABytes + kBNh * 64;      // 16 KiB
constexpr int kEpiBufBytes = 32 * 64;                // one 32 x 32 BF16 output chunk
constexpr int kEpiWarpBytes = 2 * kEpiBufBytes;
constexpr int kSmemBytes =
    kOStages * kOStageBytes + kBrBytes + kPStages * kPStageBytes + kEpiWarps * kEpiWarpBytes + 256 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory per block");
constexpr int kTmemCols = 512;
constexpr uint16_t kBoth = 3, kLeader = 1;   // multicast masks (cluster ranks)

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

__global__ void __launch_bounds__(kThreads, 1)
    k2_int4_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_xl, const __grid_constant__ CUtensorMap tm_l2,
                   const __grid_constant__ CUtensorMap tm_y, K2Int4Params p) {
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
  uint64_t* pbfull = bempty + 1;                                  // rank 0: rank 1's branch operands landed
  uint64_t* acc_full = pbfull + 1;                                // [2]
  uint64_t* acc_empty = acc_full + 2;                             // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int M = p.M, N = p.N, K = p.K;
  const uint32_t rank = dev::cluster_rank();
  const bool leader = rank == 0;
  const int tiles_m = (M + kPM - 1) / kPM;
  const int tiles_n = (N + kBN - 1) / kBN;
  const int num_tiles = tiles_m * tiles_n;
  const int pair_id = (int)blockIdx.x >> 1, npairs = (int)gridDim.x >> 1;
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
      dev::mbar_init(&ofull[s], 2 * kConvWarps);      // rank 0: the converters of both CTAs
      dev::mbar_init(&oempty[s], 1);
    }
    dev::mbar_init(bfull, 1);
    dev::mbar_init(bempty, 1);
    dev::mbar_init(pbfull, 1);
    for (int b = 0; b < 2; ++b) {
      dev::mbar_init(&acc_full[b], 1);
      dev::mbar_init(&acc_empty[b], 2 * kEpiWarps);   // rank 0: the epilogues of both CTAs
    }
    dev::mbar_init(drain, 1);
    *abort_flag = 0;
    dev::fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    dev::tmem_alloc_pair(tmem_slot, kTmemCols);
    dev::tmem_relinquish_pair();
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::cluster_sync();                               // barriers and TMEM of both CTAs exist
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
      int it = 0, tcount = 0;
      bool ok = true, deps_ready = false;
      for (int tile = pair_id; tile < num_tiles && ok; tile += npairs, ++tcount) {
        const int m0 = (tile % tiles_m) * kPM + kBM * (int)rank;     // this CTA's rows of A
        const int n0 = (tile / tiles_m) * kBN + kBNh * (int)rank;    // and of B
        const bool sa_rows = m0 < p.mpad;     // the activation scales cover these rows (else they stay
                                              // stale: their results are never stored)
        if (p.branch) {
          if (!dev::mbar_wait(bempty, ((uint32_t)tcount & 1u) ^ 1u, abort_flag, p.budget_ns)) {
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
        }
        for (int g = 0; g < G; ++g, ++it) {
          const int s = it % kPStages;
          if (!dev::mbar_wait(&pempty[s], ((uint32_t)(it / kPStages) & 1u) ^ 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x302);
            ok = false;
            break;
          }
          uint8_t* st = pring + s * kPStageBytes;
          dev::mbar_arrive_expect_tx(&pfull[s], kBM * 32 + kBNh * 32 + (sa_rows ? kBM * 2 : 0) + kBNh * 2);
          // weights first: they do not depend on the preceding kernel
          dev::tma_load_2d(st + kPB, &tm_b, &pfull[s], g * 32, n0);
          dev::bulk_load(st + kPSB, p.sb + (size_t)g * p.npad + n0, kBNh * 2, &pfull[s]);
          if (!deps_ready) {
            dev::griddep_wait();
            deps_ready = true;
          }
          dev::tma_load_2d(st + kPA, &tm_a, &pfull[s], g * 32, m0);
          if (sa_rows) dev::bulk_load(st + kPSA, p.sa + (size_t)g * p.mpad + m0, kBM * 2, &pfull[s]);
        }
      }
      // every exit path waits for the preceding grid, so that this grid never
      // completes before it (the next launch on the stream waits only for this one)
      if (!deps_ready) dev::griddep_wait();
      for (int j = max(0, it - kPStages); j < it; ++j)
        if (!dev::mbar_wait(&pfull[j % kPStages], (uint32_t)(j / kPStages) & 1u, abort_flag, p.budget_ns)) break;
      if (p.branch && tcount > 0) dev::mbar_wait(bfull, (uint32_t)(tcount - 1) & 1u, abort_flag, p.budget_ns);
    }
  } else if (warp == 1 && !leader) {
    // ------------------------------------------------------------ rank 1: forward "branch operands landed"
    dev::setmaxnreg_dec<kRegsCtl>();
    if (lane == 0 && p.branch) {
      const uint32_t pb0 = dev::map_to_rank(pbfull, 0);
      int tcount = 0;
      for (int tile = pair_id; tile < num_tiles; tile += npairs, ++tcount) {
        if (!dev::mbar_wait(bfull, (uint32_t)tcount & 1u, abort_flag, p.budget_ns)) {
          record_error(p.err, abort_flag, 0x308);
          break;
        }
        dev::mbar_arrive_remote(pb0);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ rank 0: MMA issuer
    dev::setmaxnreg_dec<kRegsCtl>();
    if (lane == 0) {
      const uint32_t id16 = idesc_f16(kPM, kBN);
      const uint32_t idbf = dev::idesc_bf16(kPM, kBN);
      int it = 0, tcount = 0;
      bool ok = true;
      for (int tile = pair_id; tile < num_tiles && ok; tile += npairs, ++tcount) {
        const int ab = tcount & 1;
        const uint32_t dacc = tmem + (uint32_t)(ab * 256);
        if (!dev::mbar_wait_cluster(&acc_empty[ab], ((uint32_t)(tcount >> 1) & 1u) ^ 1u, abort_flag, p.budget_ns)) {
          record_error(p.err, abort_flag, 0x303);
          break;
        }
        dev::tc_fence_after();
        uint32_t accumulate = 0;
        if (p.branch) {
          if (!dev::mbar_wait(bfull, (uint32_t)tcount & 1u, abort_flag, p.budget_ns) ||
              !dev::mbar_wait_cluster(pbfull, (uint32_t)tcount & 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x304);
            break;
          }
          dev::tc_fence_after();
          const uint32_t a0 = dev::smem_u32(brbuf);
          const uint32_t b0 = a0 + kBrABytes;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            dev::mma_f16_pair(dacc, dev::smem_desc(a0 + 32 * j, 16, 512, 4), dev::smem_desc(b0 + 32 * j, 16, 512, 4),
                              idbf, accumulate);
            accumulate = 1;
          }
          dev::tc_commit_pair(bempty, kBoth);
        }
        for (int g = 0; g < G; ++g, ++it) {
          const int s = it % kOStages;
          if (!dev::mbar_wait_cluster(&ofull[s], (uint32_t)(it / kOStages) & 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x305);
            ok = false;
            break;
          }
          dev::tc_fence_after();
          const uint32_t a0 = dev::smem_u32(oring + s * kOStageBytes);
          const uint32_t b0 = a0 + kOABytes;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            dev::mma_f16_pair(dacc, dev::smem_desc(a0 + 32 * j, 16, 1024, 2),
                              dev::smem_desc(b0 + 32 * j, 16, 1024, 2), id16, accumulate);
            accumulate = 1;
          }
          dev::tc_commit_pair(&oempty[s], kBoth);
        }
        if (!ok) break;
        dev::tc_commit_pair(&acc_full[ab], kBoth);
      }
      // Wait until every pair operation this thread issued has completed.
      dev::tc_commit_pair(drain, kLeader);
      dev::mbar_wait(drain, 0, abort_flag, p.budget_ns);
    }
  } else if (warp >= kConvWarp0) {
    // ------------------------------------------------------------ converters
    dev::setmaxnreg_dec<kRegsConv>();
    const int ct = threadIdx.x - kConvWarp0 * 32;   // 0 .. kConvThreads - 1
    const float xs = p.xscale;                      // 2^-ex
    const uint32_t ofull0 = dev::map_to_rank(ofull, 0);
    int it = 0;
    bool ok = true;
    for (int tile = pair_id; tile < num_tiles && ok; tile += npairs) {
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
        if (lane == 0) dev::mbar_arrive_remote(ofull0 + 8u * (uint32_t)os);   // rank 0's barrier
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
    const uint32_t acc_empty0 = dev::map_to_rank(acc_empty, 0);
    int tcount = 0, chunk = 0;
    for (int tile = pair_id; tile < num_tiles; tile += npairs, ++tcount) {
      const int m0 = (tile % tiles_m) * kPM + kBM * (int)rank;
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
        if (lane == 0 && m0 + q * 32 < M) {        // rows past M (a pair tile's tail): nothing to store
          dev::tma_store_2d(&tm_y, buf, n0 + c * 32, m0 + q * 32);
          dev::bulk_commit_group();
        }
        if (c + 1 < 8) dev::tmem_load_wait(nxt);
        if (c == 6) {
          // the last chunk is in registers: hand the accumulator back to the MMA warp
          dev::tc_fence_before();
          __syncwarp();
          if (lane == 0) dev::mbar_arrive_remote(acc_empty0 + 8u * (uint32_t)ab);   // rank 0's barrier
        }
      }
      __syncwarp();
    }
    if (lane == 0) dev::bulk_wait_group_all();
  }

  // Neither CTA leaves (nor frees TMEM) while the pair's operations may still
  // read its shared memory or write its TMEM.
  __syncwarp();                                      // single-lane roles rejoin their warps first
  dev::tc_fence_before();
  __syncthreads();
  dev::cluster_sync();
  if (warp == 1) {
    __syncwarp();
    dev::tc_fence_after();
    dev::tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace

int k2_int4_pair_rows_b() { return kBNh; }

cudaError_t launch_k2_int4_pair(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const CUtensorMap& tm_xl,
                                const CUtensorMap& tm_l2, const CUtensorMap& tm_y, const K2Int4Params& p,
                                int num_sms, cudaStream_t stream) {
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(k2_int4_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    // the warpgroups' register budgets fit the launch allocation
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, k2_int4_pair_kernel);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    configured_device = dev;
  }
  const int tiles = ((p.M + kPM - 1) / kPM) * ((p.N + kBN - 1) / kBN);
  const int pairs = tiles < num_sms / 2 ? tiles : num_sms / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, k2_int4_pair_kernel, tm_a, tm_b, tm_xl, tm_l2, tm_y, p);
}

}  // namespace svdq
