// K2 for W8A8: INT8 GEMM with exact int32 accumulation, the rank-16 low-rank
// branch in an FP32 accumulator of its own, per-token and per-channel scales in
// the epilogue.
//
// SOTA-314 practice page, "Do this": rank 16 at 8 bits.  With one scale per
// token (s_x) and per output channel (s_w) the product of the codes is exact in
// int32 (|c| <= 127, K < 2^17), so the layer is
//
//   acc_i = sum_k c_x c_w                        (tcgen05 kind::i8, K = 32 per MMA)
//   acc_b = XL L2b                               (one BF16 MMA, K = 16: the rank)
//   Y     = bf16([gelu](s_x s_w acc_i + acc_b + b))
//
// A and B types differ from the branch's, so the branch cannot share the
// integer accumulator: TMEM columns 0-255 hold acc_i, 256-511 acc_b.
//
// Structure (one CTA per SM, persistent over 128 x 256 output tiles, 16 warps):
//   warp 0     activation producer: per stage of 128 K the 128 x 128-byte code
//              block the first kernel wrote in this layout (one bulk copy);
//              per tile the XL rows into the branch buffer.
//   warp 2     weight producer: per stage the 256 x 128-byte weight block (one
//              bulk copy, tiled when the layer is prepared); per tile the L2b^T
//              rows into the branch buffer.
//   warp 1     allocates TMEM and issues the MMAs.
//   warps 8-15 epilogue: both accumulators into registers, handed back at
//              once; scales, bias, [GELU], BF16, TMA stores from swizzled
//              shared memory, overlapping the next tile's mainloop.
// Pipelines are mbarrier rings; every wait is bounded (sm100.cuh).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100.cuh"

namespace svdq {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBKBytes = 128;                // int8 codes per operand row per stage
constexpr int kStages = 3;
constexpr uint32_t kSwz = 2u;                // descriptor layout: 128-byte swizzle
constexpr uint32_t kSwzAtom = 8u * kBKBytes;
constexpr int kEpiWarps = 8;
constexpr int kProdA = 0, kMmaWarp = 1, kProdB = 2, kEpiWarp0 = 8;
constexpr int kThreads = 16 * 32;
constexpr int kRegsCtl = 56, kRegsIdle = 72, kRegsEpi = 192;
static_assert(128 * kRegsCtl + 128 * kRegsIdle + 256 * kRegsEpi == kThreads * 128, "register split");
constexpr int kABytes = kBM * kBKBytes;      // 16 KiB
constexpr int kBBytes = kBN * kBKBytes;      // 32 KiB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kBrXL = kBM * 64;              // XL rows (32 BF16, the rank in the first 16)
constexpr int kBrBytes = kBrXL + kBN * 64;
constexpr int kEpiBufBytes = 32 * 64;
constexpr int kEpiWarpBytes = 2 * kEpiBufBytes + 1024;   // two chunk buffers + 128 bias + 128 s_w floats
constexpr int kSmemBytes = kStages * kStageBytes + kBrBytes + kEpiWarps * kEpiWarpBytes + 1024 + 256;
static_assert(kSmemBytes <= 232448, "shared memory per block");
constexpr int kTmemCols = 512;
constexpr int kBranchCol = 256;

// Instruction descriptor: signed INT8 x signed INT8 -> S32, both operands K-major.
constexpr uint32_t idesc_i8(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void record_error(int* err, volatile int* abort_flag, int code) {
  atomicCAS(err, 0, code);
  *abort_flag = 1;
}

__global__ void __launch_bounds__(kThreads, 1)
    k2_int8_kernel(const __grid_constant__ CUtensorMap tm_xl, const __grid_constant__ CUtensorMap tm_l2,
                   const __grid_constant__ CUtensorMap tm_y, K2Int8Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* brbuf = smem + kStages * kStageBytes;
  uint8_t* epi_buf = brbuf + kBrBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_buf + kEpiWarps * kEpiWarpBytes);
  uint64_t* empty = full + kStages;
  uint64_t* br_full = empty + kStages;
  uint64_t* br_empty = br_full + 1;
  uint64_t* acc_full = br_empty + 1;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int M = p.M, N = p.N, K = p.K;
  const int tiles_m = (M + kBM - 1) / kBM;
  const int tiles_n = (N + kBN - 1) / kBN;
  const int num_tiles = tiles_m * tiles_n;
  const int ktiles = (K + 127) / 128;             // stages of 128 K (K is a multiple of 64)

  if (threadIdx.x == 0) {
    dev::griddep_launch_dependents();
    for (int s = 0; s < kStages; ++s) {
      dev::mbar_init(&full[s], 2);                  // the two producers
      dev::mbar_init(&empty[s], 1);
    }
    dev::mbar_init(br_full, 2);
    dev::mbar_init(br_empty, 1);
    dev::mbar_init(acc_full, 1);
    dev::mbar_init(acc_empty, kEpiWarps);
    dev::mbar_init(drain, 1);
    *abort_flag = 0;
    dev::fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    __syncwarp();
    dev::tmem_alloc(tmem_slot, kTmemCols);
    dev::tmem_relinquish();
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProdA || warp == kProdB) {
    // ------------------------------------------------------------ producers
    dev::setmaxnreg_dec<kRegsCtl>();
    if (lane == 0) {
      const bool pa = warp == kProdA;
      if (p.branch) dev::tma_prefetch_desc(pa ? &tm_xl : &tm_l2);
      if (pa) dev::griddep_wait();                  // the codes, scales and XL come from the first kernels
      int it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tcount) {
        const int m0 = (tile % tiles_m) * kBM;
        const int n0 = (tile / tiles_m) * kBN;
        if (p.branch) {
          if (!dev::mbar_wait(br_empty, ((uint32_t)tcount & 1u) ^ 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x501);
            ok = false;
            break;
          }
          if (pa) {
            dev::mbar_arrive_expect_tx(br_full, kBrXL);
            dev::tma_load_2d(brbuf, &tm_xl, br_full, 0, m0);
          } else {
            dev::mbar_arrive_expect_tx(br_full, kBN * 64);
            dev::tma_load_2d(brbuf + kBrXL, &tm_l2, br_full, 0, n0);
          }
        }
        for (int kt = 0; kt < ktiles; ++kt, ++it) {
          const int s = it % kStages;
          if (!dev::mbar_wait(&empty[s], ((uint32_t)(it / kStages) & 1u) ^ 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x502);
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kStageBytes;
          if (pa) {
            dev::mbar_arrive_expect_tx(&full[s], (uint32_t)kABytes);
            dev::bulk_load(st, p.acodes + ((size_t)(m0 >> 7) * (size_t)ktiles + (size_t)kt) * kABytes, kABytes,
                           &full[s]);
          } else {
            dev::mbar_arrive_expect_tx(&full[s], (uint32_t)kBBytes);
            dev::bulk_load(st + kABytes, p.wq + ((size_t)(n0 >> 8) * (size_t)ktiles + (size_t)kt) * kBBytes, kBBytes,
                           &full[s]);
          }
        }
      }
      // Do not leave while copies into this CTA's shared memory are in flight.
      for (int j = max(0, it - kStages); j < it; ++j)
        if (!dev::mbar_wait(&full[j % kStages], (uint32_t)(j / kStages) & 1u, abort_flag, p.budget_ns)) break;
      if (p.branch && tcount > 0) dev::mbar_wait(br_full, (uint32_t)(tcount - 1) & 1u, abort_flag, p.budget_ns);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    dev::setmaxnreg_dec<kRegsCtl>();
    if (lane == 0) {
      const uint32_t idesc8 = idesc_i8(kBM, kBN);
      const uint32_t idesc_h = dev::idesc_bf16(kBM, kBN);
      int it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tcount) {
        if (!dev::mbar_wait(acc_empty, ((uint32_t)tcount & 1u) ^ 1u, abort_flag, p.budget_ns)) {
          record_error(p.err, abort_flag, 0x503);
          ok = false;
          break;
        }
        dev::tc_fence_after();
        if (p.branch) {
          if (!dev::mbar_wait(br_full, (uint32_t)tcount & 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x504);
            ok = false;
            break;
          }
          dev::tc_fence_after();
          // rank 16: one K = 16 MMA over the first 32 bytes of each row
          const uint32_t a0 = dev::smem_u32(brbuf);
          dev::mma_bf16(tmem + kBranchCol, dev::smem_desc(a0, 16, 512, 4), dev::smem_desc(a0 + kBrXL, 16, 512, 4),
                        idesc_h, 0u);
          dev::tc_commit(br_empty);
        }
        uint32_t accumulate = 0;
        for (int kt = 0; kt < ktiles; ++kt, ++it) {
          const int s = it % kStages;
          if (!dev::mbar_wait(&full[s], (uint32_t)(it / kStages) & 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x505);
            ok = false;
            break;
          }
          dev::tc_fence_after();
          const int nks = min(4, (K - kt * 128) / 32);  // k-steps of 32 in this stage
          const uint32_t a0 = dev::smem_u32(smem + s * kStageBytes);
          const uint32_t b0 = a0 + kABytes;
          for (int j = 0; j < nks; ++j) {
            mma_i8(tmem, dev::smem_desc(a0 + 32 * j, 16, kSwzAtom, kSwz), dev::smem_desc(b0 + 32 * j, 16, kSwzAtom, kSwz),
                   idesc8, accumulate);
            accumulate = 1;
          }
          dev::tc_commit(&empty[s]);
        }
        if (!ok) break;
        dev::tc_commit(acc_full);
      }
      dev::tc_commit(drain);
      dev::mbar_wait(drain, 0, abort_flag, p.budget_ns);
    }
  } else if (warp < kEpiWarp0) {
    if (warp < 4) dev::setmaxnreg_dec<kRegsCtl>();  // idle warps of the first two warpgroups
    else dev::setmaxnreg_dec<kRegsIdle>();
  } else {
    // ------------------------------------------------------------ epilogue
    dev::setmaxnreg_inc<kRegsEpi>();
    const int q = warp & 3;                          // TMEM lane quarter
    const int half = (warp - kEpiWarp0) >> 2;       // which 128 of the 256 columns
    uint8_t* wbuf = epi_buf + (warp - kEpiWarp0) * kEpiWarpBytes;
    float* bias_s = reinterpret_cast<float*>(wbuf + 2 * kEpiBufBytes);
    float* sw_s = bias_s + 128;
    if (lane == 0) dev::tma_prefetch_desc(&tm_y);
    int tcount = 0, chunk = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tcount) {
      const int m0 = (tile % tiles_m) * kBM;
      const int n0 = (tile / tiles_m) * kBN + half * 128;
      {
        const int col = n0 + lane * 4;
        float4 b4 = make_float4(0.f, 0.f, 0.f, 0.f), w4 = b4;
        if (col < N) {
          b4 = __ldg(reinterpret_cast<const float4*>(p.bias + col));
          w4 = __ldg(reinterpret_cast<const float4*>(p.sw + col));
        }
        reinterpret_cast<float4*>(bias_s)[lane] = b4;
        reinterpret_cast<float4*>(sw_s)[lane] = w4;
      }
      const bool got = dev::mbar_wait(acc_full, (uint32_t)tcount & 1u, abort_flag, p.budget_ns);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) record_error(p.err, abort_flag, 0x506);
        break;
      }
      __syncwarp();
      dev::tc_fence_after();
      // this lane's row scale (mpad entries; padding rows are not stored)
      const float sx = p.sx[m0 + q * 32 + lane];
      const uint32_t lanebase = (uint32_t)(q * 32) << 16;
      const uint32_t taddr = tmem + lanebase + (uint32_t)(half * 128);
      uint32_t va[32], vb[32], vc[32], vd[32];
      dev::tmem_load_32cols(taddr, va);
      dev::tmem_load_32cols(taddr + 32, vb);
      dev::tmem_load_32cols(taddr + 64, vc);
      dev::tmem_load_32cols(taddr + 96, vd);
      dev::tmem_load_wait(va);
      dev::tmem_load_wait(vb);
      dev::tmem_load_wait(vc);
      dev::tmem_load_wait(vd);
      // s_x s_w acc_i, then + acc_b, in place (FP32 bits in the same registers)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t (&cur)[32] = c == 0 ? va : c == 1 ? vb : c == 2 ? vc : vd;
        uint32_t br[32];
        if (p.branch) {
          dev::tmem_load_32cols(taddr + kBranchCol + 32 * c, br);
          dev::tmem_load_wait(br);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float y = __int2float_rn((int)cur[i]) * (sx * sw_s[c * 32 + i]);
          cur[i] = __float_as_uint(p.branch ? y + __uint_as_float(br[i]) : y);
        }
      }
      dev::tc_fence_before();
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(acc_empty);
#pragma unroll
      for (int c = 0; c < 4; ++c, ++chunk) {
        uint32_t (&cur)[32] = c == 0 ? va : c == 1 ? vb : c == 2 ? vc : vd;
        if (lane == 0) dev::bulk_wait_group_read<1>();
        __syncwarp();
        uint8_t* buf = wbuf + (chunk & 1) * kEpiBufBytes;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t packed[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 b2 = reinterpret_cast<const float2*>(bias_s)[c * 16 + j * 4 + e];
            float y0 = __uint_as_float(cur[j * 8 + 2 * e]) + b2.x;
            float y1 = __uint_as_float(cur[j * 8 + 2 * e + 1]) + b2.y;
            if (p.gelu) {
              y0 = dev::gelu_tanh(y0);
              y1 = dev::gelu_tanh(y1);
            }
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
            packed[e] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          *reinterpret_cast<uint4*>(buf + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
              make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
        dev::fence_async_shared();
        __syncwarp();
        if (lane == 0) {
          dev::tma_store_2d(&tm_y, buf, n0 + c * 32, m0 + q * 32);
          dev::bulk_commit_group();
        }
      }
      __syncwarp();
    }
    if (lane == 0) dev::bulk_wait_group_all();
  }

  __syncwarp();
  dev::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    dev::tc_fence_after();
    dev::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

size_t k2_int8_weight_bytes(int N, int K) {
  return (size_t)((N + 255) / 256) * (size_t)((K + 127) / 128) * (size_t)kBBytes;
}

cudaError_t launch_k2_int8(const CUtensorMap& tm_xl, const CUtensorMap& tm_l2, const CUtensorMap& tm_y,
                           const K2Int8Params& p, int num_sms, cudaStream_t stream) {
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(k2_int8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, k2_int8_kernel);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != 128) return cudaErrorInvalidConfiguration;
    configured_device = dev;
  }
  const int tiles = ((p.M + kBM - 1) / kBM) * ((p.N + kBN - 1) / kBN);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles < num_sms ? tiles : num_sms);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k2_int8_kernel, tm_xl, tm_l2, tm_y, p);
}

}  // namespace svdq
