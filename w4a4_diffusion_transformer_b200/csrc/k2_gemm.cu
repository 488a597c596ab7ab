// K2: NVFP4 block-scaled GEMM with the low-rank up projection fused into the
// same accumulator.
//
// SOTA-314 practice page, "Do this": the fusion pairs "Up Projection with the
// 4-bit compute, because they write the same output"; NOTE-257 note page, "Key
// results": unfused, the branch costs "the extra 16-bit write in Up
// Projection".  For a 128 x 256 output tile:
//
//   acc  = XL (L2b / alpha)                        (2 BF16 MMAs, K = 32)
//   acc += sum_k (c_x s_x) (c_w s_w)               (NVFP4 MMAs, K = 64 each)
//   Y    = bf16( [gelu]( alpha * acc + b ) )       (one BF16 store)
//
// where alpha = g_x g_w is a power of two, so L2b / alpha is exact in BF16 and
// alpha * acc reproduces Q(X^)Q(R) + XL L2b.
//
// Structure (one CTA per SM, persistent over output tiles):
//   warp 0     producer: per stage a 128 x 256 E2M1 A tile and a 256 x 256 E2M1
//              B tile, each one contiguous bulk copy (the codes are stored in
//              blocks already in the 128-byte-swizzled order the tensor core
//              reads: contiguous copies reach each SM faster than row-strided
//              tensor boxes), and the E4M3 scale factors (bulk copies, already
//              in the tensor-core layout); per tile one extra stage with the XL
//              tile and the L2b^T tile (TMA, 64-byte swizzle).
//   warp 1     allocates TMEM (512 columns: accumulator 256 + per-stage scale
//              factors) and issues tcgen05.mma.
//   warps 4-7  move each stage's scale factors into TMEM as soon as they land
//              (they complete their own barrier and are loaded before the
//              operand tiles): each warp reads them from shared memory and
//              writes its TMEM lane quarter with tcgen05.st.  Issued as
//              tcgen05.cp copies instead, they would share the tensor pipe with
//              the MMAs, and 12 copies per stage cost about as much pipe time as
//              two thirds of the stage's MMAs (the copy path stays selectable).
//   warps 8-15 epilogue, two warps per TMEM lane quarter (32 rows), each owning
//              128 of the 256 columns: all 128 columns into registers with four
//              tcgen05.ld, the accumulator handed back to the MMA warp at once,
//              then alpha, bias (staged in shared memory while the mainloop
//              runs), GELU, BF16, into two 64-byte-swizzled 32 x 32 buffers per
//              warp that the warp's lane 0 stores to Y with TMA, so the stores
//              of tile t overlap the mainloop of tile t+1.
// Pipelines are mbarrier rings; every wait is bounded (sm100.cuh).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100.cuh"

namespace svdq {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
// Epilogue output path: BF16 rows stored from registers straight to global
// memory (1), or staged in shared memory and written by TMA stores (0).  The
// direct path frees the staging buffers, which makes room for a fourth stage.
#ifndef SVDQ_K2_DIRECT_STORE
#define SVDQ_K2_DIRECT_STORE 0
#endif
#ifndef SVDQ_K2_STAGES
#define SVDQ_K2_STAGES (SVDQ_K2_DIRECT_STORE ? 4 : 3)
#endif
// Epilogue drains its 128 accumulator columns into registers before any math (1),
// or loads them chunk by chunk, overlapping each load with the previous chunk's math (0).
#ifndef SVDQ_K2_FAST_DRAIN
#define SVDQ_K2_FAST_DRAIN 1
#endif
constexpr bool kFastDrain = SVDQ_K2_FAST_DRAIN != 0;
// Stage shape: 4 blocks of 64 K per pipeline stage, i.e. 128-byte operand rows
// in the 128-byte swizzle: the tiled layout the operands are stored in.
constexpr int kKB = 4;
constexpr int kBKBytes = kKB * 32;          // E2M1 bytes per operand row per stage
constexpr int kStages = SVDQ_K2_STAGES;
constexpr uint32_t kSwz = 2u;                          // descriptor layout: 128-byte swizzle
constexpr uint32_t kSwzAtom = 8u * kBKBytes;           // bytes between 8-row groups
// Scale factors reach TMEM either through tcgen05.cp issued by one warp (0),
// or from registers: four warps, one per TMEM lane quarter, read them from
// shared memory and write them with tcgen05.st (1).  A copy occupies the
// tensor pipe that the MMAs need; the register path keeps it for the MMAs.
#ifndef SVDQ_K2_SF_REGS
#define SVDQ_K2_SF_REGS 1
#endif
constexpr bool kSfRegs = SVDQ_K2_SF_REGS != 0;
constexpr int kEpiWarps = 8;
// warp roles: 0 producer, 1 MMA issuer; register path: 4-7 scale factors,
// 8-15 epilogue (2-3 idle); copy path: 2-9 epilogue, 10 scale factors
constexpr int kEpiWarp0 = kSfRegs ? 8 : 2;
constexpr int kSfWarp0 = kSfRegs ? 4 : 2 + kEpiWarps;
constexpr int kThreads = (kSfRegs ? 16 : 3 + kEpiWarps) * 32;
// Register split of the register path (per thread, by warpgroup): producer and
// MMA warpgroup, scale-factor warpgroup, the two epilogue warpgroups.  The sum
// over the block equals the launch allocation of 128 per thread, which the
// host checks before the first launch (a larger sum would make the increase
// wait forever).
constexpr int kRegsCtl = 56, kRegsSf = 72, kRegsEpi = 192;
static_assert(128 * kRegsCtl + 128 * kRegsSf + 256 * kRegsEpi == 512 * 128, "register split");
constexpr int kEpiBufBytes = 32 * 64;        // one 32 x 32 BF16 output chunk
constexpr bool kDirectStore = SVDQ_K2_DIRECT_STORE != 0;
// per epilogue warp: two chunk buffers (TMA store path only) + 128 bias floats
constexpr int kEpiWarpBytes = (kDirectStore ? 0 : 2 * kEpiBufBytes) + 512;
constexpr int kABytes = kBM * kBKBytes;      // 16 KiB
constexpr int kBBytes = kBN * kBKBytes;      // 32 KiB
constexpr int kSFABytes = kKB * 512;         // kKB K-blocks x 128 rows
constexpr int kSFBBytes = 2 * kKB * 512;     // 2 row blocks x kKB K-blocks
constexpr int kStageBytes = kABytes + kBBytes + kSFABytes + kSFBBytes;
static_assert(kStageBytes % 1024 == 0, "stage alignment");
static_assert(kABytes >= kBM * 64 && kBBytes >= kBN * 64, "the branch stage fits a pipeline stage");
constexpr int kSmemBytes = kStages * kStageBytes + kEpiWarps * kEpiWarpBytes + 1024 + 256;
constexpr int kTmemCols = 512;
// Scale factors in TMEM, one region per pipeline stage (so a region is only
// rewritten after the MMAs that read it have completed): 4 columns per 128-row
// x 64-K block, 16 for A and 32 for B per stage.
constexpr int kSFCol0 = 256;
constexpr int kSFStageCols = 12 * kKB;       // 4 columns of A + 8 of B per K block
static_assert(kSFCol0 + kStages * kSFStageCols <= kTmemCols, "TMEM budget");

__device__ __forceinline__ void record_error(int* err, volatile int* abort_flag, int code) {
  atomicCAS(err, 0, code);
  *abort_flag = 1;
}

__device__ __forceinline__ float gelu_tanh(float y) {
  const float k0 = 0.7978845608028654f;   // sqrt(2/pi)
  return 0.5f * y * (1.0f + tanhf(k0 * (y + 0.044715f * y * y * y)));
}

__global__ void __launch_bounds__(kThreads, 1)
    k2_kernel(const __grid_constant__ CUtensorMap tm_xl, const __grid_constant__ CUtensorMap tm_l2,
              const __grid_constant__ CUtensorMap tm_y, K2Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi_buf = smem + kStages * kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_buf + kEpiWarps * kEpiWarpBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint64_t* sf_ready = drain + 1;                  // [kStages], scale factors of a stage in TMEM
  uint64_t* cp_drain = sf_ready + kStages;
  uint64_t* sf_full = cp_drain + 1;                // [kStages], a stage's scale factors in shared memory
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_full + kStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int M = p.M, N = p.N, K = p.K;
  const int tiles_m = (M + kBM - 1) / kBM;
  const int tiles_n = (N + kBN - 1) / kBN;
  const int num_tiles = tiles_m * tiles_n;
  const int kblocks = K >> 6;                     // 64-element K blocks
  const int ktiles = (kblocks + kKB - 1) / kKB;

  if (threadIdx.x == 0) {
    // the next kernel on the stream may launch now; it waits for this grid's
    // completion before it touches anything this grid reads or writes
    dev::griddep_launch_dependents();
    for (int s = 0; s < kStages; ++s) {
      dev::mbar_init(&full[s], 1);
      dev::mbar_init(&empty[s], 1);
      dev::mbar_init(&sf_full[s], 1);
    }
    dev::mbar_init(acc_full, 1);
    dev::mbar_init(acc_empty, kEpiWarps);
    dev::mbar_init(drain, 1);
    for (int st = 0; st < kStages; ++st) dev::mbar_init(&sf_ready[st], kSfRegs ? 4 : 1);
    dev::mbar_init(cp_drain, 1);
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

  // (register path) each role sets its warpgroup's register budget first
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (kSfRegs) dev::setmaxnreg_dec<kRegsCtl>();
    if (lane == 0) {
      if (p.branch) {
        dev::tma_prefetch_desc(&tm_xl);
        dev::tma_prefetch_desc(&tm_l2);
      }
      int it = 0;
      bool ok = true;
      bool deps_ready = false;     // activations come from the preceding kernel (launched as a dependency)
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m0 = (tile % tiles_m) * kBM;
        const int n0 = (tile / tiles_m) * kBN;
        if (p.branch) {
          const int s = it % kStages;
          if (!dev::mbar_wait(&empty[s], ((uint32_t)(it / kStages) & 1u) ^ 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x201);
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kStageBytes;
          dev::mbar_arrive(&sf_full[s]);               // a branch stage carries no scale factors
          dev::mbar_arrive_expect_tx(&full[s], kBM * 64 + kBN * 64);
          dev::tma_load_2d(st + kABytes, &tm_l2, &full[s], 0, n0);
          if (!deps_ready) {
            dev::griddep_wait();
            deps_ready = true;
          }
          dev::tma_load_2d(st, &tm_xl, &full[s], 0, m0);
          ++it;
        }
        for (int kt = 0; kt < ktiles; ++kt) {
          const int s = it % kStages;
          if (!dev::mbar_wait(&empty[s], ((uint32_t)(it / kStages) & 1u) ^ 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x202);
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kStageBytes;
          const int nkb = min(kKB, kblocks - kKB * kt);
          const uint32_t sf_bytes = (uint32_t)nkb * 512u;
          // The scale factors complete their own barrier and are issued first:
          // the copy warp moves them into TMEM while the operand tiles are
          // still in flight, so those copies are off the stage's critical path.
          dev::mbar_arrive_expect_tx(&sf_full[s], 3u * sf_bytes);
          dev::mbar_arrive_expect_tx(&full[s], kABytes + kBBytes);
          // weights first: they do not depend on the preceding kernel
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const size_t b_chunk = (size_t)((n0 >> 7) + h) * (size_t)kblocks + (size_t)(kKB * kt);
            dev::bulk_load(st + kABytes + kBBytes + kSFABytes + h * (kKB * 512), p.sfb + b_chunk * 512, sf_bytes,
                           &sf_full[s]);
          }
          // operand blocks are stored tiled and pre-swizzled: one contiguous bulk copy each
          dev::bulk_load(st + kABytes, p.wcodes + ((size_t)(n0 >> 8) * (size_t)ktiles + (size_t)kt) * kBBytes,
                         kBBytes, &full[s]);
          if (!deps_ready) {
            dev::griddep_wait();
            deps_ready = true;
          }
          const size_t a_chunk = (size_t)(m0 >> 7) * (size_t)kblocks + (size_t)(kKB * kt);
          dev::bulk_load(st + kABytes + kBBytes, p.sfa + a_chunk * 512, sf_bytes, &sf_full[s]);
          dev::bulk_load(st, p.acodes + ((size_t)(m0 >> 7) * (size_t)ktiles + (size_t)kt) * kABytes, kABytes,
                         &full[s]);
          ++it;
        }
      }
      // every exit path waits for the preceding grid, so that this grid never
      // completes before it (the next launch on the stream waits only for this one)
      if (!deps_ready) dev::griddep_wait();
      for (int j = max(0, it - kStages); j < it; ++j)
        if (!dev::mbar_wait(&full[j % kStages], (uint32_t)(j / kStages) & 1u, abort_flag, p.budget_ns) ||
            !dev::mbar_wait(&sf_full[j % kStages], (uint32_t)(j / kStages) & 1u, abort_flag, p.budget_ns))
          break;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (kSfRegs) dev::setmaxnreg_dec<kRegsCtl>();
    if (lane == 0) {
      const uint32_t idesc_f4 = dev::idesc_nvfp4(kBM, kBN);
      const uint32_t idesc_h = dev::idesc_bf16(kBM, kBN);
      auto wait_full = [&](int slot, int code) -> bool {
        if (!dev::mbar_wait(&full[slot % kStages], (uint32_t)(slot / kStages) & 1u, abort_flag, p.budget_ns)) {
          record_error(p.err, abort_flag, code);
          return false;
        }
        dev::tc_fence_after();
        return true;
      };
      uint32_t sf_phase = 0;                          // per-stage parity of sf_ready
      auto wait_sf = [&](int slot) -> bool {
        const int st = slot % kStages;
        if (!dev::mbar_wait(&sf_ready[st], (sf_phase >> st) & 1u, abort_flag, p.budget_ns)) {
          record_error(p.err, abort_flag, 0x207);
          return false;
        }
        sf_phase ^= 1u << st;
        dev::tc_fence_after();
        return true;
      };
      int it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tcount) {
        const int kslot0 = it + (p.branch ? 1 : 0);
        if (!dev::mbar_wait(acc_empty, ((uint32_t)tcount & 1u) ^ 1u, abort_flag, p.budget_ns)) {
          record_error(p.err, abort_flag, 0x203);
          ok = false;
          break;
        }
        dev::tc_fence_after();
        uint32_t accumulate = 0;
        if (p.branch) {
          if (!(ok = wait_full(it, 0x204))) break;
          const int s = it % kStages;
          const uint32_t a0 = dev::smem_u32(smem + s * kStageBytes);
          const uint32_t b0 = a0 + kABytes;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const uint64_t ad = dev::smem_desc(a0 + 32 * j, 16, 512, 4);
            const uint64_t bd = dev::smem_desc(b0 + 32 * j, 16, 512, 4);
            dev::mma_bf16(tmem, ad, bd, idesc_h, accumulate);
            accumulate = 1;
          }
          dev::tc_commit(&empty[s]);
        }
        for (int kt = 0; kt < ktiles; ++kt) {
          const int slot = kslot0 + kt;
          const int s = slot % kStages;
          if (!(ok = wait_full(slot, 0x205))) break;
          if (!(ok = wait_sf(slot))) break;
          const int nkb = min(kKB, kblocks - kKB * kt);
          const uint32_t a0 = dev::smem_u32(smem + s * kStageBytes);
          const uint32_t b0 = a0 + kABytes;
          const uint32_t tsfa = tmem + kSFCol0 + s * kSFStageCols;
          const uint32_t tsfb = tsfa + 4 * kKB;
          for (int j = 0; j < nkb; ++j) {
            const uint64_t ad = dev::smem_desc(a0 + 32 * j, 16, kSwzAtom, kSwz);
            const uint64_t bd = dev::smem_desc(b0 + 32 * j, 16, kSwzAtom, kSwz);
            dev::mma_nvfp4(tmem, ad, bd, idesc_f4, tsfa + 4 * j, tsfb + 8 * j, accumulate);
            accumulate = 1;
          }
          dev::tc_commit(&empty[s]);
        }
        if (!ok) break;
        it = kslot0 + ktiles;
        dev::tc_commit(acc_full);
      }
      // Wait until every MMA and copy this thread issued has completed.
      dev::tc_commit(drain);
      dev::mbar_wait(drain, 0, abort_flag, p.budget_ns);
    }
  } else if (kSfRegs && warp >= kSfWarp0 && warp < kSfWarp0 + 4) {
    // ------------------------------------------------------------ scale factors, register path
    // Warp w writes TMEM lanes 32 (w % 4) .. +31.  The layout is the one the
    // 32x128b.warpx4 copy produces: lane 32 q + u holds, per 64-K block j, the
    // 16-byte unit u of A's 512-byte chunk in columns 4 j .. 4 j + 3 of the A
    // region, and unit u of B's two chunks (rows 0-127, 128-255) in columns
    // 8 j .. 8 j + 7 of the B region.
    dev::setmaxnreg_dec<kRegsSf>();
    const uint32_t lanebase = (uint32_t)((warp & 3) * 32) << 16;
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      if (p.branch) ++it;
      for (int kt = 0; kt < ktiles; ++kt, ++it) {
        const int st = it % kStages;
        const bool got = dev::mbar_wait(&sf_full[st], (uint32_t)(it / kStages) & 1u, abort_flag, p.budget_ns);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) record_error(p.err, abort_flag, 0x208);
          ok = false;
          break;
        }
        const uint8_t* sfa = smem + st * kStageBytes + kABytes + kBBytes;
        const uint8_t* sfb = sfa + kSFABytes;
        uint32_t ra[16], rb[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          // blocks past the K tail hold stale bytes that no MMA reads
          const uint4 a = *reinterpret_cast<const uint4*>(sfa + 512 * j + lane * 16);
          const uint4 b0 = *reinterpret_cast<const uint4*>(sfb + 512 * j + lane * 16);
          const uint4 b1 = *reinterpret_cast<const uint4*>(sfb + kKB * 512 + 512 * j + lane * 16);
          ra[4 * j + 0] = a.x; ra[4 * j + 1] = a.y; ra[4 * j + 2] = a.z; ra[4 * j + 3] = a.w;
          rb[8 * j + 0] = b0.x; rb[8 * j + 1] = b0.y; rb[8 * j + 2] = b0.z; rb[8 * j + 3] = b0.w;
          rb[8 * j + 4] = b1.x; rb[8 * j + 5] = b1.y; rb[8 * j + 6] = b1.z; rb[8 * j + 7] = b1.w;
        }
        const uint32_t tsfa = tmem + kSFCol0 + st * kSFStageCols;
        dev::tmem_store_16cols(tsfa + lanebase, ra);
        dev::tmem_store_32cols(tsfa + 4 * kKB + lanebase, rb);
        dev::tmem_store_wait();
        dev::tc_fence_before();
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(&sf_ready[st]);
      }
    }
  } else if (!kSfRegs && warp == kSfWarp0) {
    // ------------------------------------------------------------ scale-factor copier
    if (lane == 0) {
      int it = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        bool ok = true;
        if (p.branch) ++it;
        for (int kt = 0; kt < ktiles; ++kt, ++it) {
          const int st = it % kStages;
          if (!dev::mbar_wait(&sf_full[st], (uint32_t)(it / kStages) & 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x208);
            ok = false;
            break;
          }
          dev::tc_fence_after();
          const int nkb = min(kKB, kblocks - kKB * kt);
          const uint32_t sfa0 = dev::smem_u32(smem + st * kStageBytes) + kABytes + kBBytes;
          const uint32_t sfb0 = sfa0 + kSFABytes;
          const uint32_t tsfa = tmem + kSFCol0 + st * kSFStageCols;
          const uint32_t tsfb = tsfa + 4 * kKB;
          for (int j = 0; j < nkb; ++j) {
            dev::tmem_copy_32x128b_x4(tsfa + 4 * j, dev::smem_desc(sfa0 + 512 * j, 0, 128, 0));
            dev::tmem_copy_32x128b_x4(tsfb + 8 * j, dev::smem_desc(sfb0 + 512 * j, 0, 128, 0));
            dev::tmem_copy_32x128b_x4(tsfb + 8 * j + 4, dev::smem_desc(sfb0 + kKB * 512 + 512 * j, 0, 128, 0));
          }
          dev::tc_commit(&sf_ready[st]);
        }
        if (!ok) break;
      }
      dev::tc_commit(cp_drain);
      dev::mbar_wait(cp_drain, 0, abort_flag, p.budget_ns);
    }
  } else if (kSfRegs && warp < kSfWarp0) {
    dev::setmaxnreg_dec<kRegsCtl>();                 // idle warps of the first warpgroup
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------ epilogue
    if (kSfRegs) dev::setmaxnreg_inc<kRegsEpi>();
    const int q = warp & 3;                          // TMEM lane quarter of this warp
    const int half = (warp - kEpiWarp0) >> 2;       // which 128 of the 256 columns
    uint8_t* wbuf = epi_buf + (warp - kEpiWarp0) * kEpiWarpBytes;
    float* bias_s = reinterpret_cast<float*>(wbuf + (kDirectStore ? 0 : 2 * kEpiBufBytes));
    if (!kDirectStore && lane == 0) dev::tma_prefetch_desc(&tm_y);
    int tcount = 0, chunk = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tcount) {
      const int m0 = (tile % tiles_m) * kBM;
      const int n0 = (tile / tiles_m) * kBN + half * 128;
      // stage this tile's 128 bias values (the previous tile's reads are done:
      // every lane passed the __syncwarp after its last use)
      {
        const int col = n0 + lane * 4;
        float4 b4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (col < N) b4 = __ldg(reinterpret_cast<const float4*>(p.bias + col));
        reinterpret_cast<float4*>(bias_s)[lane] = b4;
      }
      const bool got = dev::mbar_wait(acc_full, (uint32_t)tcount & 1u, abort_flag, p.budget_ns);
      if (!__all_sync(0xffffffffu, got)) {          // warp-uniform exit (tcgen05.ld is warp-collective)
        if (lane == 0) record_error(p.err, abort_flag, 0x206);
        break;
      }
      __syncwarp();
      dev::tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(half * 128);
      uint32_t va[32], vb[32], vc[32], vd[32];
      dev::tmem_load_32cols(taddr, va);
      if (kFastDrain) {
        // all 128 columns into registers, then hand the accumulator back at once
        dev::tmem_load_32cols(taddr + 32, vb);
        dev::tmem_load_32cols(taddr + 64, vc);
        dev::tmem_load_32cols(taddr + 96, vd);
        dev::tmem_load_wait(va);
        dev::tmem_load_wait(vb);
        dev::tmem_load_wait(vc);
        dev::tmem_load_wait(vd);
        dev::tc_fence_before();
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(acc_empty);
      } else {
        dev::tmem_load_wait(va);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c, ++chunk) {
        uint32_t (&cur)[32] = kFastDrain ? (c == 0 ? va : c == 1 ? vb : c == 2 ? vc : vd) : ((c & 1) ? vb : va);
        uint32_t (&nxt)[32] = (c & 1) ? va : vb;
        if (!kFastDrain && c + 1 < 4) dev::tmem_load_32cols(taddr + (uint32_t)((c + 1) * 32), nxt);
        // the buffer of this chunk was last read by the store issued two chunks ago
        if (!kDirectStore) {
          if (lane == 0) dev::bulk_wait_group_read<1>();
          __syncwarp();
        }
        uint8_t* buf = wbuf + (chunk & 1) * kEpiBufBytes;
        const int row = m0 + q * 32 + lane;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t packed[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 b2 = reinterpret_cast<const float2*>(bias_s)[c * 16 + j * 4 + e];
            float y0 = p.alpha * __uint_as_float(cur[j * 8 + 2 * e]) + b2.x;
            float y1 = p.alpha * __uint_as_float(cur[j * 8 + 2 * e + 1]) + b2.y;
            if (p.gelu) {
              y0 = gelu_tanh(y0);
              y1 = gelu_tanh(y1);
            }
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
            packed[e] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          if (kDirectStore) {
            // 8 columns per 16-byte store; N is a multiple of 16, so a store
            // that starts inside the row ends inside it
            const int col = n0 + c * 32 + j * 8;
            if (row < M && col < N)
              *reinterpret_cast<uint4*>(p.y + (size_t)row * (size_t)N + col) =
                  make_uint4(packed[0], packed[1], packed[2], packed[3]);
          } else {
            // 64-byte swizzle: 16-byte chunk j of row `lane` sits at j ^ ((lane >> 1) & 3)
            *reinterpret_cast<uint4*>(buf + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(packed[0], packed[1], packed[2], packed[3]);
          }
        }
        if (!kDirectStore) {
          dev::fence_async_shared();                  // make the writes visible to the TMA engine
          __syncwarp();
          if (lane == 0) {
            dev::tma_store_2d(&tm_y, buf, n0 + c * 32, m0 + q * 32);
            dev::bulk_commit_group();
          }
        }
        if (!kFastDrain && c + 1 < 4) dev::tmem_load_wait(nxt);
        if (!kFastDrain && c == 2) {
          // the last chunk is in registers: hand the accumulator back to the MMA warp
          dev::tc_fence_before();
          __syncwarp();
          if (lane == 0) dev::mbar_arrive(acc_empty);
        }
      }
      __syncwarp();
    }
    if (!kDirectStore && lane == 0) dev::bulk_wait_group_all();
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

int k2_block_n() { return kBN; }

cudaError_t launch_k2(const CUtensorMap& tm_xl, const CUtensorMap& tm_l2, const CUtensorMap& tm_y,
                      const K2Params& p, int num_sms, cudaStream_t stream) {
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(k2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    if (kSfRegs) {
      // the warpgroups' register budgets add up to exactly 128 per thread
      cudaFuncAttributes fa;
      e = cudaFuncGetAttributes(&fa, k2_kernel);
      if (e != cudaSuccess) return e;
      if (fa.numRegs != 128) return cudaErrorInvalidConfiguration;
    }
    configured_device = dev;
  }
  const int tiles = ((p.M + kBM - 1) / kBM) * ((p.N + kBN - 1) / kBN);
  const int grid = tiles < num_sms ? tiles : num_sms;
  // Programmatic dependent launch: the prologue (barriers, TMEM, descriptor
  // prefetch, weight tiles) overlaps the tail of the kernel that produces the
  // activations; the producer waits for it before the first activation load.
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
  return cudaLaunchKernelEx(&cfg, k2_kernel, tm_xl, tm_l2, tm_y, p);
}

}  // namespace svdq
