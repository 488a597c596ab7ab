// K2 on CTA pairs: the NVFP4 block-scaled GEMM with the fused up projection,
// computed by two CTAs (one cluster) per 256 x 256 output tile with the
// fifth-generation tensor core's pair mode (tcgen05 cta_group::2).
//
// Same mathematics as the single-CTA kernel (SOTA-314 practice page, "Do
// this": "Up Projection with the 4-bit compute, because they write the same
// output"):
//   acc  = XL (L2b / alpha) + sum_k (c_x s_x) (c_w s_w);   Y = bf16([gelu](alpha acc + b)).
//
// Why pairs: the operand stream into each SM bounds the single-CTA kernel
// (54 KB per 128 x 256 x 256 stage).  In pair mode each CTA holds its own 128
// rows of A and only half of B's 256 rows -- the two SMs' tensor cores share
// the B halves -- so a stage is 38 KB per SM for the same work.
//
// What makes the stream fast here: a bulk copy occupies its issuing thread for
// about a tenth of a microsecond whatever its size, so each CTA moves a stage
// in two large copies from two producer warps: the weight half and the scale
// factors of all 256 weight rows are stored next to each other (one 20 KB block
// per CTA and stage, prepared once), and the activation codes (16 KB) plus
// their scales (2 KB) come from the first kernel's output.
//
// Roles (CTA rank r = 0, 1 of the pair; tile rows m0.., columns n0..):
//   both CTAs   warp 0: activation producer (A rows m0 + 128 r and their
//               scale factors; per tile the XL rows of the branch stage).
//               warp 2: weight producer (the B half n0 + 128 r with the scale
//               factors of all 256 columns; per tile the L2b / alpha rows).
//               Both complete the CTA's own `full` barrier of the stage.
//               warps 4-7: wait for the CTA's stage, write its scale factors
//               into the CTA's TMEM from registers (tcgen05.st, one warp per
//               lane quarter) and arrive on the leader's `ready` barrier of the
//               stage -- directly, across the cluster: once all eight warps of
//               both CTAs have arrived, every operand of the stage is in place.
//               warps 8-15: epilogue of the CTA's 128 accumulator rows.
//   rank 0      warp 1: the MMA issuer: pair MMAs (M = 256), whose commits
//               arrive on both CTAs' barriers (multicast): a stage is free in
//               both, an accumulator full in both.
// Every wait is bounded (sm100.cuh).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100.cuh"

namespace svdq {

namespace {

constexpr int kBM = 128;                     // rows of A per CTA
constexpr int kPM = 256;                     // rows per pair tile
constexpr int kBN = 256;                     // columns per tile
constexpr int kBNh = 128;                    // rows of B per CTA
constexpr int kKB = 4;                       // 64-element K blocks per stage
constexpr int kBKBytes = kKB * 32;           // E2M1 bytes per operand row per stage (128: 128-byte swizzle)
#ifndef SVDQ_K2P_STAGES
#define SVDQ_K2P_STAGES 5
#endif
#ifndef SVDQ_K2P_EPI_BUFS
#define SVDQ_K2P_EPI_BUFS 2
#endif
// How the MMA issuer waits on barriers that the other CTA's warps complete:
// 1 polls with test_wait, 2 with a short try_wait hint, 0 plain try_wait.
#ifndef SVDQ_K2P_REMOTE_WAIT
#define SVDQ_K2P_REMOTE_WAIT 1
#endif
constexpr int kRemoteWait = SVDQ_K2P_REMOTE_WAIT;
constexpr int kStages = SVDQ_K2P_STAGES;
constexpr int kEpiBufs = SVDQ_K2P_EPI_BUFS;  // 32 x 32 output buffers per epilogue warp
constexpr int kEpiWarps = 8;
// warp roles: 0 activation producer, 1 MMA issuer (rank 0), 2 weight producer,
// 3 idle, 4-7 scale factors / stage readiness, 8-15 epilogue
constexpr int kProdA = 0, kMmaWarp = 1, kProdB = 2, kSfWarp0 = 4, kEpiWarp0 = 8;
constexpr int kThreads = 16 * 32;
// register budgets per thread by warpgroup (control, scale factors, two
// epilogue warpgroups); they add up to the launch allocation of 128, which the
// host checks before the first launch
constexpr int kRegsCtl = 56, kRegsSf = 72, kRegsEpi = 192;
static_assert(128 * kRegsCtl + 128 * kRegsSf + 256 * kRegsEpi == kThreads * 128, "register split");
constexpr int kEpiBufBytes = 32 * 64;        // one 32 x 32 BF16 output chunk
constexpr int kEpiWarpBytes = kEpiBufs * kEpiBufBytes;
// stage: [A codes 16 KB][B half codes 16 KB][B scales, 256 rows, 4 KB][A scales 2 KB]
constexpr int kABytes = kBM * kBKBytes;      // 16 KiB
constexpr int kBBytes = kBNh * kBKBytes;     // 16 KiB
constexpr int kSFBBytes = 2 * kKB * 512;     // both 128-row halves x kKB K-blocks
constexpr int kSFABytes = kKB * 512;
constexpr int kOffB = kABytes;
constexpr int kOffSFB = kOffB + kBBytes;
constexpr int kOffSFA = kOffSFB + kSFBBytes;
constexpr int kStageBytes = kOffSFA + kSFABytes;
constexpr int kWBlockBytes = kBBytes + kSFBBytes;      // one CTA's weight block per stage (20 KB)
static_assert(kStageBytes % 1024 == 0, "stage alignment");
static_assert(kABytes >= kBM * 64 && kBBytes >= kBNh * 64, "the branch stage fits a pipeline stage");
constexpr int kBarBytes = 512;
constexpr int kSmemBytes = kStages * kStageBytes + kEpiWarps * kEpiWarpBytes + 1024 + kBarBytes;
static_assert(kSmemBytes <= 232448, "shared memory per block");
constexpr int kTmemCols = 512;
constexpr int kSFCol0 = 256;
constexpr int kSFStageCols = 12 * kKB;       // 4 columns of A + 8 of B per K block
static_assert(kSFCol0 + kStages * kSFStageCols <= kTmemCols, "TMEM budget");
constexpr uint16_t kBoth = 3, kLeader = 1;   // multicast masks (cluster ranks)

__device__ __forceinline__ void record_error(int* err, volatile int* abort_flag, int code) {
  atomicCAS(err, 0, code);
  *abort_flag = 1;
}

__global__ void __launch_bounds__(kThreads, 1)
    k2_pair_kernel(const __grid_constant__ CUtensorMap tm_xl, const __grid_constant__ CUtensorMap tm_l2,
                   const __grid_constant__ CUtensorMap tm_y, K2Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi_buf = smem + kStages * kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_buf + kEpiWarps * kEpiWarpBytes);
  uint64_t* empty = full + kStages;            // this CTA's copy of "stage consumed" (multicast commit)
  uint64_t* ready = empty + kStages;           // rank 0: the stage is in place in both CTAs
  uint64_t* acc_full = ready + kStages;
  uint64_t* acc_empty = acc_full + 1;          // rank 0: both CTAs drained the accumulator
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = dev::cluster_rank();
  const bool leader = rank == 0;
  const int M = p.M, N = p.N, K = p.K;
  const int tiles_m = (M + kPM - 1) / kPM;
  const int tiles_n = (N + kBN - 1) / kBN;
  const int num_tiles = tiles_m * tiles_n;
  const int pair_id = (int)blockIdx.x >> 1, npairs = (int)gridDim.x >> 1;
  const int kblocks = K >> 6;
  const int ktiles = (kblocks + kKB - 1) / kKB;

  if (threadIdx.x == 0) {
    // the next kernel on the stream may launch now; it waits for this grid's
    // completion before it touches anything this grid reads or writes
    dev::griddep_launch_dependents();
    for (int s = 0; s < kStages; ++s) {
      dev::mbar_init(&full[s], 2);              // the two producer warps
      dev::mbar_init(&empty[s], 1);
      dev::mbar_init(&ready[s], 8);             // the scale-factor warps of both CTAs
    }
    dev::mbar_init(acc_full, 1);
    dev::mbar_init(acc_empty, 2 * kEpiWarps);
    dev::mbar_init(drain, 1);
    *abort_flag = 0;
    dev::fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    __syncwarp();
    dev::tmem_alloc_pair(tmem_slot, kTmemCols);
    dev::tmem_relinquish_pair();
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::cluster_sync();                         // barriers and TMEM of both CTAs exist
  dev::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProdA) {
    // ------------------------------------------------------------ activation producer (both CTAs)
    dev::setmaxnreg_dec<kRegsCtl>();
    if (lane == 0) {
      if (p.branch) dev::tma_prefetch_desc(&tm_xl);
      // the activations come from the preceding kernel (launched as a dependency)
      dev::griddep_wait();
      int it = 0;
      bool ok = true;
      for (int tile = pair_id; tile < num_tiles && ok; tile += npairs) {
        const int my_m = (tile % tiles_m) * kPM + kBM * (int)rank;
        const bool rows_xl = my_m < M;                        // the branch rows exist
        const bool rows_a = my_m < p.mpad;                    // the code and scale layouts cover these rows
        // (rows that do not exist leave stale shared memory: their results are never stored)
        if (p.branch) {
          const int s = it % kStages;
          if (!dev::mbar_wait_cluster(&empty[s], ((uint32_t)(it / kStages) & 1u) ^ 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x221);
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kStageBytes;
          dev::mbar_arrive_expect_tx(&full[s], rows_xl ? kBM * 64 : 0);
          if (rows_xl) dev::tma_load_2d(st, &tm_xl, &full[s], 0, my_m);
          ++it;
        }
        for (int kt = 0; kt < ktiles; ++kt) {
          const int s = it % kStages;
          if (!dev::mbar_wait_cluster(&empty[s], ((uint32_t)(it / kStages) & 1u) ^ 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x222);
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kStageBytes;
          const uint32_t sf_bytes = (uint32_t)min(kKB, kblocks - kKB * kt) * 512u;
          dev::mbar_arrive_expect_tx(&full[s], rows_a ? (uint32_t)kABytes + sf_bytes : 0u);
          if (rows_a) {
            const size_t a_chunk = (size_t)(my_m >> 7) * (size_t)kblocks + (size_t)(kKB * kt);
            dev::bulk_load(st, p.acodes + ((size_t)(my_m >> 7) * (size_t)ktiles + (size_t)kt) * kABytes, kABytes,
                           &full[s]);
            dev::bulk_load(st + kOffSFA, p.sfa + a_chunk * 512, sf_bytes, &full[s]);
          }
          ++it;
        }
      }
      for (int j = max(0, it - kStages); j < it; ++j)
        if (!dev::mbar_wait(&full[j % kStages], (uint32_t)(j / kStages) & 1u, abort_flag, p.budget_ns)) break;
    }
  } else if (warp == kProdB) {
    // ------------------------------------------------------------ weight producer (both CTAs)
    dev::setmaxnreg_dec<kRegsCtl>();
    if (lane == 0) {
      if (p.branch) dev::tma_prefetch_desc(&tm_l2);
      int it = 0;
      bool ok = true;
      for (int tile = pair_id; tile < num_tiles && ok; tile += npairs) {
        const int n0 = (tile / tiles_m) * kBN;
        const int my_n = n0 + kBNh * (int)rank;
        if (p.branch) {
          const int s = it % kStages;
          if (!dev::mbar_wait_cluster(&empty[s], ((uint32_t)(it / kStages) & 1u) ^ 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x223);
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kStageBytes;
          const bool rows_b = my_n < N;
          dev::mbar_arrive_expect_tx(&full[s], rows_b ? kBNh * 64 : 0);
          if (rows_b) dev::tma_load_2d(st + kOffB, &tm_l2, &full[s], 0, my_n);
          ++it;
        }
        for (int kt = 0; kt < ktiles; ++kt) {
          const int s = it % kStages;
          if (!dev::mbar_wait_cluster(&empty[s], ((uint32_t)(it / kStages) & 1u) ^ 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x224);
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kStageBytes;
          // this CTA's 128-row half of the 256-row weight block followed by the
          // scale factors of all 256 rows: one contiguous 20 KB block
          dev::mbar_arrive_expect_tx(&full[s], kWBlockBytes);
          dev::bulk_load(st + kOffB,
                         p.wpair + (((size_t)(n0 >> 8) * (size_t)ktiles + (size_t)kt) * 2 + rank) * kWBlockBytes,
                         kWBlockBytes, &full[s]);
          ++it;
        }
      }
      for (int j = max(0, it - kStages); j < it; ++j)
        if (!dev::mbar_wait(&full[j % kStages], (uint32_t)(j / kStages) & 1u, abort_flag, p.budget_ns)) break;
    }
  } else if (warp == kMmaWarp && leader) {
    // ------------------------------------------------------------ rank 0: MMA issuer
    dev::setmaxnreg_dec<kRegsCtl>();
    if (lane == 0) {
      const uint32_t idesc_f4 = dev::idesc_nvfp4(kPM, kBN);
      const uint32_t idesc_h = dev::idesc_bf16(kPM, kBN);
      auto wait_ready = [&](int slot, int code) -> bool {
        if (!dev::mbar_wait_remote<kRemoteWait>(&ready[slot % kStages], (uint32_t)(slot / kStages) & 1u, abort_flag,
                                                p.budget_ns)) {
          record_error(p.err, abort_flag, code);
          return false;
        }
        dev::tc_fence_after();
        return true;
      };
      int it = 0, tcount = 0;
      bool ok = true;
      for (int tile = pair_id; tile < num_tiles && ok; tile += npairs, ++tcount) {
        if (!dev::mbar_wait_remote<kRemoteWait>(acc_empty, ((uint32_t)tcount & 1u) ^ 1u, abort_flag, p.budget_ns)) {
          record_error(p.err, abort_flag, 0x225);
          ok = false;
          break;
        }
        dev::tc_fence_after();
        uint32_t accumulate = 0;
        if (p.branch) {
          if (!(ok = wait_ready(it, 0x226))) break;
          const int s = it % kStages;
          const uint32_t a0 = dev::smem_u32(smem + s * kStageBytes);
          const uint32_t b0 = a0 + kOffB;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            dev::mma_f16_pair(tmem, dev::smem_desc(a0 + 32 * j, 16, 512, 4), dev::smem_desc(b0 + 32 * j, 16, 512, 4),
                              idesc_h, accumulate);
            accumulate = 1;
          }
          dev::tc_commit_pair(&empty[s], kBoth);
          ++it;
        }
        for (int kt = 0; kt < ktiles; ++kt, ++it) {
          const int s = it % kStages;
          if (!(ok = wait_ready(it, 0x227))) break;
          const int nkb = min(kKB, kblocks - kKB * kt);
          const uint32_t a0 = dev::smem_u32(smem + s * kStageBytes);
          const uint32_t b0 = a0 + kOffB;
          const uint32_t tsfa = tmem + kSFCol0 + s * kSFStageCols;
          const uint32_t tsfb = tsfa + 4 * kKB;
          for (int j = 0; j < nkb; ++j) {
            dev::mma_nvfp4_pair(tmem, dev::smem_desc(a0 + 32 * j, 16, 1024, 2), dev::smem_desc(b0 + 32 * j, 16, 1024, 2),
                                idesc_f4, tsfa + 4 * j, tsfb + 8 * j, accumulate);
            accumulate = 1;
          }
          dev::tc_commit_pair(&empty[s], kBoth);
        }
        if (!ok) break;
        dev::tc_commit_pair(acc_full, kBoth);
      }
      // Wait until every pair operation this thread issued has completed.
      dev::tc_commit_pair(drain, kLeader);
      dev::mbar_wait(drain, 0, abort_flag, p.budget_ns);
    }
  } else if (warp >= kSfWarp0 && warp < kSfWarp0 + 4) {
    // ------------------------------------------------------------ scale factors / stage readiness (both CTAs)
    // Warp w writes its CTA's TMEM lanes 32 (w % 4) .. +31 from registers
    // (tcgen05.st), in the layout a 32x128b.warpx4 copy produces: per 64-K
    // block j, unit `lane` of A's 512-byte chunk (this CTA's 128 rows) in
    // columns 4 j .. 4 j + 3 of the A region, and of B's two chunks (all 256
    // columns of the tile) in columns 8 j .. 8 j + 7 of the B region.  Then it
    // tells the leader that this CTA's part of the stage is in place.
    dev::setmaxnreg_dec<kRegsSf>();
    const uint32_t lanebase = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t ready0 = dev::map_to_rank(ready, 0);
    int it = 0;
    bool ok = true;
    for (int tile = pair_id; tile < num_tiles && ok; tile += npairs) {
      const int nst = ktiles + (p.branch ? 1 : 0);
      for (int u = 0; u < nst; ++u, ++it) {
        const int st = it % kStages;
        const bool got = dev::mbar_wait(&full[st], (uint32_t)(it / kStages) & 1u, abort_flag, p.budget_ns);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) record_error(p.err, abort_flag, 0x229);
          ok = false;
          break;
        }
        const bool kstage = !(p.branch && u == 0);
        if (kstage) {
          // K blocks past the tail hold stale bytes that no MMA reads; so do the
          // A scales of rows past the activations' padding
          const uint8_t* sfa = smem + st * kStageBytes + kOffSFA;
          const uint8_t* sfb = smem + st * kStageBytes + kOffSFB;
          uint32_t ra[16], rb[32];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
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
        }
        dev::tc_fence_before();
        __syncwarp();
        if (lane == 0) dev::mbar_arrive_remote(ready0 + 8u * (uint32_t)st);
      }
    }
  } else if (warp < kSfWarp0) {
    dev::setmaxnreg_dec<kRegsCtl>();                 // idle warps of the first warpgroup
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    dev::setmaxnreg_inc<kRegsEpi>();
    const int q = warp & 3;                          // TMEM lane quarter of this warp
    const int half = (warp - kEpiWarp0) >> 2;        // which 128 of the 256 columns
    uint8_t* wbuf = epi_buf + (warp - kEpiWarp0) * kEpiWarpBytes;
    const uint32_t acc_empty_leader = dev::map_to_rank(acc_empty, 0);
    if (lane == 0) dev::tma_prefetch_desc(&tm_y);
    int tcount = 0, chunk = 0;
    for (int tile = pair_id; tile < num_tiles; tile += npairs, ++tcount) {
      const int m0 = (tile % tiles_m) * kPM + kBM * (int)rank;
      const int n0 = (tile / tiles_m) * kBN + half * 128;
      const bool got = dev::mbar_wait_cluster(acc_full, (uint32_t)tcount & 1u, abort_flag, p.budget_ns);
      if (!__all_sync(0xffffffffu, got)) {          // warp-uniform exit (tcgen05.ld is warp-collective)
        if (lane == 0) record_error(p.err, abort_flag, 0x22a);
        break;
      }
      __syncwarp();
      dev::tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(half * 128);
      uint32_t va[32], vb[32], vc[32], vd[32];
      // all 128 columns into registers, then hand the accumulator back at once
      dev::tmem_load_32cols(taddr, va);
      dev::tmem_load_32cols(taddr + 32, vb);
      dev::tmem_load_32cols(taddr + 64, vc);
      dev::tmem_load_32cols(taddr + 96, vd);
      dev::tmem_load_wait(va);
      dev::tmem_load_wait(vb);
      dev::tmem_load_wait(vc);
      dev::tmem_load_wait(vd);
      dev::tc_fence_before();
      __syncwarp();
      if (lane == 0) dev::mbar_arrive_remote(acc_empty_leader);
      if (m0 >= M) continue;                         // rows past M (the pair tile's second half): nothing to store
#pragma unroll
      for (int c = 0; c < 4; ++c, ++chunk) {
        uint32_t (&cur)[32] = c == 0 ? va : c == 1 ? vb : c == 2 ? vc : vd;
        // this chunk's 32 bias values (lane-uniform addresses: broadcast loads)
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
        // the buffer of this chunk was last read by the store issued kEpiBufs chunks ago
        if (lane == 0) dev::bulk_wait_group_read<kEpiBufs - 1>();
        __syncwarp();
        uint8_t* buf = wbuf + (chunk % kEpiBufs) * kEpiBufBytes;
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
  if (warp == kMmaWarp) {
    __syncwarp();
    dev::tc_fence_after();
    dev::tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace

int k2_pair_rows_b() { return kBNh; }

size_t k2_pair_weight_bytes(int N, int K) {
  const size_t nb = (size_t)((N + 255) / 256), ktiles = (size_t)((K / 64 + kKB - 1) / kKB);
  return nb * ktiles * 2u * (size_t)kWBlockBytes;
}

void k2_pair_pack_weights(const uint8_t* tiled_codes, const uint8_t* sf, int N, int K, uint8_t* out) {
  // tiled_codes: the single-CTA layout (wgt_tile_offset), 32 KB per (256-row
  // block, stage); sf: the tensor-core scale layout, 512-byte chunks per
  // (128-row block, 64-K block), rows padded to 256
  const int nbl = (N + 255) / 256, kblocks = K / 64, ktiles = (kblocks + kKB - 1) / kKB;
  for (int b = 0; b < nbl; ++b)
    for (int t = 0; t < ktiles; ++t)
      for (int h = 0; h < 2; ++h) {
        uint8_t* dst = out + (((size_t)b * ktiles + t) * 2 + h) * kWBlockBytes;
        const uint8_t* src = tiled_codes + ((size_t)b * ktiles + t) * 32768u + (size_t)h * kBBytes;
        for (int i = 0; i < kBBytes; ++i) dst[i] = src[i];
        for (int hh = 0; hh < 2; ++hh)
          for (int j = 0; j < kKB; ++j) {
            uint8_t* d = dst + kBBytes + hh * (kKB * 512) + j * 512;
            const int kb = kKB * t + j;
            if (kb < kblocks) {
              const uint8_t* s = sf + ((size_t)(2 * b + hh) * kblocks + kb) * 512u;
              for (int i = 0; i < 512; ++i) d[i] = s[i];
            } else {
              for (int i = 0; i < 512; ++i) d[i] = 0;
            }
          }
      }
}

cudaError_t launch_k2_pair(const CUtensorMap& tm_xl, const CUtensorMap& tm_l2, const CUtensorMap& tm_y,
                           const K2Params& p, int num_sms, cudaStream_t stream) {
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(k2_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    // the warpgroups' register budgets add up to exactly 128 per thread
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, k2_pair_kernel);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != 128) return cudaErrorInvalidConfiguration;
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
  // programmatic dependent launch: the prologue and the weight stream overlap
  // the tail of the kernel that produces the activations; the activation
  // producer waits for it before its first load
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, k2_pair_kernel, tm_xl, tm_l2, tm_y, p);
}

}  // namespace svdq
