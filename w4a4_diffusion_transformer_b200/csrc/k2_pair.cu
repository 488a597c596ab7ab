// K2 on CTA pairs: the NVFP4 block-scaled GEMM with the fused up projection,
// computed by two CTAs (one cluster) per 256 x 256 output tile with the
// fifth-generation tensor core's pair mode (tcgen05 cta_group::2).
//
// Same mathematics as the single-CTA kernel (SOTA-314 practice page, "Do
// this": "Up Projection with the 4-bit compute, because they write the same
// output"):
//   acc  = XL (L2b / alpha) + sum_k (c_x s_x) (c_w s_w);   Y = bf16([gelu](alpha acc + b)).
//
// Why pairs: the single-CTA kernel is bound by the stream of its operand
// stages into each SM (54 KB per 16.8 MFLOP).  In pair mode each CTA holds its
// own 128 rows of A but only half of B's 256 rows; the tensor cores of the two
// SMs share the B halves.  A stage is then 38 KB per SM for the same work, and
// five of them fit.  On this part it measures slower than the single-CTA
// kernel all the same (pair MMAs deliver less per SM than single-CTA ones), so
// it runs only when selected.
//
// Layout of the work (CTA rank r = 0, 1 of the pair; tile rows m0.., cols n0..):
//   both CTAs   warp 0: TMA producer of this CTA's stage data: A rows m0+128r,
//               B rows n0+128r, A's scale factors (own rows) and B's (all 256
//               rows: each CTA's tensor core needs the scales of every column);
//               per tile a branch stage with XL rows m0+128r and L2b/alpha rows
//               n0+128r.  Warps 4-7: scale factors from shared memory into this
//               CTA's TMEM through registers (tcgen05.st, one warp per lane
//               quarter).  Warps 8-15: epilogue of this CTA's 128 accumulator
//               rows (the single-CTA kernel's epilogue).
//   rank 0      warp 1: MMA issuer (pair MMAs, M = 256).
//   rank 1      warp 1 forwards "stage data landed" and warp 2 "scale factors
//               in TMEM" to rank 0's barriers (remote mbarrier arrives), since
//               rank 0's pair operations read both CTAs' shared memory and TMEM.
// Rank 0's commits arrive on both CTAs' barriers (multicast commit): a stage is
// free in both, an accumulator is full in both.  Every epilogue warp of both
// CTAs hands the accumulator back through rank 0's barrier.  Every wait is
// bounded (sm100.cuh).
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
constexpr int kStages = SVDQ_K2P_STAGES;
constexpr int kEpiWarps = 8;
// warp roles: 0 producer, 1 MMA issuer (rank 0) or forwarder (rank 1), 2-3
// idle, 4-7 scale factors (one per TMEM lane quarter), 8-15 epilogue
constexpr int kSfWarp0 = 4;
constexpr int kEpiWarp0 = 8;
constexpr int kThreads = 16 * 32;
// register budgets per thread by warpgroup (control, scale factors, two
// epilogue warpgroups); they add up to the launch allocation of 128, which the
// host checks before the first launch
constexpr int kRegsCtl = 56, kRegsSf = 72, kRegsEpi = 192;
static_assert(128 * kRegsCtl + 128 * kRegsSf + 256 * kRegsEpi == kThreads * 128, "register split");
constexpr int kEpiBufBytes = 32 * 64;        // one 32 x 32 BF16 output chunk
constexpr int kEpiWarpBytes = 2 * kEpiBufBytes;
constexpr int kABytes = kBM * kBKBytes;      // 16 KiB
constexpr int kBBytes = kBNh * kBKBytes;     // 16 KiB
constexpr int kSFABytes = kKB * 512;         // kKB K-blocks x 128 rows
constexpr int kSFBBytes = 2 * kKB * 512;     // 2 row blocks (all 256 columns) x kKB K-blocks
constexpr int kStageBytes = kABytes + kBBytes + kSFABytes + kSFBBytes;
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

__device__ __forceinline__ float gelu_tanh(float y) {
  const float k0 = 0.7978845608028654f;   // sqrt(2/pi)
  return 0.5f * y * (1.0f + tanhf(k0 * (y + 0.044715f * y * y * y)));
}

__global__ void __launch_bounds__(kThreads, 1)
    k2_pair_kernel(const __grid_constant__ CUtensorMap tm_xl, const __grid_constant__ CUtensorMap tm_l2,
                   const __grid_constant__ CUtensorMap tm_y, K2Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi_buf = smem + kStages * kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_buf + kEpiWarps * kEpiWarpBytes);
  uint64_t* empty = full + kStages;
  uint64_t* sf_full = empty + kStages;         // this CTA's scale factors landed
  uint64_t* pfull = sf_full + kStages;         // rank 0: rank 1's stage data landed
  uint64_t* sf_ready = pfull + kStages;        // this CTA's scale factors of a stage are in its TMEM
  uint64_t* psf_ready = sf_ready + kStages;    // rank 0: rank 1's scale factors are in rank 1's TMEM
  uint64_t* acc_full = psf_ready + kStages;
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
      dev::mbar_init(&full[s], 1);
      dev::mbar_init(&empty[s], 1);
      dev::mbar_init(&sf_full[s], 1);
      dev::mbar_init(&pfull[s], 1);
      dev::mbar_init(&sf_ready[s], 4);          // this CTA's scale-factor warps
      dev::mbar_init(&psf_ready[s], 1);
    }
    dev::mbar_init(acc_full, 1);
    dev::mbar_init(acc_empty, 2 * kEpiWarps);
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
  dev::cluster_sync();                         // barriers and TMEM of both CTAs exist
  dev::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    dev::setmaxnreg_dec<kRegsCtl>();
    if (lane == 0) {
      if (p.branch) {
        dev::tma_prefetch_desc(&tm_xl);
        dev::tma_prefetch_desc(&tm_l2);
      }
      int it = 0;
      bool ok = true;
      bool deps_ready = false;     // activations come from the preceding kernel (launched as a dependency)
      for (int tile = pair_id; tile < num_tiles && ok; tile += npairs) {
        const int m0 = (tile % tiles_m) * kPM;
        const int n0 = (tile / tiles_m) * kBN;
        const int my_m = m0 + kBM * (int)rank, my_n = n0 + kBNh * (int)rank;
        const bool rows_a = my_m < M, rows_b = my_n < N;      // this CTA's rows exist (else they stay stale:
                                                              // their results are never stored)
        const bool sf_a = my_m < p.mpad;                      // the activation scales cover these rows
        if (p.branch) {
          const int s = it % kStages;
          if (!dev::mbar_wait_cluster(&empty[s], ((uint32_t)(it / kStages) & 1u) ^ 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x221);
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kStageBytes;
          dev::mbar_arrive(&sf_full[s]);               // a branch stage carries no scale factors
          dev::mbar_arrive_expect_tx(&full[s], (rows_a ? kBM * 64 : 0) + (rows_b ? kBNh * 64 : 0));
          if (rows_b) dev::tma_load_2d(st + kABytes, &tm_l2, &full[s], 0, my_n);
          if (!deps_ready) {
            dev::griddep_wait();
            deps_ready = true;
          }
          if (rows_a) dev::tma_load_2d(st, &tm_xl, &full[s], 0, my_m);
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
          const int nkb = min(kKB, kblocks - kKB * kt);
          const uint32_t sf_bytes = (uint32_t)nkb * 512u;
          // scale factors on their own barrier, issued first (their TMEM copies
          // then run while the operand tiles are still in flight)
          dev::mbar_arrive_expect_tx(&sf_full[s], (sf_a ? sf_bytes : 0u) + 2u * sf_bytes);
          dev::mbar_arrive_expect_tx(&full[s], (sf_a ? kABytes : 0) + kBBytes);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const size_t b_chunk = (size_t)((n0 >> 7) + h) * (size_t)kblocks + (size_t)(kKB * kt);
            dev::bulk_load(st + kABytes + kBBytes + kSFABytes + h * (kKB * 512), p.sfb + b_chunk * 512, sf_bytes,
                           &sf_full[s]);
          }
          // this CTA's 128-row half of the 256-row weight block (tiled, pre-swizzled)
          dev::bulk_load(st + kABytes,
                         p.wcodes + ((size_t)(n0 >> 8) * (size_t)ktiles + (size_t)kt) * (2 * kBBytes) + rank * kBBytes,
                         kBBytes, &full[s]);
          if (!deps_ready) {
            dev::griddep_wait();
            deps_ready = true;
          }
          if (sf_a) {
            const size_t a_chunk = (size_t)(my_m >> 7) * (size_t)kblocks + (size_t)(kKB * kt);
            dev::bulk_load(st + kABytes + kBBytes, p.sfa + a_chunk * 512, sf_bytes, &sf_full[s]);
          }
          if (sf_a)
            dev::bulk_load(st, p.acodes + ((size_t)(my_m >> 7) * (size_t)ktiles + (size_t)kt) * kABytes, kABytes,
                           &full[s]);
          ++it;
        }
      }
      for (int j = max(0, it - kStages); j < it; ++j)
        if (!dev::mbar_wait(&full[j % kStages], (uint32_t)(j / kStages) & 1u, abort_flag, p.budget_ns) ||
            !dev::mbar_wait(&sf_full[j % kStages], (uint32_t)(j / kStages) & 1u, abort_flag, p.budget_ns))
          break;
    }
  } else if (warp == 1 && !leader) {
    // ------------------------------------------------------------ rank 1: forward "stage data landed"
    dev::setmaxnreg_dec<kRegsCtl>();
    if (lane == 0) {
      const int uses = (num_tiles > pair_id ? (num_tiles - pair_id + npairs - 1) / npairs : 0) *
                       (ktiles + (p.branch ? 1 : 0));
      for (int it = 0; it < uses; ++it) {
        const int s = it % kStages;
        if (!dev::mbar_wait(&full[s], (uint32_t)(it / kStages) & 1u, abort_flag, p.budget_ns)) {
          record_error(p.err, abort_flag, 0x223);
          break;
        }
        dev::mbar_arrive_remote(dev::map_to_rank(&pfull[s], 0));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ rank 0: MMA issuer
    dev::setmaxnreg_dec<kRegsCtl>();
    if (lane == 0) {
      const uint32_t idesc_f4 = dev::idesc_nvfp4(kPM, kBN);
      const uint32_t idesc_h = dev::idesc_bf16(kPM, kBN);
      auto wait_data = [&](int slot, int code) -> bool {
        const int s = slot % kStages;
        const uint32_t ph = (uint32_t)(slot / kStages) & 1u;
        if (!dev::mbar_wait(&full[s], ph, abort_flag, p.budget_ns) ||
            !dev::mbar_wait_cluster(&pfull[s], ph, abort_flag, p.budget_ns)) {
          record_error(p.err, abort_flag, code);
          return false;
        }
        dev::tc_fence_after();
        return true;
      };
      uint32_t sf_phase = 0;                          // per-stage parity of sf_ready
      int it = 0, tcount = 0;
      bool ok = true;
      for (int tile = pair_id; tile < num_tiles && ok; tile += npairs, ++tcount) {
        const int kslot0 = it + (p.branch ? 1 : 0);
        if (!dev::mbar_wait_cluster(acc_empty, ((uint32_t)tcount & 1u) ^ 1u, abort_flag, p.budget_ns)) {
          record_error(p.err, abort_flag, 0x225);
          ok = false;
          break;
        }
        dev::tc_fence_after();
        uint32_t accumulate = 0;
        if (p.branch) {
          if (!(ok = wait_data(it, 0x226))) break;
          const int s = it % kStages;
          const uint32_t a0 = dev::smem_u32(smem + s * kStageBytes);
          const uint32_t b0 = a0 + kABytes;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            dev::mma_f16_pair(tmem, dev::smem_desc(a0 + 32 * j, 16, 512, 4), dev::smem_desc(b0 + 32 * j, 16, 512, 4),
                              idesc_h, accumulate);
            accumulate = 1;
          }
          dev::tc_commit_pair(&empty[s], kBoth);
        }
        for (int kt = 0; kt < ktiles; ++kt) {
          const int slot = kslot0 + kt;
          const int s = slot % kStages;
          if (!(ok = wait_data(slot, 0x227))) break;
          if (!dev::mbar_wait(&sf_ready[s], (sf_phase >> s) & 1u, abort_flag, p.budget_ns) ||
              !dev::mbar_wait_cluster(&psf_ready[s], (sf_phase >> s) & 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x228);
            ok = false;
            break;
          }
          sf_phase ^= 1u << s;
          dev::tc_fence_after();
          const int nkb = min(kKB, kblocks - kKB * kt);
          const uint32_t a0 = dev::smem_u32(smem + s * kStageBytes);
          const uint32_t b0 = a0 + kABytes;
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
        it = kslot0 + ktiles;
        dev::tc_commit_pair(acc_full, kBoth);
      }
      // Wait until every pair operation this thread issued has completed.
      dev::tc_commit_pair(drain, kLeader);
      dev::mbar_wait(drain, 0, abort_flag, p.budget_ns);
    }
  } else if (warp >= kSfWarp0 && warp < kSfWarp0 + 4) {
    // ------------------------------------------------------------ scale factors (both CTAs)
    // Warp w writes its CTA's TMEM lanes 32 (w % 4) .. +31 from registers
    // (tcgen05.st), in the layout a 32x128b.warpx4 copy produces: per 64-K
    // block j, unit `lane` of A's 512-byte chunk (this CTA's 128 rows) in
    // columns 4 j .. 4 j + 3 of the A region, and of B's two chunks (all 256
    // columns of the tile) in columns 8 j .. 8 j + 7 of the B region (rank 1's
    // readiness reaches rank 0 through a forwarder).  The tensor pipe stays
    // with the MMAs.
    dev::setmaxnreg_dec<kRegsSf>();
    const uint32_t lanebase = (uint32_t)((warp & 3) * 32) << 16;
    int it = 0;
    bool ok = true;
    for (int tile = pair_id; tile < num_tiles && ok; tile += npairs) {
      if (p.branch) ++it;
      for (int kt = 0; kt < ktiles; ++kt, ++it) {
        const int st = it % kStages;
        const bool got = dev::mbar_wait(&sf_full[st], (uint32_t)(it / kStages) & 1u, abort_flag, p.budget_ns);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) record_error(p.err, abort_flag, 0x229);
          ok = false;
          break;
        }
        const uint8_t* sfa = smem + st * kStageBytes + kABytes + kBBytes;
        const uint8_t* sfb = sfa + kSFABytes;
        uint32_t ra[16], rb[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          // blocks past the K tail (and the A scales of rows past the
          // activations' padding) hold stale bytes whose results are never used
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
  } else if (warp == 2 && !leader) {
    // ------------------------------------------------------------ rank 1: forward "scale factors in TMEM"
    dev::setmaxnreg_dec<kRegsCtl>();
    if (lane == 0) {
      const uint32_t psf0 = dev::map_to_rank(psf_ready, 0);
      uint32_t sf_phase = 0;                        // per-slot parity of sf_ready (k-stages only)
      int it = 0;
      bool ok = true;
      for (int tile = pair_id; tile < num_tiles && ok; tile += npairs) {
        if (p.branch) ++it;                         // branch stages carry no scale factors
        for (int kt = 0; kt < ktiles; ++kt, ++it) {
          const int s = it % kStages;
          if (!dev::mbar_wait(&sf_ready[s], (sf_phase >> s) & 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x22b);
            ok = false;
            break;
          }
          sf_phase ^= 1u << s;
          dev::tc_fence_after();
          dev::mbar_arrive_remote(psf0 + 8u * (uint32_t)s);
        }
      }
    }
  } else if (warp >= 2 && warp < kSfWarp0) {
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
              y0 = gelu_tanh(y0);
              y1 = gelu_tanh(y1);
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
  if (warp == 1) {
    __syncwarp();
    dev::tc_fence_after();
    dev::tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace

int k2_pair_rows_b() { return kBNh; }

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
  // programmatic dependent launch: the prologue overlaps the tail of the kernel
  // that produces the activations; the producers wait for it before loading them
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, k2_pair_kernel, tm_xl, tm_l2, tm_y, p);
}

}  // namespace svdq
