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
// Structure (one CTA per SM, persistent over output tiles, 16 warps):
//   warp 0     activation producer: per stage of 256 K the 128 x 256 E2M1 A
//              block (16 KB) and its scale factors (2 KB), each one contiguous
//              bulk copy (the first kernel writes both in the order the tensor
//              core reads them); per tile the XL rows into the branch buffer.
//   warp 2     weight producer: per stage one 36 KB block -- the 256 x 256
//              E2M1 B block followed by the scale factors of its 256 rows,
//              packed side by side when the layer is prepared (the scale
//              factors are copied first, then the codes); per tile the L2b^T
//              rows into the branch buffer.
//   warp 1     allocates TMEM (512 columns: accumulator 256 + per-stage scale
//              factors) and issues tcgen05.mma: per tile first the two branch
//              MMAs from the branch buffer (kept out of the ring, so a tile is
//              12 ring stages at K = 3072, not 13), then 4 NVFP4 MMAs per stage.
//   warps 4-7  move each stage's scale factors into TMEM as soon as they land
//              (their copies are issued first and complete their own barrier),
//              from registers (tcgen05.st, one warp per TMEM lane quarter; as
//              copies they would share the tensor pipe with the MMAs).
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
#include "nvfp4_quant.cuh"
#include "sm100.cuh"

namespace svdq {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
// Stage shape: 4 blocks of 64 K per pipeline stage, i.e. 128-byte operand rows
// in the 128-byte swizzle: the tiled layout the operands are stored in.
constexpr int kKB = 4;
constexpr int kBKBytes = kKB * 32;           // E2M1 bytes per operand row per stage
// Ring depth: 3 stages beside the branch buffer and the epilogue's staging.
// SVDQ_K2_DEEP=1 builds a 4-stage default mode instead (the low-rank branch
// becomes a ring stage and the epilogue stores Y straight from registers,
// which frees that shared memory); measured slower at the attention-output
// shape (31.0 vs 25.9 us): a lane holds one row, so each 16-byte store of the
// epilogue touches 32 rows, and that costs more than the deeper ring gains.
#ifndef SVDQ_K2_DEEP
#define SVDQ_K2_DEEP 0
#endif
constexpr uint32_t kSwz = 2u;                          // descriptor layout: 128-byte swizzle
constexpr uint32_t kSwzAtom = 8u * kBKBytes;           // bytes between 8-row groups
constexpr int kEpiWarps = 8;
// warp roles
constexpr int kProdA = 0, kMmaWarp = 1, kProdB = 2, kSfWarp0 = 4, kEpiWarp0 = 8;
constexpr int kThreads = 16 * 32;
// Register split (per thread, by warpgroup): control warps, scale-factor warps,
// the two epilogue warpgroups.  The sum over the block equals the launch
// allocation of 128 per thread, which the host checks before the first launch
// (a larger sum would make the increase wait forever).
constexpr int kRegsCtl = 56, kRegsSf = 72, kRegsEpi = 192;
static_assert(128 * kRegsCtl + 128 * kRegsSf + 256 * kRegsEpi == kThreads * 128, "register split");
constexpr int kEpiBufBytes = 32 * 64;        // one 32 x 32 BF16 output chunk
constexpr int kEpiWarpBytes = 2 * kEpiBufBytes + 512;   // two chunk buffers + 128 bias floats
// stage: [A 16 KB][B 32 KB][B scales 4 KB][A scales 2 KB]
constexpr int kABytes = kBM * kBKBytes;      // 16 KiB
constexpr int kBBytes = kBN * kBKBytes;      // 32 KiB
constexpr int kSFBBytes = 2 * kKB * 512;     // 2 row blocks x kKB K-blocks
constexpr int kSFABytes = kKB * 512;         // kKB K-blocks x 128 rows
constexpr int kOffB = kABytes;
constexpr int kOffSFB = kOffB + kBBytes;
constexpr int kOffSFA = kOffSFB + kSFBBytes;
constexpr int kStageBytes = kOffSFA + kSFABytes;
constexpr int kWBlockBytes = kBBytes + kSFBBytes;       // one weight block per stage (36 KB)
static_assert(kStageBytes % 1024 == 0, "stage alignment");
// branch buffer: [XL 128 rows x 64 B][L2b^T / alpha 256 rows x 64 B]
constexpr int kBrXL = kBM * 64;
constexpr int kBrBytes = kBrXL + kBN * 64;
static_assert(kBrBytes % 1024 == 0, "branch buffer alignment");

constexpr int kTmemCols = 512;
// Scale factors in TMEM, one region per pipeline stage (so a region is only
// rewritten after the MMAs that read it have completed): 4 columns per 128-row
// x 64-K block, 16 for A and 32 for B per stage.
constexpr int kSFCol0 = 256;
constexpr int kSFStageCols = 12 * kKB;       // 4 columns of A + 8 of B per K block

template <bool kChain>
struct K2Layout {
  static constexpr bool deep = !kChain && SVDQ_K2_DEEP;
  static constexpr int stages = deep ? 4 : 3;
  static constexpr int br_bytes = deep ? 0 : kBrBytes;
  static constexpr int epi_warp_bytes = deep ? 512 : kEpiWarpBytes;   // deep: 128 bias floats only
  static constexpr int smem = stages * kStageBytes + br_bytes + kEpiWarps * epi_warp_bytes + 1024 + 256;
  static_assert(smem <= 232448, "shared memory per block");
  static_assert(kSFCol0 + stages * kSFStageCols <= kTmemCols, "TMEM budget");
};

__device__ __forceinline__ void record_error(int* err, volatile int* abort_flag, int code) {
  atomicCAS(err, 0, code);
  *abort_flag = 1;
}

// Output tiles of one CTA, in order; every warp role walks the same sequence.
// Default: tile t = blockIdx.x + i gridDim.x, row block t % tiles_m (CTAs that
// run together share weight tiles).  Chain mode: work unit u = blockIdx.x +
// i gridDim.x is row block u / S and the (u % S)-th of S contiguous ranges of
// N tiles, so the epilogue can sum fc2's down projection over the unit.
template <bool kChain>
struct TileSeq {
  int tiles_m, tiles_n, S;
  __device__ int units() const { return kChain ? tiles_m * S : tiles_m * tiles_n; }
  __device__ int first(int u) const { return kChain ? (u % S) * tiles_n / S : 0; }
  __device__ int last(int u) const { return kChain ? ((u % S) + 1) * tiles_n / S : 1; }
  __device__ int m0(int u) const { return (kChain ? u / S : u % tiles_m) * kBM; }
  __device__ int n0(int u, int t) const { return (kChain ? t : u / tiles_m) * kBN; }
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <bool kChain>
__global__ void __launch_bounds__(kThreads, 1)
    k2_kernel(const __grid_constant__ CUtensorMap tm_xl, const __grid_constant__ CUtensorMap tm_l2,
              const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_xla,
              const __grid_constant__ CUtensorMap tm_l2a, K2Params p) {
  using Lay = K2Layout<kChain>;
  constexpr int kStages = Lay::stages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* brbuf = smem + kStages * kStageBytes;
  uint8_t* epi_buf = brbuf + Lay::br_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_buf + kEpiWarps * Lay::epi_warp_bytes);
  uint64_t* empty = full + kStages;
  uint64_t* sf_full = empty + kStages;             // a stage's scale factors are in shared memory
  uint64_t* sf_ready = sf_full + kStages;          // ... and in TMEM
  uint64_t* br_full = sf_ready + kStages;
  uint64_t* br_empty = br_full + 1;
  uint64_t* acc_full = br_empty + 1;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* rcp_s = reinterpret_cast<float*>(tmem_slot + 4);   // chain mode: the quantizer's constants

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int M = p.M, N = p.N, K = p.K;
  const int tiles_m = (M + kBM - 1) / kBM;
  const int tiles_n = (N + kBN - 1) / kBN;
  const TileSeq<kChain> ts{tiles_m, tiles_n, kChain ? p.chain.S : 1};
  const int kblocks = K >> 6;                     // 64-element K blocks
  const int ktiles = (kblocks + kKB - 1) / kKB;
  // Extra ring stages in front of each tile's K stages, each with XL rows in
  // the A slot and (L2 / alpha)^T rows in the B slot (64-byte rows) for two
  // BF16 MMAs; their scale-factor slots are moved but not read.  Stage 0: the
  // low-rank branch (deep mode; otherwise it has a buffer of its own); then a
  // LoRA adapter's XL_lora and (s B / alpha)^T.
  const int lora = kChain ? 0 : p.lora;
  const int br_stage = (Lay::deep && p.branch) ? 1 : 0;
  const int nextra = br_stage + lora;
  const bool br_buf = p.branch && !Lay::deep;

  if (threadIdx.x == 0) {
    // the next kernel on the stream may launch now; it waits for this grid's
    // completion before it touches anything this grid reads or writes
    dev::griddep_launch_dependents();
    for (int s = 0; s < kStages; ++s) {
      dev::mbar_init(&full[s], 2);                  // the two producers
      dev::mbar_init(&empty[s], 1);
      dev::mbar_init(&sf_full[s], 2);
      dev::mbar_init(&sf_ready[s], 4);              // the scale-factor warps
    }
    dev::mbar_init(br_full, 2);
    dev::mbar_init(br_empty, 1);
    dev::mbar_init(acc_full, 1);
    dev::mbar_init(acc_empty, kEpiWarps);
    dev::mbar_init(drain, 1);
    *abort_flag = 0;
    if (kChain) {
#pragma unroll
      for (int i = 0; i < 16; ++i) rcp_s[i] = p.chain.rcp[i];   // constant indices
    }
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
      if (lora) dev::tma_prefetch_desc(pa ? &tm_xla : &tm_l2a);
      const CUtensorMap* xmap[2] = {pa ? &tm_xl : &tm_l2, pa ? &tm_xla : &tm_l2a};
      // the activations come from the preceding kernel (launched as a
      // dependency); the weights do not, so their stream starts at once
      if (pa) dev::griddep_wait();
      int it = 0, tcount = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < ts.units() && ok; u += gridDim.x) {
        for (int t = ts.first(u); t < ts.last(u) && ok; ++t, ++tcount) {
          const int m0 = ts.m0(u);
          const int n0 = ts.n0(u, t);
          if (br_buf) {
            // the previous tile's branch MMAs have read the buffer
            if (!dev::mbar_wait(br_empty, ((uint32_t)tcount & 1u) ^ 1u, abort_flag, p.budget_ns)) {
              record_error(p.err, abort_flag, 0x201);
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
          for (int e = 0; e < nextra && ok; ++e, ++it) {
            const int s = it % kStages;
            if (!dev::mbar_wait(&empty[s], ((uint32_t)(it / kStages) & 1u) ^ 1u, abort_flag, p.budget_ns)) {
              record_error(p.err, abort_flag, 0x209);
              ok = false;
              break;
            }
            uint8_t* st = smem + s * kStageBytes;
            const CUtensorMap* map = xmap[e < br_stage ? 0 : 1];
            dev::mbar_arrive_expect_tx(&sf_full[s], 0u);   // no scale factors in this stage
            if (pa) {
              dev::mbar_arrive_expect_tx(&full[s], (uint32_t)(kBM * 64));
              dev::tma_load_2d(st, map, &full[s], 0, m0);
            } else {
              dev::mbar_arrive_expect_tx(&full[s], (uint32_t)(kBN * 64));
              dev::tma_load_2d(st + kOffB, map, &full[s], 0, n0);
            }
          }
          if (!ok) break;
          for (int kt = 0; kt < ktiles; ++kt, ++it) {
            const int s = it % kStages;
            if (!dev::mbar_wait(&empty[s], ((uint32_t)(it / kStages) & 1u) ^ 1u, abort_flag, p.budget_ns)) {
              record_error(p.err, abort_flag, 0x202);
              ok = false;
              break;
            }
            uint8_t* st = smem + s * kStageBytes;
            // The scale factors complete their own barrier and are issued first:
            // the scale-factor warps move them into TMEM while the operand
            // blocks are still in flight, off the stage's critical path.
            if (pa) {
              const uint32_t sf_bytes = (uint32_t)min(kKB, kblocks - kKB * kt) * 512u;
              const size_t a_chunk = (size_t)(m0 >> 7) * (size_t)kblocks + (size_t)(kKB * kt);
              dev::mbar_arrive_expect_tx(&sf_full[s], sf_bytes);
              dev::bulk_load(st + kOffSFA, p.sfa + a_chunk * 512, sf_bytes, &sf_full[s]);
              dev::mbar_arrive_expect_tx(&full[s], (uint32_t)kABytes);
              dev::bulk_load(st, p.acodes + ((size_t)(m0 >> 7) * (size_t)ktiles + (size_t)kt) * kABytes, kABytes,
                             &full[s]);
            } else {
              const uint8_t* wb = p.wmerged + ((size_t)(n0 >> 8) * (size_t)ktiles + (size_t)kt) * kWBlockBytes;
              dev::mbar_arrive_expect_tx(&sf_full[s], kSFBBytes);
              dev::bulk_load(st + kOffSFB, wb + kBBytes, kSFBBytes, &sf_full[s]);
              dev::mbar_arrive_expect_tx(&full[s], kBBytes);
              dev::bulk_load(st + kOffB, wb, kBBytes, &full[s]);
            }
          }
        }
      }
      // Do not leave while copies into this CTA's shared memory are in flight.
      for (int j = max(0, it - kStages); j < it; ++j)
        if (!dev::mbar_wait(&full[j % kStages], (uint32_t)(j / kStages) & 1u, abort_flag, p.budget_ns) ||
            !dev::mbar_wait(&sf_full[j % kStages], (uint32_t)(j / kStages) & 1u, abort_flag, p.budget_ns))
          break;
      if (br_buf && tcount > 0) dev::mbar_wait(br_full, (uint32_t)(tcount - 1) & 1u, abort_flag, p.budget_ns);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    dev::setmaxnreg_dec<kRegsCtl>();
    if (lane == 0) {
      const uint32_t idesc_f4 = dev::idesc_nvfp4(kBM, kBN);
      const uint32_t idesc_h = dev::idesc_bf16(kBM, kBN);
      int it = 0, tcount = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < ts.units() && ok; u += gridDim.x) {
        for (int t = ts.first(u); t < ts.last(u) && ok; ++t, ++tcount) {
          if (!dev::mbar_wait(acc_empty, ((uint32_t)tcount & 1u) ^ 1u, abort_flag, p.budget_ns)) {
            record_error(p.err, abort_flag, 0x203);
            ok = false;
            break;
          }
          dev::tc_fence_after();
          uint32_t accumulate = 0;
          if (br_buf) {
            if (!dev::mbar_wait(br_full, (uint32_t)tcount & 1u, abort_flag, p.budget_ns)) {
              record_error(p.err, abort_flag, 0x204);
              ok = false;
              break;
            }
            dev::tc_fence_after();
            const uint32_t a0 = dev::smem_u32(brbuf);
            const uint32_t b0 = a0 + kBrXL;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const uint64_t ad = dev::smem_desc(a0 + 32 * j, 16, 512, 4);
              const uint64_t bd = dev::smem_desc(b0 + 32 * j, 16, 512, 4);
              dev::mma_bf16(tmem, ad, bd, idesc_h, accumulate);
              accumulate = 1;
            }
            dev::tc_commit(br_empty);
          }
          for (int e = 0; e < nextra && ok; ++e, ++it) {
            const int s = it % kStages;
            if (!dev::mbar_wait(&full[s], (uint32_t)(it / kStages) & 1u, abort_flag, p.budget_ns) ||
                !dev::mbar_wait(&sf_ready[s], (uint32_t)(it / kStages) & 1u, abort_flag, p.budget_ns)) {
              record_error(p.err, abort_flag, 0x20A);
              ok = false;
              break;
            }
            dev::tc_fence_after();
            const uint32_t a0 = dev::smem_u32(smem + s * kStageBytes);
            const uint32_t b0 = a0 + kOffB;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const uint64_t ad = dev::smem_desc(a0 + 32 * j, 16, 512, 4);
              const uint64_t bd = dev::smem_desc(b0 + 32 * j, 16, 512, 4);
              dev::mma_bf16(tmem, ad, bd, idesc_h, accumulate);
              accumulate = 1;
            }
            dev::tc_commit(&empty[s]);
          }
          if (!ok) break;
          for (int kt = 0; kt < ktiles; ++kt, ++it) {
            const int s = it % kStages;
            if (!dev::mbar_wait(&full[s], (uint32_t)(it / kStages) & 1u, abort_flag, p.budget_ns) ||
                !dev::mbar_wait(&sf_ready[s], (uint32_t)(it / kStages) & 1u, abort_flag, p.budget_ns)) {
              record_error(p.err, abort_flag, 0x205);
              ok = false;
              break;
            }
            dev::tc_fence_after();
            const int nkb = min(kKB, kblocks - kKB * kt);
            const uint32_t a0 = dev::smem_u32(smem + s * kStageBytes);
            const uint32_t b0 = a0 + kOffB;
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
          dev::tc_commit(acc_full);
        }
      }
      // Wait until every MMA this thread issued has completed.
      dev::tc_commit(drain);
      dev::mbar_wait(drain, 0, abort_flag, p.budget_ns);
    }
  } else if (warp >= kSfWarp0 && warp < kSfWarp0 + 4) {
    // ------------------------------------------------------------ scale factors
    // Warp w writes TMEM lanes 32 (w % 4) .. +31.  The layout is the one the
    // 32x128b.warpx4 copy produces: lane 32 q + u holds, per 64-K block j, the
    // 16-byte unit u of A's 512-byte chunk in columns 4 j .. 4 j + 3 of the A
    // region, and unit u of B's two chunks (rows 0-127, 128-255) in columns
    // 8 j .. 8 j + 7 of the B region.
    dev::setmaxnreg_dec<kRegsSf>();
    const uint32_t lanebase = (uint32_t)((warp & 3) * 32) << 16;
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < ts.units() && ok; u += gridDim.x) {
      for (int t = ts.first(u); t < ts.last(u) && ok; ++t) {
        for (int kt = 0; kt < ktiles + nextra; ++kt, ++it) {   // the extra stages' slots are moved too, unread
          const int st = it % kStages;
          const bool got = dev::mbar_wait(&sf_full[st], (uint32_t)(it / kStages) & 1u, abort_flag, p.budget_ns);
          if (!__all_sync(0xffffffffu, got)) {
            if (lane == 0) record_error(p.err, abort_flag, 0x208);
            ok = false;
            break;
          }
          const uint8_t* sfa = smem + st * kStageBytes + kOffSFA;
          const uint8_t* sfb = smem + st * kStageBytes + kOffSFB;
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
    }
  } else if (warp < kSfWarp0) {
    dev::setmaxnreg_dec<kRegsCtl>();                 // idle warp of the first warpgroup
  } else {
    // ------------------------------------------------------------ epilogue
    dev::setmaxnreg_inc<kRegsEpi>();
    const int q = warp & 3;                          // TMEM lane quarter of this warp
    const int half = (warp - kEpiWarp0) >> 2;       // which 128 of the 256 columns
    if (!kChain) {
      uint8_t* wbuf = epi_buf + (warp - kEpiWarp0) * Lay::epi_warp_bytes;
      float* bias_s = reinterpret_cast<float*>(Lay::deep ? wbuf : wbuf + 2 * kEpiBufBytes);
      if (!Lay::deep && lane == 0) dev::tma_prefetch_desc(&tm_y);
      int tcount = 0, chunk = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < ts.units() && ok; u += gridDim.x) {
        for (int t = ts.first(u); t < ts.last(u) && ok; ++t, ++tcount) {
          const int m0 = ts.m0(u);
          const int n0 = ts.n0(u, t) + half * 128;
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
            ok = false;
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
          if (lane == 0) dev::mbar_arrive(acc_empty);
          if (Lay::deep) {
            // each lane stores its row's 128 columns, 16 bytes at a time
            const int row = m0 + q * 32 + lane;
            __nv_bfloat16* yrow = p.y + (size_t)row * N;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t (&cur)[32] = c == 0 ? va : c == 1 ? vb : c == 2 ? vc : vd;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                uint32_t packed[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float2 b2 = reinterpret_cast<const float2*>(bias_s)[c * 16 + j * 4 + e];
                  float y0 = p.alpha * __uint_as_float(cur[j * 8 + 2 * e]) + b2.x;
                  float y1 = p.alpha * __uint_as_float(cur[j * 8 + 2 * e + 1]) + b2.y;
                  if (p.gelu) {
                    y0 = dev::gelu_tanh(y0);
                    y1 = dev::gelu_tanh(y1);
                  }
                  const __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
                  packed[e] = *reinterpret_cast<const uint32_t*>(&h2);
                }
                const int col = n0 + c * 32 + j * 8;     // N is a multiple of 16: chunks are whole
                if (row < M && col < N)
                  *reinterpret_cast<uint4*>(yrow + col) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
              }
            }
            __syncwarp();                                 // bias_s is restaged for the next tile
          } else {
#pragma unroll
          for (int c = 0; c < 4; ++c, ++chunk) {
            uint32_t (&cur)[32] = c == 0 ? va : c == 1 ? vb : c == 2 ? vc : vd;
            // the buffer of this chunk was last read by the store issued two chunks ago
            if (lane == 0) dev::bulk_wait_group_read<1>();
            __syncwarp();
            uint8_t* buf = wbuf + (chunk & 1) * kEpiBufBytes;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t packed[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 b2 = reinterpret_cast<const float2*>(bias_s)[c * 16 + j * 4 + e];
                float y0 = p.alpha * __uint_as_float(cur[j * 8 + 2 * e]) + b2.x;
                float y1 = p.alpha * __uint_as_float(cur[j * 8 + 2 * e + 1]) + b2.y;
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
        }
      }
      if (!Lay::deep && lane == 0) dev::bulk_wait_group_all();
    } else {
      // ---------------------------------------------- chain: fc2's input
      // Shared memory of the epilogue in this mode: one 32 x 32 BF16 chunk
      // buffer per warp (the A operand of the down projection), and per column
      // half -- shared by its four warps -- fc2's L1d^T rows for the half's 128
      // input channels (two 128-byte-swizzled 32 x 64 sub-tiles) plus the
      // half's bias and fc2 1/lam values.  The four warps fetch their shares
      // with cp.async before they wait for the accumulator, so the loads are
      // hidden behind the mainloop.
      uint8_t* cbuf = epi_buf + (warp - kEpiWarp0) * 2048;
      uint8_t* l1s = epi_buf + 8 * 2048 + half * 8192;
      float* bias_h = reinterpret_cast<float*>(epi_buf + 8 * 2048 + 2 * 8192 + half * 1024);
      float* inv_h = bias_h + 128;
      const int bar_id = 1 + half;                   // named barrier of the half's 128 threads
      const bool br2 = p.chain.l1t != nullptr;
      const int K2 = p.chain.K2;
      float acc2[2][4][4];                           // this warp's share of y L1d2 over the unit
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc2[a][b][e] = 0.f;
      int tcount = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < ts.units() && ok; u += gridDim.x) {
        for (int t = ts.first(u); t < ts.last(u) && ok; ++t, ++tcount) {
          const int m0 = ts.m0(u);
          const int n0 = ts.n0(u, t) + half * 128;    // the half's first column = fc2 input channel
          dev::named_barrier(bar_id, 128);           // the previous tile's staged values are no longer read
          if (br2) {
            // rows 8q..8q+7 of fc2's L1d^T, 16 chunks of 8 channels each
            const int j = 8 * q + (lane >> 2);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int c16 = (lane & 3) * 4 + i;
              const int col = n0 + c16 * 8;
              const bool valid = col < K2;
              dev::cp_async16(l1s + (c16 >> 3) * 4096 + j * 128 + (((c16 & 7) ^ (j & 7)) << 4),
                              p.chain.l1t + (valid ? (size_t)j * K2 + col : 0), valid ? 16u : 0u);
            }
          }
          if (lane < 16) {
            // columns 32q..32q+31 of the half: bias (lanes 0-7), fc2 1/lam (lanes 8-15)
            const int col = n0 + 32 * q + 4 * (lane & 7);
            const bool valid = col < N;
            const float* src = lane < 8 ? p.bias : p.chain.inv_lam;
            float* dst = (lane < 8 ? bias_h : inv_h) + 32 * q + 4 * (lane & 7);
            dev::cp_async16(dst, src + (valid ? col : 0), valid ? 16u : 0u);
          }
          const bool got = dev::mbar_wait(acc_full, (uint32_t)tcount & 1u, abort_flag, p.budget_ns);
          // the half's four warps leave together or not at all
          if (!dev::named_barrier_and(bar_id, 128, __all_sync(0xffffffffu, got))) {
            if (lane == 0) record_error(p.err, abort_flag, 0x206);
            dev::cp_async_wait_all();
            ok = false;
            break;
          }
          dev::tc_fence_after();
          const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(half * 128);
          uint32_t va[32], vb[32], vc[32], vd[32];
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
          if (lane == 0) dev::mbar_arrive(acc_empty);
          dev::cp_async_wait_all();
          dev::named_barrier(bar_id, 128);           // every share of the staged values has landed
          // y = [gelu](alpha acc + b) rounded to BF16 -- the value fc2 would
          // read -- for all 128 columns first (halves the live registers)
          uint32_t hb[64];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t (&cur)[32] = c == 0 ? va : c == 1 ? vb : c == 2 ? vc : vd;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float2 b2 = reinterpret_cast<const float2*>(bias_h)[c * 16 + i];
              float y0 = p.alpha * __uint_as_float(cur[2 * i]) + b2.x;
              float y1 = p.alpha * __uint_as_float(cur[2 * i + 1]) + b2.y;
              if (p.gelu) {
                y0 = dev::gelu_tanh(y0);
                y1 = dev::gelu_tanh(y1);
              }
              const __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
              hb[c * 16 + i] = *reinterpret_cast<const uint32_t*>(&h2);
            }
          }
          const int row = m0 + q * 32 + lane;           // < mpad: the operand layouts hold padded rows
          const bool live = row < M;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int kc = n0 + c * 32;                  // fc2 input channel of the chunk's first value
            if (kc >= K2) break;                         // warp-uniform; K2 is a multiple of 64
            // x_hat = fp32(y * inv_lam2), then fc2's NVFP4 quantizer
            float2 v[16];
            const float2* inv2 = reinterpret_cast<const float2*>(inv_h) + c * 16;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const uint32_t w = hb[c * 16 + i];
              v[i] = __fmul2_rn(make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)), inv2[i]);
            }
            uint32_t packed[4];
            uint32_t sb2 = dev::nvfp4_quant32(v, p.chain.c_x, p.chain.g_x_exp, rcp_s, packed);
            if (!live) {                                  // padding rows: zero codes and scales
              sb2 = 0u;
              packed[0] = packed[1] = packed[2] = packed[3] = 0u;
            }
            *reinterpret_cast<uint4*>(p.chain.codes + act_tile_offset(row, kc >> 8, (kc & 255) >> 5, p.chain.nst)) =
                make_uint4(packed[0], packed[1], packed[2], packed[3]);
            *reinterpret_cast<uint16_t*>(p.chain.scales + sf_offset(row, kc >> 4, K2)) = (uint16_t)(sb2 & 0xFFFFu);
            if (br2) {
              // the 32 x 32 BF16 chunk into this warp's buffer (64-byte rows,
              // swizzled so that ldmatrix reads are conflict-free), then y L1d2
              // on the tensor cores: 2 row tiles x 4 column tiles x 2 k-steps
              __syncwarp();                              // the previous chunk's ldmatrix reads are done
#pragma unroll
              for (int j = 0; j < 4; ++j)
                *reinterpret_cast<uint4*>(cbuf + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
                    make_uint4(hb[c * 16 + 4 * j], hb[c * 16 + 4 * j + 1], hb[c * 16 + 4 * j + 2],
                               hb[c * 16 + 4 * j + 3]);
              __syncwarp();
              const uint32_t abase = dev::smem_u32(cbuf);
              const uint32_t bbase = dev::smem_u32(l1s) + (c >> 1) * 4096;
#pragma unroll
              for (int ks = 0; ks < 2; ++ks) {
                uint32_t a[2][4], b[2][4];
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                  const int r = mt * 16 + (lane & 15);
                  const int kch = 2 * ks + (lane >> 4);
                  ldsm_x4(abase + r * 64 + ((kch ^ ((r >> 1) & 3)) << 4), a[mt]);
                }
                const int c0 = (c & 1) * 4 + 2 * ks;       // 16-byte chunk of the k-step in the sub-tile row
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                  // n-tiles 2np, 2np+1: matrices (n 0-7, k lo), (n 0-7, k hi), (n 8-15, k lo), (n 8-15, k hi)
                  const int brow = np * 16 + (lane & 7) + ((lane >> 4) << 3);
                  const int bch = c0 + ((lane >> 3) & 1);
                  ldsm_x4(bbase + brow * 128 + ((bch ^ (brow & 7)) << 4), b[np]);
                }
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                  for (int np = 0; np < 2; ++np) {
                    mma_16816(acc2[mt][2 * np], a[mt], b[np][0], b[np][1]);
                    mma_16816(acc2[mt][2 * np + 1], a[mt], b[np][2], b[np][3]);
                  }
              }
            }
          }
          if (br2 && t == ts.last(u) - 1) {
            // the unit's partial sums for this warp's 32 rows: slot 2 (u % S) + half
            const int S2 = 2 * p.chain.S;
            const int slot = 2 * (u % p.chain.S) + half;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
              for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                  const int r = m0 + q * 32 + mt * 16 + (lane >> 2) + 8 * hh;
                  const int j = nt * 8 + 2 * (lane & 3);
                  *reinterpret_cast<float2*>(p.chain.partials + ((size_t)r * S2 + slot) * 32 + j) =
                      make_float2(acc2[mt][nt][2 * hh], acc2[mt][nt][2 * hh + 1]);
                  acc2[mt][nt][2 * hh] = 0.f;
                  acc2[mt][nt][2 * hh + 1] = 0.f;
                }
          }
          __syncwarp();
        }
      }
    }
  }

  __syncwarp();                                      // single-lane roles rejoin their warps first
  dev::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    dev::tc_fence_after();
    dev::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

int k2_block_n() { return kBN; }

size_t k2_weight_bytes(int N, int K) {
  const size_t nb = (size_t)((N + 255) / 256), ktiles = (size_t)((K / 64 + kKB - 1) / kKB);
  return nb * ktiles * (size_t)kWBlockBytes;
}

void k2_pack_weights(const uint8_t* tiled_codes, const uint8_t* sf, int N, int K, uint8_t* out) {
  // tiled_codes: 32 KB per (256-row block, stage) (wgt_tile_offset); sf: the
  // tensor-core scale layout, 512-byte chunks per (128-row block, 64-K block)
  const int nbl = (N + 255) / 256, kblocks = K / 64, ktiles = (kblocks + kKB - 1) / kKB;
  for (int b = 0; b < nbl; ++b)
    for (int t = 0; t < ktiles; ++t) {
      uint8_t* dst = out + ((size_t)b * ktiles + t) * kWBlockBytes;
      const uint8_t* src = tiled_codes + ((size_t)b * ktiles + t) * 32768u;
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

namespace {

template <bool kChain>
cudaError_t configure_k2() {
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device == dev) return cudaSuccess;
  cudaError_t e =
      cudaFuncSetAttribute(k2_kernel<kChain>, cudaFuncAttributeMaxDynamicSharedMemorySize, K2Layout<kChain>::smem);
  if (e != cudaSuccess) return e;
  // the warpgroups' register budgets add up to exactly 128 per thread
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, k2_kernel<kChain>);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != 128) return cudaErrorInvalidConfiguration;
  configured_device = dev;
  return cudaSuccess;
}

template <bool kChain>
cudaError_t launch_k2_impl(const CUtensorMap& tm_xl, const CUtensorMap& tm_l2, const CUtensorMap& tm_y,
                           const CUtensorMap& tm_xla, const CUtensorMap& tm_l2a, const K2Params& p, int grid,
                           cudaStream_t stream) {
  cudaError_t e = configure_k2<kChain>();
  if (e != cudaSuccess) return e;
  // Programmatic dependent launch: the prologue (barriers, TMEM, descriptor
  // prefetch, weight stream) overlaps the tail of the kernel that produces the
  // activations; the activation producer waits for it before its first load.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = K2Layout<kChain>::smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k2_kernel<kChain>, tm_xl, tm_l2, tm_y, tm_xla, tm_l2a, p);
}

}  // namespace

cudaError_t launch_k2(const CUtensorMap& tm_xl, const CUtensorMap& tm_l2, const CUtensorMap& tm_y,
                      const CUtensorMap& tm_xla, const CUtensorMap& tm_l2a, const K2Params& p, int num_sms,
                      cudaStream_t stream) {
  const int tiles = ((p.M + kBM - 1) / kBM) * ((p.N + kBN - 1) / kBN);
  return launch_k2_impl<false>(tm_xl, tm_l2, tm_y, tm_xla, tm_l2a, p, tiles < num_sms ? tiles : num_sms, stream);
}

int k2_chain_splits(int M, int N, int num_sms) {
  const int tm = (M + kBM - 1) / kBM, tn = (N + kBN - 1) / kBN;
  int S = num_sms / tm;
  if (S < 1) S = 1;
  if (S > tn) S = tn;
  return S;
}

cudaError_t launch_k2_chain(const CUtensorMap& tm_xl, const CUtensorMap& tm_l2, const K2Params& p, int num_sms,
                            cudaStream_t stream) {
  const int units = ((p.M + kBM - 1) / kBM) * p.chain.S;
  // tm_y and the LoRA maps are not used in chain mode: any valid map fills the slots
  return launch_k2_impl<true>(tm_xl, tm_l2, tm_l2, tm_l2, tm_l2, p, units < num_sms ? units : num_sms, stream);
}

}  // namespace svdq
