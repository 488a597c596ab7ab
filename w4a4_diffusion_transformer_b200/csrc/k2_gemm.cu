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
#include "sm100.cuh"

namespace svdq {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
// Stage shape: 4 blocks of 64 K per pipeline stage, i.e. 128-byte operand rows
// in the 128-byte swizzle: the tiled layout the operands are stored in.
constexpr int kKB = 4;
constexpr int kBKBytes = kKB * 32;           // E2M1 bytes per operand row per stage
constexpr int kStages = 3;
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
constexpr int kSmemBytes = kStages * kStageBytes + kBrBytes + kEpiWarps * kEpiWarpBytes + 1024 + 256;
static_assert(kSmemBytes <= 232448, "shared memory per block");
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
  uint8_t* brbuf = smem + kStages * kStageBytes;
  uint8_t* epi_buf = brbuf + kBrBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_buf + kEpiWarps * kEpiWarpBytes);
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
      // the activations come from the preceding kernel (launched as a
      // dependency); the weights do not, so their stream starts at once
      if (pa) dev::griddep_wait();
      int it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tcount) {
        const int m0 = (tile % tiles_m) * kBM;
        const int n0 = (tile / tiles_m) * kBN;
        if (p.branch) {
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
      // Do not leave while copies into this CTA's shared memory are in flight.
      for (int j = max(0, it - kStages); j < it; ++j)
        if (!dev::mbar_wait(&full[j % kStages], (uint32_t)(j / kStages) & 1u, abort_flag, p.budget_ns) ||
            !dev::mbar_wait(&sf_full[j % kStages], (uint32_t)(j / kStages) & 1u, abort_flag, p.budget_ns))
          break;
      if (p.branch && tcount > 0) dev::mbar_wait(br_full, (uint32_t)(tcount - 1) & 1u, abort_flag, p.budget_ns);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    dev::setmaxnreg_dec<kRegsCtl>();
    if (lane == 0) {
      const uint32_t idesc_f4 = dev::idesc_nvfp4(kBM, kBN);
      const uint32_t idesc_h = dev::idesc_bf16(kBM, kBN);
      int it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tcount) {
        if (!dev::mbar_wait(acc_empty, ((uint32_t)tcount & 1u) ^ 1u, abort_flag, p.budget_ns)) {
          record_error(p.err, abort_flag, 0x203);
          ok = false;
          break;
        }
        dev::tc_fence_after();
        uint32_t accumulate = 0;
        if (p.branch) {
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
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      for (int kt = 0; kt < ktiles; ++kt, ++it) {
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
  } else if (warp < kSfWarp0) {
    dev::setmaxnreg_dec<kRegsCtl>();                 // idle warp of the first warpgroup
  } else {
    // ------------------------------------------------------------ epilogue
    dev::setmaxnreg_inc<kRegsEpi>();
    const int q = warp & 3;                          // TMEM lane quarter of this warp
    const int half = (warp - kEpiWarp0) >> 2;       // which 128 of the 256 columns
    uint8_t* wbuf = epi_buf + (warp - kEpiWarp0) * kEpiWarpBytes;
    float* bias_s = reinterpret_cast<float*>(wbuf + 2 * kEpiBufBytes);
    if (lane == 0) dev::tma_prefetch_desc(&tm_y);
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

cudaError_t launch_k2(const CUtensorMap& tm_xl, const CUtensorMap& tm_l2, const CUtensorMap& tm_y,
                      const K2Params& p, int num_sms, cudaStream_t stream) {
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(k2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    // the warpgroups' register budgets add up to exactly 128 per thread
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, k2_kernel);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != 128) return cudaErrorInvalidConfiguration;
    configured_device = dev;
  }
  const int tiles = ((p.M + kBM - 1) / kBM) * ((p.N + kBN - 1) / kBN);
  const int grid = tiles < num_sms ? tiles : num_sms;
  // Programmatic dependent launch: the prologue (barriers, TMEM, descriptor
  // prefetch, weight stream) overlaps the tail of the kernel that produces the
  // activations; the activation producer waits for it before its first load.
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
