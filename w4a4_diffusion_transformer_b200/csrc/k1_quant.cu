// K1: fused low-rank down projection + activation quantization.
//
// SOTA-314 practice page, "Do this": the fusion pairs "Down Projection with
// Quantize, because they read the same input"; NOTE-257 note page, "Key
// results": unfused, the branch costs "the extra 16-bit read in Down
// Projection".  One pass over X (BF16, [M][K]) produces
//   * the NVFP4 activation codes of x_hat = fp32(x * inv_lam) in groups of 16
//     along K (E4M3 scale per group, power-of-two tensor scale g_x), packed two
//     per byte with the even k in the low nibble, and the E4M3 scales in the
//     tensor-core scale-factor layout the GEMM reads directly;
//   * XL = bf16(X L1d) (rank 32; 1/lam is folded into L1d).
//
// Layout of the work: a CTA owns 32 token rows and streams the whole K range in
// stages of 256 columns.  Two producer warps load with TMA (one 3D copy per
// stage over a 64-column-chunk view): one feeds a 6-deep ring of X tiles
// (+ 256 floats of inv_lam) from HBM, the other a 5-deep ring of the matching
// 256 x 32 slices of L1d^T, which every CTA reads from L2.  The consumer warps
// are specialized and never wait for each other inside the loop:
//   * 8 quantizer warps: warp w owns columns 32w..32w+31 of the stage (two
//     groups) and lane l owns row l, so the inv_lam reads are broadcasts and
//     the swizzled X reads are conflict-free.  Each lane stores its 16 code
//     bytes straight from registers into the GEMM's tiled, pre-swizzled operand
//     layout; the two scale bytes of a lane are stored as one 2-byte word;
//   * 8 down-projection warps on the tensor cores (mma.sync BF16; the
//     projection is 32 columns wide and the pass is bound by memory, not by the
//     tensor pipe): warp w owns k-steps 2w, 2w+1 of every stage for all 32 rows
//     and all 32 output columns, so every operand fragment is read from shared
//     memory once; the eight partial sums are added through shared memory at
//     the end.
//
// The INT4 variant (groups of 64, BF16 scales, codes in [-7, 7]; SOTA-314
// "Do this") runs 4 quantizer warps of 64 columns each, stores each warp's
// 32 x 32-byte code tile (row-major [M][K/2]) with its own TMA store, and writes
// its scales group-major, [K/64][M padded to 128] BF16, the order the INT4 GEMM
// stages them in.
//
// NVFP4 quantizer arithmetic per group of 16 (bit-exact with the CPU oracle; the
// device code is nvfp4_quant32 in nvfp4_quant.cuh): a = max|v|; t = fp32(a *
// c_x) with c_x = fp32(1/6) 2^-gx; s = E4M3_rn_satfinite(t); s == 0 -> all
// codes +0; inv = fp32(1 / (s * g_x)); code = E2M1_rn_satfinite(fp32(v *
// inv)).  The reciprocal is exact without a division: for s = (1 + m/8)
// 2^(e-7) (or m 2^-9 when e = 0) it equals fp32(1/(1 + m/8)) 2^(7-e-gx) (or
// fp32(1/m) 2^(9-gx)), a power-of-two scaling of one of 15 correctly rounded
// constants computed on the host.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "nvfp4_quant.cuh"
#include "sm100.cuh"

namespace svdq {

namespace {

constexpr int kRows = 32;
constexpr int kBK = 256;
// Ring depths (measured at the attention-output shape: 6 X + 5 L1d^T stages
// 12.8 us per launch back to back, 8 + 3 stages 13.1 us).
#ifndef SVDQ_K1_XSTAGES
#define SVDQ_K1_XSTAGES 6
#endif
#ifndef SVDQ_K1_LSTAGES
#define SVDQ_K1_LSTAGES 5
#endif
constexpr int kXStages = SVDQ_K1_XSTAGES;     // X + inv_lam ring (HBM stream)
constexpr int kLStages = SVDQ_K1_LSTAGES;     // L1d^T ring (L2-resident)
constexpr int kMmaWarps = 8;
constexpr int kXBytes = kRows * kBK * 2;     // 4 sub-tiles of 32 rows x 128 B
constexpr int kLBytes = 32 * kBK * 2;        // 4 sub-tiles of 32 rows x 128 B
constexpr int kIBytes = kBK * 4;
constexpr int kXStageBytes = kXBytes + kIBytes;            // 17 KiB, 1 KiB multiple
constexpr int kCodeBytes = 8 * 1024;                       // code staging tiles, double-buffered per warp
// Quantizer warps per format: NVFP4 warps own 32 columns of a stage (two
// groups of 16), INT4 warps own 64 columns (one group of 64).
template <int F>
struct K1Shape {
  static constexpr int quant_warps = F == kFmtInt4 ? 4 : 8;
  static constexpr int cols = kBK / quant_warps;                     // columns per quantizer warp
  static constexpr int code_tile = kRows * cols / 2;                 // its codes: 32 rows x cols/2 B
  static constexpr int consumer_warps = quant_warps + kMmaWarps;
  static constexpr int threads = (consumer_warps + 2) * 32;
  static_assert(quant_warps * 2 * code_tile == kCodeBytes, "code staging size");
};
constexpr int kPartBytes = kMmaWarps * 32 * 32 * 4;         // down-projection partial sums
static_assert(kPartBytes <= kLStages * kLBytes, "partial sums reuse the L1d^T ring");
constexpr int kSmemBytes = kXStages * kXStageBytes + kLStages * kLBytes + kCodeBytes + 1024 + 256 + 16 * 4;

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

// Byte offset of 16-byte chunk `c` of row `r` in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

__device__ __forceinline__ void record_error(int* err, volatile int* abort_flag, int code) {
  atomicCAS(err, 0, code);
  *abort_flag = 1;
}

__device__ __forceinline__ void mma_warps_sync() { dev::named_barrier(1, kMmaWarps * 32); }

template <int kFmt, bool kQuant, bool kDown>
__global__ void __launch_bounds__(K1Shape<kFmt>::threads, 1)
    k1_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l,
              const __grid_constant__ CUtensorMap tm_c, K1Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* lring = smem + kXStages * kXStageBytes;              // L1d^T ring (1 KiB aligned)
  uint8_t* cbuf = lring + kLStages * kLBytes;                    // code staging tiles
  float4* part = reinterpret_cast<float4*>(lring);               // partial sums, after the loop
  uint64_t* xfull = reinterpret_cast<uint64_t*>(cbuf + kCodeBytes);
  uint64_t* xempty = xfull + kXStages;
  uint64_t* lfull = xempty + kXStages;
  uint64_t* lempty = lfull + kLStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(lempty + kLStages);
  float* rcp = reinterpret_cast<float*>(cbuf + kCodeBytes + 256);   // reciprocal table
  constexpr int kQuantWarps = K1Shape<kFmt>::quant_warps;
  constexpr int kConsumerWarps = K1Shape<kFmt>::consumer_warps;
  constexpr int kCodeTile = K1Shape<kFmt>::code_tile;
  constexpr int kActiveWarps = (kQuant ? kQuantWarps : 0) + (kDown ? kMmaWarps : 0);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * kRows;
  const int K = p.K;
  const int nk = (K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    // the GEMM that consumes this kernel's outputs may start its prologue now;
    // it waits for this grid's completion before reading them
    dev::griddep_launch_dependents();
    for (int s = 0; s < kXStages; ++s) {
      dev::mbar_init(&xfull[s], 1);
      dev::mbar_init(&xempty[s], kActiveWarps);
    }
    for (int s = 0; s < kLStages; ++s) {
      dev::mbar_init(&lfull[s], 1);
      dev::mbar_init(&lempty[s], kMmaWarps);
    }
    *abort_flag = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) rcp[i] = p.rcp[i];     // constant indices: stays in parameter space
    dev::fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ X producer
    if (lane == 0) {
      dev::tma_prefetch_desc(&tm_x);
      // This kernel is itself a programmatic dependent launch: X may be the
      // output of the preceding kernel, and that kernel may still read the
      // buffers this one writes.  Every write here follows an X stage, so
      // waiting before the first X load covers both.
      dev::griddep_wait();
      int issued = 0;
      for (int it = 0; it < nk; ++it) {
        const int s = it % kXStages;
        if (!dev::mbar_wait(&xempty[s], ((uint32_t)(it / kXStages) & 1u) ^ 1u, abort_flag, p.budget_ns)) {
          record_error(p.err, abort_flag, 0x101);
          break;
        }
        uint8_t* st = smem + s * kXStageBytes;
        const int k0 = it * kBK;
        const int kvalid = min(kBK, K - k0);
        // one box brings the stage's four 64-column sub-tiles (past K they
        // are zero-filled, and no consumer reads them)
        dev::mbar_arrive_expect_tx(&xfull[s], (uint32_t)kXBytes + (kQuant ? (uint32_t)kvalid * 4u : 0u));
        dev::tma_load_3d(st, &tm_x, &xfull[s], 0, row0, k0 >> 6);
        if (kQuant) dev::bulk_load(st + kXBytes, p.inv_lam + k0, (uint32_t)kvalid * 4u, &xfull[s]);
        issued = it + 1;
      }
      // Do not leave while copies into this CTA's shared memory are in flight.
      for (int it = max(0, issued - kXStages); it < issued; ++it)
        if (!dev::mbar_wait(&xfull[it % kXStages], (uint32_t)(it / kXStages) & 1u, abort_flag, p.budget_ns)) break;
    }
    return;
  }
  if (warp == kConsumerWarps + 1) {
    // ------------------------------------------------------------ L1d^T producer
    if (kDown && lane == 0) {
      dev::tma_prefetch_desc(&tm_l);
      int issued = 0;
      for (int it = 0; it < nk; ++it) {
        const int s = it % kLStages;
        if (!dev::mbar_wait(&lempty[s], ((uint32_t)(it / kLStages) & 1u) ^ 1u, abort_flag, p.budget_ns)) {
          record_error(p.err, abort_flag, 0x104);
          break;
        }
        const int k0 = it * kBK;
        dev::mbar_arrive_expect_tx(&lfull[s], (uint32_t)kLBytes);
        dev::tma_load_3d(lring + s * kLBytes, &tm_l, &lfull[s], 0, 0, k0 >> 6);
        issued = it + 1;
      }
      for (int it = max(0, issued - kLStages); it < issued; ++it)
        if (!dev::mbar_wait(&lfull[it % kLStages], (uint32_t)(it / kLStages) & 1u, abort_flag, p.budget_ns)) break;
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const bool quant_warp = warp < kQuantWarps;
  if ((quant_warp && !kQuant) || (!quant_warp && !kDown)) return;   // role not used by this variant

  if (quant_warp && kFmt == kFmtInt4) {
    // ---------------------------------------------------------- INT4 quantizer
    // Warp w owns sub-tile w of each stage (columns 64w..64w+63: one group of
    // 64) and lane l owns row l.  Per group: a = max|v|; s = bf16(fp32(a *
    // fp32(1/7))); s == 0 -> all codes 0; inv = fp32(1/s) (correctly rounded
    // reciprocal); code = rint_even(fp32(v * inv)).  |v * inv| <= 7 (1 + 2^-8)
    // because s is a > 0 divided by 7 and rounded to 8 significant bits, so the
    // clamp to [-7, 7] never changes a code.  Rounding adds 1.5 * 2^23: the
    // sum's low mantissa bits are then the rounded integer in two's
    // complement, so its low nibble is the 4-bit code.
    const int grow = row0 + lane;                     // < mpad: the grid covers the padded rows
    uint16_t* srow = reinterpret_cast<uint16_t*>(p.scales) + grow;   // scales [K/64][mpad]
    uint8_t* ctile = cbuf + warp * 2 * kCodeTile;
    if (lane == 0) dev::tma_prefetch_desc(&tm_c);
    for (int it = 0; it < nk; ++it) {
      const int s = it % kXStages;
      if (!dev::mbar_wait(&xfull[s], (uint32_t)(it / kXStages) & 1u, abort_flag, p.budget_ns)) {
        record_error(p.err, abort_flag, 0x102);
        break;
      }
      const uint8_t* st = smem + s * kXStageBytes;
      const int k0 = it * kBK;
      const bool active = warp * 64 < min(kBK, K - k0);
      uint32_t packed[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      uint32_t sbits = 0u;
      if (active) {
        const uint8_t* xt = st + warp * 4096;
        const float4* inv4 = reinterpret_cast<const float4*>(st + kXBytes) + warp * 16;
        float2 v[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 raw = *reinterpret_cast<const uint4*>(xt + sw128(lane, i));
          const float4 ia = inv4[2 * i], ib = inv4[2 * i + 1];
          const float2 iv[4] = {make_float2(ia.x, ia.y), make_float2(ia.z, ia.w), make_float2(ib.x, ib.y),
                                make_float2(ib.z, ib.w)};
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            v[i * 4 + e] = __fmul2_rn(make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u)),
                                      iv[e]);
        }
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) a = dev::fmax3(a, fabsf(v[i].x), fabsf(v[i].y));
        const __nv_bfloat16 sb = __float2bfloat16_rn(__fmul_rn(a, 1.0f / 7.0f));
        sbits = __bfloat16_as_ushort(sb);
        const float sc = __bfloat162float(sb);
        if (sc != 0.f) {
          const float inv = __frcp_rn(sc);
          const float2 inv2 = make_float2(inv, inv);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            // codes 8j..8j+7: even ones form byte-lanes A, odd ones B; byte i of
            // the word holds code 8j+2i in its low nibble and 8j+2i+1 in its high
            uint32_t t[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              // q = fp32(v * inv) must be rounded before the integer rounding:
              // the scalar __fadd_rn is never contracted with the multiply into
              // a fused multiply-add (a packed add can be, which rounds the
              // exact product and moves ties such as 2.5000000326 -> 3)
              const float2 q = __fmul2_rn(v[4 * j + e], inv2);
              t[2 * e] = __float_as_uint(__fadd_rn(q.x, 12582912.0f));
              t[2 * e + 1] = __float_as_uint(__fadd_rn(q.y, 12582912.0f));
            }
            const uint32_t A = __byte_perm(__byte_perm(t[0], t[2], 0x0040), __byte_perm(t[4], t[6], 0x0040), 0x5410);
            const uint32_t B = __byte_perm(__byte_perm(t[1], t[3], 0x0040), __byte_perm(t[5], t[7], 0x0040), 0x5410);
            packed[j] = (A & 0x0F0F0F0Fu) | ((B << 4) & 0xF0F0F0F0u);
          }
        }
      }
      // the stage's inputs have been read
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&xempty[s]);
      if (active) {
        srow[(size_t)((k0 >> 6) + warp) * (size_t)p.mpad] = (uint16_t)sbits;
        // codes: this warp's 32 x 32-byte tile, stored with TMA once the store
        // that last read this buffer (two stages ago) is done reading
        uint8_t* ct = ctile + (it & 1) * kCodeTile;
        if (lane == 0) dev::bulk_wait_group_read<1>();
        __syncwarp();
        *reinterpret_cast<uint4*>(ct + lane * 32) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        *reinterpret_cast<uint4*>(ct + lane * 32 + 16) = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        dev::fence_async_shared();
        __syncwarp();
        if (lane == 0) {
          dev::tma_store_2d(&tm_c, ct, (k0 + warp * 64) >> 1, row0);
          dev::bulk_commit_group();
        }
      }
    }
    if (lane == 0) dev::bulk_wait_group_all();
    return;
  }
  if (quant_warp && kFmt == kFmtInt8) {
    // ---------------------------------------------------------- INT8 quantizer
    // Warp w owns columns 32w..32w+31 of each 256-column stage, lane l row l;
    // code = clamp(rint_even(fp32(v * inv_sx)), -127, 127) with v = fp32(x *
    // inv_lam) and the row's 1/s_x from the per-token scale pass.  The 32
    // codes go to the GEMM's tiled layout in 128-column stages: stage 2 it +
    // w / 4, 16-byte chunks 2 (w % 4) and 2 (w % 4) + 1.
    const int grow = row0 + lane;                     // < mpad
    const int nst8 = (K + 127) / 128;
    float invs = 0.f;
    for (int it = 0; it < nk; ++it) {
      const int s = it % kXStages;
      if (!dev::mbar_wait(&xfull[s], (uint32_t)(it / kXStages) & 1u, abort_flag, p.budget_ns)) {
        record_error(p.err, abort_flag, 0x105);
        break;
      }
      // the per-token scales come from the preceding kernel: read them only
      // after the first X stage, which the X producer loads after waiting for it
      if (it == 0) invs = p.inv_sx[grow];             // zero for padding rows: zero codes
      const uint8_t* st = smem + s * kXStageBytes;
      const int k0 = it * kBK;
      const int kvalid = min(kBK, K - k0);
      const int col0 = warp * 32;
      const bool active = col0 < kvalid;              // kvalid is a multiple of 64
      uint32_t w8[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      if (active) {
        const uint8_t* xt = st + (col0 >> 6) * 4096;
        const int c0 = (col0 & 63) >> 3;
        const float4* inv4 = reinterpret_cast<const float4*>(st + kXBytes) + (col0 >> 2);
        const float2 is2 = make_float2(invs, invs);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 raw = *reinterpret_cast<const uint4*>(xt + sw128(lane, c0 + i));
          const float4 ia = inv4[2 * i], ib = inv4[2 * i + 1];
          const float2 iv[4] = {make_float2(ia.x, ia.y), make_float2(ia.z, ia.w), make_float2(ib.x, ib.y),
                                make_float2(ib.z, ib.w)};
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            // four codes (columns 8i + 2e .. +3) into one 32-bit word
            const float2 v0 = __fmul2_rn(
                make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u)), iv[e]);
            const float2 v1 = __fmul2_rn(
                make_float2(__uint_as_float(w[e + 1] << 16), __uint_as_float(w[e + 1] & 0xFFFF0000u)), iv[e + 1]);
            const float2 q0 = __fmul2_rn(v0, is2), q1 = __fmul2_rn(v1, is2);
            const int c[4] = {max(-127, min(127, __float2int_rn(q0.x))), max(-127, min(127, __float2int_rn(q0.y))),
                              max(-127, min(127, __float2int_rn(q1.x))), max(-127, min(127, __float2int_rn(q1.y)))};
            w8[2 * i + (e >> 1)] = (uint32_t)(c[0] & 0xFF) | ((uint32_t)(c[1] & 0xFF) << 8) |
                                   ((uint32_t)(c[2] & 0xFF) << 16) | ((uint32_t)(c[3] & 0xFF) << 24);
          }
        }
      }
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&xempty[s]);
      if (active) {
        const int t8 = 2 * it + (warp >> 2);
        const int ch = (warp & 3) * 2;
        *reinterpret_cast<uint4*>(p.codes + act_tile_offset(grow, t8, ch, nst8)) = make_uint4(w8[0], w8[1], w8[2], w8[3]);
        *reinterpret_cast<uint4*>(p.codes + act_tile_offset(grow, t8, ch + 1, nst8)) =
            make_uint4(w8[4], w8[5], w8[6], w8[7]);
      }
    }
    return;
  }
  if (quant_warp) {
    // ---------------------------------------------------------- NVFP4 quantizer
    const int grow = row0 + lane;                     // this lane's row (may be >= M: zero padding)
    const int col0 = warp * 32;                       // 2 groups of 16 columns of each stage
    uint16_t* scale_pair = reinterpret_cast<uint16_t*>(p.scales + sf_offset(grow, 2 * warp, K));
    for (int it = 0; it < nk; ++it) {
      const int s = it % kXStages;
      if (!dev::mbar_wait(&xfull[s], (uint32_t)(it / kXStages) & 1u, abort_flag, p.budget_ns)) {
        record_error(p.err, abort_flag, 0x102);
        break;
      }
      const uint8_t* st = smem + s * kXStageBytes;
      const int k0 = it * kBK;
      const int kvalid = min(kBK, K - k0);
      const bool active = col0 < kvalid;              // kvalid is a multiple of 64
      uint32_t packed[4] = {0u, 0u, 0u, 0u}, sb2 = 0u;
      if (active) {
        const uint8_t* xt = st + (col0 >> 6) * 4096;
        const int c0 = (col0 & 63) >> 3;               // first 16-byte chunk of the columns in a row
        const float4* inv4 = reinterpret_cast<const float4*>(st + kXBytes) + (col0 >> 2);
        // v = fp32(x * inv_lam), two elements per packed multiply (each lane
        // of the pair is an IEEE round-to-nearest product)
        float2 v[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 raw = *reinterpret_cast<const uint4*>(xt + sw128(lane, c0 + i));
          const float4 ia = inv4[2 * i], ib = inv4[2 * i + 1];
          const float2 iv[4] = {make_float2(ia.x, ia.y), make_float2(ia.z, ia.w), make_float2(ib.x, ib.y),
                                make_float2(ib.z, ib.w)};
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            v[i * 4 + e] = __fmul2_rn(make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u)),
                                      iv[e]);
        }
        sb2 = dev::nvfp4_quant32(v, p.c_x, p.g_x_exp, rcp, packed);
      }
      // the stage's inputs have been read
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&xempty[s]);
      if (active) {
        scale_pair[(size_t)(k0 >> 6) * 256] = (uint16_t)(sb2 & 0xFFFFu);   // next 64 columns: next 512-byte chunk
        // codes: 16 bytes = chunk `warp` of this row's 128-byte stage row, in the
        // tiled layout the GEMM loads with one bulk copy per stage (see
        // act_tile_offset): block (row / 128, stage), swizzled by row % 8
        *reinterpret_cast<uint4*>(p.codes + act_tile_offset(grow, it, warp, p.nst)) =
            make_uint4(packed[0], packed[1], packed[2], packed[3]);
      }
    }
    return;
  }

  // ------------------------------------------------------------ down projection
  const int mw = warp - kQuantWarps;                  // k-steps 2mw, 2mw+1 of each stage
  float acc[2][4][4] = {};                            // 2 row tiles x 4 column tiles
  bool ok = true;
  for (int it = 0; it < nk; ++it) {
    const int s = it % kXStages;
    const int ls = it % kLStages;
    const bool got = dev::mbar_wait(&xfull[s], (uint32_t)(it / kXStages) & 1u, abort_flag, p.budget_ns) &&
                     dev::mbar_wait(&lfull[ls], (uint32_t)(it / kLStages) & 1u, abort_flag, p.budget_ns);
    if (!__all_sync(0xffffffffu, got)) {            // warp-uniform exit (ldmatrix/mma are warp-collective)
      if (lane == 0) record_error(p.err, abort_flag, 0x103);
      ok = false;
      break;
    }
    const int kvalid = min(kBK, K - it * kBK);
    const uint32_t xbase = dev::smem_u32(smem + s * kXStageBytes);
    const uint32_t lbase = dev::smem_u32(lring + ls * kLBytes);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int kk = 2 * mw + h;
      if (kk * 16 < kvalid) {
        const int sub = kk >> 2;
        const int c0 = (kk & 3) * 2;                  // first 16-byte chunk of the k-step
        uint32_t b[2][4];
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          // n-tiles 2np, 2np+1: matrices (n 0-7, k lo), (n 0-7, k hi), (n 8-15, k lo), (n 8-15, k hi)
          const int brow = np * 16 + (lane & 7) + ((lane >> 4) << 3);
          ldsm_x4(lbase + sub * 4096 + sw128(brow, c0 + ((lane >> 3) & 1)), b[np]);
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          uint32_t a[4];
          ldsm_x4(xbase + sub * 4096 + sw128(mt * 16 + (lane & 15), c0 + (lane >> 4)), a);
#pragma unroll
          for (int np = 0; np < 2; ++np) {
            mma_16816(acc[mt][2 * np], a, b[np][0], b[np][1]);
            mma_16816(acc[mt][2 * np + 1], a, b[np][2], b[np][3]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) {
      dev::mbar_arrive(&xempty[s]);
      dev::mbar_arrive(&lempty[ls]);
    }
  }

  // Sum the eight partials through shared memory, in the L1d^T ring: only the
  // down-projection warps read it and the producer issues no copy beyond the
  // last k-tile, which every one of them has consumed once all of them reach
  // this barrier.  Every down-projection warp reaches both barriers.
  mma_warps_sync();
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int n = 0; n < 4; ++n)
      part[(mw * 32 + lane) * 8 + mt * 4 + n] = make_float4(acc[mt][n][0], acc[mt][n][1], acc[mt][n][2], acc[mt][n][3]);
  mma_warps_sync();
  if (ok && !*abort_flag) {
    // thread t sums one fragment (4 values) over the eight partials
    const int t = mw * 32 + lane;                      // 0..255
    const int fm = t >> 7, fl = (t >> 2) & 31, fn = t & 3;
    const float4* src = part + fl * 8 + fm * 4 + fn;
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int g = 0; g < kMmaWarps; ++g) {
      const float4 v = src[g * 32 * 8];
      sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
    }
    const int row = row0 + fm * 16 + (fl >> 2);
    const int col = fn * 8 + 2 * (fl & 3);
    if (row < p.M)
      *reinterpret_cast<__nv_bfloat162*>(p.xl + (size_t)row * p.xl_stride + col) = __floats2bfloat162_rn(sum.x, sum.y);
    if (row + 8 < p.M)
      *reinterpret_cast<__nv_bfloat162*>(p.xl + (size_t)(row + 8) * p.xl_stride + col) =
          __floats2bfloat162_rn(sum.z, sum.w);
  }
}

template <int F, bool Q, bool D>
cudaError_t launch_k1_t(const CUtensorMap& tm_x, const CUtensorMap& tm_l, const CUtensorMap& tm_c,
                        const K1Params& p, cudaStream_t stream) {
  auto kern = k1_kernel<F, Q, D>;
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  const int mpad = (p.M + 127) / 128 * 128;
  dim3 grid(mpad / kRows);
  // programmatic dependent launch: the prologue overlaps the preceding kernel's tail
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(K1Shape<F>::threads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tm_x, tm_l, tm_c, p);
}

}  // namespace

int k1_rows_per_cta() { return kRows; }

cudaError_t launch_k1(const CUtensorMap& tm_x, const CUtensorMap& tm_l, const CUtensorMap& tm_c,
                      const K1Params& p, int fmt, int mode, cudaStream_t stream) {
  if (mode == 2) return launch_k1_t<kFmtNvfp4, false, true>(tm_x, tm_l, tm_c, p, stream);   // no quantizer
  if (fmt == kFmtNvfp4) {
    if (mode == 0) return launch_k1_t<kFmtNvfp4, true, true>(tm_x, tm_l, tm_c, p, stream);
    if (mode == 1) return launch_k1_t<kFmtNvfp4, true, false>(tm_x, tm_l, tm_c, p, stream);
  } else if (fmt == kFmtInt4) {
    if (mode == 0) return launch_k1_t<kFmtInt4, true, true>(tm_x, tm_l, tm_c, p, stream);
    if (mode == 1) return launch_k1_t<kFmtInt4, true, false>(tm_x, tm_l, tm_c, p, stream);
  } else if (fmt == kFmtInt8) {
    if (mode == 0) return launch_k1_t<kFmtInt8, true, true>(tm_x, tm_l, tm_c, p, stream);
    if (mode == 1) return launch_k1_t<kFmtInt8, true, false>(tm_x, tm_l, tm_c, p, stream);
  }
  return cudaErrorInvalidValue;
}

namespace {

// One warp per row: the row's largest |fp32(x * inv_lam)| (the same IEEE
// products the quantizer forms), then s = fp32(a fp32(1/127)) and the
// correctly rounded reciprocal.
__global__ void __launch_bounds__(256) rowscale_kernel(const __nv_bfloat16* __restrict__ x,
                                                       const float* __restrict__ inv_lam, int M, int K, int mpad,
                                                       float* __restrict__ sx, float* __restrict__ inv_sx) {
  // X may be the preceding kernel's output
  dev::griddep_wait();
  dev::griddep_launch_dependents();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= mpad) return;
  float a = 0.f;
  if (row < M) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)row * K);
    const float4* il = reinterpret_cast<const float4*>(inv_lam);
#pragma unroll 4
    for (int c = lane; c < K / 8; c += 32) {        // 8 columns per 16-byte chunk (4 chunks in flight per lane)
      const uint4 raw = xr[c];
      const float4 i0 = il[2 * c], i1 = il[2 * c + 1];
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
      const float2 iv[4] = {make_float2(i0.x, i0.y), make_float2(i0.z, i0.w), make_float2(i1.x, i1.y),
                            make_float2(i1.z, i1.w)};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 v = __fmul2_rn(make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u)),
                                    iv[e]);
        a = dev::fmax3(a, fabsf(v.x), fabsf(v.y));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  }
  if (lane == 0) {
    const float s = __fmul_rn(a, 1.0f / 127.0f);
    sx[row] = s;
    inv_sx[row] = s == 0.f ? 0.f : __frcp_rn(s);
  }
}

}  // namespace

cudaError_t launch_rowscale(const __nv_bfloat16* x, const float* inv_lam, int M, int K, int mpad, float* sx,
                            float* inv_sx, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((mpad + 7) / 8);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, rowscale_kernel, x, inv_lam, M, K, mpad, sx, inv_sx);
}

}  // namespace svdq
