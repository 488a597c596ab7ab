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
// stages of 256 columns.  One producer warp loads each stage with TMA (X tile,
// the matching 256 x 32 slice of L1d^T and 256 floats of inv_lam) into a
// 4-deep shared-memory ring.  Sixteen consumer warps share each stage:
//   * quantization: warp w owns the 16-column group w of the stage and lane l
//     owns row l, so the inv_lam reads are broadcasts and the swizzled X reads
//     are conflict-free;
//   * down projection on the tensor cores (mma.sync BF16; the projection is 32
//     columns wide and the pass is bound by memory, not by the tensor pipe):
//     warp w computes the 16x8 tile (w & 1, (w >> 1) & 3) over half of the
//     stage's 256 columns (w >> 3); the two halves are summed at the end.
//
// Quantizer arithmetic per group of 16 (bit-exact with the CPU oracle): a =
// max|v|; t = fp32(a * c_x) with c_x = fp32(1/6) 2^-gx; s = E4M3_rn_satfinite(t);
// s == 0 -> all codes +0; inv = fp32(1 / (s * g_x)); code =
// E2M1_rn_satfinite(fp32(v * inv)).  The reciprocal is exact without a
// division: for s = (1 + m/8) 2^(e-7) (or m 2^-9 when e = 0) it equals
// fp32(1/(1 + m/8)) 2^(7-e-gx) (or fp32(1/m) 2^(9-gx)), a power-of-two scaling
// of one of 15 correctly rounded constants computed on the host.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100.cuh"

namespace svdq {

namespace {

constexpr int kRows = 32;
constexpr int kBK = 256;
constexpr int kStages = 4;
constexpr int kConsumerWarps = 16;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kXBytes = kRows * kBK * 2;     // 4 sub-tiles of 32 rows x 128 B
constexpr int kLBytes = 32 * kBK * 2;        // 4 sub-tiles of 32 rows x 128 B
constexpr int kIBytes = kBK * 4;
constexpr int kStageBytes = kXBytes + kLBytes + kIBytes;   // 33 KiB, 1 KiB multiple
constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 256 + (2 * 4 * 32 * 4 + 16) * 4;

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

template <bool kQuant, bool kDown>
__global__ void __launch_bounds__(kThreads, 1)
    k1_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l, K1Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kStages);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * kRows;
  const int K = p.K;
  const int nk = (K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      dev::mbar_init(&full[s], 1);
      dev::mbar_init(&empty[s], kConsumerWarps);
    }
    *abort_flag = 0;
    dev::fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      dev::tma_prefetch_desc(&tm_x);
      if (kDown) dev::tma_prefetch_desc(&tm_l);
      int issued = 0;
      for (int it = 0; it < nk; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        if (!dev::mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.budget_ns)) {
          record_error(p.err, abort_flag, 0x101);
          break;
        }
        uint8_t* st = smem + s * kStageBytes;
        const int k0 = it * kBK;
        const int kvalid = min(kBK, K - k0);
        const int nsub = kvalid >> 6;
        uint32_t bytes = (uint32_t)nsub * 4096u;
        if (kDown) bytes += (uint32_t)nsub * 4096u;
        if (kQuant) bytes += (uint32_t)kvalid * 4u;
        dev::mbar_arrive_expect_tx(&full[s], bytes);
        for (int j = 0; j < nsub; ++j) dev::tma_load_2d(st + j * 4096, &tm_x, &full[s], k0 + 64 * j, row0);
        if (kDown)
          for (int j = 0; j < nsub; ++j) dev::tma_load_2d(st + kXBytes + j * 4096, &tm_l, &full[s], k0 + 64 * j, 0);
        if (kQuant) dev::bulk_load(st + kXBytes + kLBytes, p.inv_lam + k0, (uint32_t)kvalid * 4u, &full[s]);
        issued = it + 1;
      }
      // Do not leave while copies into this CTA's shared memory are in flight.
      for (int it = max(0, issued - kStages); it < issued; ++it) {
        const int s = it % kStages;
        if (!dev::mbar_wait(&full[s], (uint32_t)(it / kStages) & 1u, abort_flag, p.budget_ns)) break;
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  float* red = reinterpret_cast<float*>(smem + kStages * kStageBytes + 256);   // k-half partial sums
  float* rcp = red + 2 * 4 * 32 * 4;                                           // reciprocal table
  if (threadIdx.x == 0) {
#pragma unroll
    for (int i = 0; i < 16; ++i) rcp[i] = p.rcp[i];     // constant indices: stays in parameter space
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32));
  const int grow = row0 + lane;         // quantizer: this lane's row (may be >= M: zero padding)
  const int qcol = warp * 16;           //            16-column group of the stage
  const int mt = warp & 1;              // down projection: 16-row tile
  const int nt = (warp >> 1) & 3;       //                  8-column tile of XL
  const int kh = warp >> 3;             //                  half of the stage's k-steps
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  bool ok = true;

  for (int it = 0; it < nk; ++it) {
    const int s = it % kStages;
    const uint32_t ph = (uint32_t)(it / kStages) & 1u;
    const bool got = dev::mbar_wait(&full[s], ph, abort_flag, p.budget_ns);
    if (!__all_sync(0xffffffffu, got)) {            // warp-uniform exit (ldmatrix/mma are warp-collective)
      if (lane == 0) record_error(p.err, abort_flag, 0x102);
      ok = false;
      break;
    }
    const uint8_t* st = smem + s * kStageBytes;
    const int k0 = it * kBK;
    const int kvalid = min(kBK, K - k0);

    if (kQuant && qcol < kvalid) {
      const uint8_t* xt = st + (qcol >> 6) * 4096;
      const int c0 = (qcol & 63) >> 3;                  // first 16-byte chunk of the group in its row
      const float4* inv4 = reinterpret_cast<const float4*>(st + kXBytes + kLBytes) + (qcol >> 2);
      float v[16];
      float a = 0.f;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint4 raw = *reinterpret_cast<const uint4*>(xt + sw128(lane, c0 + i));
        const float4 ia = inv4[2 * i], ib = inv4[2 * i + 1];
        const float iv[8] = {ia.x, ia.y, ia.z, ia.w, ib.x, ib.y, ib.z, ib.w};
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[i * 8 + 2 * e] = __fmul_rn(__uint_as_float(w[e] << 16), iv[2 * e]);
          v[i * 8 + 2 * e + 1] = __fmul_rn(__uint_as_float(w[e] & 0xFFFF0000u), iv[2 * e + 1]);
        }
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(v[i]));
      const uint32_t sb = dev::cvt_e4m3x2(__fmul_rn(a, p.c_x), 0.0f) & 0xFFu;
      uint32_t packed0 = 0u, packed1 = 0u;
      if (sb != 0u) {
        const uint32_t e = sb >> 3, m = sb & 7u;
        const int p2 = (e ? 7 - (int)e : 9) - p.g_x_exp;
        const float invs = rcp[(e ? 0 : 8) + m] * __int_as_float((p2 + 127) << 23);
        float q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(v[i], invs);
        packed0 = dev::cvt_e2m1x8(q);
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(v[8 + i], invs);
        packed1 = dev::cvt_e2m1x8(q);
      }
      if (grow < p.M)
        *reinterpret_cast<uint2*>(p.codes + (size_t)grow * (size_t)(K >> 1) + ((k0 + qcol) >> 1)) =
            make_uint2(packed0, packed1);
      p.scales[sf_offset(grow, (k0 + qcol) >> 4, K)] = (uint8_t)sb;
    }

    if (kDown) {
      const uint32_t xbase = dev::smem_u32(st);
      const uint32_t lbase = dev::smem_u32(st + kXBytes);
      const int nsteps = kvalid >> 4;
      const int arow = mt * 16 + (lane & 15);
      const int brow = nt * 8 + (lane & 7);
#pragma unroll 2
      for (int kk = kh * 8; kk < min(nsteps, kh * 8 + 8); kk += 2) {
        const int sub = kk >> 2;
        const int cpair = (kk & 3) * 2;                 // 16B chunk of this k-step pair
        uint32_t b[4];
        ldsm_x4(lbase + sub * 4096 + sw128(brow, cpair + (lane >> 3)), b);
        uint32_t a[4];
        ldsm_x4(xbase + sub * 4096 + sw128(arow, cpair + (lane >> 4)), a);
        mma_16816(acc, a, b[0], b[1]);
        ldsm_x4(xbase + sub * 4096 + sw128(arow, cpair + 2 + (lane >> 4)), a);
        mma_16816(acc, a, b[2], b[3]);
      }
    }

    __syncwarp();
    if (lane == 0) dev::mbar_arrive(&empty[s]);
  }

  if (kDown) {
    // sum the two k-halves; every consumer warp reaches this barrier (no early exit)
    float* slot = red + ((mt * 4 + nt) * 32 + lane) * 4;
    if (kh == 1) {
#pragma unroll
      for (int i = 0; i < 4; ++i) slot[i] = acc[i];
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32));
    if (kh == 0 && ok && !*abort_flag) {
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] += slot[i];
      const int r_a = row0 + mt * 16 + (lane >> 2);
      const int col = nt * 8 + 2 * (lane & 3);
      if (r_a < p.M)
        *reinterpret_cast<__nv_bfloat162*>(p.xl + (size_t)r_a * 32 + col) = __floats2bfloat162_rn(acc[0], acc[1]);
      if (r_a + 8 < p.M)
        *reinterpret_cast<__nv_bfloat162*>(p.xl + (size_t)(r_a + 8) * 32 + col) =
            __floats2bfloat162_rn(acc[2], acc[3]);
    }
  }
}

template <bool Q, bool D>
cudaError_t launch_k1_t(const CUtensorMap& tm_x, const CUtensorMap& tm_l, const K1Params& p, cudaStream_t stream) {
  auto kern = k1_kernel<Q, D>;
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
  kern<<<grid, kThreads, kSmemBytes, stream>>>(tm_x, tm_l, p);
  return cudaGetLastError();
}

}  // namespace

int k1_rows_per_cta() { return kRows; }

cudaError_t launch_k1(const CUtensorMap& tm_x, const CUtensorMap& tm_l, const K1Params& p, int mode,
                      cudaStream_t stream) {
  switch (mode) {
    case 0: return launch_k1_t<true, true>(tm_x, tm_l, p, stream);
    case 1: return launch_k1_t<true, false>(tm_x, tm_l, p, stream);
    case 2: return launch_k1_t<false, true>(tm_x, tm_l, p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace svdq
