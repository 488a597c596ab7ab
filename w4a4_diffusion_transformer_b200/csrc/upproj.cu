// Unfused low-rank up projection (measurement variant only).
//
// The SOTA-314 practice page ("Do this") reports that running the rank-32
// branch as separate 16-bit kernels adds 57% latency, from "the extra 16-bit
// read in Down Projection and the extra 16-bit write in Up Projection" (NOTE-257
// note page, "Key results").  This kernel is that separate up projection:
// Y <- bf16([gelu](Y + XL L2b)), reading and rewriting the BF16 output of the
// bare W4A4 GEMM.  Tensor cores via mma.sync (K = 32 is two k-steps).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"

namespace svdq {

namespace {

constexpr int kTileM = 64;     // 4 warps x 16 rows
constexpr int kTileN = 64;     // 8 n-tiles of 8

__device__ __forceinline__ float gelu_tanh(float y) {
  const float k0 = 0.7978845608028654f;
  return 0.5f * y * (1.0f + tanhf(k0 * (y + 0.044715f * y * y * y)));
}

__device__ __forceinline__ uint32_t ld32(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }

__global__ void __launch_bounds__(128) upproj_kernel(UpParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int m0 = blockIdx.y * kTileM + warp * 16;
  const int n0 = blockIdx.x * kTileN;
  const int ra = m0 + g, rb = m0 + g + 8;
  // A fragments of XL rows (16 x 32): two k-steps
  uint32_t a[2][4];
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    const int k = ks * 16 + 2 * t4;
    a[ks][0] = ra < p.M ? ld32(p.xl + (size_t)ra * 32 + k) : 0u;
    a[ks][1] = rb < p.M ? ld32(p.xl + (size_t)rb * 32 + k) : 0u;
    a[ks][2] = ra < p.M ? ld32(p.xl + (size_t)ra * 32 + k + 8) : 0u;
    a[ks][3] = rb < p.M ? ld32(p.xl + (size_t)rb * 32 + k + 8) : 0u;
  }
#pragma unroll
  for (int j = 0; j < kTileN / 8; ++j) {
    const int nb = n0 + j * 8;
    if (nb >= p.N) break;
    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const uint32_t b0 = ld32(p.l2t + (size_t)(nb + g) * 32 + ks * 16 + 2 * t4);
      const uint32_t b1 = ld32(p.l2t + (size_t)(nb + g) * 32 + ks * 16 + 2 * t4 + 8);
      asm volatile(
          "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
          "{%0, %1, %2, %3};"
          : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
          : "r"(a[ks][0]), "r"(a[ks][1]), "r"(a[ks][2]), "r"(a[ks][3]), "r"(b0), "r"(b1));
    }
    const int col = nb + 2 * t4;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = h ? rb : ra;
      if (row >= p.M) continue;
      __nv_bfloat162* yp = reinterpret_cast<__nv_bfloat162*>(p.y + (size_t)row * p.N + col);
      const float2 y = __bfloat1622float2(*yp);
      float y0 = y.x + c[2 * h], y1 = y.y + c[2 * h + 1];
      if (p.gelu) {
        y0 = gelu_tanh(y0);
        y1 = gelu_tanh(y1);
      }
      *yp = __floats2bfloat162_rn(y0, y1);
    }
  }
}

}  // namespace

cudaError_t launch_upproj(const UpParams& p, cudaStream_t stream) {
  dim3 grid((p.N + kTileN - 1) / kTileN, (p.M + kTileM - 1) / kTileM);
  upproj_kernel<<<grid, 128, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace svdq
