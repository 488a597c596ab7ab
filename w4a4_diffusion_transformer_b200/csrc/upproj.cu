// Unfused low-rank up projection (measurement variant only).  With a LoRA
// adapter the branch is 64 wide ([XL | X A] times [L2b ; bf16(s B)]), one pass.
//
// The SOTA-314 practice page ("Do this") reports that running the rank-32
// branch as separate 16-bit kernels adds 57% latency, from "the extra 16-bit
// read in Down Projection and the extra 16-bit write in Up Projection" (NOTE-257
// note page, "Key results").  This kernel is that separate up projection:
// Y <- bf16([gelu](Y + XL L2b)), reading and rewriting the BF16 output of the
// bare W4A4 GEMM.  Its floor is that extra traffic: Y read once and written
// once (2 x 28.3 MB at the attention-output shape).
//
// A CTA owns a 64 x 128 tile of Y.  One thread loads the tile with two TMA
// boxes (64 rows x 64 columns, 128-byte swizzle) while the four warps fetch
// their XL rows (A fragments) and L2b^T rows (B fragments); each warp then
// computes its 16 x 128 branch values with mma.sync (K = 32: two k-steps per
// 8-column tile), adds them to the Y values in shared memory -- in the MMA's
// fragment order, which the swizzle makes free of bank conflicts -- applies
// GELU when asked, and writes the BF16 results back in place; one thread
// stores the tile with two TMA stores.  Small tiles and 16 KB of shared memory
// keep about a dozen CTAs on each SM, so many tiles' loads are in flight.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100.cuh"

namespace svdq {

namespace {

constexpr int kTileM = 64;     // 4 warps x 16 rows
constexpr int kTileN = 128;    // two 64-column TMA boxes
constexpr int kBoxBytes = 64 * 128;

__device__ __forceinline__ uint32_t ld32(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }

// kKS k-steps of 16: the branch width is 32 (2) or, with a LoRA adapter
// concatenated into it, 64 (4); l2t rows are then kKS * 16 wide.
template <int kKS>
__global__ void __launch_bounds__(128) upproj_kernel(const __grid_constant__ CUtensorMap tm_y, UpParams p) {
  __shared__ __align__(1024) uint8_t tile[2 * kBoxBytes];
  __shared__ uint64_t full;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int m0 = blockIdx.y * kTileM;
  const int n0 = blockIdx.x * kTileN;
  const int nbox = (n0 + 64 < p.N) ? 2 : 1;                 // the second box lies inside Y
  if (threadIdx.x == 0) {
    abort_flag = 0;
    dev::mbar_init(&full, 1);
    dev::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    dev::mbar_arrive_expect_tx(&full, (uint32_t)(nbox * kBoxBytes));
    for (int b = 0; b < nbox; ++b) dev::tma_load_2d(tile + b * kBoxBytes, &tm_y, &full, n0 + 64 * b, m0);
  }
  // A fragments of this warp's 16 XL rows (kKS k-steps of 16)
  const int ra = m0 + warp * 16 + g, rb = ra + 8;
  constexpr int kW = kKS * 16;                                // branch width
  uint32_t a[kKS][4];
#pragma unroll
  for (int ks = 0; ks < kKS; ++ks) {
    const int k = ks * 16 + 2 * t4;
    a[ks][0] = ra < p.M ? ld32(p.xl + (size_t)ra * p.xl_stride + k) : 0u;
    a[ks][1] = rb < p.M ? ld32(p.xl + (size_t)rb * p.xl_stride + k) : 0u;
    a[ks][2] = ra < p.M ? ld32(p.xl + (size_t)ra * p.xl_stride + k + 8) : 0u;
    a[ks][3] = rb < p.M ? ld32(p.xl + (size_t)rb * p.xl_stride + k + 8) : 0u;
  }
  const bool got = dev::mbar_wait(&full, 0, &abort_flag, p.budget_ns);
  if (!__syncthreads_and(got)) {
    if (threadIdx.x == 0) atomicCAS(p.err, 0, 0x401);
    return;                                                  // the copies were not seen to land: no store
  }
#pragma unroll 4
  for (int j = 0; j < kTileN / 8; ++j) {
    const int nb = n0 + j * 8;
    if (j >= 8 * nbox) break;
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    const bool bv = nb + g < p.N;
#pragma unroll
    for (int ks = 0; ks < kKS; ++ks) {
      const uint32_t b0 = bv ? ld32(p.l2t + (size_t)(nb + g) * kW + ks * 16 + 2 * t4) : 0u;
      const uint32_t b1 = bv ? ld32(p.l2t + (size_t)(nb + g) * kW + ks * 16 + 2 * t4 + 8) : 0u;
      asm volatile(
          "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
          "{%0, %1, %2, %3};"
          : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
          : "r"(a[ks][0]), "r"(a[ks][1]), "r"(a[ks][2]), "r"(a[ks][3]), "r"(b0), "r"(b1));
    }
    // element (row r, column 8 j + 2 t4 .. +1) of the tile: box j / 8, 16-byte
    // chunk j % 8 of the row, swizzled by r % 8
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = warp * 16 + g + 8 * h;
      uint8_t* e = tile + (j >> 3) * kBoxBytes + r * 128 + ((((j & 7) ^ (r & 7))) << 4) + 4 * t4;
      const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(e));
      float y0 = y.x + c[2 * h], y1 = y.y + c[2 * h + 1];
      if (p.gelu) {
        y0 = dev::gelu_tanh(y0);
        y1 = dev::gelu_tanh(y1);
      }
      *reinterpret_cast<__nv_bfloat162*>(e) = __floats2bfloat162_rn(y0, y1);
    }
  }
  dev::fence_async_shared();                                 // the TMA engine reads what the threads wrote
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int b = 0; b < nbox; ++b) dev::tma_store_2d(&tm_y, tile + b * kBoxBytes, n0 + 64 * b, m0);
    dev::bulk_commit_group();
    dev::bulk_wait_group_read<0>();                          // the tile stays valid until the stores read it
  }
}

}  // namespace

cudaError_t launch_upproj(const CUtensorMap& tm_y, const UpParams& p, cudaStream_t stream) {
  dim3 grid((p.N + kTileN - 1) / kTileN, (p.M + kTileM - 1) / kTileM);
  if (p.width == 64)
    upproj_kernel<4><<<grid, 128, 0, stream>>>(tm_y, p);
  else if (p.width == 32)
    upproj_kernel<2><<<grid, 128, 0, stream>>>(tm_y, p);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

int upproj_box_rows() { return kTileM; }

}  // namespace svdq
