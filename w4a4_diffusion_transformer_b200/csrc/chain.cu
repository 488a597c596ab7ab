// fc1 -> fc2 chain: the fixed-order sum of fc2's down-projection partials.
//
// In chain mode the NVFP4 GEMM of fc1 produces fc2's input already quantized
// (the NOTE-257 note page, "Key results", pairs the down projection with the
// quantizer because they read the same input; here that input never reaches
// HBM) and, per CTA, the partial sums of y L1d2 over the N-tile range the CTA
// owns.  This kernel adds the 2 S partials of each row in slot order and rounds
// once to BF16: XL2 = bf16(sum_i partials[m][i][:]).  The order is fixed, so the
// result does not depend on which CTA finished first.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100.cuh"

namespace svdq {

namespace {

__global__ void __launch_bounds__(256) xl_reduce_kernel(const float* __restrict__ partials, int nparts, int M,
                                                        __nv_bfloat16* __restrict__ xl) {
  // the GEMM that reads XL2 may launch now; it waits for this grid to complete
  dev::griddep_launch_dependents();
  // the partials come from the preceding grid
  dev::griddep_wait();
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;   // (row, column pair)
  if (idx >= M * 16) return;
  const int m = idx >> 4, j = (idx & 15) * 2;
  const float* src = partials + (size_t)m * nparts * 32 + j;
  float2 acc = *reinterpret_cast<const float2*>(src);
  for (int i = 1; i < nparts; ++i) {
    const float2 v = *reinterpret_cast<const float2*>(src + (size_t)i * 32);
    acc.x += v.x;
    acc.y += v.y;
  }
  *reinterpret_cast<__nv_bfloat162*>(xl + (size_t)m * 32 + j) = __floats2bfloat162_rn(acc.x, acc.y);
}

}  // namespace

cudaError_t launch_xl_reduce(const float* partials, int nparts, int M, __nv_bfloat16* xl, cudaStream_t stream) {
  const int threads = 256, total = M * 16;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((total + threads - 1) / threads);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, xl_reduce_kernel, partials, nparts, M, xl);
}

}  // namespace svdq
