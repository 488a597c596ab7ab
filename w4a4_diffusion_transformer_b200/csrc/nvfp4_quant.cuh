// NVFP4 activation quantizer of 32 consecutive values of one row (two groups of
// 16), shared by the first kernel and by the GEMM epilogue that hands the next
// layer its input already quantized.  One definition keeps both bit-identical.
//
// SOTA-314 practice page, "Do this": NVFP4 with groups of 16 and FP8 scales.
// Per group: a = max|v|; t = fp32(a * c_x) with c_x = fp32(1/6) 2^-g_x;
// s = E4M3_rn_satfinite(t); s == 0 -> all codes +0; inv = fp32(1 / (s * g_x));
// code = E2M1_rn_satfinite(fp32(v * inv)).  The reciprocal needs no division:
// for s = (1 + m/8) 2^(e-7) (or m 2^-9 when e = 0) it equals
// fp32(1/(1 + m/8)) 2^(7-e-g_x) (or fp32(1/m) 2^(9-g_x)), a power-of-two
// scaling of one of the 15 correctly rounded constants rcp[0..7] (normal
// mantissas) and rcp[9..15] (subnormal m) computed on the host.
#pragma once

#include <cstdint>

#include "sm100.cuh"

namespace svdq {
namespace dev {

// v: the 32 values x_hat = fp32(x * inv_lam) as 16 pairs (pair i holds
// columns 2i, 2i+1).  Returns the two E4M3 scale bytes (group 0 in the low
// byte) and the 32 E2M1 codes in packed[0..3] (group 0 in packed[0..1]; two
// codes per byte, the even column in the low nibble).
__device__ __forceinline__ uint32_t nvfp4_quant32(const float2 (&v)[16], float c_x, int g_x_exp,
                                                  const float* rcp, uint32_t (&packed)[4]) {
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    a0 = fmax3(a0, fabsf(v[i].x), fabsf(v[i].y));
    a1 = fmax3(a1, fabsf(v[8 + i].x), fabsf(v[8 + i].y));
  }
  const uint32_t sb2 = cvt_e4m3x2(__fmul_rn(a0, c_x), __fmul_rn(a1, c_x));
#pragma unroll
  for (int i = 0; i < 4; ++i) packed[i] = 0u;
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    const uint32_t sb = (sb2 >> (8 * g)) & 0xFFu;
    if (sb != 0u) {
      const uint32_t e = sb >> 3, m = sb & 7u;
      const int p2 = (e ? 7 - (int)e : 9) - g_x_exp;
      const float invs = rcp[(e ? 0 : 8) + m] * __int_as_float((p2 + 127) << 23);
      const float2 inv2 = make_float2(invs, invs);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int b = g * 8 + h * 4;
        packed[2 * g + h] = cvt_e2m1x8(__fmul2_rn(v[b], inv2), __fmul2_rn(v[b + 1], inv2),
                                       __fmul2_rn(v[b + 2], inv2), __fmul2_rn(v[b + 3], inv2));
      }
    }
  }
  return sb2;
}

}  // namespace dev
}  // namespace svdq
