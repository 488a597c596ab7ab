// Internal declarations shared by the host preparation code and the CUDA
// launch code of the SVDQuant W4A4 library.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>

#include "svdq.h"   // include/ is on the include path

#ifdef __CUDACC__
#define SVDQ_HD __host__ __device__
#else
#define SVDQ_HD
#endif

namespace svdq {

// Host results of the offline preparation (logical layouts).
struct HostPrep {
  int K = 0, N = 0, rank = 0, format = 0;
  float alpha = 0.5f;
  std::vector<float> lam, inv_lam;          // [K]
  std::vector<double> L1;                   // [K][r]
  std::vector<double> L2;                   // [r][N]
  std::vector<double> sigma;                // [r]
  std::vector<uint16_t> L1d;                // [K][r] BF16 bits
  std::vector<uint16_t> L2b;                // [r][N] BF16 bits
  std::vector<float> R;                     // [K][N]
  int g_x_exp = 0, g_w_exp = 0;
  float x_amax = 0.0f;                      // max |fp32(Xc / lam)| over the calibration batch
  float w_amax = 0.0f;                      // largest group maximum the residual quantizer saw
  std::vector<double> gptq_U;               // [K][K] GPTQ factor (kept only on request)
  int lora_r = 0;                           // LoRA adapter rank (0: none)
  std::vector<uint16_t> lora_A;             // [K][lora_r] BF16 bits, as given
  std::vector<uint16_t> lora_B;             // [lora_r][N] BF16 bits of bf16(scale * B)
  std::vector<uint8_t> w_codes;             // [N][K/2] (4-bit formats), [N][K] int8 (W8A8)
  std::vector<uint8_t> w_scales_e4m3;       // [N][K/16]   (NVFP4)
  std::vector<uint16_t> w_scales_bf16;      // [N][K/64]   (INT4 / W4A16)
  std::vector<float> w_scales_f32;          // [N]         (W8A8: one scale per output channel)
  std::vector<float> bias;                  // [N]
  int svd_iterations = 0;
  double svd_tail_energy = 0.0;
};

// Runs the offline pipeline on the host.  Returns SVDQ_OK or an error status.
svdq_status host_prepare(const svdq_config& cfg, int K, int N, const uint16_t* W,
                         const uint16_t* bias, const uint16_t* calib, int M_calib,
                         HostPrep& out);

// Number-format helpers (host).
float bf16_to_float(uint16_t b);
uint16_t bf16_from_double(double x);       // single round-to-nearest-even
uint8_t e4m3_from_nonneg(float t);         // RNE, saturating at 448
float e4m3_to_float(uint8_t b);
uint8_t e2m1_code(float q);                // RNE (ties to even code), sat 6, sign kept
int pow2_ceil_exponent(double x);          // smallest e with 2^e >= x; 0 for x <= 0

// Offset in bytes of scale (row r, group-of-16 g) inside the tensor-core
// scale-factor layout of a [rows][K] operand (see svdq_act_scale_bytes).
SVDQ_HD inline size_t sf_offset(int r, int g, int K) {
  const size_t kb = (size_t)(g >> 2);                 // 64-element K block
  const size_t chunk = (size_t)(r >> 7) * (size_t)(K >> 6) + kb;
  return chunk * 512 + (size_t)(r & 31) * 16 + (size_t)((r >> 5) & 3) * 4 + (size_t)(g & 3);
}

// Tiled layout of NVFP4 activation codes (the GEMM's A operand): for row
// block b = r / 128 and K stage t (256 codes = 128 bytes of each row), a
// contiguous 16 KiB block at (b * nst + t) * 16384 holding the block's 128 rows
// as the tensor core reads them (128-byte swizzle): 16-byte chunk c of row
// r % 128 at (r % 128) * 128 + ((c ^ (r % 8)) * 16).  nst = ceil(K / 256).
SVDQ_HD inline size_t act_tile_offset(int r, int t, int c, int nst) {
  return ((size_t)(r >> 7) * (size_t)nst + (size_t)t) * 16384u + (size_t)(r & 127) * 128u +
         (size_t)(((c ^ (r & 7)) & 7) << 4);
}

// The same layout for the weight codes (the GEMM's B operand) in blocks of 256
// rows: block (r / 256, t) at (b * nst + t) * 32768.
SVDQ_HD inline size_t wgt_tile_offset(int r, int t, int c, int nst) {
  return ((size_t)(r >> 8) * (size_t)nst + (size_t)t) * 32768u + (size_t)(r & 255) * 128u +
         (size_t)(((c ^ (r & 7)) & 7) << 4);
}

}  // namespace svdq
