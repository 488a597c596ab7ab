// Kernel parameter blocks and launchers (internal to the library).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "svdq_internal.h"

namespace svdq {

// Activation/weight formats of the W4A4 kernels.
constexpr int kFmtNvfp4 = 0;
constexpr int kFmtInt4 = 1;
constexpr int kFmtInt8 = 2;    // W8A8: one scale per token

struct K1Params {
  int M, K;
  int mpad;                     // M rounded up to 128 (rows of the INT4 scale array)
  int nst;                      // K stages of 256 codes (rows of 128 bytes) in the NVFP4 tiled code layout
  float c_x;                    // fp32(1/6) * 2^-g_x_exp
  int g_x_exp;                  // activation tensor scale g_x = 2^g_x_exp
  float rcp[16];                // fp32(1/(1 + m/8)) for m = 0..7, then fp32(1/m) (index 8 + m)
  const float* inv_lam;         // [K]
  const float* inv_sx;          // INT8: per-token 1/s_x [mpad] (zero for padding rows)
  uint8_t* codes;               // NVFP4: tiled layout (act_tile_offset); INT4: [M][K/2];
                                // INT8: tiled in 128-column stages (act_tile_offset, nst = ceil(K/128))
  uint8_t* scales;              // NVFP4: tensor-core scale layout, mpad rows; INT4: BF16 [K/64][mpad]
  __nv_bfloat16* xl;            // [M][32] with row stride xl_stride elements
  int xl_stride;                // 32, or 64 when a LoRA adapter's XL_lora shares the rows
  int* err;                     // device error word
  unsigned long long budget_ns; // bound on each wait
};

// fc1 -> fc2 chain: the NVFP4 GEMM of fc1 hands fc2 its input already
// quantized (fc1's N is fc2's K).  Per output tile the epilogue rounds
// y = [gelu](alpha acc + b) to BF16 -- the value fc2 would read -- quantizes
// x_hat = fp32(y * inv_lam2) into fc2's activation codes and scales (the first
// kernel's layouts and arithmetic), and accumulates y L1d2 (fc2's down
// projection) over the tiles of one 128-row block that the CTA owns; the
// per-CTA partial sums are added in a fixed order by launch_xl_reduce.
struct K2Chain {
  uint8_t* codes;               // fc2 activation codes, tiled layout (act_tile_offset over K2), mpad rows
  uint8_t* scales;              // fc2 activation scales, tensor-core layout over K2, mpad rows
  const float* inv_lam;         // fc2's 1/lam, [K2]
  const __nv_bfloat16* l1t;     // fc2's L1d^T, [32][K2]; null when fc2 has no branch
  float* partials;              // [mpad][2 S][32] partial sums of y L1d2 (with l1t)
  int K2;                       // = N of this GEMM
  int nst;                      // ceil(K2 / 256)
  int S;                        // CTAs that share one 128-row block (N-tile ranges)
  int g_x_exp;                  // fc2's activation tensor scale 2^g_x_exp
  float c_x;                    // fp32(1/6) * 2^-g_x_exp
  float rcp[16];                // the quantizer's reciprocal constants (K1Params::rcp)
};

struct K2Params {
  int M, N, K;
  int mpad;                     // rows of the activation scale layout (M rounded up to 128)
  const uint8_t* acodes;        // activation codes, tiled layout (act_tile_offset), mpad rows
  float alpha;                  // g_x * g_w (power of two)
  const uint8_t* sfa;           // activation scales, tensor-core layout
  const uint8_t* wmerged;       // single-CTA GEMM: weight codes and scales merged (k2_pack_weights)
  const uint8_t* wpair;         // CTA-pair GEMM: weight codes and scales merged (k2_pair_pack_weights)
  const float* bias;            // [N]
  __nv_bfloat16* y;             // [M][N]
  int* err;
  unsigned long long budget_ns;
  int branch;                   // 1: add XL (L2b / alpha) into the accumulator
  int gelu;                     // 1: tanh-GELU epilogue
  int lora;                     // 1: one more ring stage per tile adds XL_lora (s B / alpha) (tm_xla, tm_l2a)
  K2Chain chain;                // launch_k2_chain only
};

struct K2Int4Params {
  int M, N, K;
  int mpad, npad;               // rows of the activation / weight scale arrays (multiples of 128 / 256)
  float alpha;                  // 2^(ex + ew): undoes the FP16 range exponents
  float xscale;                 // 2^-ex, applied to the BF16 activation scales
  const uint16_t* sa;           // activation scales, BF16 [K/64][mpad]
  const uint16_t* sb;           // weight scales times 2^-ew, FP16 [K/64][npad]
  const float* bias;            // [N]
  __nv_bfloat16* y;             // [M][N]
  int* err;
  unsigned long long budget_ns;
  int branch;                   // 1: add XL (L2b / alpha) into the accumulator
  int gelu;                     // 1: tanh-GELU epilogue
  int lora;                     // 1: add XL_lora (s B / alpha) too (tm_xla, tm_l2a), same accumulator
};

struct K2Int8Params {
  int M, N, K;
  const uint8_t* acodes;        // int8 activation codes, tiled in 128-column stages (act_tile_offset), mpad rows
  const uint8_t* wq;            // int8 weight codes, tiled in (256-row, 128-column) blocks (wgt_tile_offset)
  const float* sx;              // per-token scales [mpad]
  const float* sw;              // per-output-channel scales [N]
  const float* bias;            // [N]
  __nv_bfloat16* y;             // [M][N]
  int* err;
  unsigned long long budget_ns;
  int branch;                   // 1: add XL L2b (rank 16) from its own accumulator
  int gelu;
};

struct UpParams {
  int M, N;
  int width;                    // branch width: 32, or 64 with a LoRA adapter
  const __nv_bfloat16* xl;      // [M][width], row stride xl_stride elements
  int xl_stride;
  const __nv_bfloat16* l2t;     // [N][width] = L2b^T (with bf16(s B)^T beside it)
  int gelu;
  int* err;                     // device error word (a wait that ran out)
  unsigned long long budget_ns;
};

struct W4A16Params {
  int M, N, K;
  const __nv_bfloat16* x;       // [M][K]
  const uint8_t* wt;            // codes and scales packed by w4a16_pack
  const float* bias;            // [N]
  __nv_bfloat16* y;             // [M][N]
  int* err;                     // set to 1 if a bounded wait gave up
  unsigned long long budget_ns;
};

// Device layout of W4A16 weights: from codes [N][K/2] (two's complement
// nibbles, even k low) and BF16 scales [N][K/64] to the tile-packed stream the
// GEMV reads (w4a16_packed_bytes(N, K) bytes).
size_t w4a16_packed_bytes(int N, int K);
bool w4a16_supported(int K);   // shared-memory bound on K
void w4a16_pack(const uint8_t* codes, const uint16_t* scales, int N, int K, uint8_t* out);
cudaError_t launch_w4a16(const W4A16Params& p, cudaStream_t stream);

// fmt = kFmtNvfp4 or kFmtInt4; mode 0 = fused, 1 = quantize only, 2 = down projection only
cudaError_t launch_k1(const CUtensorMap& tm_x, const CUtensorMap& tm_l, const CUtensorMap& tm_c,
                      const K1Params& p, int fmt, int mode, cudaStream_t stream);
int k1_rows_per_cta();
// Per-token INT8 scales of x_hat = fp32(x * inv_lam): a = max_k |x_hat|,
// s = fp32(a fp32(1/127)), inv = fp32(1/s) (0 when s == 0); sx and inv_sx get
// mpad entries (padding rows zero).
cudaError_t launch_rowscale(const __nv_bfloat16* x, const float* inv_lam, int M, int K, int mpad, float* sx,
                            float* inv_sx, cudaStream_t stream);

// NVFP4 GEMM: operands from p.acodes / p.sfa (the first kernel's layouts) and
// p.wmerged; tm_xl / tm_l2 the branch tiles, tm_y the output; with p.lora,
// tm_xla / tm_l2a the LoRA tiles (XL_lora [M][32], (s B / alpha)^T [N][32]; the
// same boxes and swizzle as tm_xl / tm_l2).
cudaError_t launch_k2(const CUtensorMap& tm_xl, const CUtensorMap& tm_l2, const CUtensorMap& tm_y,
                      const CUtensorMap& tm_xla, const CUtensorMap& tm_l2a, const K2Params& p, int num_sms,
                      cudaStream_t stream);
int k2_block_n();
// The same GEMM in chain mode (p.chain; Y is not written): CTA c owns 128-row
// block c / S and the c % S-th of S contiguous ranges of N tiles.
// k2_chain_splits gives S for an M x N GEMM on num_sms SMs.
cudaError_t launch_k2_chain(const CUtensorMap& tm_xl, const CUtensorMap& tm_l2, const K2Params& p, int num_sms,
                            cudaStream_t stream);
int k2_chain_splits(int M, int N, int num_sms);
// xl[m][j] = bf16(sum_{i < nparts} partials[m][i][j]) in order i = 0, 1, ...
// (m < M, j < 32); launched as a programmatic dependent of the chain GEMM.
cudaError_t launch_xl_reduce(const float* partials, int nparts, int M, __nv_bfloat16* xl, cudaStream_t stream);
// The single-CTA GEMM's weight layout: per (256-row block, 256-K stage) the 32 KB
// of tiled codes (wgt_tile_offset) followed by the 4 KB of scale factors of the
// block's 256 rows (tensor-core layout, zero past K): one contiguous copy per stage.
size_t k2_weight_bytes(int N, int K);
void k2_pack_weights(const uint8_t* tiled_codes, const uint8_t* sf, int N, int K, uint8_t* out);
// The same GEMM on CTA pairs (256 x 256 tiles, tcgen05 cta_group::2, clusters of
// two): tm_l2 has 128-row boxes (each CTA holds half of B).
cudaError_t launch_k2_pair(const CUtensorMap& tm_xl, const CUtensorMap& tm_l2, const CUtensorMap& tm_y,
                           const K2Params& p, int num_sms, cudaStream_t stream);
int k2_pair_rows_b();
// The pair GEMM's weight layout: per (256-row block, 256-K stage) and CTA half
// h, the half's 16 KB of tiled codes followed by the 4 KB of scale factors of
// all 256 rows (tensor-core layout, zero past K), so that each CTA moves its
// weights of a stage in one contiguous copy.  Built from the single-CTA tiled
// codes (wgt_tile_offset) and the tensor-core scale layout (rows padded to 256).
size_t k2_pair_weight_bytes(int N, int K);
void k2_pair_pack_weights(const uint8_t* tiled_codes, const uint8_t* sf, int N, int K, uint8_t* out);

// INT4 GEMM: A = activation codes [M][K/2] (box 32 B x 128 rows), B = weight
// codes [N][K/2] (box 32 B x 256 rows), both unswizzled.
cudaError_t launch_k2_int4(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const CUtensorMap& tm_xl,
                           const CUtensorMap& tm_l2, const CUtensorMap& tm_y, const CUtensorMap& tm_xla,
                           const CUtensorMap& tm_l2a, const K2Int4Params& p, int num_sms, cudaStream_t stream);
// The INT4 GEMM on CTA pairs (256 x 256 tiles, clusters of two): tm_b and tm_l2
// with boxes of k2_int4_pair_rows_b() rows.
int k2_int4_pair_rows_b();
cudaError_t launch_k2_int4_pair(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const CUtensorMap& tm_xl,
                                const CUtensorMap& tm_l2, const CUtensorMap& tm_y, const K2Int4Params& p,
                                int num_sms, cudaStream_t stream);

// W8A8 GEMM (tcgen05 kind::i8): tm_xl / tm_l2 the branch tiles (as for the
// NVFP4 GEMM, L2b unscaled), tm_y the output.
cudaError_t launch_k2_int8(const CUtensorMap& tm_xl, const CUtensorMap& tm_l2, const CUtensorMap& tm_y,
                           const K2Int8Params& p, int num_sms, cudaStream_t stream);
size_t k2_int8_weight_bytes(int N, int K);

// Y is read and rewritten through tm_y: a BF16 [M][N] map with boxes of 64
// columns x upproj_box_rows() rows and the 128-byte swizzle.
cudaError_t launch_upproj(const CUtensorMap& tm_y, const UpParams& p, cudaStream_t stream);
int upproj_box_rows();

// One-thread kernel whose only wait can never complete: it gives up after
// budget_ns and sets *err (failure-detection self-test).
cudaError_t launch_wait_selftest(int* err, unsigned long long budget_ns, cudaStream_t stream);

}  // namespace svdq
