// C ABI of the SVDQuant W4A4 library: layer lifetime, device upload, tensor
// maps, workspace layout and the forward launches (see include/svdq.h).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "kernels.h"
#include "svdq_internal.h"

using namespace svdq;

struct svdq_layer {
  HostPrep host;
  int device = -1;
  int num_sms = 0;
  unsigned long long budget_ns = 2000000000ull;
  // device buffers (owned)
  float* d_inv_lam = nullptr;
  __nv_bfloat16* d_l1t = nullptr;    // [32][K]   L1d^T
  __nv_bfloat16* d_l2s = nullptr;    // [N][32]   (L2b / alpha)^T
  __nv_bfloat16* d_l2t = nullptr;    // [N][32]   L2b^T (unfused up projection)
  uint8_t* d_wq = nullptr;           // INT4: codes [N][K/2]; W4A16: the GEMV's packed weights
  uint8_t* d_ws = nullptr;           // INT4: weight scales, FP16 [K/64][npad] (times 2^-ew)
  uint8_t* d_wmerged = nullptr;      // NVFP4: codes and scales merged for the single-CTA GEMM
  uint8_t* d_wpair = nullptr;        // NVFP4: codes and scales merged for the CTA-pair GEMM
  int i4_ex = 0, i4_ew = 0;          // INT4: power-of-two range exponents of the FP16 GEMM operands
  float* d_bias = nullptr;           // [N]
  int* d_err = nullptr;
  CUtensorMap tm_wq, tm_l2s, tm_l1t;     // tm_wq: INT4 weight codes [N][K/2]
  CUtensorMap tm_l2s_pair;               // 128-row boxes for the CTA-pair GEMMs
  CUtensorMap tm_wq_pair;                // INT4 weight codes, 128-row boxes (CTA-pair INT4 GEMM)
  int k2_kernel = 0;                     // NVFP4 GEMM: 0 = by size, 1 = single-CTA, 2 = CTA pairs
  // LoRA adapter (svdq_set_lora): A^T rows for the down pass, (s B)^T rows for the up pass
  __nv_bfloat16* d_lora_l1t = nullptr;   // [32][K]   A^T, zero rows past r
  __nv_bfloat16* d_lora_l2s = nullptr;   // [N][32]   (bf16(s B) / alpha)^T (NVFP4 GEMM)
  __nv_bfloat16* d_lora_l2t = nullptr;   // [N][64]   [L2b^T | bf16(s B)^T] (unfused up projection)
  CUtensorMap tm_lora_l1t, tm_lora_l2s;
};

namespace {

// ------------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2D tensor [rows][cols] of `elem` bytes with rows `row_bytes` apart, box [box_rows][box_cols].
bool make_map_strided(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t cols, uint64_t rows,
                      uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D row-major tensor [rows][cols] of `elem` bytes, box [box_rows][box_cols].
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem, uint64_t cols, uint64_t rows,
              uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * (uint64_t)elem};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// BF16 matrix [rows][cols] seen as 64-column chunks: dimensions (64 columns,
// rows, cols / 64 chunks), so that one box of (64, box_rows, 4) brings 4
// consecutive chunks of box_rows rows, chunk-major, each chunk a [box_rows][128 B]
// tile in the 128-byte swizzle: the layout four 2D boxes of (64, box_rows) give,
// in one copy instead of four.  cols % 64 == 0.
bool make_map_kchunks(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {64, rows, cols / 64};
  const cuuint64_t strides[2] = {cols * 2, 128};
  const cuuint32_t box[3] = {64, box_rows, 4};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ helpers

struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) { ok = false; return; }
    if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }


// Formats with quantized activations (the two-kernel forward): NVFP4, INT4, W8A8.
bool w4a4(const svdq_layer* L) {
  return L->host.format == SVDQ_NVFP4 || L->host.format == SVDQ_INT4 || L->host.format == SVDQ_W8A8_INT8;
}
bool w8a8(const HostPrep& h) { return h.format == SVDQ_W8A8_INT8; }
int int8_stages(int K) { return (K + 127) / 128; }   // K stages of 128 int8 codes (128-byte rows)

int pad_rows(int M) { return (M + 127) / 128 * 128; }
int nvfp4_stages(int K) { return (K + 255) / 256; }   // K stages of 256 codes (128-byte rows)

// Bytes of the activation codes for M tokens: NVFP4 tiled (act_tile_offset),
// INT4 row-major [M][K/2].
size_t act_code_bytes(const HostPrep& h, int M) {
  if (h.format == SVDQ_NVFP4) return (size_t)pad_rows(M) * (size_t)nvfp4_stages(h.K) * 128u;
  if (h.format == SVDQ_W8A8_INT8) return (size_t)pad_rows(M) * (size_t)int8_stages(h.K) * 128u;
  return (size_t)M * (size_t)(h.K / 2);
}

// FP16 bits of a value that is exact in float32, rounded to nearest even.
uint16_t f16_from_double(double v) { return __half_as_ushort(__float2half_rn((float)v)); }
int pad_cols_int4(int N) { return (N + 255) / 256 * 256; }

size_t act_scale_bytes(const HostPrep& h, int M) {
  if (h.format == SVDQ_NVFP4) return (size_t)((M + 127) / 128) * (size_t)(h.K / 64) * 512;
  if (h.format == SVDQ_INT4) return (size_t)(h.K / 64) * (size_t)pad_rows(M) * 2;   // BF16 [K/64][mpad]
  if (h.format == SVDQ_W8A8_INT8) return (size_t)pad_rows(M) * 8;                   // s_x [mpad], 1/s_x [mpad]
  return 0;
}

// FP16 range exponents of the INT4 GEMM's dequantized operands: the largest
// |c s| of the weights maps to at most 2^14 (4x below FP16's maximum), the
// largest smoothed calibration activation to at most 2^8, so that a runtime
// group scale up to about 220x the calibration batch's largest stays below the
// GEMM's clamp of 8192, while every group scale down to 2^-24 of that largest
// value stays at or above 2^-17, where FP16 holds all of its 8 bits exactly.
void int4_range_exponents(const HostPrep& h, int* ex, int* ew) {
  // w_amax: the largest group maximum the quantizer saw (amax |R| for
  // round-to-nearest; GPTQ's updated values may move it either way)
  *ew = pow2_ceil_exponent((double)h.w_amax) - 14;
  *ex = pow2_ceil_exponent((double)h.x_amax) - 8;
}

struct WsLayout {
  size_t codes = 0, scales = 0, xl = 0, total = 0;
};

// Columns of the down projection XL: 32, plus 32 for X A when a LoRA adapter is attached.
int xl_width(const HostPrep& h) { return h.lora_r > 0 ? 64 : 32; }

WsLayout ws_layout(const HostPrep& h, int M) {
  WsLayout w;
  w.codes = 0;
  w.scales = align_up(act_code_bytes(h, M), 256);
  w.xl = w.scales + align_up(act_scale_bytes(h, M), 256);
  w.total = w.xl + align_up((size_t)M * xl_width(h) * 2, 256);
  return w;
}

template <class T>
cudaError_t upload(T** dst, const void* src, size_t bytes) {
  cudaError_t e = cudaMalloc(reinterpret_cast<void**>(dst), std::max<size_t>(bytes, 16));
  if (e != cudaSuccess) return e;
  if (bytes) e = cudaMemcpy(*dst, src, bytes, cudaMemcpyHostToDevice);
  return e;
}

void free_device(svdq_layer* L) {
  if (L->device < 0) return;
  DeviceGuard g(L->device);
  cudaFree(L->d_inv_lam);
  cudaFree(L->d_l1t);
  cudaFree(L->d_l2s);
  cudaFree(L->d_l2t);
  cudaFree(L->d_wq);
  cudaFree(L->d_ws);
  cudaFree(L->d_wmerged);
  cudaFree(L->d_wpair);
  cudaFree(L->d_bias);
  cudaFree(L->d_err);
  cudaFree(L->d_lora_l1t);
  cudaFree(L->d_lora_l2s);
  cudaFree(L->d_lora_l2t);
  L->d_inv_lam = nullptr;
  L->d_lora_l1t = L->d_lora_l2s = L->d_lora_l2t = nullptr;
}

svdq_status upload_layer(svdq_layer* L, int device) {
  DeviceGuard g(device);
  if (!g.ok) return SVDQ_ECUDA;
  const HostPrep& h = L->host;
  const int K = h.K, N = h.N, r = h.rank;
  L->device = device;
  if (cudaDeviceGetAttribute(&L->num_sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
    return SVDQ_ECUDA;
  if (const char* b = std::getenv("SVDQ_WAIT_BUDGET_MS")) {
    const double ms = std::atof(b);
    if (ms > 0) L->budget_ns = (unsigned long long)(ms * 1e6);
  }
  cudaError_t e = cudaSuccess;
  auto chk = [&](cudaError_t x) {
    if (x != cudaSuccess && e == cudaSuccess) e = x;
  };
  chk(cudaMalloc(reinterpret_cast<void**>(&L->d_err), sizeof(int)));
  if (e == cudaSuccess) chk(cudaMemset(L->d_err, 0, sizeof(int)));
  chk(upload(&L->d_bias, h.bias.data(), sizeof(float) * N));
  if (h.format == SVDQ_NVFP4 || h.format == SVDQ_INT4 || h.format == SVDQ_W8A8_INT8) {
    chk(upload(&L->d_inv_lam, h.inv_lam.data(), sizeof(float) * K));
    std::vector<uint8_t> tiled;
    if (h.format == SVDQ_W8A8_INT8) {
      // int8 weight codes in (256-row, 128-column) blocks of the GEMM's tiled
      // layout (wgt_tile_offset over 128-byte rows), rows padded with zeros
      const int nst8 = (K + 127) / 128;
      tiled.assign(k2_int8_weight_bytes(N, K), 0);
      for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k)
          tiled[wgt_tile_offset(n, k >> 7, (k & 127) >> 4, nst8) + (k & 15)] = h.w_codes[(size_t)n * K + k];
      chk(upload(&L->d_wq, tiled.data(), tiled.size()));
      chk(upload(&L->d_ws, h.w_scales_f32.data(), sizeof(float) * N));
    } else if (h.format == SVDQ_NVFP4) {
      // weight codes in the GEMM's tiled layout (wgt_tile_offset), rows padded to 256 with zeros
      const int nst = nvfp4_stages(K);
      tiled.assign((size_t)((N + 255) / 256) * (size_t)nst * 32768u, 0);
      for (int n = 0; n < N; ++n)
        for (int b = 0; b < K / 2; ++b)
          tiled[wgt_tile_offset(n, b >> 7, (b & 127) >> 4, nst) + (b & 15)] = h.w_codes[(size_t)n * (K / 2) + b];
    } else {
      chk(upload(&L->d_wq, h.w_codes.data(), h.w_codes.size()));
    }
    // the branch's up factor is divided by the GEMM's accumulator unit alpha
    // (NVFP4: g_x g_w; INT4: 2^(ex + ew)); W8A8 keeps a branch accumulator of its own
    int alpha_exp = h.format == SVDQ_W8A8_INT8 ? 0 : h.g_x_exp + h.g_w_exp;
    if (h.format == SVDQ_W8A8_INT8) {
      // nothing more: codes and scales are uploaded above
    } else if (h.format == SVDQ_NVFP4) {
      // weight scales in the tensor-core layout, rows padded to a multiple of 256
      const int npad = (N + 255) / 256 * 256;
      std::vector<uint8_t> ws((size_t)(npad / 128) * (K / 64) * 512, 0);
      for (int n = 0; n < N; ++n)
        for (int gi = 0; gi < K / 16; ++gi) ws[sf_offset(n, gi, K)] = h.w_scales_e4m3[(size_t)n * (K / 16) + gi];
      // codes and scales merged, one layout per GEMM variant
      std::vector<uint8_t> wm(k2_weight_bytes(N, K));
      k2_pack_weights(tiled.data(), ws.data(), N, K, wm.data());
      chk(upload(&L->d_wmerged, wm.data(), wm.size()));
      std::vector<uint8_t> wpair(k2_pair_weight_bytes(N, K));
      k2_pair_pack_weights(tiled.data(), ws.data(), N, K, wpair.data());
      chk(upload(&L->d_wpair, wpair.data(), wpair.size()));
    } else {
      // weight scales times 2^-ew as FP16, group-major [K/64][npad] (zero padding)
      int4_range_exponents(h, &L->i4_ex, &L->i4_ew);
      alpha_exp = L->i4_ex + L->i4_ew;
      const int npad = pad_cols_int4(N), G = K / 64;
      std::vector<uint16_t> ws((size_t)G * npad, 0);
      for (int n = 0; n < N; ++n)
        for (int gi = 0; gi < G; ++gi) {
          const double v = std::ldexp((double)bf16_to_float(h.w_scales_bf16[(size_t)n * G + gi]), -L->i4_ew);
          ws[(size_t)gi * npad + n] = f16_from_double(v);
        }
      chk(upload(&L->d_ws, ws.data(), ws.size() * 2));
    }
    // low-rank branch: L1d^T for the first kernel, (L2b / alpha)^T and L2b^T for the second
    std::vector<uint16_t> l1t((size_t)32 * K, 0), l2s((size_t)N * 32, 0), l2t((size_t)N * 32, 0);
    const double inv_alpha = std::ldexp(1.0, -alpha_exp);
    for (int i = 0; i < r; ++i) {
      for (int k = 0; k < K; ++k) l1t[(size_t)i * K + k] = h.L1d[(size_t)k * r + i];
      for (int n = 0; n < N; ++n) {
        const uint16_t b = h.L2b[(size_t)i * N + n];
        l2t[(size_t)n * 32 + i] = b;
        l2s[(size_t)n * 32 + i] = bf16_from_double((double)bf16_to_float(b) * inv_alpha);
      }
    }
    chk(upload(&L->d_l1t, l1t.data(), l1t.size() * 2));
    chk(upload(&L->d_l2s, l2s.data(), l2s.size() * 2));
    chk(upload(&L->d_l2t, l2t.data(), l2t.size() * 2));
    if (e != cudaSuccess) return SVDQ_ECUDA;
    const bool nv = h.format == SVDQ_NVFP4;
    {
      const bool ok2 = make_map(&L->tm_l2s_pair, L->d_l2s, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 32, N, 32,
                                (uint32_t)(nv ? k2_pair_rows_b() : k2_int4_pair_rows_b()), CU_TENSOR_MAP_SWIZZLE_64B);
      if (!ok2) return SVDQ_ECUDA;
      if (const char* k = std::getenv("SVDQ_K2_KERNEL")) {
        if (!std::strcmp(k, "single")) L->k2_kernel = 1;
        if (!std::strcmp(k, "pair")) L->k2_kernel = 2;
      }
    }
    // INT4 weight codes stay row-major [N][K/2] (the INT4 GEMM loads them with TMA)
    bool ok = (nv || (make_map(&L->tm_wq, L->d_wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, N, 32, 256,
                               CU_TENSOR_MAP_SWIZZLE_NONE) &&
                      make_map(&L->tm_wq_pair, L->d_wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, N, 32,
                               (uint32_t)k2_int4_pair_rows_b(), CU_TENSOR_MAP_SWIZZLE_NONE))) &&
              make_map(&L->tm_l2s, L->d_l2s, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 32, N, 32, 256,
                       CU_TENSOR_MAP_SWIZZLE_64B) &&
              make_map_kchunks(&L->tm_l1t, L->d_l1t, K, 32, 32);
    if (!ok) return SVDQ_ECUDA;
  } else if (h.format == SVDQ_W4A16_INT4) {
    std::vector<uint8_t> packed(w4a16_packed_bytes(N, K));
    w4a16_pack(h.w_codes.data(), h.w_scales_bf16.data(), N, K, packed.data());
    chk(upload(&L->d_wq, packed.data(), packed.size()));
  }
  return e == cudaSuccess ? SVDQ_OK : SVDQ_ECUDA;
}

// Arguments first (SVDQ_EINVAL), then the layer's state (SVDQ_ESTATE).
svdq_status check_forward_args(const svdq_layer* L, const void* X, int M, const void* Y) {
  if (!L || !X || !Y || M < 1) return SVDQ_EINVAL;
  if ((reinterpret_cast<uintptr_t>(X) & 15) || (reinterpret_cast<uintptr_t>(Y) & 15)) return SVDQ_EINVAL;
  if (L->device < 0) return SVDQ_ESTATE;
  return SVDQ_OK;
}

K1Params k1_params(const svdq_layer* L, int M, void* codes, void* scales, void* xl) {
  const HostPrep& h = L->host;
  K1Params p;
  p.M = M;
  p.K = h.K;
  p.mpad = pad_rows(M);
  p.nst = nvfp4_stages(h.K);
  p.c_x = (float)std::ldexp((double)(1.0f / 6.0f), -h.g_x_exp);
  p.g_x_exp = h.g_x_exp;
  for (int m = 0; m < 8; ++m) {
    p.rcp[m] = (float)(1.0 / (1.0 + m / 8.0));
    p.rcp[8 + m] = m ? (float)(1.0 / m) : 0.0f;
  }
  p.inv_lam = L->d_inv_lam;
  p.inv_sx = nullptr;
  p.codes = static_cast<uint8_t*>(codes);
  p.scales = static_cast<uint8_t*>(scales);
  p.xl = static_cast<__nv_bfloat16*>(xl);
  p.xl_stride = xl_width(h);
  p.err = L->d_err;
  p.budget_ns = L->budget_ns;
  return p;
}

svdq_status run_k1(const svdq_layer* L, const void* X, int M, void* codes, void* scales, void* xl,
                   cudaStream_t stream, int mode) {
  const HostPrep& h = L->host;
  CUtensorMap tm_x, tm_c;
  if (!make_map_kchunks(&tm_x, X, h.K, M, 32))
    return SVDQ_ECUDA;
  // activation codes are written in 32-row tiles, one per quantizer warp and stage:
  // 16 bytes wide for NVFP4 (32 columns), 32 bytes for INT4 (64 columns)
  // NVFP4 codes are written tiled from registers; INT4 codes in 32-row x 32-byte
  // tiles by TMA (one per quantizer warp and stage)
  const bool nv = h.format == SVDQ_NVFP4, i8 = w8a8(h);
  if (mode != 2 && !nv && !i8 &&
      !make_map(&tm_c, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, h.K / 2, M, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE))
    return SVDQ_ECUDA;
  if (mode == 2 || nv || i8) tm_c = tm_x;   // unused
  K1Params p = k1_params(L, M, codes, scales, xl);
  if (i8 && mode != 2) {
    // W8A8: the per-token scales first ([s_x | 1/s_x] in the scales buffer)
    const int mpad = pad_rows(M);
    float* sx = static_cast<float*>(scales);
    if (launch_rowscale(static_cast<const __nv_bfloat16*>(X), L->d_inv_lam, M, h.K, mpad, sx, sx + mpad, stream) !=
        cudaSuccess)
      return SVDQ_ECUDA;
    p.inv_sx = sx + mpad;
  }
  const int fmt = nv ? kFmtNvfp4 : i8 ? kFmtInt8 : kFmtInt4;
  return launch_k1(tm_x, L->tm_l1t, tm_c, p, fmt, mode, stream) == cudaSuccess ? SVDQ_OK : SVDQ_ECUDA;
}

svdq_status run_k2_int8(const svdq_layer* L, const void* codes, const void* scales, const void* xl, int M, void* Y,
                        cudaStream_t stream, bool branch, bool gelu) {
  const HostPrep& h = L->host;
  CUtensorMap tm_xl, tm_y;
  if (!make_map(&tm_y, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, h.N, M, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return SVDQ_ECUDA;
  if (branch) {
    if (!make_map_strided(&tm_xl, xl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 32, M, (uint64_t)xl_width(h) * 2, 32, 128,
                          CU_TENSOR_MAP_SWIZZLE_64B))
      return SVDQ_ECUDA;
  } else {
    tm_xl = tm_y;   // unused by the kernel
  }
  K2Int8Params p;
  p.M = M;
  p.N = h.N;
  p.K = h.K;
  p.acodes = static_cast<const uint8_t*>(codes);
  p.wq = L->d_wq;
  p.sx = static_cast<const float*>(scales);
  p.sw = reinterpret_cast<const float*>(L->d_ws);
  p.bias = L->d_bias;
  p.y = static_cast<__nv_bfloat16*>(Y);
  p.err = L->d_err;
  p.budget_ns = L->budget_ns;
  p.branch = branch ? 1 : 0;
  p.gelu = gelu ? 1 : 0;
  return launch_k2_int8(tm_xl, L->tm_l2s, tm_y, p, L->num_sms, stream) == cudaSuccess ? SVDQ_OK : SVDQ_ECUDA;
}

// The LoRA adapter's down pass: XL columns 32..63 = bf16(X A), the first
// kernel's down-projection-only mode over A^T.
svdq_status run_k1_lora(const svdq_layer* L, const void* X, int M, void* xl, cudaStream_t stream) {
  const HostPrep& h = L->host;
  CUtensorMap tm_x;
  if (!make_map_kchunks(&tm_x, X, h.K, M, 32)) return SVDQ_ECUDA;
  K1Params p = k1_params(L, M, nullptr, nullptr, static_cast<__nv_bfloat16*>(xl) + 32);
  return launch_k1(tm_x, L->tm_lora_l1t, tm_x, p, kFmtNvfp4, 2, stream) == cudaSuccess ? SVDQ_OK : SVDQ_ECUDA;
}

// The up-projection kernel adding xl ([M][width], row stride xlw) times l2t^T
// ([N][width]) into Y [+ GELU].
svdq_status run_upproj(const svdq_layer* L, const void* xl, int xlw, int width, const __nv_bfloat16* l2t, int M,
                       void* Y, cudaStream_t stream, bool gelu) {
  UpParams up;
  up.M = M;
  up.N = L->host.N;
  up.width = width;
  up.xl = static_cast<const __nv_bfloat16*>(xl);
  up.xl_stride = xlw;
  up.l2t = l2t;
  up.gelu = gelu ? 1 : 0;
  up.err = L->d_err;
  up.budget_ns = L->budget_ns;
  CUtensorMap tm_up;
  if (!make_map(&tm_up, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, L->host.N, M, 64, (uint32_t)upproj_box_rows(),
                CU_TENSOR_MAP_SWIZZLE_128B))
    return SVDQ_ECUDA;
  return launch_upproj(tm_up, up, stream) == cudaSuccess ? SVDQ_OK : SVDQ_ECUDA;
}

svdq_status run_k2_int4(const svdq_layer* L, const void* codes, const void* scales, const void* xl, int M,
                        void* Y, cudaStream_t stream, bool branch, bool gelu, bool lora_on) {
  const HostPrep& h = L->host;
  const bool lora = h.lora_r > 0 && lora_on;
  CUtensorMap tm_a, tm_xl, tm_y, tm_xla;
  if (!make_map(&tm_a, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, h.K / 2, M, 32, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
    return SVDQ_ECUDA;
  if (!make_map(&tm_y, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, h.N, M, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return SVDQ_ECUDA;
  if (branch) {
    if (!make_map_strided(&tm_xl, xl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 32, M, (uint64_t)xl_width(h) * 2, 32, 128,
                          CU_TENSOR_MAP_SWIZZLE_64B))
      return SVDQ_ECUDA;
  } else {
    tm_xl = tm_a;   // unused by the kernel
  }
  if (lora) {
    // XL columns 32..63 (X A): the same rows, 64 bytes in
    if (!make_map_strided(&tm_xla, static_cast<const __nv_bfloat16*>(xl) + 32, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 32,
                          M, (uint64_t)xl_width(h) * 2, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B))
      return SVDQ_ECUDA;
  } else {
    tm_xla = tm_a;  // unused by the kernel
  }
  K2Int4Params p;
  p.M = M;
  p.N = h.N;
  p.K = h.K;
  p.mpad = pad_rows(M);
  p.npad = pad_cols_int4(h.N);
  p.alpha = (float)std::ldexp(1.0, L->i4_ex + L->i4_ew);
  p.xscale = (float)std::ldexp(1.0, -L->i4_ex);
  p.sa = static_cast<const uint16_t*>(scales);
  p.sb = reinterpret_cast<const uint16_t*>(L->d_ws);
  p.bias = L->d_bias;
  p.y = static_cast<__nv_bfloat16*>(Y);
  p.err = L->d_err;
  p.budget_ns = L->budget_ns;
  p.branch = branch ? 1 : 0;
  p.gelu = gelu ? 1 : 0;
  p.lora = lora ? 1 : 0;
  const cudaError_t e =
      L->k2_kernel == 2 && !lora
          ? launch_k2_int4_pair(tm_a, L->tm_wq_pair, tm_xl, L->tm_l2s_pair, tm_y, p, L->num_sms, stream)
          : launch_k2_int4(tm_a, L->tm_wq, tm_xl, L->tm_l2s, tm_y, tm_xla, lora ? L->tm_lora_l2s : L->tm_l2s, p,
                           L->num_sms, stream);
  return e == cudaSuccess ? SVDQ_OK : SVDQ_ECUDA;
}

// The second kernel.  With a LoRA adapter (and lora_on) the NVFP4 GEMM adds
// XL_lora (s B) in its own ring stage, the INT4 GEMM by reloading its branch
// buffer within the tile; either way into the same accumulator.
svdq_status run_k2(const svdq_layer* L, const void* codes, const void* scales, const void* xl, int M, void* Y,
                   cudaStream_t stream, bool branch, bool gelu, bool lora_on = true) {
  if (L->host.format == SVDQ_INT4) return run_k2_int4(L, codes, scales, xl, M, Y, stream, branch, gelu, lora_on);
  if (w8a8(L->host)) return run_k2_int8(L, codes, scales, xl, M, Y, stream, branch, gelu);
  const HostPrep& h = L->host;
  const bool lora = h.lora_r > 0 && lora_on;
  CUtensorMap tm_xl, tm_y, tm_xla;
  if (!make_map(&tm_y, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, h.N, M, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return SVDQ_ECUDA;
  const uint64_t xl_row = (uint64_t)xl_width(h) * 2;
  if (branch) {
    if (!make_map_strided(&tm_xl, xl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 32, M, xl_row, 32, 128,
                          CU_TENSOR_MAP_SWIZZLE_64B))
      return SVDQ_ECUDA;
  } else {
    tm_xl = tm_y;   // unused by the kernel
  }
  if (lora) {
    // XL columns 32..63 (X A): the same rows, 64 bytes in
    if (!make_map_strided(&tm_xla, static_cast<const __nv_bfloat16*>(xl) + 32, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 32,
                          M, xl_row, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B))
      return SVDQ_ECUDA;
  } else {
    tm_xla = tm_y;   // unused by the kernel
  }
  K2Params p;
  p.M = M;
  p.N = h.N;
  p.K = h.K;
  p.mpad = pad_rows(M);
  p.acodes = static_cast<const uint8_t*>(codes);
  p.alpha = (float)std::ldexp(1.0, h.g_x_exp + h.g_w_exp);
  p.sfa = static_cast<const uint8_t*>(scales);
  p.wmerged = L->d_wmerged;
  p.wpair = L->d_wpair;
  p.bias = L->d_bias;
  p.y = static_cast<__nv_bfloat16*>(Y);
  p.err = L->d_err;
  p.budget_ns = L->budget_ns;
  p.branch = branch ? 1 : 0;
  p.gelu = gelu ? 1 : 0;
  p.lora = lora ? 1 : 0;
  // The CTA-pair kernel (256 x 256 tiles) is exact but measured slower than the
  // single-CTA kernel on this part; it runs only when SVDQ_K2_KERNEL=pair, and
  // only for layers without a LoRA adapter.
  const bool pair = L->k2_kernel == 2 && !lora;
  const cudaError_t e = pair ? launch_k2_pair(tm_xl, L->tm_l2s_pair, tm_y, p, L->num_sms, stream)
                             : launch_k2(tm_xl, L->tm_l2s, tm_y, tm_xla, L->tm_lora_l2s, p, L->num_sms, stream);
  return e == cudaSuccess ? SVDQ_OK : SVDQ_ECUDA;
}

// (Re)build a layer's LoRA device buffers from the host copies (none when
// lora_r == 0).  The device must be current and idle for this layer.
svdq_status upload_lora(svdq_layer* L) {
  const HostPrep& h = L->host;
  const int K = h.K, N = h.N, r = h.lora_r;
  cudaFree(L->d_lora_l1t);
  cudaFree(L->d_lora_l2s);
  cudaFree(L->d_lora_l2t);
  L->d_lora_l1t = L->d_lora_l2s = L->d_lora_l2t = nullptr;
  if (r == 0) return SVDQ_OK;
  // the GEMM's accumulator unit: alpha = g_x g_w (NVFP4) or 2^(ex + ew) (INT4)
  const int alpha_exp = h.format == SVDQ_NVFP4 ? h.g_x_exp + h.g_w_exp : L->i4_ex + L->i4_ew;
  // l2t: the unfused up projection's [N][64] = [L2b^T | bf16(s B)^T]
  std::vector<uint16_t> l1t((size_t)32 * K, 0), l2s((size_t)N * 32, 0), l2t((size_t)N * 64, 0);
  for (int i = 0; i < h.rank; ++i)
    for (int n = 0; n < N; ++n) l2t[(size_t)n * 64 + i] = h.L2b[(size_t)i * N + n];
  for (int i = 0; i < r; ++i) {
    for (int k = 0; k < K; ++k) l1t[(size_t)i * K + k] = h.lora_A[(size_t)k * r + i];
    for (int n = 0; n < N; ++n) {
      const uint16_t v = h.lora_B[(size_t)i * N + n];
      l2t[(size_t)n * 64 + 32 + i] = v;
      l2s[(size_t)n * 32 + i] = bf16_from_double(std::ldexp((double)bf16_to_float(v), -alpha_exp));
    }
  }
  cudaError_t e = upload(&L->d_lora_l1t, l1t.data(), l1t.size() * 2);
  if (e == cudaSuccess) e = upload(&L->d_lora_l2s, l2s.data(), l2s.size() * 2);
  if (e == cudaSuccess) e = upload(&L->d_lora_l2t, l2t.data(), l2t.size() * 2);
  if (e != cudaSuccess || !make_map_kchunks(&L->tm_lora_l1t, L->d_lora_l1t, K, 32, 32) ||
      !make_map(&L->tm_lora_l2s, L->d_lora_l2s, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 32, N, 32, 256,
                CU_TENSOR_MAP_SWIZZLE_64B)) {
    cudaFree(L->d_lora_l1t);
    cudaFree(L->d_lora_l2s);
    cudaFree(L->d_lora_l2t);
    L->d_lora_l1t = L->d_lora_l2s = L->d_lora_l2t = nullptr;
    return e == cudaErrorMemoryAllocation ? SVDQ_ENOMEM : SVDQ_ECUDA;
  }
  return SVDQ_OK;
}

// ------------------------------------------------------------------ serialization
//
// A prepared layer as bytes: "SVDQ", version, the scalar fields, then each
// array as a 64-bit byte count followed by its bytes (lam, inv_lam, sigma,
// L1d, L2b, w_codes, w_scales_e4m3, w_scales_bf16, w_scales_f32, bias,
// lora_A, lora_B), then a 64-bit FNV-1a checksum of everything before it.
// The preparation-only intermediates (R, L1, L2, the GPTQ factor) are not
// part of it.

constexpr uint32_t kSerialMagic = 0x51445653u;   // "SVDQ"
constexpr uint32_t kSerialVersion = 2;

// FNV-1a, 64-bit (Fowler, Noll and Vo): xor in each byte, then multiply by
// the FNV prime, starting from the offset basis.
uint64_t fnv1a64(const uint8_t* p, size_t n) {
  uint64_t h = 0xCBF29CE484222325ull;
  for (size_t i = 0; i < n; ++i) {
    h ^= p[i];
    h *= 0x100000001B3ull;
  }
  return h;
}

struct SerialHeader {
  uint32_t magic, version;
  int32_t K, N, rank, format, g_x_exp, g_w_exp, lora_r, svd_iterations;
  float alpha, x_amax, w_amax, pad;
  double svd_tail_energy;
};

// f(array) for every serialized array of h, in order (h const or not).
template <class F, class H>
void serial_arrays(F&& f, H& h) {
  f(h.lam);
  f(h.inv_lam);
  f(h.sigma);
  f(h.L1d);
  f(h.L2b);
  f(h.w_codes);
  f(h.w_scales_e4m3);
  f(h.w_scales_bf16);
  f(h.w_scales_f32);
  f(h.bias);
  f(h.lora_A);
  f(h.lora_B);
}

size_t serialized_bytes(const HostPrep& h) {
  size_t n = sizeof(SerialHeader) + 8;   // header and checksum
  serial_arrays([&](const auto& v) { n += 8 + v.size() * sizeof(v[0]); }, h);
  return n;
}

// ------------------------------------------------------------------ fc1 -> fc2 chain

bool chainable(const svdq_layer* L1, const svdq_layer* L2) {
  return L1->host.format == SVDQ_NVFP4 && L2->host.format == SVDQ_NVFP4 && L1->host.N == L2->host.K &&
         L1->device == L2->device && L1->host.lora_r == 0 && L2->host.lora_r == 0;
}

// Workspace of the fused chain: [fc1's forward workspace][fc2 codes][fc2 scales]
// [XL2][partials]; of the unfused chain: [fc1's workspace][Y1 BF16][fc2's workspace].
struct ChainLayout {
  size_t codes2 = 0, scales2 = 0, xl2 = 0, partials = 0, y1 = 0, ws2 = 0, total = 0;
  int S = 1;
};

ChainLayout chain_layout(const svdq_layer* L1, const svdq_layer* L2, int M, bool unfused) {
  ChainLayout c;
  const size_t w1 = align_up(ws_layout(L1->host, M).total, 256);
  if (unfused) {
    c.y1 = w1;
    c.ws2 = c.y1 + align_up((size_t)M * L1->host.N * 2, 256);
    c.total = c.ws2 + ws_layout(L2->host, M).total;
    return c;
  }
  c.S = k2_chain_splits(M, L1->host.N, L1->num_sms);
  c.codes2 = w1;
  c.scales2 = c.codes2 + align_up(act_code_bytes(L2->host, M), 256);
  c.xl2 = c.scales2 + align_up(act_scale_bytes(L2->host, M), 256);
  c.partials = c.xl2 + align_up((size_t)M * 32 * 2, 256);
  c.total = c.partials + (size_t)pad_rows(M) * 2 * c.S * 32 * 4;
  return c;
}

// fc1's first kernel, then its GEMM in chain mode (fc2's codes, scales and
// down-projection partials), then the fixed-order sum of the partials into XL2.
svdq_status run_chain_fc1(const svdq_layer* L1, const svdq_layer* L2, const void* X, int M, void* codes2,
                          void* scales2, void* xl2, void* partials, int S, uint8_t* ws1, cudaStream_t s, bool gelu) {
  const HostPrep& h1 = L1->host;
  const HostPrep& h2 = L2->host;
  const WsLayout w = ws_layout(h1, M);
  void* codes1 = ws1 + w.codes;
  void* scales1 = ws1 + w.scales;
  void* xl1 = ws1 + w.xl;
  const bool branch1 = h1.rank > 0, branch2 = h2.rank > 0;
  svdq_status st = run_k1(L1, X, M, codes1, scales1, xl1, s, branch1 ? 0 : 1);
  if (st != SVDQ_OK) return st;
  CUtensorMap tm_xl;
  if (branch1) {
    if (!make_map(&tm_xl, xl1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 32, M, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B))
      return SVDQ_ECUDA;
  } else {
    tm_xl = L1->tm_l2s;   // unused by the kernel
  }
  K2Params p;
  p.M = M;
  p.N = h1.N;
  p.K = h1.K;
  p.mpad = pad_rows(M);
  p.acodes = static_cast<const uint8_t*>(codes1);
  p.alpha = (float)std::ldexp(1.0, h1.g_x_exp + h1.g_w_exp);
  p.sfa = static_cast<const uint8_t*>(scales1);
  p.wmerged = L1->d_wmerged;
  p.wpair = L1->d_wpair;
  p.bias = L1->d_bias;
  p.y = nullptr;
  p.err = L1->d_err;
  p.budget_ns = L1->budget_ns;
  p.branch = branch1 ? 1 : 0;
  p.gelu = gelu ? 1 : 0;
  K2Chain& c = p.chain;
  c.codes = static_cast<uint8_t*>(codes2);
  c.scales = static_cast<uint8_t*>(scales2);
  c.inv_lam = L2->d_inv_lam;
  c.l1t = branch2 ? L2->d_l1t : nullptr;
  c.partials = static_cast<float*>(partials);
  c.K2 = h2.K;
  c.nst = nvfp4_stages(h2.K);
  c.S = S;
  c.g_x_exp = h2.g_x_exp;
  c.c_x = (float)std::ldexp((double)(1.0f / 6.0f), -h2.g_x_exp);
  for (int m = 0; m < 8; ++m) {
    c.rcp[m] = (float)(1.0 / (1.0 + m / 8.0));
    c.rcp[8 + m] = m ? (float)(1.0 / m) : 0.0f;
  }
  if (launch_k2_chain(tm_xl, L1->tm_l2s, p, L1->num_sms, s) != cudaSuccess) return SVDQ_ECUDA;
  if (branch2 && launch_xl_reduce(static_cast<const float*>(partials), 2 * S, M,
                                  static_cast<__nv_bfloat16*>(xl2), s) != cudaSuccess)
    return SVDQ_ECUDA;
  return SVDQ_OK;
}

// The second kernel (the adapter, if any, is added inside it).
svdq_status run_gemm_stage(const svdq_layer* L, const void* codes, const void* scales, const void* xl, int M,
                           void* Y, cudaStream_t s, bool branch, bool gelu, bool lora_on) {
  return run_k2(L, codes, scales, xl, M, Y, s, branch, gelu, lora_on);
}

}  // namespace

// ====================================================================== ABI

extern "C" {

const char* svdq_status_string(svdq_status s) {
  switch (s) {
    case SVDQ_OK: return "ok";
    case SVDQ_EINVAL: return "invalid argument";
    case SVDQ_EUNSUPPORTED: return "unsupported shape or option";
    case SVDQ_ENOMEM: return "out of memory";
    case SVDQ_ECUDA: return "CUDA error";
    case SVDQ_ENOCONVERGE: return "truncated SVD did not converge";
    case SVDQ_ETIMEOUT: return "device wait timed out";
    case SVDQ_ESTATE: return "layer has no device copy";
  }
  return "unknown status";
}

svdq_status svdq_prepare(const svdq_config* cfg, int K, int N, const uint16_t* W_bf16, const uint16_t* bias_bf16,
                         const uint16_t* calib_bf16, int M_calib, int device, svdq_layer** out) {
  if (!out) return SVDQ_EINVAL;
  *out = nullptr;
  if (!cfg || !W_bf16 || K <= 0 || N <= 0 || device < -1) return SVDQ_EINVAL;
  if (cfg->format < SVDQ_NVFP4 || cfg->format > SVDQ_W8A8_INT8) return SVDQ_EINVAL;
  const bool wo = cfg->format == SVDQ_W4A16_INT4;
  if (cfg->flags & ~(SVDQ_PREP_GPTQ | SVDQ_PREP_KEEP_GPTQ_FACTOR)) return SVDQ_EINVAL;
  if ((cfg->flags & SVDQ_PREP_KEEP_GPTQ_FACTOR) && !(cfg->flags & SVDQ_PREP_GPTQ)) return SVDQ_EINVAL;
  if (wo && (cfg->flags & SVDQ_PREP_GPTQ)) return SVDQ_EINVAL;   // GPTQ needs the calibration batch
  if (!wo) {
    if (!calib_bf16 || M_calib < 1) return SVDQ_EINVAL;
    if (!(cfg->alpha > 0.0f && cfg->alpha < 1.0f)) return SVDQ_EINVAL;
    // rank 32 at 4 bits, 16 at 8 bits (or no branch)
    const int want = cfg->format == SVDQ_W8A8_INT8 ? 16 : 32;
    if (cfg->rank != 0 && cfg->rank != want) return SVDQ_EUNSUPPORTED;
    if (cfg->format == SVDQ_W8A8_INT8 && (cfg->flags & SVDQ_PREP_GPTQ)) return SVDQ_EUNSUPPORTED;
  }
  // W4A4 needs N % 16 for its TMA tiles; the weight-only GEMV takes any N
  if (K % 64 != 0 || (!wo && N % 16 != 0)) return SVDQ_EUNSUPPORTED;
  if (wo && !w4a16_supported(K)) return SVDQ_EUNSUPPORTED;
  svdq_layer* L = new (std::nothrow) svdq_layer();
  if (!L) return SVDQ_ENOMEM;
  svdq_status st = host_prepare(*cfg, K, N, W_bf16, bias_bf16, calib_bf16, M_calib, L->host);
  // The first kernel's division-free reciprocal of the NVFP4 scales equals the
  // IEEE quotient for activation tensor-scale exponents in [-40, 30], i.e.
  // calibration maxima between about 3e-10 and 7e11.
  if (st == SVDQ_OK && L->host.format == SVDQ_NVFP4 && (L->host.g_x_exp < -40 || L->host.g_x_exp > 30))
    st = SVDQ_EUNSUPPORTED;
  if (st == SVDQ_OK && device >= 0) {
    st = upload_layer(L, device);
    if (st != SVDQ_OK) free_device(L);
  }
  if (st != SVDQ_OK) {
    delete L;
    return st;
  }
  *out = L;
  return SVDQ_OK;
}

void svdq_destroy(svdq_layer* L) {
  if (!L) return;
  free_device(L);
  delete L;
}

svdq_status svdq_get_info(const svdq_layer* L, svdq_layer_info* info) {
  if (!L || !info) return SVDQ_EINVAL;
  info->K = L->host.K;
  info->N = L->host.N;
  info->rank = L->host.rank;
  info->format = L->host.format;
  info->device = L->device;
  info->g_x_exp = L->host.g_x_exp;
  info->g_w_exp = L->host.g_w_exp;
  info->svd_iterations = L->host.svd_iterations;
  info->svd_tail_energy = L->host.svd_tail_energy;
  return SVDQ_OK;
}

size_t svdq_tensor_bytes(const svdq_layer* L, int id) {
  if (!L) return 0;
  const HostPrep& h = L->host;
  switch (id) {
    case SVDQ_T_LAMBDA:
    case SVDQ_T_INV_LAMBDA: return h.lam.size() * 4;
    case SVDQ_T_L1: return h.L1.size() * 8;
    case SVDQ_T_L2: return h.L2.size() * 8;
    case SVDQ_T_L1D: return h.L1d.size() * 2;
    case SVDQ_T_L2B: return h.L2b.size() * 2;
    case SVDQ_T_RESIDUAL: return h.R.size() * 4;
    case SVDQ_T_SIGMA: return h.sigma.size() * 8;
    case SVDQ_T_W_CODES: return h.w_codes.size();
    case SVDQ_T_W_SCALES:
      return h.format == SVDQ_NVFP4 ? h.w_scales_e4m3.size()
             : w8a8(h)              ? h.w_scales_f32.size() * 4
                                    : h.w_scales_bf16.size() * 2;
    case SVDQ_T_BIAS: return h.bias.size() * 4;
    case SVDQ_T_GPTQ_U: return h.gptq_U.size() * 8;
    case SVDQ_T_LORA_A: return h.lora_A.size() * 2;
    case SVDQ_T_LORA_B: return h.lora_B.size() * 2;
  }
  return 0;
}

svdq_status svdq_export(const svdq_layer* L, int id, void* dst, size_t bytes) {
  if (!L || !dst) return SVDQ_EINVAL;
  const size_t need = svdq_tensor_bytes(L, id);
  if (need == 0 || bytes != need) return SVDQ_EINVAL;
  const HostPrep& h = L->host;
  const void* src = nullptr;
  switch (id) {
    case SVDQ_T_LAMBDA: src = h.lam.data(); break;
    case SVDQ_T_INV_LAMBDA: src = h.inv_lam.data(); break;
    case SVDQ_T_L1: src = h.L1.data(); break;
    case SVDQ_T_L2: src = h.L2.data(); break;
    case SVDQ_T_L1D: src = h.L1d.data(); break;
    case SVDQ_T_L2B: src = h.L2b.data(); break;
    case SVDQ_T_RESIDUAL: src = h.R.data(); break;
    case SVDQ_T_SIGMA: src = h.sigma.data(); break;
    case SVDQ_T_W_CODES: src = h.w_codes.data(); break;
    case SVDQ_T_W_SCALES:
      src = h.format == SVDQ_NVFP4 ? (const void*)h.w_scales_e4m3.data()
            : w8a8(h)              ? (const void*)h.w_scales_f32.data()
                                   : (const void*)h.w_scales_bf16.data();
      break;
    case SVDQ_T_BIAS: src = h.bias.data(); break;
    case SVDQ_T_GPTQ_U: src = h.gptq_U.data(); break;
    case SVDQ_T_LORA_A: src = h.lora_A.data(); break;
    case SVDQ_T_LORA_B: src = h.lora_B.data(); break;
    default: return SVDQ_EINVAL;
  }
  std::memcpy(dst, src, bytes);
  return SVDQ_OK;
}

size_t svdq_workspace_bytes(const svdq_layer* L, int M) {
  if (!L || M < 1) return 0;
  if (!w4a4(L)) return 0;
  return ws_layout(L->host, M).total;
}

size_t svdq_act_scale_bytes(const svdq_layer* L, int M) {
  if (!L || M < 1) return 0;
  return act_scale_bytes(L->host, M);
}

size_t svdq_act_code_bytes(const svdq_layer* L, int M) {
  if (!L || M < 1 || !w4a4(L)) return 0;
  return act_code_bytes(L->host, M);
}

svdq_status svdq_act_codes_to_logical(const svdq_layer* L, const void* device_layout, int M, void* logical) {
  if (!L || !device_layout || !logical || M < 1) return SVDQ_EINVAL;
  const HostPrep& h = L->host;
  if (!w4a4(L)) return SVDQ_EUNSUPPORTED;
  const uint8_t* src = static_cast<const uint8_t*>(device_layout);
  uint8_t* dst = static_cast<uint8_t*>(logical);
  if (w8a8(h)) {
    const int nst8 = int8_stages(h.K);
    for (int r = 0; r < M; ++r)
      for (int k = 0; k < h.K; ++k)
        dst[(size_t)r * h.K + k] = src[act_tile_offset(r, k >> 7, (k & 127) >> 4, nst8) + (k & 15)];
    return SVDQ_OK;
  }
  const size_t row = (size_t)(h.K / 2);
  if (h.format == SVDQ_INT4) {
    std::memcpy(dst, src, (size_t)M * row);
    return SVDQ_OK;
  }
  const int nst = nvfp4_stages(h.K);
  for (int r = 0; r < M; ++r)
    for (size_t b = 0; b < row; ++b)
      dst[(size_t)r * row + b] = src[act_tile_offset(r, (int)(b >> 7), (int)((b & 127) >> 4), nst) + (b & 15)];
  return SVDQ_OK;
}

svdq_status svdq_act_scales_to_logical(const svdq_layer* L, const void* device_layout, int M, void* logical) {
  if (!L || !device_layout || !logical || M < 1) return SVDQ_EINVAL;
  const HostPrep& h = L->host;
  if (h.format == SVDQ_INT4) {
    const uint16_t* src = static_cast<const uint16_t*>(device_layout);
    uint16_t* dst = static_cast<uint16_t*>(logical);
    const int G = h.K / 64, mpad = pad_rows(M);
    for (int r = 0; r < M; ++r)
      for (int gi = 0; gi < G; ++gi) dst[(size_t)r * G + gi] = src[(size_t)gi * mpad + r];
    return SVDQ_OK;
  }
  if (w8a8(h)) {
    std::memcpy(logical, device_layout, (size_t)M * sizeof(float));   // s_x, one per token
    return SVDQ_OK;
  }
  if (h.format != SVDQ_NVFP4) return SVDQ_EUNSUPPORTED;
  const uint8_t* src = static_cast<const uint8_t*>(device_layout);
  uint8_t* dst = static_cast<uint8_t*>(logical);
  const int G = h.K / 16;
  for (int r = 0; r < M; ++r)
    for (int gi = 0; gi < G; ++gi) dst[(size_t)r * G + gi] = src[sf_offset(r, gi, h.K)];
  return SVDQ_OK;
}

svdq_status svdq_quantize_act(const svdq_layer* L, const void* X, int M, void* codes, void* scales, void* xl,
                              void* stream, int mode) {
  if ((reinterpret_cast<uintptr_t>(scales) & 15) || (reinterpret_cast<uintptr_t>(xl) & 15)) return SVDQ_EINVAL;
  svdq_status st = check_forward_args(L, X, M, codes);
  if (st != SVDQ_OK) return st;
  if (!w4a4(L)) return SVDQ_EUNSUPPORTED;
  if (mode < 0 || mode > 2) return SVDQ_EINVAL;
  if (!scales && mode != 2) return SVDQ_EINVAL;
  const bool rank = L->host.rank > 0, lora = L->host.lora_r > 0;
  const bool has_xl = rank || lora;
  if (!has_xl && mode == 2) return SVDQ_EINVAL;
  if (!has_xl && mode == 0) mode = 1;
  if (has_xl && mode != 1 && !xl) return SVDQ_EINVAL;
  DeviceGuard g(L->device);
  if (!g.ok) return SVDQ_ECUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (rank || mode != 2) st = run_k1(L, X, M, codes, scales, xl, s, rank ? mode : 1);
  if (st == SVDQ_OK && lora && mode != 1) st = run_k1_lora(L, X, M, xl, s);
  return st;
}

svdq_status svdq_gemm(const svdq_layer* L, const void* codes, const void* scales, const void* xl, int M, void* Y,
                      void* stream, unsigned flags) {
  if ((reinterpret_cast<uintptr_t>(scales) & 15) || (reinterpret_cast<uintptr_t>(xl) & 15)) return SVDQ_EINVAL;
  svdq_status st = check_forward_args(L, codes, M, Y);
  if (st != SVDQ_OK) return st;
  if (!w4a4(L)) return SVDQ_EUNSUPPORTED;
  if (!scales) return SVDQ_EINVAL;
  const bool bare = (flags & SVDQ_FWD_NO_BRANCH) != 0;
  const bool branch = L->host.rank > 0 && !bare;
  const bool lora = L->host.lora_r > 0 && !bare;
  if ((branch || lora) && !xl) return SVDQ_EINVAL;
  DeviceGuard g(L->device);
  if (!g.ok) return SVDQ_ECUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = run_gemm_stage(L, codes, scales, xl, M, Y, s, branch, (flags & SVDQ_FWD_GELU) != 0, lora);
  if (st == SVDQ_OK && (flags & SVDQ_FWD_CHECK)) st = svdq_check(L, stream);
  return st;
}

svdq_status svdq_linear_forward(const svdq_layer* L, const void* X, int M, void* Y, void* workspace,
                                size_t workspace_bytes, void* stream, unsigned flags) {
  svdq_status st = check_forward_args(L, X, M, Y);
  if (st != SVDQ_OK) return st;
  if (L->host.format == SVDQ_W4A16_INT4) {
    // weight-only path: one kernel, no workspace
    if (flags & (SVDQ_FWD_GELU | SVDQ_FWD_UNFUSED | SVDQ_FWD_NO_BRANCH)) return SVDQ_EUNSUPPORTED;
    DeviceGuard g(L->device);
    if (!g.ok) return SVDQ_ECUDA;
    W4A16Params p;
    p.M = M;
    p.N = L->host.N;
    p.K = L->host.K;
    p.x = static_cast<const __nv_bfloat16*>(X);
    p.wt = L->d_wq;
    p.bias = L->d_bias;
    p.y = static_cast<__nv_bfloat16*>(Y);
    p.err = L->d_err;
    p.budget_ns = L->budget_ns;
    st = launch_w4a16(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SVDQ_OK : SVDQ_ECUDA;
    if (st == SVDQ_OK && (flags & SVDQ_FWD_CHECK)) st = svdq_check(L, stream);
    return st;
  }
  if (!w4a4(L)) return SVDQ_EUNSUPPORTED;
  const WsLayout w = ws_layout(L->host, M);
  if (!workspace || workspace_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return SVDQ_EINVAL;
  DeviceGuard g(L->device);
  if (!g.ok) return SVDQ_ECUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* codes = ws + w.codes;
  void* scales = ws + w.scales;
  void* xl = ws + w.xl;
  const bool gelu = (flags & SVDQ_FWD_GELU) != 0;
  const bool bare = (flags & SVDQ_FWD_NO_BRANCH) != 0;
  const bool has_branch = L->host.rank > 0;
  const bool lora = L->host.lora_r > 0 && !bare;
  const int xlw = xl_width(L->host);
  if ((flags & SVDQ_FWD_UNFUSED) && (has_branch || lora) && !bare) {
    // measurement variant: down projection(s), quantize, bare GEMM, up projection.
    // A rank-0 layer's L1d^T is all zero: its pass writes zero XL columns for
    // the 64-wide up projection to read.
    st = run_k1(L, X, M, codes, scales, xl, s, 2);
    if (st == SVDQ_OK && lora) st = run_k1_lora(L, X, M, xl, s);
    if (st == SVDQ_OK) st = run_k1(L, X, M, codes, scales, xl, s, 1);
    if (st == SVDQ_OK) st = run_k2(L, codes, scales, xl, M, Y, s, false, false, false);
    // one up projection over the whole branch: [L2b^T | bf16(s B)^T] with an adapter
    if (st == SVDQ_OK) st = run_upproj(L, xl, xlw, lora ? 64 : 32, lora ? L->d_lora_l2t : L->d_l2t, M, Y, s, gelu);
  } else {
    const bool branch = has_branch && !bare;
    st = run_k1(L, X, M, codes, scales, xl, s, branch ? 0 : 1);
    if (st == SVDQ_OK && lora) st = run_k1_lora(L, X, M, xl, s);
    if (st == SVDQ_OK) st = run_gemm_stage(L, codes, scales, xl, M, Y, s, branch, gelu, lora);
  }
  if (st == SVDQ_OK && (flags & SVDQ_FWD_CHECK)) st = svdq_check(L, stream);
  return st;
}

size_t svdq_serialized_bytes(const svdq_layer* L) { return L ? serialized_bytes(L->host) : 0; }

svdq_status svdq_serialize(const svdq_layer* L, void* dst, size_t bytes) {
  if (!L || !dst) return SVDQ_EINVAL;
  const HostPrep& h = L->host;
  if (bytes != serialized_bytes(h)) return SVDQ_EINVAL;
  SerialHeader hd = {};
  hd.magic = kSerialMagic;
  hd.version = kSerialVersion;
  hd.K = h.K;
  hd.N = h.N;
  hd.rank = h.rank;
  hd.format = h.format;
  hd.g_x_exp = h.g_x_exp;
  hd.g_w_exp = h.g_w_exp;
  hd.lora_r = h.lora_r;
  hd.svd_iterations = h.svd_iterations;
  hd.alpha = h.alpha;
  hd.x_amax = h.x_amax;
  hd.w_amax = h.w_amax;
  hd.svd_tail_energy = h.svd_tail_energy;
  uint8_t* o = static_cast<uint8_t*>(dst);
  std::memcpy(o, &hd, sizeof(hd));
  o += sizeof(hd);
  serial_arrays(
      [&](const auto& v) {
        const uint64_t n = v.size() * sizeof(v[0]);
        std::memcpy(o, &n, 8);
        if (n) std::memcpy(o + 8, v.data(), n);
        o += 8 + n;
      },
      h);
  const uint64_t sum = fnv1a64(static_cast<const uint8_t*>(dst), (size_t)(o - static_cast<uint8_t*>(dst)));
  std::memcpy(o, &sum, 8);
  return SVDQ_OK;
}

svdq_status svdq_deserialize(const void* src, size_t bytes, int device, svdq_layer** out) {
  if (!out) return SVDQ_EINVAL;
  *out = nullptr;
  if (!src || bytes < sizeof(SerialHeader) + 8 || device < -1) return SVDQ_EINVAL;
  SerialHeader hd;
  std::memcpy(&hd, src, sizeof(hd));
  if (hd.magic != kSerialMagic || hd.version != kSerialVersion) return SVDQ_EINVAL;
  uint64_t sum = 0;
  std::memcpy(&sum, static_cast<const uint8_t*>(src) + bytes - 8, 8);
  if (sum != fnv1a64(static_cast<const uint8_t*>(src), bytes - 8)) return SVDQ_EINVAL;   // corrupted
  if (hd.format < SVDQ_NVFP4 || hd.format > SVDQ_W8A8_INT8 || hd.K <= 0 || hd.N <= 0 || hd.K % 64 ||
      hd.rank < 0 || hd.rank > 32 || hd.lora_r < 0 || hd.lora_r > 32)
    return SVDQ_EINVAL;
  svdq_layer* L = new (std::nothrow) svdq_layer();
  if (!L) return SVDQ_ENOMEM;
  HostPrep& h = L->host;
  h.K = hd.K;
  h.N = hd.N;
  h.rank = hd.rank;
  h.format = hd.format;
  h.g_x_exp = hd.g_x_exp;
  h.g_w_exp = hd.g_w_exp;
  h.lora_r = hd.lora_r;
  h.svd_iterations = hd.svd_iterations;
  h.alpha = hd.alpha;
  h.x_amax = hd.x_amax;
  h.w_amax = hd.w_amax;
  h.svd_tail_energy = hd.svd_tail_energy;
  const uint8_t* in = static_cast<const uint8_t*>(src) + sizeof(hd);
  const uint8_t* end = static_cast<const uint8_t*>(src) + bytes - 8;
  bool ok = true;
  try {
    serial_arrays(
        [&](auto& v) {
          uint64_t n = 0;
          if (!ok || end - in < 8) {
            ok = false;
            return;
          }
          std::memcpy(&n, in, 8);
          in += 8;
          if (n % sizeof(v[0]) || (uint64_t)(end - in) < n) {
            ok = false;
            return;
          }
          v.resize(n / sizeof(v[0]));
          if (n) std::memcpy(v.data(), in, n);
          in += n;
        },
        h);
  } catch (const std::bad_alloc&) {
    delete L;
    return SVDQ_ENOMEM;
  }
  // every array must have the size the shape and format imply
  const size_t K = h.K, N = h.N, r = h.rank, lr = h.lora_r;
  const bool nv = h.format == SVDQ_NVFP4, i4 = h.format == SVDQ_INT4 || h.format == SVDQ_W4A16_INT4,
             i8 = h.format == SVDQ_W8A8_INT8;
  ok = ok && in == end && h.lam.size() == K && h.inv_lam.size() == K && h.sigma.size() == r &&
       h.L1d.size() == K * r && h.L2b.size() == r * N && h.bias.size() == N &&
       h.w_codes.size() == (i8 ? N * K : N * K / 2) && h.w_scales_e4m3.size() == (nv ? N * K / 16 : 0) &&
       h.w_scales_bf16.size() == (i4 ? N * K / 64 : 0) && h.w_scales_f32.size() == (i8 ? N : 0) &&
       h.lora_A.size() == K * lr && h.lora_B.size() == lr * N;
  if (!ok) {
    delete L;
    return SVDQ_EINVAL;
  }
  svdq_status st = SVDQ_OK;
  if (device >= 0) {
    st = upload_layer(L, device);
    if (st == SVDQ_OK && h.lora_r > 0) {
      DeviceGuard g(device);
      st = g.ok ? upload_lora(L) : SVDQ_ECUDA;
    }
    if (st != SVDQ_OK) free_device(L);
  }
  if (st != SVDQ_OK) {
    delete L;
    return st;
  }
  *out = L;
  return SVDQ_OK;
}

svdq_status svdq_set_lora(svdq_layer* L, int r, const uint16_t* A_bf16, const uint16_t* B_bf16, float scale) {
  if (!L) return SVDQ_EINVAL;
  if (L->host.format == SVDQ_W4A16_INT4 || L->host.format == SVDQ_W8A8_INT8) return SVDQ_EUNSUPPORTED;
  if (r < 0) return SVDQ_EINVAL;
  if (r > 32) return SVDQ_EUNSUPPORTED;
  if (r > 0 && (!A_bf16 || !B_bf16 || !std::isfinite(scale))) return SVDQ_EINVAL;
  HostPrep& h = L->host;
  const int K = h.K, N = h.N;
  try {
    std::vector<uint16_t> a, b;
    if (r > 0) {
      a.assign(A_bf16, A_bf16 + (size_t)K * r);
      b.resize((size_t)r * N);
      for (size_t i = 0; i < b.size(); ++i)
        b[i] = bf16_from_double((double)bf16_to_float(B_bf16[i]) * (double)scale);   // one rounding of s B
    }
    h.lora_r = r;
    h.lora_A.swap(a);
    h.lora_B.swap(b);
    if (L->device >= 0) {
      DeviceGuard g(L->device);
      if (!g.ok) return SVDQ_ECUDA;
      // no forward of this layer may be pending: the old buffers are released
      if (cudaDeviceSynchronize() != cudaSuccess) return SVDQ_ECUDA;
      const svdq_status st = upload_lora(L);
      if (st != SVDQ_OK) {
        h.lora_r = 0;
        h.lora_A.clear();
        h.lora_B.clear();
        return st;
      }
    }
    return SVDQ_OK;
  } catch (const std::bad_alloc&) {
    return SVDQ_ENOMEM;
  }
  return SVDQ_OK;
}

size_t svdq_mlp_workspace_bytes(const svdq_layer* fc1, const svdq_layer* fc2, int M, unsigned flags) {
  if (!fc1 || !fc2 || M < 1 || fc1->device < 0 || !chainable(fc1, fc2)) return 0;
  return chain_layout(fc1, fc2, M, (flags & SVDQ_FWD_UNFUSED) != 0).total;
}

svdq_status svdq_mlp_fc1(const svdq_layer* fc1, const svdq_layer* fc2, const void* X, int M, void* codes2,
                         void* scales2, void* xl2, void* workspace, size_t workspace_bytes, void* stream,
                         unsigned flags) {
  svdq_status st = check_forward_args(fc1, X, M, codes2);
  if (st != SVDQ_OK) return st;
  if (!fc2 || !scales2) return SVDQ_EINVAL;
  if (fc2->device < 0) return SVDQ_ESTATE;
  if (!chainable(fc1, fc2)) return SVDQ_EUNSUPPORTED;
  if (flags & ~(SVDQ_FWD_GELU | SVDQ_FWD_CHECK)) return SVDQ_EUNSUPPORTED;
  if (fc2->host.rank > 0 && !xl2) return SVDQ_EINVAL;
  if ((reinterpret_cast<uintptr_t>(codes2) & 15) || (reinterpret_cast<uintptr_t>(scales2) & 15) ||
      (reinterpret_cast<uintptr_t>(xl2) & 15))
    return SVDQ_EINVAL;
  const ChainLayout c = chain_layout(fc1, fc2, M, false);
  if (!workspace || workspace_bytes < c.total || (reinterpret_cast<uintptr_t>(workspace) & 255)) return SVDQ_EINVAL;
  DeviceGuard g(fc1->device);
  if (!g.ok) return SVDQ_ECUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  st = run_chain_fc1(fc1, fc2, X, M, codes2, scales2, xl2, ws + c.partials, c.S, ws, s,
                     (flags & SVDQ_FWD_GELU) != 0);
  if (st == SVDQ_OK && (flags & SVDQ_FWD_CHECK)) st = svdq_check(fc1, stream);
  return st;
}

svdq_status svdq_mlp_forward(const svdq_layer* fc1, const svdq_layer* fc2, const void* X, int M, void* Y,
                             void* workspace, size_t workspace_bytes, void* stream, unsigned flags) {
  svdq_status st = check_forward_args(fc1, X, M, Y);
  if (st != SVDQ_OK) return st;
  if (!fc2) return SVDQ_EINVAL;
  if (fc2->device < 0) return SVDQ_ESTATE;
  if (!chainable(fc1, fc2)) return SVDQ_EUNSUPPORTED;
  if (flags & ~(SVDQ_FWD_GELU | SVDQ_FWD_CHECK | SVDQ_FWD_UNFUSED)) return SVDQ_EUNSUPPORTED;
  const bool unfused = (flags & SVDQ_FWD_UNFUSED) != 0;
  const ChainLayout c = chain_layout(fc1, fc2, M, unfused);
  if (!workspace || workspace_bytes < c.total || (reinterpret_cast<uintptr_t>(workspace) & 255)) return SVDQ_EINVAL;
  DeviceGuard g(fc1->device);
  if (!g.ok) return SVDQ_ECUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const bool gelu = (flags & SVDQ_FWD_GELU) != 0;
  const bool branch2 = fc2->host.rank > 0;
  if (unfused) {
    // the two layers one after the other, fc1's output through HBM in BF16
    const WsLayout w1 = ws_layout(fc1->host, M), w2 = ws_layout(fc2->host, M);
    uint8_t* ws2 = ws + c.ws2;
    void* y1 = ws + c.y1;
    const bool branch1 = fc1->host.rank > 0;
    st = run_k1(fc1, X, M, ws + w1.codes, ws + w1.scales, ws + w1.xl, s, branch1 ? 0 : 1);
    if (st == SVDQ_OK) st = run_k2(fc1, ws + w1.codes, ws + w1.scales, ws + w1.xl, M, y1, s, branch1, gelu);
    if (st == SVDQ_OK) st = run_k1(fc2, y1, M, ws2 + w2.codes, ws2 + w2.scales, ws2 + w2.xl, s, branch2 ? 0 : 1);
    if (st == SVDQ_OK) st = run_k2(fc2, ws2 + w2.codes, ws2 + w2.scales, ws2 + w2.xl, M, Y, s, branch2, false);
  } else {
    st = run_chain_fc1(fc1, fc2, X, M, ws + c.codes2, ws + c.scales2, ws + c.xl2, ws + c.partials, c.S, ws, s,
                       gelu);
    if (st == SVDQ_OK) st = run_k2(fc2, ws + c.codes2, ws + c.scales2, ws + c.xl2, M, Y, s, branch2, false);
  }
  if (st == SVDQ_OK && (flags & SVDQ_FWD_CHECK)) {
    st = svdq_check(fc1, stream);
    const svdq_status st2 = svdq_check(fc2, stream);
    if (st == SVDQ_OK) st = st2;
  }
  return st;
}

svdq_status svdq_selftest_wait_timeout(const svdq_layer* L, unsigned budget_us, void* stream) {
  if (!L || budget_us == 0 || budget_us > 10000000u) return SVDQ_EINVAL;
  if (L->device < 0) return SVDQ_ESTATE;
  DeviceGuard g(L->device);
  if (!g.ok) return SVDQ_ECUDA;
  return launch_wait_selftest(L->d_err, (unsigned long long)budget_us * 1000ull, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? SVDQ_OK
             : SVDQ_ECUDA;
}

svdq_status svdq_check(const svdq_layer* L, void* stream) {
  if (!L) return SVDQ_EINVAL;
  if (L->device < 0) return SVDQ_ESTATE;
  DeviceGuard g(L->device);
  if (!g.ok) return SVDQ_ECUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int err = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SVDQ_ECUDA;
  if (cudaMemcpy(&err, L->d_err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SVDQ_ECUDA;
  if (err != 0) {
    cudaMemset(L->d_err, 0, sizeof(int));
    return SVDQ_ETIMEOUT;
  }
  return SVDQ_OK;
}

}  // extern "C"
