// Weight-only INT4 GEMV for the adaptive-normalization linears (W4A16).
//
// SOTA-314 practice page, "Do this": the linear layers inside FLUX.1's adaptive
// normalization stay W4A16.  They run on a handful of conditioning rows
// (M <= 16 per pass), so the layer is a matrix-vector product whose floor is
// reading the 4-bit weights from HBM:
//     Y[m][n] = sum_g s[n][g] * sum_{k in g} X[m][k] * c[n][k]  + b[n]
// with symmetric INT4 codes c and BF16 scales s per group g of 64 k.
//
// Why tensor cores: at M = 4 the product is 4 N K multiply-adds.  On the FP32
// pipes that (plus unpacking the nibbles) takes about twice as long as reading
// the weights, so the dot products go to mma.sync m16n8k16 (BF16 in, FP32
// accumulate) on register fragments, and the kernel stays bound by the weight
// stream.
//
// Weight layout on the device (built once by w4a16_pack): rows are cut into
// tiles of 16 (the MMA's M side; rows past N are zero) and each tile is stored
// group by group, 544 bytes per (tile, group):
//   bytes   0..511  lane-major: lane l = 4 g + q holds 16 bytes = the 16 codes
//                   k = 64 gi + 16 q .. +15 of row g (8 bytes) then of row g+8;
//                   inside each 32-bit word (8 codes, pairs j = 0..3) the first
//                   code of pair j sits at bits 4j and the second at bits 16+4j,
//                   so (word >> 4j) & 0x000F000F is a BF16x2-ready pair;
//   bytes 512..543  scales (row g, row g+8) for g = 0..7.
// A tile is therefore one contiguous stream, and any range of its groups is one
// bulk copy.
//
// Tiling.  A CTA owns one tile and all of K; its 8 warps take contiguous ranges
// of groups (split K) and are reduced through shared memory at the end.  Each
// warp streams its range through a private ring of shared-memory stages with
// cp.async.bulk (one elected lane issues; an mbarrier per stage counts the
// bytes), so up to 4 stages per warp are in flight without holding registers.
// Inside a group the k order is permuted so that the 16 codes a thread reads
// are exactly its A-fragment elements for the group's 4 MMAs, and the
// activation fragments (8 consecutive BF16 pairs of X, read through L1) use the
// same permutation; a sum over k is order-free.  Each group accumulates into a
// fresh FP32 fragment that is then scaled by the row's group scale, so the BF16
// operands are the exact codes.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstddef>
#include <mutex>
#include <vector>

#include "kernels.h"
#include "sm100.cuh"

namespace svdq {

namespace {

using namespace dev;

constexpr int kWarps = 8;
constexpr int kRows = 16;                              // weight rows per tile (MMA M)
constexpr int kGroupBytes = 544;                       // 512 bytes of codes + 32 of scales
constexpr int kStageGroups = 2;
constexpr int kStages = 4;                             // ring depth per warp
constexpr int kStageBytes = kStageGroups * kGroupBytes;
static_assert(kGroupBytes % 16 == 0 && kStageBytes % 16 == 0, "bulk copies move 16-byte multiples");

// Codes pair (bits 0-3, 16-19 of y) as an exact bf16x2 of (c + 136): the
// biased nibble (n ^ 8) = c + 8 in the mantissa of 128.0.  The bias is removed
// once per group through the activation sums (see the kernel).
__device__ __forceinline__ uint32_t codes_pair(uint32_t y) { return (y & 0x000F000Fu) ^ 0x43084308u; }

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 lds128(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_u32(p)));
  return v;
}
__device__ __forceinline__ uint32_t lds32(const void* p) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)));
  return v;
}
__device__ __forceinline__ float2 lds64f(const void* p) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(smem_u32(p)));
  return v;
}

template <int MT>
struct W4A16Smem {
  uint8_t ring[kWarps][kStages][kStageBytes];
  uint64_t full[kWarps][kStages];
  float red[2][kWarps][MT][32][4];
  int abort_flag, never;
  float xsum[1];   // [G][8 MT]: sum of X over each group of 64 k, per activation column
};

template <int MT>
size_t w4a16_smem_bytes(int G) {
  return offsetof(W4A16Smem<MT>, xsum) + sizeof(float) * (size_t)G * 8 * MT;
}

// MT = number of 8-row activation tiles in this pass (1: M <= 8, 2: M <= 16).
// Persistent: CTA c takes weight tiles c, c + gridDim.x, ...; each warp's ring
// streams its group range of one tile after the other, so the next tile's
// weights are in flight while this one is reduced.
template <int MT>
__global__ void __launch_bounds__(kWarps * 32, MT == 1 ? 4 : 3) w4a16_kernel(W4A16Params p, int m0) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  W4A16Smem<MT>& sm = *reinterpret_cast<W4A16Smem<MT>*>(smem_raw);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int K = p.K, G = K >> 6;
  const int ntiles = (p.N + kRows - 1) / kRows;
  const int my_tiles = (ntiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
  const int gb = warp * G / kWarps, ge = (warp + 1) * G / kWarps;   // this warp's groups in every tile
  const int ng = ge - gb, st_per_tile = (ng + kStageGroups - 1) / kStageGroups;
  const int nst = my_tiles * st_per_tile;

  // Producer state (lane 0): the next stage to issue as (tile of this CTA, stage in tile, ring slot).
  int issued = 0, p_lt = 0, p_si = 0, p_slot = 0;
  auto issue_next = [&]() {
    const int ngr = min(kStageGroups, ng - p_si * kStageGroups);
    const size_t tile = (size_t)blockIdx.x + (size_t)p_lt * gridDim.x;
    const uint8_t* src = p.wt + (tile * G + gb + (size_t)p_si * kStageGroups) * kGroupBytes;
    mbar_arrive_expect_tx(&sm.full[warp][p_slot], (uint32_t)ngr * kGroupBytes);
    bulk_load(sm.ring[warp][p_slot], src, (uint32_t)ngr * kGroupBytes, &sm.full[warp][p_slot]);
    ++issued;
    if (++p_si == st_per_tile) {
      p_si = 0;
      ++p_lt;
    }
    if (++p_slot == kStages) p_slot = 0;
  };

  if (threadIdx.x == 0) {
    sm.abort_flag = 0;
    sm.never = 0;
  }
  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&sm.full[warp][s], 1);
    fence_mbar_init();
    while (issued < nst && issued < kStages) issue_next();
  }
  // Activation sums per (group, column) while the first weights stream in.
  for (int i = threadIdx.x; i < G * 8 * MT; i += kWarps * 32) {
    const int gi = i / (8 * MT), c = i % (8 * MT), m = m0 + c;
    float sum = 0.f;
    if (m < p.M) {
      const uint4* xs = reinterpret_cast<const uint4*>(p.x + (size_t)m * K + 64 * (size_t)gi);
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const uint4 u = __ldg(xs + v);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) sum += __uint_as_float(w[e] << 16) + __uint_as_float(w[e] & 0xFFFF0000u);
      }
    }
    sm.xsum[i] = sum;
  }
  __syncthreads();

  // activation row of this thread in each n8 tile (column g)
  const __nv_bfloat16* xr[MT];
  bool xv[MT];
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    const int m = m0 + 8 * t + g;
    xv[t] = m < p.M;
    xr[t] = p.x + (size_t)(xv[t] ? m : 0) * K + 16 * q;
  }
  // X[m][64 gi + 16 q .. +16] as 8 BF16 pairs P[i] = (x[2i], x[2i+1]) (zeros for unused columns)
  auto load_x = [&](int gi, uint32_t (&P)[MT][8]) {
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      if (xv[t]) {
        const uint4* xs = reinterpret_cast<const uint4*>(xr[t] + 64 * (size_t)gi);
        const uint4 a = __ldg(xs), b = __ldg(xs + 1);
        P[t][0] = a.x; P[t][1] = a.y; P[t][2] = a.z; P[t][3] = a.w;
        P[t][4] = b.x; P[t][5] = b.y; P[t][6] = b.z; P[t][7] = b.w;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) P[t][i] = 0u;
      }
    }
  };

  bool aborted = false;
  int consumed = 0, slot = 0;
  uint32_t phase = 0;
  for (int lt = 0; lt < my_tiles; ++lt) {
    const int tile = (int)blockIdx.x + lt * (int)gridDim.x;
    float acc[MT][4];
#pragma unroll
    for (int t = 0; t < MT; ++t)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[t][j] = 0.f;

    int gi0 = gb;
    for (int si = 0; si < st_per_tile && !aborted; ++si, gi0 += kStageGroups) {
      const int n_here = min(kStageGroups, ge - gi0);
      uint32_t P[MT][8];
      load_x(gi0, P);   // in flight during the wait
      const bool ok = mbar_wait(&sm.full[warp][slot], phase, &sm.abort_flag, p.budget_ns);
      if (!__all_sync(0xffffffffu, ok)) {
        aborted = true;
        if (lane == 0) {
          sm.abort_flag = 1;
          atomicExch(p.err, 1);
        }
        break;
      }
      uint4 cw[kStageGroups];
      uint32_t sw[kStageGroups];
#pragma unroll
      for (int j = 0; j < kStageGroups; ++j) {
        if (j < n_here) {
          cw[j] = lds128(sm.ring[warp][slot] + j * kGroupBytes + lane * 16);
          sw[j] = lds32(sm.ring[warp][slot] + j * kGroupBytes + 512 + g * 4);
        }
      }
      __syncwarp();
      if (lane == 0 && issued < nst) {   // refill this slot
        fence_async_shared();
        issue_next();
      }
      ++consumed;
      if (++slot == kStages) {
        slot = 0;
        phase ^= 1u;
      }
#pragma unroll
      for (int j = 0; j < kStageGroups; ++j) {
        if (j >= n_here) break;
        uint32_t Pn[MT][8];
        if (j + 1 < n_here) load_x(gi0 + j + 1, Pn);   // next group's activations
        // start from -136 * sum(x) so the biased codes (c + 136) give sum(x c)
        float part[MT][4];
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          const float2 xs = lds64f(&sm.xsum[(gi0 + j) * 8 * MT + 8 * t + 2 * q]);
          part[t][0] = -136.f * xs.x;
          part[t][1] = -136.f * xs.y;
          part[t][2] = -136.f * xs.x;
          part[t][3] = -136.f * xs.y;
        }
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          // MMA step s: positions (2q, 2q+1) <- codes 4s, 4s+1 and (2q+8, 2q+9) <- 4s+2, 4s+3
          // of this thread's 16; those are pairs 2(s&1) and 2(s&1)+1 of word s>>1.
          const uint32_t wa = (s < 2) ? cw[j].x : cw[j].y;   // row g
          const uint32_t wb = (s < 2) ? cw[j].z : cw[j].w;   // row g + 8
          const int sh = 8 * (s & 1);
          const uint32_t a[4] = {codes_pair(wa >> sh), codes_pair(wb >> sh), codes_pair(wa >> (sh + 4)),
                                 codes_pair(wb >> (sh + 4))};
#pragma unroll
          for (int t = 0; t < MT; ++t) mma_bf16_16816(part[t], a, P[t][2 * s], P[t][2 * s + 1]);
        }
        const float s0 = __uint_as_float(sw[j] << 16), s1 = __uint_as_float(sw[j] & 0xFFFF0000u);
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          acc[t][0] = fmaf(s0, part[t][0], acc[t][0]);
          acc[t][1] = fmaf(s0, part[t][1], acc[t][1]);
          acc[t][2] = fmaf(s1, part[t][2], acc[t][2]);
          acc[t][3] = fmaf(s1, part[t][3], acc[t][3]);
        }
        if (j + 1 < n_here) {
#pragma unroll
          for (int t = 0; t < MT; ++t)
#pragma unroll
            for (int i = 0; i < 8; ++i) P[t][i] = Pn[t][i];
        }
      }
    }

    // split-K reduction of this tile over the 8 warps (double-buffered by tile parity)
#pragma unroll
    for (int t = 0; t < MT; ++t)
#pragma unroll
      for (int j = 0; j < 4; ++j) sm.red[lt & 1][warp][t][lane][j] = acc[t][j];
    __syncthreads();
    // warp t finishes activation tile t: fragment element j is (row g + 8 (j>>1), column 2q + (j&1))
    if (warp < MT && !sm.abort_flag) {
      const int t = warp;
      float v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int w = 0; w < kWarps; ++w)
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] += sm.red[lt & 1][w][t][lane][j];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = tile * kRows + g + ((j & 2) ? 8 : 0);
        const int m = m0 + 8 * t + 2 * q + (j & 1);
        if (n < p.N && m < p.M) p.y[(size_t)m * p.N + n] = __float2bfloat16_rn(v[j] + p.bias[n]);
      }
    }
  }
  // After an abort, let this warp's copies still in flight land before the CTA exits.
  if (lane == 0) {
    for (; consumed < issued; ++consumed) {
      mbar_wait(&sm.full[warp][slot], phase, &sm.never, p.budget_ns);
      if (++slot == kStages) {
        slot = 0;
        phase ^= 1u;
      }
    }
  }
}

}  // namespace

bool w4a16_supported(int K) { return w4a16_smem_bytes<2>(K / 64) <= 200u * 1024u; }

size_t w4a16_packed_bytes(int N, int K) {
  return (size_t)((N + kRows - 1) / kRows) * (size_t)(K / 64) * kGroupBytes;
}

void w4a16_pack(const uint8_t* codes, const uint16_t* scales, int N, int K, uint8_t* out) {
  const int G = K / 64, tiles = (N + kRows - 1) / kRows;
  for (size_t i = 0; i < w4a16_packed_bytes(N, K); ++i) out[i] = 0;
  for (int t = 0; t < tiles; ++t)
    for (int gi = 0; gi < G; ++gi) {
      uint8_t* base = out + ((size_t)t * G + gi) * kGroupBytes;
      for (int g = 0; g < 8; ++g)
        for (int h = 0; h < 2; ++h) {
          const int n = t * kRows + g + 8 * h;
          if (n >= N) continue;
          for (int q = 0; q < 4; ++q) {
            const uint8_t* b = codes + (size_t)n * (K / 2) + (size_t)gi * 32 + q * 8;   // 16 codes, natural order
            for (int w = 0; w < 2; ++w) {
              uint32_t word = 0;
              for (int j = 0; j < 4; ++j) {
                const uint32_t byte = b[4 * w + j];   // codes (2j, 2j+1) of this word: low, high nibble
                word |= (byte & 0xFu) << (4 * j);
                word |= (byte >> 4) << (16 + 4 * j);
              }
              uint8_t* dst = base + (4 * g + q) * 16 + h * 8 + w * 4;
              for (int e = 0; e < 4; ++e) dst[e] = (uint8_t)(word >> (8 * e));
            }
          }
          const uint16_t s = scales[(size_t)n * G + gi];
          base[512 + g * 4 + h * 2] = (uint8_t)(s & 0xFF);
          base[512 + g * 4 + h * 2 + 1] = (uint8_t)(s >> 8);
        }
    }
}

namespace {

// Blocks per SM for this kernel at `smem` bytes, cached per device.
template <int MT>
cudaError_t grid_size(size_t smem, int ntiles, int* grid) {
  struct Entry {
    size_t smem = 0;
    int sms = 0, per_sm = 0;
  };
  static Entry cache[64];
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  Entry& c = cache[dev];
  if (c.smem != smem) {
    if ((e = cudaFuncSetAttribute(w4a16_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
        cudaSuccess)
      return e;
    if ((e = cudaDeviceGetAttribute(&c.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&c.per_sm, w4a16_kernel<MT>, kWarps * 32, smem)) !=
        cudaSuccess)
      return e;
    if (c.per_sm < 1) return cudaErrorInvalidConfiguration;
    c.smem = smem;
  }
  *grid = std::min(ntiles, c.sms * c.per_sm);
  return cudaSuccess;
}

template <int MT>
cudaError_t launch_pass(const W4A16Params& p, int m0, cudaStream_t stream) {
  const int G = p.K / 64, ntiles = (p.N + kRows - 1) / kRows;
  const size_t smem = w4a16_smem_bytes<MT>(G);
  int grid = 0;
  cudaError_t e = grid_size<MT>(smem, ntiles, &grid);
  if (e != cudaSuccess) return e;
  w4a16_kernel<MT><<<grid, kWarps * 32, smem, stream>>>(p, m0);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_w4a16(const W4A16Params& p, cudaStream_t stream) {
  for (int m0 = 0; m0 < p.M; m0 += 16) {
    cudaError_t e = (p.M - m0 <= 8) ? launch_pass<1>(p, m0, stream) : launch_pass<2>(p, m0, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace svdq
