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
// A tile is therefore one contiguous block of G * 544 bytes.
//
// Work layout: one CTA per SM with sixteen warps in eight pairs; each pair
// owns whole weight tiles (persistent over the tiles) and splits K between its
// two warps.  A warp streams its groups through a private ring of four chunk
// slots (four groups each) in shared memory with 16-byte cp.async copies (its
// 32 lanes copy one group's 512 code bytes, two lanes its 32 scale bytes),
// three chunks ahead of the one it computes, without holding registers; the
// weights are read once.  The two partial sums of a tile meet in shared memory
// behind a barrier of the pair alone, so no warp waits for the rest of the CTA.
// Inside a group the k order is permuted so that the 16 codes a thread reads
// are exactly its A-fragment elements for the group's 4 MMAs, and the
// activation fragments (8 consecutive BF16 pairs of X, read through L1) use the
// same permutation; a sum over k is order-free.  The four MMAs of a group
// accumulate into independent fragments (the MMA's latency is long) that are
// summed and scaled by the row's group scale, so the BF16 operands are the
// exact codes.
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

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 16;                              // weight rows per tile (MMA M)
constexpr int kGroupBytes = 544;                       // 512 bytes of codes + 32 of scales
constexpr int kChunk = 6;                              // groups per chunk (one bulk copy)
constexpr int kRing = 3;                               // chunk slots per warp (all of them in flight)
constexpr int kChunkBytes = kChunk * kGroupBytes;
constexpr int kSmemBudget = 227 * 1024;                 // dynamic shared memory per CTA

// Codes pair (bits 0-3, 16-19 of y) as an exact bf16x2 of (c + 136): the
// biased nibble (n ^ 8) = c + 8 in the mantissa of 128.0.  The bias is removed
// once per group through the activation sums (see the kernel): one multiply-add
// per output instead of a subtraction per code pair.
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

constexpr int kPairs = kWarps / 2;

// Shared memory: the warps' chunk rings, the second warp's partial sums per
// pair (double-buffered by tile parity), the per-group activation sums, one
// mbarrier per chunk slot and, when it fits (XS), the pass's 8 MT activation
// rows (rows padded by 16 bytes, so that the eight rows a fragment load reads
// fall into different banks).
template <int MT>
__host__ __device__ inline size_t smem_fixed(int G) {
  return (size_t)kWarps * kRing * kChunkBytes +
         sizeof(float) * ((size_t)kPairs * 2 * MT * 32 * 4 + (size_t)G * 8 * MT) + 8u * kWarps * kRing + 8u;
}
__host__ __device__ inline size_t xs_stride(int G) { return (size_t)G * 128 + 16; }
template <int MT, bool XS>
__host__ __device__ inline size_t smem_bytes(int G) {
  return (smem_fixed<MT>(G) + 15) / 16 * 16 + (XS ? (size_t)8 * MT * xs_stride(G) : 0);
}

// MT = number of 8-row activation tiles in this pass (1: M <= 8, 2: M <= 16);
// XS: the activation rows are staged in shared memory once per CTA (else every
// group's fragments are read from global memory, on the critical path).
template <int MT, bool XS>
__global__ void __launch_bounds__(kThreads, 1) w4a16_kernel(W4A16Params p, int m0) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int K = p.K, G = K >> 6;
  uint8_t* ring = smem_raw + (size_t)(threadIdx.x >> 5) * kRing * kChunkBytes;   // this warp's chunk slots
  float* red = reinterpret_cast<float*>(smem_raw + (size_t)kWarps * kRing * kChunkBytes);   // [kPairs][2][MT][32][4]
  float* xsum = red + (size_t)kPairs * 2 * MT * 32 * 4;                    // [G][8 MT]
  uint64_t* bars = reinterpret_cast<uint64_t*>(xsum + (size_t)G * 8 * MT) + (threadIdx.x >> 5) * kRing;
  uint8_t* xs_smem = smem_raw + (smem_fixed<MT>(G) + 15) / 16 * 16;      // [8 MT][xs_stride] (XS)
  int dummy_abort = 0;
  const volatile int* no_abort = &dummy_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int ntiles = (p.N + kRows - 1) / kRows;
  const int pair = warp >> 1, half = warp & 1;
  const int gpair = (int)blockIdx.x * kPairs + pair, npairs = (int)gridDim.x * kPairs;
  const int my_tiles = gpair < ntiles ? (ntiles - gpair + npairs - 1) / npairs : 0;
  const int gb = half * G / 2, ge = (half + 1) * G / 2;             // this warp's groups in every tile
  const int ng = ge - gb, nchunks = (ng + kChunk - 1) / kChunk;

  // Chunk i of this warp's sequence = (tile i / nchunks, chunk i % nchunks): up to
  // kChunk groups, which are contiguous in the packed layout, so lane 0 moves
  // them with one bulk copy into ring slot i % kRing, completing that slot's
  // mbarrier.  (Issued one by one from each of the 32 lanes, the copies made
  // the kernel bound by instruction issue rather than by the weight stream.)
  const int nseq = my_tiles * nchunks;
  if (lane == 0) {
    for (int s = 0; s < kRing; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  auto issue_chunk = [&](int i) {
    if (i < nseq && lane == 0) {
      const int lt = i / nchunks, c = i - lt * nchunks;
      const size_t tile = (size_t)gpair + (size_t)lt * npairs;
      const uint8_t* src = p.wt + (tile * G + gb + (size_t)c * kChunk) * kGroupBytes;
      const uint32_t bytes = (uint32_t)min(kChunk, ng - c * kChunk) * kGroupBytes;
      uint64_t* bar = &bars[i % kRing];
      mbar_arrive_expect_tx(bar, bytes);
      bulk_load(ring + (size_t)(i % kRing) * kChunkBytes, src, bytes, bar);
    }
  };
  // Activation sums per (group, column).  Each thread's first group of X is
  // requested before the first weight chunks, so that it does not queue behind
  // them; the sums are formed while the chunks are in flight.
  auto group_sum = [&](const uint4 (&u)[8]) {
    float sum = 0.f;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const uint32_t w[4] = {u[v].x, u[v].y, u[v].z, u[v].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) sum += __uint_as_float(w[e] << 16) + __uint_as_float(w[e] & 0xFFFF0000u);
    }
    return sum;
  };
  auto load_group = [&](int i, uint4 (&u)[8]) {
    const int gi = i / (8 * MT), m = m0 + i % (8 * MT);
    if (m < p.M) {
      const uint4* xs = reinterpret_cast<const uint4*>(p.x + (size_t)m * K + 64 * (size_t)gi);
#pragma unroll
      for (int v = 0; v < 8; ++v) u[v] = __ldg(xs + v);
    } else {
#pragma unroll
      for (int v = 0; v < 8; ++v) u[v] = make_uint4(0u, 0u, 0u, 0u);
    }
  };
  if (XS) {
    // the pass's activation rows into shared memory (zeros past M), then the
    // group sums from there.  Each thread's loads (eight at a time) go out
    // before the weight copies, which would otherwise put them behind tens of
    // megabytes of weights; the copies then fly while the rows are stored.
    const int cpr = K / 8;                                          // 16-byte pieces per row
    const int total = 8 * MT * cpr;
    uint4 v[8];
    auto load_batch = [&](int base) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = base + u * kThreads;
        const int r = i / cpr, c = i - r * cpr;
        v[u] = (i < total && m0 + r < p.M) ? __ldg(reinterpret_cast<const uint4*>(p.x + (size_t)(m0 + r) * K) + c)
                                           : make_uint4(0u, 0u, 0u, 0u);
      }
    };
    auto store_batch = [&](int base) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = base + u * kThreads;
        const int r = i / cpr, c = i - r * cpr;
        if (i < total) *reinterpret_cast<uint4*>(xs_smem + (size_t)r * xs_stride(G) + (size_t)c * 16) = v[u];
      }
    };
    load_batch(threadIdx.x);
    // every warp, whatever its share of X: the first chunk now, the rest of
    // the ring once the rows are stored, so that the first chunks of all warps
    // are not held up behind everyone's later ones
    issue_chunk(0);
    store_batch(threadIdx.x);
    for (int base = threadIdx.x + 8 * kThreads; base < total; base += 8 * kThreads) {
      load_batch(base);
      store_batch(base);
    }
#pragma unroll
    for (int i = 1; i < kRing; ++i) issue_chunk(i);
    __syncthreads();
    for (int i = threadIdx.x; i < G * 8 * MT; i += kThreads) {
      const int gi = i / (8 * MT), r = i % (8 * MT);
      uint4 u[8];
#pragma unroll
      for (int v = 0; v < 8; ++v) u[v] = lds128(xs_smem + (size_t)r * xs_stride(G) + (size_t)gi * 128 + v * 16);
      xsum[i] = group_sum(u);
    }
  } else {
    uint4 u0[8];
    const bool first = (int)threadIdx.x < G * 8 * MT;
    if (first) load_group(threadIdx.x, u0);
#pragma unroll
    for (int i = 0; i < kRing; ++i) issue_chunk(i);
    if (first) xsum[threadIdx.x] = group_sum(u0);
    for (int i = threadIdx.x + kThreads; i < G * 8 * MT; i += kThreads) {
      uint4 u[8];
      load_group(i, u);
      xsum[i] = group_sum(u);
    }
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
      if (XS) {
        const uint8_t* xp = xs_smem + (size_t)(8 * t + g) * xs_stride(G) + (size_t)gi * 128 + q * 32;
        const uint4 a = lds128(xp), b = lds128(xp + 16);
        P[t][0] = a.x; P[t][1] = a.y; P[t][2] = a.z; P[t][3] = a.w;
        P[t][4] = b.x; P[t][5] = b.y; P[t][6] = b.z; P[t][7] = b.w;
      } else if (xv[t]) {
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

  bool ok = true;
  for (int lt = 0; lt < my_tiles; ++lt) {
    const int tile = gpair + lt * npairs;
    float acc[MT][4];
#pragma unroll
    for (int t = 0; t < MT; ++t)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[t][j] = 0.f;
    for (int c = 0; c < nchunks; ++c) {
      const int i = lt * nchunks + c;
      // chunk i has landed (bounded wait: a copy that never completes ends the
      // kernel with the error word set instead of hanging it)
      if (!ok || !__all_sync(0xffffffffu, mbar_wait(&bars[i % kRing], (uint32_t)(i / kRing) & 1u, no_abort,
                                                     p.budget_ns))) {
        // the warp stops computing but still meets its partner at the
        // reduction barrier below, so neither warp of the pair is left waiting
        if (ok && lane == 0) atomicExch(p.err, 1);
        ok = false;
        break;
      }
      const uint8_t* slot = ring + (size_t)(i % kRing) * kChunkBytes;
      const int n = min(kChunk, ng - c * kChunk);
#pragma unroll
      for (int j = 0; j < kChunk; ++j) {
        if (j < n) {
          const int gi = gb + c * kChunk + j;
          uint32_t P[MT][8];
          load_x(gi, P);
          const uint4 cw = lds128(slot + j * kGroupBytes + lane * 16);
          const uint32_t swj = lds32(slot + j * kGroupBytes + 512 + g * 4);
          // the four MMA steps of a group accumulate into one fragment: with
          // sixteen warps per SM the chain's latency is hidden by the other
          // warps, and the kernel is bound by instruction issue, so fewer
          // instructions per group is what counts
          float pst[MT][4];
#pragma unroll
          for (int t = 0; t < MT; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) pst[t][e] = 0.f;
#pragma unroll
          for (int st = 0; st < 4; ++st) {
            // MMA step st: positions (2q, 2q+1) <- codes 4st, 4st+1 and (2q+8, 2q+9) <- 4st+2, 4st+3
            // of this thread's 16; those are pairs 2(st&1) and 2(st&1)+1 of word st>>1.
            const uint32_t wa = (st < 2) ? cw.x : cw.y;   // row g
            const uint32_t wb = (st < 2) ? cw.z : cw.w;   // row g + 8
            const int sh = 8 * (st & 1);
            const uint32_t a[4] = {codes_pair(wa >> sh), codes_pair(wb >> sh), codes_pair(wa >> (sh + 4)),
                                   codes_pair(wb >> (sh + 4))};
#pragma unroll
            for (int t = 0; t < MT; ++t) mma_bf16_16816(pst[t], a, P[t][2 * st], P[t][2 * st + 1]);
          }
          const float s0 = __uint_as_float(swj << 16), s1 = __uint_as_float(swj & 0xFFFF0000u);
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            // minus 136 * sum(x): the biased codes (c + 136) give sum(x c)
            const float2 xs = lds64f(&xsum[gi * 8 * MT + 8 * t + 2 * q]);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              acc[t][e] = fmaf((e & 2) ? s1 : s0, pst[t][e] - 136.f * ((e & 1) ? xs.y : xs.x), acc[t][e]);
          }
        }
      }
      // every lane is done with the slot before the copy engine refills it
      fence_async_shared();
      __syncwarp();
      issue_chunk(i + kRing);
    }
    // the pair's split-K reduction (double-buffered by tile parity): the second
    // warp hands its partials over, the first adds and stores; fragment element
    // e is (row g + 8 (e>>1), column 2q + (e&1)) of activation tile t
    float* r = red + ((size_t)pair * 2 + (lt & 1)) * MT * 32 * 4;
    if (half == 1) {
#pragma unroll
      for (int t = 0; t < MT; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) r[(t * 32 + lane) * 4 + e] = acc[t][e];
    }
    named_barrier(1 + pair, 64);
    if (half == 0) {
#pragma unroll
      for (int t = 0; t < MT; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int n = tile * kRows + g + ((e & 2) ? 8 : 0);
          const int m = m0 + 8 * t + 2 * q + (e & 1);
          const float v = acc[t][e] + r[(t * 32 + lane) * 4 + e];
          if (ok && n < p.N && m < p.M) p.y[(size_t)m * p.N + n] = __float2bfloat16_rn(v + p.bias[n]);
        }
    }
  }
}

}  // namespace

bool w4a16_supported(int K) { return smem_bytes<2, false>(K / 64) <= (size_t)kSmemBudget; }

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

// Grid size (one CTA per SM), configured once per device and shared-memory size.
template <int MT, bool XS>
cudaError_t grid_size(size_t smem, int ntiles, int* grid) {
  struct Entry {
    size_t smem = 0;
    int sms = 0;
  };
  static Entry cache[64];
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  Entry& c = cache[dev];
  if (c.smem < smem) {
    if ((e = cudaFuncSetAttribute(w4a16_kernel<MT, XS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
        cudaSuccess)
      return e;
    if ((e = cudaDeviceGetAttribute(&c.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    c.smem = smem;
  }
  *grid = std::min((ntiles + kPairs - 1) / kPairs, c.sms);
  return cudaSuccess;
}

template <int MT, bool XS>
cudaError_t launch_pass_t(const W4A16Params& p, int m0, cudaStream_t stream) {
  const int ntiles = (p.N + kRows - 1) / kRows;
  const size_t smem = smem_bytes<MT, XS>(p.K / 64);
  int grid = 0;
  cudaError_t e = grid_size<MT, XS>(smem, ntiles, &grid);
  if (e != cudaSuccess) return e;
  w4a16_kernel<MT, XS><<<grid, kThreads, smem, stream>>>(p, m0);
  return cudaGetLastError();
}

template <int MT>
cudaError_t launch_pass(const W4A16Params& p, int m0, cudaStream_t stream) {
  // activations staged in shared memory whenever they fit beside the rings
  return smem_bytes<MT, true>(p.K / 64) <= (size_t)kSmemBudget ? launch_pass_t<MT, true>(p, m0, stream)
                                                                : launch_pass_t<MT, false>(p, m0, stream);
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
