// Offline preparation of an SVDQuant W4A4 layer on the host.
//
// SOTA-314 practice page, "Do this": smooth the activation outliers into the
// weights, compute the SVD of the smoothed weight W_hat, keep the top r
// singular directions in 16 bits and quantize only the residual
// R = W_hat - L1 L2 (rank 32 at 4 bits; INT4 groups of 64 with 16-bit scales,
// NVFP4 groups of 16 with FP8 scales).  NOTE-257 note page, "Key results":
// L1 = U Sigma[:, :r], L2 = V^T[:r, :]; Eckart-Young makes the truncated SVD the
// optimal rank-r reduction.
//
// Choices where the pages are silent (all documented for users of the ABI):
//  * lam_k = max|Xc[:,k]|^alpha / max|W[k,:]|^(1-alpha); alpha = 0.5 is computed
//    as fp32(sqrt(ax)) / fp32(sqrt(aw)) in float32; a zero maximum gives lam = 1.
//  * the down factor carries 1/lam: L1d = bf16(diag(1/lam) L1), L2b = bf16(L2),
//    and the residual subtracts that stored branch: R = fp32(W_hat - diag(lam) L1d L2b).
//  * NVFP4 tensor scales are powers of two: g_w = 2^ceil(log2(amax|R| / 2688)),
//    g_x = 2^ceil(log2(4 amax|fp32(Xc / lam)| / 2688)) from the calibration batch.
//  * RTN = round to nearest, ties to even, saturating.
//
// The truncated SVD is a block subspace iteration in float64 (block r + 32,
// Gaussian start, re-orthonormalised every half step) with a Rayleigh-Ritz
// extraction; it stops when the captured energy sum_{i<r} sigma_i^2 stops
// changing.  On a slowly converging (flat) spectrum it steps on the Gram
// matrix of the smaller side instead and returns to W_hat for the extraction.
// Every reduction adds its partial sums in a fixed order, so the prepared
// bytes are the same for any number of host threads.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <memory>
#include <new>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif
#if defined(__AVX2__) && defined(__FMA__)
#include <immintrin.h>
#endif

#include "svdq_internal.h"

namespace svdq {

// ------------------------------------------------------------------ formats

float bf16_to_float(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

uint16_t bf16_from_double(double x) {
  if (x == 0.0) return std::signbit(x) ? 0x8000 : 0x0000;
  int e;
  std::frexp(x, &e);                                   // |x| = m 2^e, m in [0.5, 1)
  const double q = std::ldexp(1.0, std::max(e - 8, -133));
  const double r = std::nearbyint(x / q) * q;          // ties to even
  const float f = (float)r;                            // exact: <= 8 significant bits
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

uint8_t e4m3_from_nonneg(float t) {
  if (!(t > 0.0f)) return 0;
  if (t >= 448.0f) return 0x7E;
  int e;
  std::frexp((double)t, &e);
  const double q = std::ldexp(1.0, std::max(e - 4, -9));
  double r = std::nearbyint((double)t / q) * q;
  if (r > 448.0) r = 448.0;
  if (r == 0.0) return 0;
  if (r < 0.015625) return (uint8_t)(r / 0.001953125);         // subnormal, quantum 2^-9
  int re;
  const double m = std::frexp(r, &re);                          // r = m 2^re
  const int ebits = (re - 1) + 7;
  const int mbits = (int)((2.0 * m - 1.0) * 8.0);
  return (uint8_t)(ebits * 8 + mbits);
}

float e4m3_to_float(uint8_t b) {
  const int e = (b >> 3) & 0xF, m = b & 7;
  const double v = e == 0 ? m * 0.001953125 : (1.0 + m / 8.0) * std::ldexp(1.0, e - 7);
  return (float)((b & 0x80) ? -v : v);
}

uint8_t e2m1_code(float q) {
  const float a = std::fabs(q);
  uint8_t mag;
  if (a <= 0.25f) mag = 0;
  else if (a < 0.75f) mag = 1;
  else if (a <= 1.25f) mag = 2;
  else if (a < 1.75f) mag = 3;
  else if (a <= 2.5f) mag = 4;
  else if (a < 3.5f) mag = 5;
  else if (a <= 5.0f) mag = 6;
  else mag = 7;
  return (uint8_t)((std::signbit(q) ? 8 : 0) | mag);
}

int pow2_ceil_exponent(double x) {
  if (!(x > 0.0)) return 0;
  int e;
  const double m = std::frexp(x, &e);
  return m == 0.5 ? e - 1 : e;
}

// ------------------------------------------------------------------ dense helpers

namespace {

// Deterministic standard normals: splitmix64 + Box-Muller.
struct Rng {
  uint64_t s;
  explicit Rng(uint64_t seed) : s(seed) {}
  uint64_t next() {
    uint64_t z = (s += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }
  double uniform() { return ((next() >> 11) + 0.5) * (1.0 / 9007199254740992.0); }
  double normal() {
    const double u1 = uniform(), u2 = uniform();
    return std::sqrt(-2.0 * std::log(u1)) * std::cos(6.283185307179586 * u2);
  }
};

// Row blocks of a fixed size for reductions over rows: the partial sums of each
// block are added in block order, so the result does not depend on the thread
// count.
constexpr int kRowChunk = 256;

inline int row_chunks(int rows) { return (rows + kRowChunk - 1) / kRowChunk; }

// sum_r x[r] y[r] over [0, n) with four interleaved partial sums.
inline double dot4(const double* x, const double* y, int n) {
  double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
  int r = 0;
  for (; r + 4 <= n; r += 4) {
    s0 += x[r] * y[r];
    s1 += x[r + 1] * y[r + 1];
    s2 += x[r + 2] * y[r + 2];
    s3 += x[r + 3] * y[r + 3];
  }
  for (; r < n; ++r) s0 += x[r] * y[r];
  return (s0 + s1) + (s2 + s3);
}

// ---- packed float64 GEMM
//
// C[m][n] = op(A) op(B) with op(A)(i, p) = A[i * ars + p * acs] and
// op(B)(p, j) = B[p * brs + j * bcs]; C is row-major with leading dimension
// ldc.  Panels of op(A) (kMR rows) and op(B) (kNR columns) are packed per
// kKC-deep slice; a 4 x 8 register tile accumulates each slice with fused
// multiply-adds in ascending p and is then added to C, slice after slice.  Each
// element of C belongs to one thread, so the result is the same for every
// thread count.
constexpr int kMR = 4, kNR = 8, kMC = 64, kKC = 256, kNC = 1024;

inline void micro_tile(const double* ap, const double* bp, int kc, double* c) {
#if defined(__AVX2__) && defined(__FMA__)
  __m256d c00 = _mm256_setzero_pd(), c01 = _mm256_setzero_pd(), c10 = _mm256_setzero_pd(),
          c11 = _mm256_setzero_pd(), c20 = _mm256_setzero_pd(), c21 = _mm256_setzero_pd(),
          c30 = _mm256_setzero_pd(), c31 = _mm256_setzero_pd();
  for (int p = 0; p < kc; ++p) {
    const __m256d b0 = _mm256_loadu_pd(bp + kNR * p), b1 = _mm256_loadu_pd(bp + kNR * p + 4);
    __m256d a = _mm256_broadcast_sd(ap + kMR * p);
    c00 = _mm256_fmadd_pd(a, b0, c00);
    c01 = _mm256_fmadd_pd(a, b1, c01);
    a = _mm256_broadcast_sd(ap + kMR * p + 1);
    c10 = _mm256_fmadd_pd(a, b0, c10);
    c11 = _mm256_fmadd_pd(a, b1, c11);
    a = _mm256_broadcast_sd(ap + kMR * p + 2);
    c20 = _mm256_fmadd_pd(a, b0, c20);
    c21 = _mm256_fmadd_pd(a, b1, c21);
    a = _mm256_broadcast_sd(ap + kMR * p + 3);
    c30 = _mm256_fmadd_pd(a, b0, c30);
    c31 = _mm256_fmadd_pd(a, b1, c31);
  }
  _mm256_storeu_pd(c, c00);
  _mm256_storeu_pd(c + 4, c01);
  _mm256_storeu_pd(c + 8, c10);
  _mm256_storeu_pd(c + 12, c11);
  _mm256_storeu_pd(c + 16, c20);
  _mm256_storeu_pd(c + 20, c21);
  _mm256_storeu_pd(c + 24, c30);
  _mm256_storeu_pd(c + 28, c31);
#else
  for (int i = 0; i < kMR * kNR; ++i) c[i] = 0.0;
  for (int p = 0; p < kc; ++p)
    for (int i = 0; i < kMR; ++i)
      for (int j = 0; j < kNR; ++j) c[i * kNR + j] = std::fma(ap[kMR * p + i], bp[kNR * p + j], c[i * kNR + j]);
#endif
}

// Pack op(A)[i0, i0+mc) x [p0, p0+kc) into kMR-row micro-panels Ap[ip][p][kMR]
// (zero rows past mc).
void pack_a(const double* A, size_t ars, size_t acs, int i0, int mc, int p0, int kc, double* Ap) {
  const int mp = (mc + kMR - 1) / kMR;
  for (int ip = 0; ip < mp; ++ip)
    for (int p = 0; p < kc; ++p)
      for (int ii = 0; ii < kMR; ++ii) {
        const int i = ip * kMR + ii;
        Ap[((size_t)ip * kc + p) * kMR + ii] = i < mc ? A[(size_t)(i0 + i) * ars + (size_t)(p0 + p) * acs] : 0.0;
      }
}

// Pack micro-panels [jp0, jp1) of op(B)[p0, p0+kc) x [j0, j0+nc) into
// Bp[jp][p][kNR] (zero columns past nc).
void pack_b(const double* B, size_t brs, size_t bcs, int p0, int kc, int j0, int nc, int jp0, int jp1,
            double* Bp) {
  for (int jp = jp0; jp < jp1; ++jp) {
    double* dst = Bp + (size_t)jp * kc * kNR;
    for (int p = 0; p < kc; ++p)
      for (int jj = 0; jj < kNR; ++jj) {
        const int j = jp * kNR + jj;
        dst[(size_t)p * kNR + jj] = j < nc ? B[(size_t)(p0 + p) * brs + (size_t)(j0 + j) * bcs] : 0.0;
      }
  }
}

// C[0, mc) x [0, nc) += (or -=) Ap Bp over one packed slice of depth kc.
void slice_tiles(const double* Ap, int mc, const double* Bp, int nc, int kc, bool subtract, double* C,
                 size_t ldc) {
  double tile[kMR * kNR];
  const int mp = (mc + kMR - 1) / kMR, np = (nc + kNR - 1) / kNR;
  for (int jp = 0; jp < np; ++jp)
    for (int ip = 0; ip < mp; ++ip) {
      micro_tile(Ap + (size_t)ip * kc * kMR, Bp + (size_t)jp * kc * kNR, kc, tile);
      const int ie = std::min(kMR, mc - ip * kMR), je = std::min(kNR, nc - jp * kNR);
      for (int ii = 0; ii < ie; ++ii) {
        double* c = C + (size_t)(ip * kMR + ii) * ldc + jp * kNR;
        if (subtract)
          for (int jj = 0; jj < je; ++jj) c[jj] -= tile[ii * kNR + jj];
        else
          for (int jj = 0; jj < je; ++jj) c[jj] += tile[ii * kNR + jj];
      }
    }
}

// C = op(A) op(B) on the calling thread alone (for use inside parallel tasks);
// with `update` set, C -= op(A) op(B) instead.  Ap and Bp are scratch.
void gemm_serial(int m, int n, int k, const double* A, size_t ars, size_t acs, const double* B, size_t brs,
                 size_t bcs, double* C, size_t ldc, bool update, std::vector<double>& Ap,
                 std::vector<double>& Bp) {
  if (!update)
    for (int i = 0; i < m; ++i) std::fill(C + (size_t)i * ldc, C + (size_t)i * ldc + n, 0.0);
  if (k <= 0 || m <= 0 || n <= 0) return;
  for (int ic = 0; ic < m; ic += kMC) {
    const int mc = std::min(kMC, m - ic);
    for (int jc = 0; jc < n; jc += kNC) {
      const int nc = std::min(kNC, n - jc);
      for (int pc = 0; pc < k; pc += kKC) {
        const int kc = std::min(kKC, k - pc);
        Ap.resize((size_t)kMC * kc);
        Bp.resize((size_t)((nc + kNR - 1) / kNR) * kc * kNR);
        pack_a(A, ars, acs, ic, mc, pc, kc, Ap.data());
        pack_b(B, brs, bcs, pc, kc, jc, nc, 0, (nc + kNR - 1) / kNR, Bp.data());
        slice_tiles(Ap.data(), mc, Bp.data(), nc, kc, update, C + (size_t)ic * ldc + jc, ldc);
      }
    }
  }
}

// C[m][n] = op(A) op(B), the row blocks of C spread over the threads.
void gemm(int m, int n, int k, const double* A, size_t ars, size_t acs, const double* B, size_t brs,
          size_t bcs, double* C, size_t ldc) {
#pragma omp parallel for schedule(static)
  for (int i = 0; i < m; ++i) std::fill(C + (size_t)i * ldc, C + (size_t)i * ldc + n, 0.0);
  if (k <= 0 || m <= 0 || n <= 0) return;
  const int npan_max = (std::min(n, kNC) + kNR - 1) / kNR;
  std::vector<double> Bp((size_t)npan_max * kKC * kNR);
  for (int jc = 0; jc < n; jc += kNC) {
    const int nc = std::min(kNC, n - jc);
    const int np = (nc + kNR - 1) / kNR;
    for (int pc = 0; pc < k; pc += kKC) {
      const int kc = std::min(kKC, k - pc);
#pragma omp parallel
      {
#pragma omp for schedule(static)
        for (int jp = 0; jp < np; ++jp) pack_b(B, brs, bcs, pc, kc, jc, nc, jp, jp + 1, Bp.data());
        std::vector<double> Ap((size_t)kMC * kc);
#pragma omp for schedule(static)
        for (int ib = 0; ib < (m + kMC - 1) / kMC; ++ib) {
          const int ic = ib * kMC, mc = std::min(kMC, m - ic);
          pack_a(A, ars, acs, ic, mc, pc, kc, Ap.data());
          slice_tiles(Ap.data(), mc, Bp.data(), nc, kc, false, C + (size_t)ic * ldc + jc, ldc);
        }
      }
    }
  }
}

// Orthonormalise the b columns of row-major X[rows][b] in place: classical
// Gram-Schmidt with one re-orthogonalisation (twice is enough), the inner
// products summed in fixed row blocks.  A column that vanishes is replaced by
// a random direction orthogonal to the previous ones.
void orthonormalize(double* X, int rows, int b, Rng& rng) {
  std::vector<double> C((size_t)rows * b);
  const int nch = row_chunks(rows);
  std::vector<double> part((size_t)nch * (b + 1)), d(b + 1);
  double n0 = 0.0, nn = 0.0;
  bool done = false;
#pragma omp parallel
  {
#pragma omp for schedule(static)
    for (int j = 0; j < b; ++j)
      for (int r = 0; r < rows; ++r) C[(size_t)j * rows + r] = X[(size_t)r * b + j];
    for (int j = 0; j < b; ++j) {
      double* cj = C.data() + (size_t)j * rows;
#pragma omp for schedule(static)
      for (int ch = 0; ch < nch; ++ch) {
        const int r0 = ch * kRowChunk, r1 = std::min(rows, r0 + kRowChunk);
        part[ch] = dot4(cj + r0, cj + r0, r1 - r0);
      }
#pragma omp single
      {
        double s = 0.0;
        for (int ch = 0; ch < nch; ++ch) s += part[ch];
        n0 = std::sqrt(s);
        done = false;
      }
      for (int attempt = 0; attempt < 4 && !done; ++attempt) {
        for (int pass = 0; pass < 2; ++pass) {              // c_j -= C_{<j} (C_{<j}^T c_j)
#pragma omp for schedule(static)
          for (int ch = 0; ch < nch; ++ch) {
            const int r0 = ch * kRowChunk, r1 = std::min(rows, r0 + kRowChunk);
            for (int i = 0; i < j; ++i)
              part[(size_t)ch * (b + 1) + i] = dot4(C.data() + (size_t)i * rows + r0, cj + r0, r1 - r0);
          }
#pragma omp single
          for (int i = 0; i < j; ++i) {
            double s = 0.0;
            for (int ch = 0; ch < nch; ++ch) s += part[(size_t)ch * (b + 1) + i];
            d[i] = s;
          }
#pragma omp for schedule(static)
          for (int ch = 0; ch < nch; ++ch) {
            const int r0 = ch * kRowChunk, r1 = std::min(rows, r0 + kRowChunk);
            for (int i = 0; i < j; ++i) {
              const double* ci = C.data() + (size_t)i * rows;
              const double di = d[i];
              for (int r = r0; r < r1; ++r) cj[r] -= di * ci[r];
            }
          }
        }
#pragma omp for schedule(static)
        for (int ch = 0; ch < nch; ++ch) {
          const int r0 = ch * kRowChunk, r1 = std::min(rows, r0 + kRowChunk);
          part[ch] = dot4(cj + r0, cj + r0, r1 - r0);
        }
#pragma omp single
        {
          double s = 0.0;
          for (int ch = 0; ch < nch; ++ch) s += part[ch];
          nn = std::sqrt(s);
          if (nn > 1e-10 * std::max(n0, 1e-300) && nn > 1e-200) {
            for (int r = 0; r < rows; ++r) cj[r] /= nn;
            done = true;
          } else {
            for (int r = 0; r < rows; ++r) cj[r] = rng.normal();
            s = 0.0;
            for (int ch = 0; ch < nch; ++ch) {
              const int r0 = ch * kRowChunk, r1 = std::min(rows, r0 + kRowChunk);
              s += dot4(cj + r0, cj + r0, r1 - r0);
            }
            n0 = std::sqrt(s);
          }
        }
      }
    }
#pragma omp for schedule(static)
    for (int r = 0; r < rows; ++r)
      for (int j = 0; j < b; ++j) X[(size_t)r * b + j] = C[(size_t)j * rows + r];
  }
}

// Symmetric eigen-decomposition of T[b][b] (cyclic Jacobi).  On return the
// eigenvalues are in w (descending) and, when `vectors` is set, the
// eigenvectors are the columns of E.  A rotation in the (p, q) plane rotates
// rows p and q, mirrors them into columns p and q, and sets the 2 x 2 block
// from the rotation's tangent t: T'pp = Tpp - t Tpq, T'qq = Tqq + t Tpq,
// T'pq = 0.  The eigenvectors are kept as rows so that each rotation touches
// two contiguous rows.
void sym_eig(std::vector<double> T, int b, std::vector<double>& w, std::vector<double>& E, bool vectors) {
  std::vector<double> V;
  if (vectors) {
    V.assign((size_t)b * b, 0.0);
    for (int i = 0; i < b; ++i) V[(size_t)i * b + i] = 1.0;
  }
  auto at = [&](int i, int j) -> double& { return T[(size_t)i * b + j]; };
  for (int sweep = 0; sweep < 100; ++sweep) {
    double off = 0.0, tot = 0.0;
    for (int i = 0; i < b; ++i)
      for (int j = 0; j < b; ++j) {
        tot += at(i, j) * at(i, j);
        if (i != j) off += at(i, j) * at(i, j);
      }
    if (off <= 1e-30 * tot || off == 0.0) break;
    for (int p = 0; p < b - 1; ++p)
      for (int q = p + 1; q < b; ++q) {
        const double apq = at(p, q);
        if (std::fabs(apq) < 1e-300) continue;
        const double theta = (at(q, q) - at(p, p)) / (2.0 * apq);
        const double t = (theta >= 0 ? 1.0 : -1.0) / (std::fabs(theta) + std::sqrt(theta * theta + 1.0));
        const double c = 1.0 / std::sqrt(t * t + 1.0), s = t * c;
        const double app = at(p, p) - t * apq, aqq = at(q, q) + t * apq;
        double* rp = &at(p, 0);
        double* rq = &at(q, 0);
        for (int k = 0; k < b; ++k) {
          const double x = rp[k], y = rq[k];
          rp[k] = c * x - s * y;
          rq[k] = s * x + c * y;
        }
        rp[p] = app;
        rq[q] = aqq;
        rp[q] = rq[p] = 0.0;
        for (int k = 0; k < b; ++k) {
          if (k == p || k == q) continue;
          at(k, p) = rp[k];
          at(k, q) = rq[k];
        }
        if (vectors) {
          double* vp = V.data() + (size_t)p * b;
          double* vq = V.data() + (size_t)q * b;
          for (int k = 0; k < b; ++k) {
            const double x = vp[k], y = vq[k];
            vp[k] = c * x - s * y;
            vq[k] = s * x + c * y;
          }
        }
      }
  }
  std::vector<int> idx(b);
  for (int i = 0; i < b; ++i) idx[i] = i;
  std::sort(idx.begin(), idx.end(), [&](int x, int y) { return at(x, x) > at(y, y); });
  w.resize(b);
  for (int c = 0; c < b; ++c) w[c] = at(idx[c], idx[c]);
  if (vectors) {
    E.assign((size_t)b * b, 0.0);
    for (int c = 0; c < b; ++c)
      for (int k = 0; k < b; ++k) E[(size_t)k * b + c] = V[(size_t)idx[c] * b + k];
  }
}

// G[b][b] = X^T Y for row-major X[rows][b] and Y[rows][b], summed in fixed row
// blocks.
void gram_xy(const double* X, const double* Y, int rows, int b, std::vector<double>& G) {
  const int nch = row_chunks(rows);
  std::vector<double> part((size_t)nch * b * b, 0.0);
#pragma omp parallel for schedule(static)
  for (int ch = 0; ch < nch; ++ch) {
    double* g = part.data() + (size_t)ch * b * b;
    const int r0 = ch * kRowChunk, r1 = std::min(rows, r0 + kRowChunk);
    for (int r = r0; r < r1; ++r) {
      const double* x = X + (size_t)r * b;
      const double* y = Y + (size_t)r * b;
      for (int i = 0; i < b; ++i) {
        const double xi = x[i];
        for (int j = 0; j < b; ++j) g[(size_t)i * b + j] += xi * y[j];
      }
    }
  }
  G.assign((size_t)b * b, 0.0);
  for (int ch = 0; ch < nch; ++ch)
    for (size_t i = 0; i < (size_t)b * b; ++i) G[i] += part[(size_t)ch * b * b + i];
}

// Top-r SVD of A[K][N]: L1 = U Sigma[:, :r] ([K][r]), L2 = V^T[:r, :] ([r][N]).
//
// Block subspace iteration (block b = r + 32): Q = orth(A Z), Z = orth(A^T Q),
// with the Ritz values of B B^T (B = Q^T A) after every step; it stops when
// the captured energy sum_{i<r} sigma_i^2 stops changing.  The energy settles
// like (sigma_{b+1} / sigma_r)^(2t), which is slow when the spectrum is flat
// around sigma_r.  When the observed rate says the remaining steps on A cost
// more than forming the Gram matrix of the smaller side (G = A^T A or A A^T,
// min(K, N)^2 entries) and stepping on it (2 min(K,N)^2 b flops a step against
// 4 K N b), the iteration moves to G.  The last step and the extraction run on
// A itself, so the factors keep the accuracy of the plain iteration.
svdq_status truncated_svd(const std::vector<double>& A, int K, int N, int r,
                          std::vector<double>& L1, std::vector<double>& L2,
                          std::vector<double>& sigma, int& iters, double& tail) {
  constexpr double kTol = 1e-13;                        // relative change of the energy
  constexpr int kMaxSteps = 300, kMaxGramSteps = 1000;
  const int b = std::min(std::min(r + 32, K), N);
  const int re = std::min(r, b);                        // directions beyond rank(A) stay zero
  Rng rng(0x5EED5EEDull);
  std::vector<double> Z((size_t)N * b), Zraw((size_t)N * b), Q((size_t)K * b), T, w, E;
  for (auto& z : Z) z = rng.normal();
  orthonormalize(Z.data(), N, b, rng);
  const bool exact_block = (b == std::min(K, N));      // the block spans the whole range
  auto top_energy = [&]() {
    double e = 0.0;
    for (int i = 0; i < re; ++i) e += std::max(w[i], 0.0);
    return e;
  };
  auto step_on_A = [&](bool from_Z) {
    if (from_Z) {
      gemm(K, b, N, A.data(), N, 1, Z.data(), b, 1, Q.data(), b);    // Q <- A Z
      orthonormalize(Q.data(), K, b, rng);
    }
    gemm(N, b, K, A.data(), 1, N, Q.data(), b, 1, Zraw.data(), b);   // Zraw <- A^T Q (= B^T)
    gram_xy(Zraw.data(), Zraw.data(), N, b, T);                       // B B^T
    sym_eig(T, b, w, E, false);
  };
  const int ns = std::min(K, N);
  const double cost_a = 4.0 * K * N * b, cost_g = 2.0 * ns * ns * b, cost_form = 2.0 * ns * ns * std::max(K, N);
  double prev = -1.0, delta_prev = -1.0, energy = 0.0;
  bool converged = false, to_gram = false;
  int steps = 0;
  for (int it = 0; it < kMaxSteps; ++it) {
    step_on_A(true);
    ++steps;
    energy = top_energy();
    if (exact_block || (it >= 3 && std::fabs(energy - prev) <= kTol * energy)) {
      converged = true;
      break;
    }
    const double delta = std::fabs(energy - prev);
    if (it >= 4 && delta_prev > 0.0) {
      const double rho = delta / delta_prev;
      const double left = (rho > 0.0 && rho < 1.0) ? std::log(kTol * energy / delta) / std::log(rho) : 1e30;
      to_gram = left * (cost_a - cost_g) > cost_form;
    }
    delta_prev = it >= 1 ? delta : -1.0;
    prev = energy;
    if (to_gram) break;
    Z = Zraw;
    orthonormalize(Z.data(), N, b, rng);
  }
  if (to_gram) {
    // Gram of the smaller side, started from the basis on that side
    const bool right = N <= K;
    std::vector<double> G((size_t)ns * ns), S, Y((size_t)ns * b);
    if (right) {
      gemm(N, N, K, A.data(), 1, N, A.data(), N, 1, G.data(), N);   // A^T A
      S = Zraw;
    } else {
      gemm(K, K, N, A.data(), N, 1, A.data(), 1, N, G.data(), K);   // A A^T
      S = Q;
    }
    orthonormalize(S.data(), ns, b, rng);
    double gprev = -1.0;
    for (int it = 0; it < kMaxGramSteps; ++it) {
      gemm(ns, b, ns, G.data(), ns, 1, S.data(), b, 1, Y.data(), b);   // Y <- G S
      ++steps;
      gram_xy(S.data(), Y.data(), ns, b, T);                          // S^T G S
      sym_eig(T, b, w, E, false);
      energy = top_energy();
      if (it >= 1 && std::fabs(energy - gprev) <= kTol * energy) {
        converged = true;
        break;
      }
      prev = gprev = energy;
      S = Y;
      orthonormalize(S.data(), ns, b, rng);
    }
    // last step and Rayleigh-Ritz on A
    if (right) {
      Z = Y;
      orthonormalize(Z.data(), N, b, rng);
      step_on_A(true);
    } else {
      Q = Y;
      orthonormalize(Q.data(), K, b, rng);
      step_on_A(false);
    }
    ++steps;
    energy = top_energy();
  }
  iters = steps;
  if (!converged && std::fabs(energy - prev) > 1e-8 * std::max(energy, 1e-300))
    return SVDQ_ENOCONVERGE;
  sym_eig(T, b, w, E, true);
  const std::vector<double>& Zf = Zraw;
  // Rayleigh-Ritz: B = Q^T A = Z^T, B B^T = E diag(w) E^T.
  // U = Q E, sigma = sqrt(w), V^T rows = E^T B / sigma = (Z E)^T / sigma.
  sigma.assign(r, 0.0);
  L1.assign((size_t)K * r, 0.0);
  L2.assign((size_t)r * N, 0.0);
  for (int i = 0; i < re; ++i) sigma[i] = std::sqrt(std::max(w[i], 0.0));
#pragma omp parallel for schedule(static)
  for (int k = 0; k < K; ++k)
    for (int i = 0; i < re; ++i) {
      double u = 0.0;
      for (int j = 0; j < b; ++j) u += Q[(size_t)k * b + j] * E[(size_t)j * b + i];
      L1[(size_t)k * r + i] = u * sigma[i];
    }
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n)
    for (int i = 0; i < re; ++i) {
      double v = 0.0;
      for (int j = 0; j < b; ++j) v += Zf[(size_t)n * b + j] * E[(size_t)j * b + i];
      L2[(size_t)i * N + n] = sigma[i] > 0 ? v / sigma[i] : 0.0;
    }
  const int nch = row_chunks(K);
  std::vector<double> part(nch);
#pragma omp parallel for schedule(static)
  for (int ch = 0; ch < nch; ++ch) {
    const int r0 = ch * kRowChunk, r1 = std::min(K, r0 + kRowChunk);
    const double* a = A.data() + (size_t)r0 * N;
    part[ch] = dot4(a, a, (r1 - r0) * N);
  }
  double total = 0.0;
  for (int ch = 0; ch < nch; ++ch) total += part[ch];
  double kept = 0.0;
  for (int i = 0; i < r; ++i) kept += sigma[i] * sigma[i];
  tail = total - kept;
  return SVDQ_OK;
}

// NVFP4 quantization of one group of 16 float32 values (same steps as the
// kernel): a = max|v|, t = fp32(a c), s = E4M3(t), inv = fp32(1/(s g)),
// code = E2M1(fp32(v inv)).  `codes` receives 16 nibbles.
uint8_t nvfp4_group(const float* v, float c, float g, uint8_t* codes) {
  float a = 0.0f;
  for (int i = 0; i < 16; ++i) a = std::max(a, std::fabs(v[i]));
  volatile float t = a * c;
  const uint8_t sb = e4m3_from_nonneg(t);
  const float s = e4m3_to_float(sb);
  if (s == 0.0f) {
    for (int i = 0; i < 16; ++i) codes[i] = 0;
    return sb;
  }
  volatile float sg = s * g;
  volatile float inv = 1.0f / sg;
  for (int i = 0; i < 16; ++i) {
    volatile float q = v[i] * inv;
    codes[i] = e2m1_code(q);
  }
  return sb;
}

// INT4 quantization of one group of 64: s = bf16(fp32(a fp32(1/7))),
// code = clamp(rint(fp32(v fp32(1/s))), -7, 7).
uint16_t int4_group(const float* v, int8_t* codes) {
  float a = 0.0f;
  for (int i = 0; i < 64; ++i) a = std::max(a, std::fabs(v[i]));
  const float seventh = 1.0f / 7.0f;
  volatile float t = a * seventh;
  const uint16_t sb = bf16_from_double((double)t);
  const float s = bf16_to_float(sb);
  if (s == 0.0f) {
    for (int i = 0; i < 64; ++i) codes[i] = 0;
    return sb;
  }
  volatile float inv = 1.0f / s;
  for (int i = 0; i < 64; ++i) {
    volatile float q = v[i] * inv;
    float rq = std::nearbyint((float)q);
    rq = std::min(7.0f, std::max(-7.0f, rq));
    codes[i] = (int8_t)rq;
  }
  return sb;
}

// ------------------------------------------------------------------ GPTQ
//
// SOTA-314 practice page, "Do this": the residual is quantized with GPTQ rather
// than round-to-nearest.  The published algorithm (Frantar et al. 2022) in its
// column-by-column form; its lazy block updates only reorder the same
// arithmetic.  The loss of output column n is ||X_hat (r_n - q_n)||^2, so one
// Hessian H = X_hat^T X_hat serves every column.

constexpr double kGptqDamp = 0.01;          // fraction of the mean diagonal added to H

// Damped Hessian of the smoothed calibration activations X_hat = fp32(Xc * inv_lam).
void gptq_hessian(const uint16_t* calib, int M, int K, const std::vector<float>& inv_lam,
                  std::vector<double>& H) {
  std::vector<double> xt((size_t)K * M);    // X_hat^T, [K][M]
#pragma omp parallel for schedule(static)
  for (int k = 0; k < K; ++k)
    for (int m = 0; m < M; ++m) {
      volatile float v = bf16_to_float(calib[(size_t)m * K + k]) * inv_lam[k];
      xt[(size_t)k * M + m] = (double)(float)v;
    }
  H.assign((size_t)K * K, 0.0);
  constexpr int T = 32;
  const int nb = (K + T - 1) / T;
  std::vector<int> ti, tj;
  for (int i = 0; i < nb; ++i)
    for (int j = i; j < nb; ++j) {
      ti.push_back(i);
      tj.push_back(j);
    }
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < (int)ti.size(); ++t) {
    const int i0 = ti[t] * T, j0 = tj[t] * T;
    for (int i = i0; i < std::min(K, i0 + T); ++i) {
      const double* xi = xt.data() + (size_t)i * M;
      for (int j = std::max(i, j0); j < std::min(K, j0 + T); ++j) {
        const double* xj = xt.data() + (size_t)j * M;
        double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
        int m = 0;
        for (; m + 4 <= M; m += 4) {
          s0 += xi[m] * xj[m];
          s1 += xi[m + 1] * xj[m + 1];
          s2 += xi[m + 2] * xj[m + 2];
          s3 += xi[m + 3] * xj[m + 3];
        }
        for (; m < M; ++m) s0 += xi[m] * xj[m];
        H[(size_t)i * K + j] = H[(size_t)j * K + i] = (s0 + s1) + (s2 + s3);
      }
    }
  }
  double tr = 0.0;
  for (int k = 0; k < K; ++k) {
    double& d = H[(size_t)k * K + k];
    if (d == 0.0) d = 1.0;                  // a channel the calibration never fires
    tr += d;
  }
  const double add = kGptqDamp * (tr / K);
  for (int k = 0; k < K; ++k) H[(size_t)k * K + k] += add;
}

// The GPTQ factor U (upper triangular, positive diagonal, H^-1 = U^T U) of the
// damped Hessian H ([K][K], symmetric positive definite), blocked for the cache
// and the cores.  With J the order reversal, P = J H J = L L^T (lower
// Cholesky), so H = T T^T with T = J L J upper and U = T^-1 = J L^-1 J.
//   * L: right-looking blocked Cholesky of P in place (the diagonal block by
//     the textbook loop, the panel by a triangular solve, the trailing lower
//     triangle by packed block products, one block pair per task);
//   * X = L^-1: one block column per task; each block row takes the product
//     of L's row block with the rows of X above it (a packed product), then a
//     forward substitution through L's diagonal block.
// false if a pivot is not positive.
constexpr int kFactorBlock = 128;

bool gptq_factor(const std::vector<double>& H, int K, std::vector<double>& U) {
  const int B = kFactorBlock;
  const int nb = (K + B - 1) / B;
  std::vector<double> P((size_t)K * K);
  // P = J H J (the lower triangle is what the factorization uses)
#pragma omp parallel for schedule(static)
  for (int i = 0; i < K; ++i)
    for (int j = 0; j < K; ++j) P[(size_t)i * K + j] = H[(size_t)(K - 1 - i) * K + (K - 1 - j)];
  auto at = [&](int i, int j) -> double& { return P[(size_t)i * K + j]; };
  bool ok = true;
  for (int kb = 0; kb < nb && ok; ++kb) {
    const int k0 = kb * B, k1 = std::min(K, k0 + B), w = k1 - k0;
    // diagonal block
    for (int j = k0; j < k1 && ok; ++j) {
      double d = at(j, j);
      for (int k = k0; k < j; ++k) d -= at(j, k) * at(j, k);
      if (!(d > 0.0) || !std::isfinite(d)) {
        ok = false;
        break;
      }
      const double ljj = std::sqrt(d);
      at(j, j) = ljj;
      for (int i = j + 1; i < k1; ++i) {
        double v = at(i, j);
        for (int k = k0; k < j; ++k) v -= at(i, k) * at(j, k);
        at(i, j) = v / ljj;
      }
    }
    if (!ok) break;
    // panel: rows below the block, L[i, k0:k1] = P[i, k0:k1] L[k0:k1, k0:k1]^-T
#pragma omp parallel for schedule(static)
    for (int i = k1; i < K; ++i)
      for (int j = k0; j < k1; ++j) {
        double v = at(i, j);
        for (int k = k0; k < j; ++k) v -= at(i, k) * at(j, k);
        at(i, j) = v / at(j, j);
      }
    // trailing lower triangle: P[I, J] -= L[I, k0:k1] L[J, k0:k1]^T for block
    // rows I and block columns J <= I (a diagonal block is updated whole; its
    // upper part is never read)
    const int rem = nb - kb - 1;
    if (rem > 0) {
#pragma omp parallel
      {
        std::vector<double> Ap, Bp;
#pragma omp for schedule(dynamic, 1)
        for (int t = 0; t < rem * (rem + 1) / 2; ++t) {
          int ib = 0;
          while ((ib + 1) * (ib + 2) / 2 <= t) ++ib;     // block row ib, block column jb <= ib
          const int jb = t - ib * (ib + 1) / 2;
          const int i0 = k1 + ib * B, i1 = std::min(K, i0 + B);
          const int j0 = k1 + jb * B, j1 = std::min(K, j0 + B);
          gemm_serial(i1 - i0, j1 - j0, w, &P[(size_t)i0 * K + k0], K, 1, &P[(size_t)j0 * K + k0], 1, K,
                      &P[(size_t)i0 * K + j0], K, true, Ap, Bp);
        }
      }
    }
  }
  if (!ok) return false;
  U.assign((size_t)K * K, 0.0);
#pragma omp parallel
  {
    std::vector<double> X, Ap, Bp;
#pragma omp for schedule(dynamic, 1)
    for (int jb = 0; jb < nb; ++jb) {
      const int j0 = jb * B, w = std::min(K, j0 + B) - j0;
      X.assign((size_t)(K - j0) * w, 0.0);               // rows j0.., row-major [K - j0][w]
      for (int ib = jb; ib < nb; ++ib) {
        const int i0 = ib * B, i1 = std::min(K, i0 + B);
        double* xi0 = &X[(size_t)(i0 - j0) * w];
        // S = L[i0:i1, j0:i0] X[j0:i0, :], kept negated in the rows' slots
        if (i0 > j0)
          gemm_serial(i1 - i0, w, i0 - j0, &P[(size_t)i0 * K + j0], K, 1, X.data(), w, 1, xi0, w, true, Ap, Bp);
        for (int i = i0; i < i1; ++i) {
          double* xr = &X[(size_t)(i - j0) * w];
          if (i - j0 < w) xr[i - j0] += 1.0;             // the identity's column
          const double* li = &P[(size_t)i * K];
          for (int k = i0; k < i; ++k) {
            const double lik = li[k];
            const double* xk = &X[(size_t)(k - j0) * w];
            for (int c = 0; c < w; ++c) xr[c] -= lik * xk[c];
          }
          for (int c = 0; c < w; ++c) xr[c] = xr[c] / li[i];
          double* urow = &U[(size_t)(K - 1 - i) * K];
          for (int c = 0; c < w; ++c) urow[K - 1 - (j0 + c)] = xr[c];
        }
      }
    }
  }
  return true;
}

// Magnitude of a 3-bit E2M1 code.
double e2m1_magnitude(uint8_t c) {
  static const double grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  return grid[c & 7];
}

// GPTQ over the columns of the residual R [K][N] with factor U; writes codes and
// scales into P exactly where round-to-nearest writes them.  Columns are
// independent given U; each thread carries kNB of them through the K steps.
void gptq_columns(const std::vector<float>& R, int K, int N, const std::vector<double>& U, bool nvfp4,
                  HostPrep& P) {
  constexpr int kNB = 16;
  const int G = nvfp4 ? 16 : 64;
  const float g = nvfp4 ? (float)std::ldexp(1.0, P.g_w_exp) : 1.0f;
  const float cc = nvfp4 ? (float)std::ldexp((double)(1.0f / 6.0f), -P.g_w_exp) : 0.0f;
  const double gd = (double)g;
  float amax_all = 0.0f;
#pragma omp parallel for schedule(dynamic, 1) reduction(max : amax_all)
  for (int b = 0; b < (N + kNB - 1) / kNB; ++b) {
    const int n0 = b * kNB, nc = std::min(kNB, N - n0);
    std::vector<double> w((size_t)K * kNB, 0.0);      // working values, [K][kNB]
    for (int k = 0; k < K; ++k)
      for (int c = 0; c < nc; ++c) w[(size_t)k * kNB + c] = (double)R[(size_t)k * N + n0 + c];
    float inv[kNB], sc[kNB];
    double err[kNB];
    for (int k = 0; k < K; ++k) {
      if (k % G == 0) {
        for (int c = 0; c < nc; ++c) {
          float a = 0.0f;
          for (int i = 0; i < G; ++i) a = std::max(a, std::fabs((float)w[(size_t)(k + i) * kNB + c]));
          amax_all = std::max(amax_all, a);
          const int n = n0 + c;
          if (nvfp4) {
            volatile float t = a * cc;
            const uint8_t sb = e4m3_from_nonneg(t);
            sc[c] = e4m3_to_float(sb);
            P.w_scales_e4m3[(size_t)n * (K / 16) + k / 16] = sb;
            if (sc[c] == 0.0f) {
              inv[c] = 0.0f;
            } else {
              volatile float sg = sc[c] * g;
              volatile float iv = 1.0f / sg;
              inv[c] = iv;
            }
          } else {
            const float seventh = 1.0f / 7.0f;
            volatile float t = a * seventh;
            const uint16_t sb = bf16_from_double((double)t);
            sc[c] = bf16_to_float(sb);
            P.w_scales_bf16[(size_t)n * (K / 64) + k / 64] = sb;
            if (sc[c] == 0.0f) {
              inv[c] = 0.0f;
            } else {
              volatile float iv = 1.0f / sc[c];
              inv[c] = iv;
            }
          }
        }
      }
      const double ukk = U[(size_t)k * K + k];
      for (int c = 0; c < nc; ++c) {
        const double wk = w[(size_t)k * kNB + c];
        const float v = (float)wk;
        uint8_t nib;
        double deq;
        if (nvfp4) {
          if (sc[c] == 0.0f) {
            nib = 0;
            deq = 0.0;
          } else {
            volatile float q = v * inv[c];
            nib = e2m1_code(q);
            const double mag = e2m1_magnitude(nib) * ((double)sc[c] * gd);
            deq = (nib & 8) ? -mag : mag;
          }
        } else {
          volatile float q = v * inv[c];
          float rq = std::nearbyint((float)q);
          rq = std::min(7.0f, std::max(-7.0f, rq));
          const int code = (int)rq;
          nib = (uint8_t)(code & 0xF);
          deq = (double)code * (double)sc[c];
        }
        uint8_t& byte = P.w_codes[(size_t)(n0 + c) * (K / 2) + k / 2];
        byte = (k & 1) ? (uint8_t)((byte & 0x0F) | (nib << 4)) : (uint8_t)((byte & 0xF0) | nib);
        err[c] = (wk - deq) / ukk;
      }
      const double* uk = U.data() + (size_t)k * K;
      for (int j = k + 1; j < K; ++j) {
        const double ukj = uk[j];
        double* wj = w.data() + (size_t)j * kNB;
        for (int c = 0; c < nc; ++c) wj[c] = wj[c] - ukj * err[c];
      }
    }
  }
  P.w_amax = amax_all;
}

}  // namespace

// ------------------------------------------------------------------ pipeline

svdq_status host_prepare(const svdq_config& cfg, int K, int N, const uint16_t* W,
                         const uint16_t* bias, const uint16_t* calib, int M_calib,
                         HostPrep& P) {
  try {
    const bool w4a16 = cfg.format == SVDQ_W4A16_INT4;
    // NaN or infinity anywhere in the inputs (all exponent bits set) would only
    // stall the iterations below: refuse it up front.
    auto finite = [](const uint16_t* p, size_t n) {
      for (size_t i = 0; i < n; ++i)
        if ((p[i] & 0x7F80u) == 0x7F80u) return false;
      return true;
    };
    if (!finite(W, (size_t)K * N) || (bias && !finite(bias, (size_t)N)) ||
        (!w4a16 && calib && !finite(calib, (size_t)M_calib * K)))
      return SVDQ_EINVAL;
    P.K = K; P.N = N; P.format = cfg.format;
    P.rank = w4a16 ? 0 : cfg.rank;
    P.alpha = cfg.alpha;
    const int r = P.rank;
    P.bias.assign(N, 0.0f);
    if (bias)
      for (int n = 0; n < N; ++n) P.bias[n] = bf16_to_float(bias[n]);

    // ---- smoothing factors (float32)
    P.lam.assign(K, 1.0f);
    P.inv_lam.assign(K, 1.0f);
    if (!w4a16) {
      std::vector<float> ax(K, 0.0f), aw(K, 0.0f);
      for (int m = 0; m < M_calib; ++m)
        for (int k = 0; k < K; ++k)
          ax[k] = std::max(ax[k], std::fabs(bf16_to_float(calib[(size_t)m * K + k])));
#pragma omp parallel for schedule(static)
      for (int k = 0; k < K; ++k) {
        float mx = 0.0f;
        for (int n = 0; n < N; ++n) mx = std::max(mx, std::fabs(bf16_to_float(W[(size_t)k * N + n])));
        aw[k] = mx;
      }
      for (int k = 0; k < K; ++k) {
        float lam;
        if (ax[k] == 0.0f || aw[k] == 0.0f) {
          lam = 1.0f;
        } else if (cfg.alpha == 0.5f) {
          volatile float sx = std::sqrt(ax[k]);
          volatile float sw = std::sqrt(aw[k]);
          lam = sx / sw;
        } else {
          lam = (float)(std::pow((double)ax[k], (double)cfg.alpha) /
                        std::pow((double)aw[k], 1.0 - (double)cfg.alpha));
        }
        P.lam[k] = lam;
        volatile float inv = 1.0f / lam;
        P.inv_lam[k] = inv;
      }
    }

    // ---- W_hat = diag(lam) W (float64)
    std::vector<double> Wh((size_t)K * N);
#pragma omp parallel for schedule(static)
    for (int k = 0; k < K; ++k)
      for (int n = 0; n < N; ++n)
        Wh[(size_t)k * N + n] = (double)P.lam[k] * (double)bf16_to_float(W[(size_t)k * N + n]);

    // ---- truncated SVD, stored 16-bit branch, residual
    P.R.assign((size_t)K * N, 0.0f);
    if (r > 0) {
      svdq_status st = truncated_svd(Wh, K, N, r, P.L1, P.L2, P.sigma, P.svd_iterations, P.svd_tail_energy);
      if (st != SVDQ_OK) return st;
      P.L1d.resize((size_t)K * r);
      P.L2b.resize((size_t)r * N);
      for (int k = 0; k < K; ++k)
        for (int i = 0; i < r; ++i)
          P.L1d[(size_t)k * r + i] = bf16_from_double((double)P.inv_lam[k] * P.L1[(size_t)k * r + i]);
      for (size_t i = 0; i < P.L2b.size(); ++i) P.L2b[i] = bf16_from_double(P.L2[i]);
      std::vector<double> L2v((size_t)r * N);
      for (size_t i = 0; i < L2v.size(); ++i) L2v[i] = bf16_to_float(P.L2b[i]);
      // each element sums its r products in ascending i; a whole row at a
      // time, so that the inner loop runs along contiguous columns
#pragma omp parallel
      {
        std::vector<double> br(N);
#pragma omp for schedule(static)
        for (int k = 0; k < K; ++k) {
          std::fill(br.begin(), br.end(), 0.0);
          for (int i = 0; i < r; ++i) {
            const double lki = (double)P.lam[k] * (double)bf16_to_float(P.L1d[(size_t)k * r + i]);
            const double* l2 = &L2v[(size_t)i * N];
            for (int n = 0; n < N; ++n) br[n] += lki * l2[n];
          }
          for (int n = 0; n < N; ++n) P.R[(size_t)k * N + n] = (float)(Wh[(size_t)k * N + n] - br[n]);
        }
      }
    } else {
#pragma omp parallel for schedule(static)
      for (int k = 0; k < K; ++k)
        for (int n = 0; n < N; ++n) P.R[(size_t)k * N + n] = (float)Wh[(size_t)k * N + n];
      if (!w4a16) {
        const int nch = row_chunks(K);
        std::vector<double> part(nch);
#pragma omp parallel for schedule(static)
        for (int ch = 0; ch < nch; ++ch) {
          const int r0 = ch * kRowChunk, r1 = std::min(K, r0 + kRowChunk);
          const double* a = Wh.data() + (size_t)r0 * N;
          part[ch] = dot4(a, a, (r1 - r0) * N);
        }
        double tot = 0.0;
        for (int ch = 0; ch < nch; ++ch) tot += part[ch];
        P.svd_tail_energy = tot;
      }
    }

    // ---- largest smoothed calibration activation, amax |fp32(Xc / lam)|
    P.x_amax = 0.0f;
    if (!w4a16)
      for (int m = 0; m < M_calib; ++m)
        for (int k = 0; k < K; ++k) {
          volatile float v = bf16_to_float(calib[(size_t)m * K + k]) * P.inv_lam[k];
          P.x_amax = std::max(P.x_amax, std::fabs((float)v));
        }

    // ---- residual quantization, groups along K for each output column n
    float amax = 0.0f;                      // a maximum: exact in any order
#pragma omp parallel for schedule(static) reduction(max : amax)
    for (size_t i = 0; i < P.R.size(); ++i) amax = std::max(amax, std::fabs(P.R[i]));
    P.w_amax = amax;
    if (cfg.format == SVDQ_W8A8_INT8) {
      // INT8, one group per output channel: s = fp32(a fp32(1/127)),
      // code = clamp(rint(fp32(v fp32(1/s))), -127, 127)
      P.w_codes.assign((size_t)N * K, 0);
      P.w_scales_f32.assign(N, 0.0f);
#pragma omp parallel for schedule(static)
      for (int n = 0; n < N; ++n) {
        float a = 0.0f;
        for (int k = 0; k < K; ++k) a = std::max(a, std::fabs(P.R[(size_t)k * N + n]));
        const float c127 = 1.0f / 127.0f;
        volatile float t = a * c127;
        const float sc = t;
        P.w_scales_f32[n] = sc;
        if (sc == 0.0f) continue;
        volatile float iv = 1.0f / sc;
        const float inv = iv;
        for (int k = 0; k < K; ++k) {
          volatile float q = P.R[(size_t)k * N + n] * inv;
          float rq = std::nearbyint((float)q);
          rq = std::min(127.0f, std::max(-127.0f, rq));
          P.w_codes[(size_t)n * K + k] = (uint8_t)(int8_t)rq;
        }
      }
      return SVDQ_OK;
    }
    P.w_codes.assign((size_t)N * K / 2, 0);
    if (cfg.flags & SVDQ_PREP_GPTQ) {
      const bool nvfp4 = cfg.format == SVDQ_NVFP4;
      if (nvfp4) {
        P.g_w_exp = pow2_ceil_exponent((double)amax / 2688.0);
        P.w_scales_e4m3.assign((size_t)N * K / 16, 0);
      } else {
        P.w_scales_bf16.assign((size_t)N * K / 64, 0);
      }
      std::vector<double> H, U;
      gptq_hessian(calib, M_calib, K, P.inv_lam, H);
      if (!gptq_factor(H, K, U)) return SVDQ_ENOCONVERGE;
      std::vector<double>().swap(H);
      gptq_columns(P.R, K, N, U, nvfp4, P);
      if (nvfp4) P.g_x_exp = pow2_ceil_exponent(4.0 * (double)P.x_amax / 2688.0);
      if (cfg.flags & SVDQ_PREP_KEEP_GPTQ_FACTOR) P.gptq_U.swap(U);
      return SVDQ_OK;
    }
    if (cfg.format == SVDQ_NVFP4) {
      P.g_w_exp = pow2_ceil_exponent((double)amax / 2688.0);
      const float g = (float)std::ldexp(1.0, P.g_w_exp);
      const float c = (float)std::ldexp((double)(1.0f / 6.0f), -P.g_w_exp);
      P.w_scales_e4m3.assign((size_t)N * K / 16, 0);
      // 16 output columns per task, so that each group's 16 rows are read as
      // contiguous 64-byte row segments
#pragma omp parallel for schedule(static)
      for (int nb = 0; nb < (N + 15) / 16; ++nb) {
        const int n0 = nb * 16, nc = std::min(16, N - n0);
        float blk[16][16];
        uint8_t codes[16];
        for (int g16 = 0; g16 < K / 16; ++g16) {
          for (int i = 0; i < 16; ++i)
            for (int j = 0; j < nc; ++j) blk[j][i] = P.R[(size_t)(g16 * 16 + i) * N + n0 + j];
          for (int j = 0; j < nc; ++j) {
            const int n = n0 + j;
            P.w_scales_e4m3[(size_t)n * (K / 16) + g16] = nvfp4_group(blk[j], c, g, codes);
            for (int i = 0; i < 8; ++i)
              P.w_codes[(size_t)n * (K / 2) + g16 * 8 + i] = (uint8_t)(codes[2 * i] | (codes[2 * i + 1] << 4));
          }
        }
      }
      // activation tensor scale from the calibration batch, 4x headroom
      P.g_x_exp = pow2_ceil_exponent(4.0 * (double)P.x_amax / 2688.0);
    } else {
      P.w_scales_bf16.assign((size_t)N * K / 64, 0);
      // 16 output columns per task (contiguous 64-byte row segments)
#pragma omp parallel for schedule(static)
      for (int nb = 0; nb < (N + 15) / 16; ++nb) {
        const int n0 = nb * 16, nc = std::min(16, N - n0);
        float blk[16][64];
        int8_t codes[64];
        for (int g64 = 0; g64 < K / 64; ++g64) {
          for (int i = 0; i < 64; ++i)
            for (int j = 0; j < nc; ++j) blk[j][i] = P.R[(size_t)(g64 * 64 + i) * N + n0 + j];
          for (int j = 0; j < nc; ++j) {
            const int n = n0 + j;
            P.w_scales_bf16[(size_t)n * (K / 64) + g64] = int4_group(blk[j], codes);
            for (int i = 0; i < 32; ++i)
              P.w_codes[(size_t)n * (K / 2) + g64 * 32 + i] =
                  (uint8_t)((codes[2 * i] & 0xF) | ((codes[2 * i + 1] & 0xF) << 4));
          }
        }
      }
    }
    return SVDQ_OK;
  } catch (const std::bad_alloc&) {
    return SVDQ_ENOMEM;
  } catch (...) {
    return SVDQ_EINVAL;
  }
}

}  // namespace svdq
