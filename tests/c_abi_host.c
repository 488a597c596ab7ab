/*
 * The C ABI (include/svdq.h) used from plain C, without Python: prepare a
 * small layer on the host (device -1), read its description and tensors,
 * round-trip it through a checkpoint, and check the documented status codes of
 * bad calls.  No GPU work is issued.  Built and run by tests/test_c_abi_host.py;
 * prints "ok" and returns 0, or names the first failed check and returns 1.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "svdq.h"

static int failures = 0;

#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "check failed (line %d): %s\n", __LINE__, #cond); \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

/* splitmix64 and Box-Muller: deterministic normals */
static uint64_t rng_state = 0x243F6A8885A308D3ull;
static double uniform01(void) {
  uint64_t z = (rng_state += 0x9E3779B97F4A7C15ull);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  z ^= z >> 31;
  return ((double)(z >> 11) + 0.5) / 9007199254740992.0;
}
static double normal(void) {
  const double u1 = uniform01(), u2 = uniform01();
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

/* float -> BF16 bits, round to nearest even (finite inputs) */
static uint16_t bf16_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

int main(void) {
  enum { K = 256, N = 64, MC = 32, R = 32 };
  uint16_t* W = malloc(sizeof(uint16_t) * K * N);
  uint16_t* bias = malloc(sizeof(uint16_t) * N);
  uint16_t* calib = malloc(sizeof(uint16_t) * MC * K);
  if (!W || !bias || !calib) return 1;
  for (int i = 0; i < K * N; ++i) W[i] = bf16_bits((float)(normal() / 16.0));
  for (int n = 0; n < N; ++n) bias[n] = bf16_bits((float)(0.1 * normal()));
  for (int i = 0; i < MC * K; ++i) calib[i] = bf16_bits((float)normal());

  svdq_config cfg = {SVDQ_NVFP4, R, 0.5f, 0u};
  svdq_layer* L = NULL;
  CHECK(svdq_prepare(&cfg, K, N, W, bias, calib, MC, -1, &L) == SVDQ_OK);
  CHECK(L != NULL);
  if (!L) return 1;

  svdq_layer_info info;
  CHECK(svdq_get_info(L, &info) == SVDQ_OK);
  CHECK(info.K == K && info.N == N && info.rank == R && info.format == SVDQ_NVFP4 && info.device == -1);
  CHECK(info.svd_iterations > 0 && info.svd_tail_energy >= 0.0);

  /* tensor sizes as the header documents them */
  CHECK(svdq_tensor_bytes(L, SVDQ_T_LAMBDA) == (size_t)K * 4);
  CHECK(svdq_tensor_bytes(L, SVDQ_T_INV_LAMBDA) == (size_t)K * 4);
  CHECK(svdq_tensor_bytes(L, SVDQ_T_L1) == (size_t)K * R * 8);
  CHECK(svdq_tensor_bytes(L, SVDQ_T_L2) == (size_t)R * N * 8);
  CHECK(svdq_tensor_bytes(L, SVDQ_T_L1D) == (size_t)K * R * 2);
  CHECK(svdq_tensor_bytes(L, SVDQ_T_L2B) == (size_t)R * N * 2);
  CHECK(svdq_tensor_bytes(L, SVDQ_T_RESIDUAL) == (size_t)K * N * 4);
  CHECK(svdq_tensor_bytes(L, SVDQ_T_SIGMA) == (size_t)R * 8);
  CHECK(svdq_tensor_bytes(L, SVDQ_T_W_CODES) == (size_t)N * K / 2);
  CHECK(svdq_tensor_bytes(L, SVDQ_T_W_SCALES) == (size_t)N * K / 16);
  CHECK(svdq_tensor_bytes(L, SVDQ_T_BIAS) == (size_t)N * 4);
  CHECK(svdq_tensor_bytes(L, SVDQ_T_GPTQ_U) == 0);
  CHECK(svdq_tensor_bytes(L, SVDQ_T_LORA_A) == 0);
  CHECK(svdq_tensor_bytes(L, SVDQ_T_COUNT) == 0);
  CHECK(svdq_tensor_bytes(NULL, SVDQ_T_LAMBDA) == 0);

  /* exports: lambda * inv_lambda = 1 to float rounding; sigma sorted, positive */
  float lam[K], inv[K];
  double sigma[R];
  CHECK(svdq_export(L, SVDQ_T_LAMBDA, lam, sizeof lam) == SVDQ_OK);
  CHECK(svdq_export(L, SVDQ_T_INV_LAMBDA, inv, sizeof inv) == SVDQ_OK);
  CHECK(svdq_export(L, SVDQ_T_SIGMA, sigma, sizeof sigma) == SVDQ_OK);
  for (int k = 0; k < K; ++k) CHECK(lam[k] > 0.0f && fabs((double)lam[k] * inv[k] - 1.0) < 1e-6);
  for (int i = 0; i + 1 < R; ++i) CHECK(sigma[i] >= sigma[i + 1] && sigma[i + 1] > 0.0);
  CHECK(svdq_export(L, SVDQ_T_LAMBDA, lam, sizeof lam - 4) == SVDQ_EINVAL);   /* size must match */
  CHECK(svdq_export(L, SVDQ_T_GPTQ_U, lam, sizeof lam) == SVDQ_EINVAL);       /* no such tensor */
  CHECK(svdq_export(L, SVDQ_T_LAMBDA, NULL, sizeof lam) == SVDQ_EINVAL);

  /* checkpoint round trip: the rebuilt layer serializes to the same bytes */
  const size_t nb = svdq_serialized_bytes(L);
  CHECK(nb > 0);
  unsigned char* a = malloc(nb);
  unsigned char* b = malloc(nb);
  if (!a || !b) return 1;
  CHECK(svdq_serialize(L, a, nb) == SVDQ_OK);
  CHECK(svdq_serialize(L, a, nb - 1) == SVDQ_EINVAL);
  svdq_layer* L2 = NULL;
  CHECK(svdq_deserialize(a, nb, -1, &L2) == SVDQ_OK && L2 != NULL);
  if (L2) {
    CHECK(svdq_serialized_bytes(L2) == nb);
    CHECK(svdq_serialize(L2, b, nb) == SVDQ_OK);
    CHECK(memcmp(a, b, nb) == 0);
    CHECK(svdq_tensor_bytes(L2, SVDQ_T_RESIDUAL) == 0);   /* preparation-only, not stored */
    svdq_destroy(L2);
  }
  L2 = (svdq_layer*)a;                                    /* any non-NULL value */
  CHECK(svdq_deserialize(a, nb - 1, -1, &L2) == SVDQ_EINVAL && L2 == NULL);
  a[0] ^= 0xFF;                                           /* not a checkpoint */
  CHECK(svdq_deserialize(a, nb, -1, &L2) == SVDQ_EINVAL && L2 == NULL);

  /* a host-only layer has no forward */
  CHECK(svdq_workspace_bytes(L, 16) > 0);
  CHECK(svdq_linear_forward(L, (void*)16, 16, (void*)16, (void*)256, 1u << 20, NULL, 0) == SVDQ_ESTATE);
  CHECK(svdq_linear_forward_static(L, (void*)16, 16, (void*)16, NULL, 0) == SVDQ_ESTATE);
  CHECK(svdq_check(L, NULL) == SVDQ_ESTATE);
  CHECK(svdq_selftest_wait_timeout(L, 1000, NULL) == SVDQ_ESTATE);

  /* documented argument errors of svdq_prepare; *out is NULL after each */
  svdq_layer* bad = (svdq_layer*)W;
  CHECK(svdq_prepare(NULL, K, N, W, bias, calib, MC, -1, &bad) == SVDQ_EINVAL && bad == NULL);
  bad = (svdq_layer*)W;
  CHECK(svdq_prepare(&cfg, K, N, W, bias, NULL, 0, -1, &bad) == SVDQ_EINVAL && bad == NULL);
  svdq_config badfmt = {7, R, 0.5f, 0u};
  CHECK(svdq_prepare(&badfmt, K, N, W, bias, calib, MC, -1, &bad) == SVDQ_EINVAL);
  svdq_config flags = {SVDQ_NVFP4, R, 0.5f, 0x80u};
  CHECK(svdq_prepare(&flags, K, N, W, bias, calib, MC, -1, &bad) == SVDQ_EINVAL);
  CHECK(svdq_prepare(&cfg, 96, N, W, bias, calib, MC, -1, &bad) == SVDQ_EUNSUPPORTED);   /* K % 64 */
  CHECK(svdq_prepare(&cfg, K, 24, W, bias, calib, MC, -1, &bad) == SVDQ_EUNSUPPORTED);   /* N % 16 */
  svdq_config r17 = {SVDQ_NVFP4, 17, 0.5f, 0u};
  CHECK(svdq_prepare(&r17, K, N, W, bias, calib, MC, -1, &bad) == SVDQ_EUNSUPPORTED);
  const uint16_t keep = W[5];
  W[5] = 0x7FC0u;                                         /* a NaN in the weight */
  CHECK(svdq_prepare(&cfg, K, N, W, bias, calib, MC, -1, &bad) == SVDQ_EINVAL && bad == NULL);
  W[5] = keep;

  /* W4A16 needs no calibration and keeps no branch */
  svdq_config w16 = {SVDQ_W4A16_INT4, 0, 0.5f, 0u};
  svdq_layer* L3 = NULL;
  CHECK(svdq_prepare(&w16, K, N, W, bias, NULL, 0, -1, &L3) == SVDQ_OK && L3 != NULL);
  if (L3) {
    CHECK(svdq_get_info(L3, &info) == SVDQ_OK && info.rank == 0 && info.format == SVDQ_W4A16_INT4);
    CHECK(svdq_workspace_bytes(L3, 4) == 0);
    svdq_destroy(L3);
  }

  /* status strings and NULL handling */
  for (int s = SVDQ_OK; s <= SVDQ_ESTATE; ++s) {
    const char* t = svdq_status_string((svdq_status)s);
    CHECK(t != NULL && strlen(t) > 0 && strcmp(t, "unknown status") != 0);
  }
  CHECK(strcmp(svdq_status_string((svdq_status)99), "unknown status") == 0);
  CHECK(svdq_get_info(NULL, &info) == SVDQ_EINVAL);
  CHECK(svdq_get_info(L, NULL) == SVDQ_EINVAL);
  svdq_destroy(NULL);

  svdq_destroy(L);
  free(a);
  free(b);
  free(W);
  free(bias);
  free(calib);
  if (failures) {
    fprintf(stderr, "%d check(s) failed\n", failures);
    return 1;
  }
  printf("ok\n");
  return 0;
}
