/* A plain C consumer of the library: includes vark.h, links libvark.so and
 * drives the host-side calls (no Python, no torch).  Reads an S-CAS array from
 * stdin ("L H S n_sinks budget_bp", the S sides, then L*H*S values), prints
 * the status of each call and the results, one item per line:
 *   version V
 *   schedule STATUS k0 k1 ...            (keep[L][H][S])
 *   finalize STATUS x0 x1 ...            (S-CAS of a mass array built from the input)
 *   cache STATUS b0 b1 ...               (bytes[S][L] for B = 2, D = 64)
 *   args A B C                           (argument errors of three device calls)
 *   device STATUS                         (only with the argument "device", given on a
 *                                         host without a GPU: a device call whose
 *                                         placeholder pointers would otherwise be used)
 */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "vark.h"

int main(int argc, char** argv) {
  const int device_call = argc > 1 && strcmp(argv[1], "device") == 0;
  int L, H, S, n_sinks;
  unsigned budget;
  if (scanf("%d %d %d %d %u", &L, &H, &S, &n_sinks, &budget) != 5) return 2;
  if (L < 1 || H < 1 || S < 1 || S > VARK_MAX_SCALES) return 2;
  int32_t sides[VARK_MAX_SCALES];
  for (int s = 0; s < S; ++s)
    if (scanf("%d", &sides[s]) != 1) return 2;
  const int n = L * H * S;
  double* scas = malloc(sizeof(double) * n);
  uint8_t* keep = malloc((size_t)n);
  float* mass = calloc((size_t)L * H * S * S, sizeof(float));
  double* fin = malloc(sizeof(double) * n);
  int64_t* bytes = malloc(sizeof(int64_t) * (size_t)S * L);
  if (!scas || !keep || !mass || !fin || !bytes) return 3;
  for (int i = 0; i < n; ++i)
    if (scanf("%lf", &scas[i]) != 1) return 2;

  printf("version %d\n", vark_version());

  int rc = vark_build_schedule(scas, L, H, S, sides, budget, n_sinks, keep);
  printf("schedule %d", rc);
  if (rc == VARK_OK)
    for (int i = 0; i < n; ++i) printf(" %d", keep[i]);
  printf("\n");

  /* mass[l][h][s][k] = scas[l][h][s] for k = S-1 only: S-CAS of s < S-1 is then scas[l][h][s] */
  for (int l = 0; l < L; ++l)
    for (int h = 0; h < H; ++h)
      for (int s = 0; s < S; ++s)
        mass[(((size_t)l * H + h) * S + s) * S + (S - 1)] = (float)scas[((size_t)l * H + h) * S + s];
  rc = vark_scas_finalize(mass, L, H, S, 1, fin);
  printf("finalize %d", rc);
  if (rc == VARK_OK)
    for (int i = 0; i < n; ++i) printf(" %.17g", fin[i]);
  printf("\n");

  rc = vark_cache_size_after_layer(keep, L, H, S, sides, 2, 64, bytes);
  printf("cache %d", rc);
  if (rc == VARK_OK)
    for (int i = 0; i < S * L; ++i) printf(" %lld", (long long)bytes[i]);
  printf("\n");

  /* argument errors of the attention-over-codes calls come back before any
   * device work, on any host: a missing query, 3-bit rows of 24 bytes
   * (D = 64), and 8-bit codes off the 16-byte boundary */
  {
    static _Alignas(16) unsigned char buf[256];
    const uint16_t* p = (const uint16_t*)buf;
    uint16_t* o = (uint16_t*)buf;
    int32_t* st = (int32_t*)buf;
    const int32_t* t = (const int32_t*)buf;
    const float* f = (const float*)buf;
    int a = vark_pruned_attention_int4(NULL, buf, buf, p, p, 8, p, p, 1, 1, S, 128, sides, -1, t, t, t, f, NULL, o,
                                       st, NULL);
    int b = vark_pruned_attention_int3(p, buf, buf, p, p, 8, p, p, 1, 1, S, 64, sides, -1, t, t, t, f, NULL, o, st,
                                       NULL);
    int c = vark_pruned_attention_int8(p, (const int8_t*)(buf + 8), (const int8_t*)buf, f, f, 8, p, p, 1, 1, S, 64,
                                       sides, -1, t, t, t, f, NULL, o, st, NULL);
    printf("args %d %d %d\n", a, b, c);
  }

  /* a device call with aligned placeholder pointers: on a host without a GPU
   * this reports VARK_E_DEVICE; the strings come from the library */
  if (device_call) {
    int32_t* dummy = aligned_alloc(64, 4096);
    rc = vark_build_offsets(keep, L, H, S, sides, 1, 64, dummy, dummy, dummy, (int64_t*)dummy, NULL);
    printf("device %d %s\n", rc, vark_status_string(rc));
    free(dummy);
  }
  free(scas); free(keep); free(mass); free(fin); free(bytes);
  return 0;
}
