/* A plain C11 program against include/qvla.h and libqvla.so: the boundary is
 * a C ABI (no C++ or torch types), and its host-only entry points work with
 * no GPU present.  Prints one "key values..." line per check. */
#include <stdio.h>
#include <string.h>

#include "qvla.h"

int main(void) {
  printf("abi %d %d\n", qvla_abi_version(), QVLA_ABI_VERSION);
  printf("status %s|%s\n", qvla_status_str(QVLA_OK), qvla_status_str(QVLA_ERR_SHAPE));

  size_t wq = 0, rot = 0, tc = 0, ws = 0, b = 0;
  qvla_status st = qvla_packed_sizes(256, 1024, 64, &wq, &rot, &tc, &ws);
  printf("sizes %d %zu %zu %zu\n", (int)st, wq, rot, tc);
  printf("badshape %d\n", (int)qvla_packed_sizes(256, 1000, 64, &wq, &rot, &tc, &ws));
  st = qvla_rotate_quant_workspace_bytes(50, 2048, 64, QVLA_DTYPE_BF16, &b);
  printf("rqws %d %zu\n", (int)st, b);
  st = qvla_rotate_quant_a8_workspace_bytes(50, 1024, &b);
  printf("a8ws %d %zu\n", (int)st, b);

  /* GPTQ on the host with H = I and no damping: U = I, every error update
   * is zero, and each code is clamp(rint(w / s)) with the quotient in fp64
   * (the RTN rule, except where fp32 division would round onto a tie:
   * 0.35 / 0.1 in row 1). */
  enum { N = 3, K = 8 };
  const float Wr[N * K] = {0.5f,  -1.25f, 3.5f,  0.0f,   -2.0f, 1.0f,  0.75f, -3.5f,
                           0.1f,  0.2f,   -0.3f, 0.4f,   -0.5f, 0.6f,  -0.7f, 0.35f,
                           0.0f,  0.0f,   0.0f,  0.0f,   0.0f,  0.0f,  0.0f,  0.0f};
  double H[K * K];
  memset(H, 0, sizeof(H));
  for (int i = 0; i < K; ++i) H[i * K + i] = 1.0;
  int8_t q[N * K];
  float s[N];
  st = qvla_gptq_quantize_host(Wr, N, K, H, 0.0, NULL, q, s);
  printf("gptq %d", (int)st);
  for (int i = 0; i < N * K; ++i) printf(" %d", (int)q[i]);
  printf("\nscales %.9g %.9g %.9g\n", s[0], s[1], s[2]);

  /* H = X'^T X' of two rows, on the host */
  const float xr[2 * 2] = {1.0f, 2.0f, 3.0f, -1.0f};
  double Hx[4];
  st = qvla_gptq_hessian_host(xr, 2, 2, Hx);
  printf("hessian %d %g %g %g %g\n", (int)st, Hx[0], Hx[1], Hx[2], Hx[3]);

  /* argument errors are found before any CUDA call */
  st = qvla_rotate_quant_act(NULL, QVLA_DTYPE_BF16, 4, 64, NULL, QVLA_SCALE_DYNAMIC, NULL, 0, 0,
                             NULL, 0, 0, NULL, NULL, NULL, 0, NULL);
  printf("nulllinear %d\n", (int)st);
  printf("gptqshape %d\n", (int)qvla_gptq_quantize_host(Wr, N, 5000, H, 0.0, NULL, q, s));
  return 0;
}
