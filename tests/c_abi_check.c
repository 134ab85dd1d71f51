/* Calls the library through include/nshb.h from C (no GPU needed: argument checking and
 * workspace sizing only) and prints what tests/test_c_abi.py compares with the ctypes
 * binding.  Built as C11 and as C++17 with -pedantic -Wall -Wextra -Werror. */
#include <stddef.h>
#include <stdint.h>
#include <stdio.h>

#include "nshb.h"

static void fake(nshb_matrix *m, int64_t rows, int64_t cols, uintptr_t base) {
  m->rows = rows;
  m->cols = cols;
  m->ld = cols;
  m->w_dtype = NSHB_BF16;
  m->z_index = -1;
  m->W = (void *)base;
  m->G = (const void *)(base + 0x4000000u);
  m->M = (float *)(base + 0x8000000u);
  m->O_out = NULL;
}

int main(void) {
  nshb_params p;
  nshb_adam_params a;
  nshb_matrix m[3];
  size_t bytes = 0, adam_bytes = 0;
  if (nshb_default_params(&p) != NSHB_OK || nshb_default_adam_params(&a) != NSHB_OK) return 1;
  printf("sizeof_matrix %zu\n", sizeof(nshb_matrix));
  printf("sizeof_params %zu\n", sizeof(nshb_params));
  printf("sizeof_adam %zu\n", sizeof(nshb_adam_params));
  printf("offset_coeffs %zu\n", offsetof(nshb_params, coeffs));
  printf("offset_rho %zu\n", offsetof(nshb_params, rho));
  printf("defaults %.4f %d %d %d %.4f\n", p.beta, p.ns_steps, p.tile, a.step, a.beta2);
  fake(&m[0], 768, 768, 0x10000000u);
  fake(&m[1], 3072, 768, 0x20000000u);
  fake(&m[2], 5, 7, 0x30000000u);
  printf("ws_status %d\n", (int)nshb_workspace_size(m, 3, &p, NSHB_OP_HYPERBALL, NULL, 0, 0, &bytes));
  printf("ws_bytes %zu\n", bytes);
  printf("adam_status %d\n", (int)nshb_workspace_size(m, 3, &p, NSHB_OP_ADAMH, NULL, 0, 0, &adam_bytes));
  printf("adam_bytes %zu\n", adam_bytes);
  printf("null_ws %s\n", nshb_status_string(hyperball_step(m, 3, &p, NULL, bytes, NULL)));
  printf("short_ws %s\n", nshb_status_string(muon_step(m, 3, &p, (void *)0x40000000u, bytes - 256, NULL)));
  m[2].cols = 0;
  printf("bad_shape %s\n", nshb_status_string(nshb_workspace_size(m, 3, &p, NSHB_OP_MUON, NULL, 0, 0, &bytes)));
  printf("version %d\n", (int)nshb_version());
  return 0;
}
