/* A plain C99 caller of the library's C ABI: it includes only nvfp4rac.h, links the shared
 * library, and uses the calls that need no device (sizes, status strings, host-side argument
 * checks).  Built and run by tests/test_c_abi_cpu.py. */
#include <stdio.h>
#include <string.h>

#include "nvfp4rac.h"

static int fails = 0;
#define CHECK(cond)                                                 \
  do {                                                              \
    if (!(cond)) {                                                  \
      printf("FAIL line %d: %s\n", __LINE__, #cond);                \
      ++fails;                                                      \
    }                                                               \
  } while (0)

int main(void) {
  CHECK(nvfp4_version() >= 100);
  CHECK(strcmp(nvfp4_status_string(NVFP4_OK), "ok") == 0);
  CHECK(nvfp4_codes_bytes(128, 256) == 128 * 128);
  CHECK(nvfp4_sf_bytes(128, 256) == 128 * 16);
  CHECK(nvfp4_sf_bytes_layout(48, 256, NVFP4_SF_SLAB16) == 3 * 4 * 512);
  CHECK(nvfp4_kp_from_ratio(2048, 0.5) == 1024);
  CHECK(mxfp8_codes_bytes(128, 256) == 128 * 256 && mxfp8_sf_bytes(128, 256) == 128 * 8);
  CHECK(rac_calibrate_grouped_workspace_size(64, 128, 3) > rac_calibrate_workspace_size(64, 128));

  /* a K that is not a multiple of 64 is refused on the host, before any device work */
  nvfp4_tensor q;
  memset(&q, 0, sizeof(q));
  q.codes = (uint8_t*)16;
  q.sf = (uint8_t*)16;
  q.s_g = (float*)16;
  q.slabs = 1;
  q.rows = 64;
  q.rows_padded = 128;
  q.cols = 100;
  nvfp4_status st = nvfp4_quantize((const uint16_t*)16, 64, 100, 104, NULL, 64, NULL, 0, NULL, &q, NULL,
                                   (void*)16, 1024, NULL, NULL);
  CHECK(st == NVFP4_ERR_UNSUPPORTED_SHAPE);
  CHECK(strlen(nvfp4_last_error_string()) > 0);

  mxfp8_tensor m;
  memset(&m, 0, sizeof(m));
  m.codes = (uint8_t*)16;
  m.sf = (uint8_t*)16;
  m.slabs = 1;
  m.rows = 64;
  m.rows_padded = 128;
  m.cols = 192;
  CHECK(mxfp8_quantize((const uint16_t*)16, 64, 192, 192, NULL, 64, &m, NULL, NULL) == NVFP4_ERR_UNSUPPORTED_SHAPE);
  CHECK(moe_row_groups(NULL, 4, 0, NULL, NULL) == NVFP4_OK);

  if (fails == 0) printf("c abi ok\n");
  return fails == 0 ? 0 : 1;
}
