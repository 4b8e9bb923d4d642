/* A plain C99 client of libnectar.so: includes only nectar.h and calls the
 * entry points that need no GPU -- version, status strings, the packed size
 * of a module set (the parameter count of Eq. (3.6) laid out in tiles) and
 * the host-side argument checks, which must fail before touching a device.
 * Prints "ok" and exits 0, or names the first failed check and exits 1. */
#include <stdio.h>
#include <string.h>

#include "nectar.h"

#define CHECK(c)                                   \
  do {                                             \
    if (!(c)) {                                    \
      printf("FAIL line %d: %s\n", __LINE__, #c); \
      return 1;                                    \
    }                                              \
  } while (0)

int main(void) {
  const char *v = nectar_version();
  nectar_dims dims = {2, 2, 4, 128};
  nectar_dims bad_d = {2, 2, 4, 64};
  int32_t widths[2] = {256, 512};
  int32_t bad_widths[2] = {256, 500};
  int64_t elems;
  int64_t elems_wider;
  float scale = 0.08838834764831845f;
  nectar_status st;

  CHECK(v != NULL && strchr(v, '.') != NULL);
  CHECK(nectar_status_string(NECTAR_OK) != NULL);
  CHECK(nectar_status_string(NECTAR_ERR_WORKSPACE) != NULL);

  elems = nectar_module_packed_elems(dims, 2, widths);
  CHECK(elems > 0);
  /* at least the bf16 parameters of both nets, 2 H^2 + 645 H + 129 per pair */
  CHECK(elems >= (int64_t)dims.Hkv * ((2 * 256 * 256 + 645 * 256 + 129) + (2 * 512 * 512 + 645 * 512 + 129)));
  widths[1] = 1024;
  elems_wider = nectar_module_packed_elems(dims, 2, widths);
  CHECK(elems_wider > elems);
  CHECK(nectar_module_packed_elems(dims, 2, bad_widths) <= 0);
  CHECK(nectar_last_error()[0] != '\0');

  /* host validation comes first: no device is touched for these */
  st = nectar_cache_attn_lse(bad_d, NULL, NULL, 10, NULL, 1, scale, NULL, NULL, NULL, 0, NULL);
  CHECK(st == NECTAR_ERR_UNSUPPORTED);
  st = nectar_cache_attn_lse(dims, NULL, NULL, -1, NULL, 1, scale, NULL, NULL, NULL, 0, NULL);
  CHECK(st == NECTAR_ERR_INVALID_ARG);
  st = nectar_cache_attn_lse(dims, NULL, NULL, 10, NULL, 0, scale, NULL, NULL, NULL, 0, NULL);
  CHECK(st == NECTAR_OK); /* nq == 0: nothing to do */
  st = nectar_merge_local(dims, NULL, NULL, NULL, 1, NULL, NULL, NULL, NULL, 1, 4, NULL, scale, NULL, NULL);
  CHECK(st == NECTAR_ERR_INVALID_ARG);
  CHECK(nectar_cache_attn_workspace_size(bad_d, 10, 1) == 0);

  printf("ok %s\n", v);
  return 0;
}
