/* A plain C99 client of libnectar.so: includes only nectar.h and calls the
 * entry points that need no GPU -- version, status strings, the packed size
 * of a module set (the parameter count of Eq. (3.6) laid out in tiles) and
 * the host-side argument checks, which must fail before touching a device,
 * and the per-thread error text (two threads failing at once each read
 * their own reason).
 * Prints "ok" and exits 0, or names the first failed check and exits 1. */
#include <pthread.h>
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

/* Fails one call per iteration, in one of two ways, and checks that this
 * thread's error text names its own reason every time. */
static void *fail_repeatedly(void *arg) {
  const int kind = *(const int *)arg;
  nectar_dims dims = {1, 1, 1, 128};
  nectar_dims bad_d = {1, 1, 1, 64};
  int i;
  for (i = 0; i < 20000; ++i) {
    nectar_status st = kind == 0
        ? nectar_cache_attn_lse(bad_d, NULL, NULL, 1, NULL, 1, 1.0f, NULL, NULL, NULL, 0, NULL)
        : nectar_cache_attn_lse(dims, NULL, NULL, -1, NULL, 1, 1.0f, NULL, NULL, NULL, 0, NULL);
    const char *msg = nectar_last_error();
    if (st == NECTAR_OK) return (void *)1;
    if (kind == 0 && strstr(msg, "d = 64") == NULL) return (void *)1;
    if (kind == 1 && strstr(msg, ">= 0") == NULL) return (void *)1;
  }
  return NULL;
}

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

  {
    pthread_t t[2];
    int kinds[2] = {0, 1};
    void *r0 = NULL, *r1 = NULL;
    CHECK(pthread_create(&t[0], NULL, fail_repeatedly, &kinds[0]) == 0);
    CHECK(pthread_create(&t[1], NULL, fail_repeatedly, &kinds[1]) == 0);
    CHECK(pthread_join(t[0], &r0) == 0 && pthread_join(t[1], &r1) == 0);
    CHECK(r0 == NULL && r1 == NULL);
  }

  printf("ok %s\n", v);
  return 0;
}
