/* Plain C use of the ditango C ABI (no Python, no torch): geometry checks,
 * active units, slot tables with and without KV groups, status strings, and
 * argument validation of the launching calls.  Needs no GPU: every call here
 * is host-side or fails validation before anything launches.
 * Prints one "key value" line per result; exits non-zero on a mismatch. */
#include <stdio.h>
#include <string.h>

#include "ditango.h"

static int fails = 0;
#define CHECK(cond, msg)                          \
  do {                                            \
    if (!(cond)) {                                \
      printf("FAIL %s\n", msg);                   \
      ++fails;                                    \
    }                                             \
  } while (0)

int main(void) {
  /* 8 frames of 3600 tokens, one partition per frame, frame f attends
   * frames f-1, f, f+1 and 0 */
  enum { F = 8, L = 3600 };
  int32_t off[F + 1];
  uint8_t mask[F * F];
  for (int f = 0; f <= F; ++f) off[f] = f * L;
  for (int f = 0; f < F; ++f)
    for (int g = 0; g < F; ++g) mask[f * F + g] = (f - g <= 1 && g - f <= 1) || g == 0;
  ditango_geom geo;
  memset(&geo, 0, sizeof(geo));
  geo.B = 1;
  geo.H = 24;
  geo.N = F * L;
  geo.d = 96;
  geo.P = F;
  geo.F = F;
  geo.part_off = off;
  geo.frame_off = off;
  geo.frame_mask = mask;
  for (int k = 0; k < 3; ++k) {
    geo.q_strides[k] = geo.k_strides[k] = geo.v_strides[k] =
        k == 0 ? (int64_t)geo.H * geo.N * geo.d : (k == 1 ? (int64_t)geo.N * geo.d : geo.d);
  }
  printf("version %d\n", ditango_version());
  CHECK(ditango_check_geom(&geo) == DITANGO_OK, "frame-tile geometry");
  const int64_t active = ditango_num_active(&geo);
  printf("active_pairs %lld\n", (long long)active);
  CHECK(active == 4 * F - 4, "4F-4 active pairs");
  CHECK(ditango_state_rows(&geo) == L, "state rows");
  int32_t slots[F * F];
  CHECK(ditango_slot_table(&geo, slots) == DITANGO_OK, "slot table");
  CHECK(slots[0] == 0 && slots[1] == 1 && slots[2] == -1, "row 0 slots");
  CHECK(slots[(F - 1) * F + 0] == active - 3 && slots[(F - 1) * F + F - 1] == active - 1, "last row slots");

  /* KV groups {0}, {1, 2, 3}, {4, 5, 6, 7}: row 5 attends 0, 4, 5, 6 */
  int32_t groups[4] = {0, 1, 4, 8};
  geo.G = 3;
  geo.group_off = groups;
  CHECK(ditango_check_geom(&geo) == DITANGO_OK, "grouped geometry");
  int32_t gslots[F * 3];
  CHECK(ditango_slot_table(&geo, gslots) == DITANGO_OK, "grouped slot table");
  CHECK(gslots[5 * 3 + 0] >= 0 && gslots[5 * 3 + 1] == -1 && gslots[5 * 3 + 2] >= 0, "row 5 units");
  printf("active_units %lld\n", (long long)ditango_num_active(&geo));

  /* bad groupings and shapes are refused */
  int32_t bad_groups[3] = {0, 5, 7};   /* does not end at P */
  geo.group_off = bad_groups;
  geo.G = 2;
  CHECK(ditango_check_geom(&geo) == DITANGO_ERR_INVALID, "groups not ending at P");
  geo.G = 0;
  geo.group_off = NULL;
  geo.d = 80;
  CHECK(ditango_check_geom(&geo) == DITANGO_ERR_UNSUPPORTED, "d = 80");
  geo.d = 96;

  /* launching calls validate their arguments first (no GPU needed to fail) */
  CHECK(ditango_plan(&geo, NULL, NULL, 1, 0.5, 0, NULL, NULL, NULL, NULL, NULL, 0, NULL) ==
            DITANGO_ERR_INVALID, "plan without buffers");
  CHECK(ditango_merge(&geo, NULL, NULL, NULL, NULL, NULL, NULL, 0, 0, NULL, 1, NULL, NULL, NULL, NULL) ==
            DITANGO_ERR_INVALID, "merge without buffers");
  CHECK(ditango_plan_error(&geo, NULL, NULL, 1, 0.5, 1, 0, NULL, NULL, NULL, NULL, NULL, NULL, 0,
                           NULL) == DITANGO_ERR_INVALID, "error plan without its state");
  {
    /* a plan from mass partials needs the partials, of the plan workspace's size */
    void *fake = (void *)(uintptr_t)4096;   /* never dereferenced: refused first */
    CHECK(ditango_plan_from_mass(&geo, NULL, 0, NULL, 1, 0.5, (int8_t *)fake, (int32_t *)fake,
                                 (int32_t *)fake, NULL, NULL) == DITANGO_ERR_INVALID,
          "plan from mass without partials");
    CHECK(ditango_plan_from_mass(&geo, (float *)fake, ditango_plan_workspace_size(&geo) - 4,
                                 NULL, 1, 0.5, (int8_t *)fake, (int32_t *)fake, (int32_t *)fake,
                                 NULL, NULL) == DITANGO_ERR_INVALID,
          "plan from mass partials that are too small");
  }
  {
    /* composing into groups that are not a coarsening of the fine ones */
    ditango_geom fine = geo, coarse = geo;
    int32_t fine_groups[3] = {0, 4, 8}, coarse_groups[3] = {0, 2, 8};
    fine.G = 2;
    fine.group_off = fine_groups;
    coarse.G = 2;
    coarse.group_off = coarse_groups;
    void *fake = (void *)(uintptr_t)4096;   /* never dereferenced: refused first */
    CHECK(ditango_cache_compose(&fine, &coarse, fake, (const float *)fake, NULL, fake,
                                (float *)fake, NULL, 0, NULL) == DITANGO_ERR_INVALID,
          "compose into a grouping that is not coarser");
  }
  CHECK(ditango_selftest_bounded_wait(0, NULL, NULL) == DITANGO_ERR_INVALID, "selftest limit 0");
  CHECK(strcmp(ditango_status_string(DITANGO_ERR_TIMEOUT), "device wait timed out") == 0, "status string");
  ditango_set_wait_limit_ns(2000000);
  printf("fails %d\n", fails);
  return fails != 0;
}
