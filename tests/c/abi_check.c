/* A C program against the library's C ABI: include/moe.h compiles as C99 (and
 * as C++), the library links from C, and the host-side checks behave as the
 * header states.  Every call made here returns before anything touches a GPU:
 * plan building, status strings, and argument checks that fail before the
 * first launch. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "moe.h"

static int failures = 0;

#define EXPECT(cond)                                             \
  do {                                                           \
    if (!(cond)) {                                               \
      printf("FAILED line %d: %s\n", __LINE__, #cond);           \
      ++failures;                                                \
    }                                                            \
  } while (0)

static moe_status plan_status(int T, int H, int I, int E, int k, int w_dtype) {
  moe_dtypes dt;
  moe_act_params act;
  moe_plan_t p = NULL;
  moe_status s;
  dt.w_dtype = w_dtype;
  act.kind = MOE_ACT_SWIGLU;
  act.alpha = 1.0f;
  act.up_bias = 0.0f;
  act.limit = INFINITY;
  s = moe_plan(T, H, I, E, k, dt, act, &p);
  EXPECT((s == MOE_OK) == (p != NULL));
  moe_plan_destroy(p);
  return s;
}

int main(void) {
  moe_dtypes dt;
  moe_act_params act;
  moe_plan_t plan = NULL;
  /* Never dereferenced: every call below fails its checks before any launch. */
  void *ws = (void *)(uintptr_t)0x10000000u;
  void *ws_misaligned = (void *)(uintptr_t)0x10000010u;
  const void *dev = (const void *)(uintptr_t)0x20000000u;
  const uint8_t *u8 = (const uint8_t *)(uintptr_t)0x20000000u;
  const int32_t *i32 = (const int32_t *)(uintptr_t)0x20000000u;
  const float *f32 = (const float *)(uintptr_t)0x20000000u;
  int32_t *o32 = (int32_t *)ws;
  int code;

  /* Plan checks, with the status each requirement returns. */
  EXPECT(plan_status(64, 512, 256, 8, 2, MOE_W_E4M3_UE8M0_128x128) == MOE_OK);
  EXPECT(plan_status(64, 512, 256, 8, 2, MOE_W_E2M1_UE8M0_1x32) == MOE_OK);
  EXPECT(plan_status(64, 512, 256, 8, 2, MOE_W_BF16) == MOE_OK);
  EXPECT(plan_status(0, 512, 256, 8, 2, 0) == MOE_ERR_INVALID_ARG);    /* T >= 1 */
  EXPECT(plan_status(4, 512, 256, 2, 3, 0) == MOE_ERR_INVALID_ARG);    /* k <= E */
  EXPECT(plan_status(4, 384, 256, 8, 2, 0) == MOE_ERR_UNSUPPORTED);    /* H % 256 */
  EXPECT(plan_status(4, 512, 200, 8, 2, 0) == MOE_ERR_UNSUPPORTED);    /* I % 128 */
  EXPECT(plan_status(4, 512, 256, 300, 2, 0) == MOE_ERR_UNSUPPORTED);  /* E <= 256 */
  EXPECT(plan_status(4, 512, 256, 8, 2, 7) == MOE_ERR_INVALID_ARG);    /* w_dtype */

  dt.w_dtype = MOE_W_E4M3_UE8M0_128x128;
  act.kind = MOE_ACT_SWIGLU_OAI;
  act.alpha = 1.702f;
  act.up_bias = 1.0f;
  act.limit = -1.0f;
  EXPECT(moe_plan(4, 512, 256, 8, 2, dt, act, &plan) == MOE_ERR_INVALID_ARG && plan == NULL);
  act.limit = 7.0f;
  EXPECT(moe_plan(4, 512, 256, 8, 2, dt, act, NULL) == MOE_ERR_INVALID_ARG);
  EXPECT(moe_plan(4, 512, 256, 8, 2, dt, act, &plan) == MOE_OK && plan != NULL);

  EXPECT(moe_workspace_bytes(plan) > 0);
  EXPECT(moe_workspace_bytes(NULL) == 0);
  EXPECT(moe_forward_launch_count(plan) > 0);

  /* Argument checks of moe_forward, all before the first launch. */
  EXPECT(moe_forward(NULL, dev, u8, i32, f32, dev, u8, dev, u8, ws, ws, NULL) ==
         MOE_ERR_INVALID_ARG);
  EXPECT(moe_forward(plan, dev, u8, i32, f32, dev, u8, dev, u8, ws, NULL, NULL) ==
         MOE_ERR_INVALID_ARG);
  EXPECT(moe_forward(plan, dev, u8, i32, f32, dev, u8, dev, u8, ws, ws_misaligned, NULL) ==
         MOE_ERR_ALIGNMENT);
  EXPECT(moe_forward(plan, NULL, u8, i32, f32, dev, u8, dev, u8, ws, ws, NULL) ==
         MOE_ERR_INVALID_ARG);
  EXPECT(moe_forward(plan, dev, NULL, i32, f32, dev, u8, dev, u8, ws, ws, NULL) ==
         MOE_ERR_INVALID_ARG);
  EXPECT(moe_forward(plan, u8 + 8, u8, i32, f32, dev, u8, dev, u8, ws, ws, NULL) ==
         MOE_ERR_ALIGNMENT);

  /* Plan settings outside their ranges. */
  EXPECT(moe_plan_set_swap_ab(plan, 3) == MOE_ERR_INVALID_ARG);
  EXPECT(moe_plan_set_swap_ab(NULL, 0) == MOE_ERR_INVALID_ARG);
  EXPECT(moe_plan_set_cta_pairs(plan, -1) == MOE_ERR_INVALID_ARG);
  EXPECT(moe_plan_set_debug(plan, 4) == MOE_ERR_INVALID_ARG);
  EXPECT(moe_plan_set_weight_layout(plan, 9) == MOE_ERR_INVALID_ARG);
  EXPECT(moe_plan_set_weight_layout(plan, MOE_WEIGHTS_SCALES_CHUNKED) == MOE_ERR_UNSUPPORTED);
  EXPECT(moe_plan_cta_pairs_active(NULL) == 0);

  /* moe_route_static refuses sizes beyond its static scratch before launching. */
  EXPECT(moe_route_static(i32, MOE_ROUTE_STATIC_MAX_SLOTS, 2, 8, o32, o32, o32, o32, NULL) ==
         MOE_ERR_UNSUPPORTED);

  /* Every status has a name. */
  for (code = MOE_OK; code <= MOE_ERR_BAD_ROUTING; ++code) {
    const char *name = moe_status_str((moe_status)code);
    EXPECT(name != NULL && strncmp(name, "MOE_", 4) == 0);
  }
  EXPECT(strcmp(moe_status_str(MOE_OK), "MOE_OK") == 0);

  moe_plan_destroy(plan);
  moe_plan_destroy(NULL);
  if (failures == 0) printf("abi ok\n");
  return failures == 0 ? 0 : 1;
}
