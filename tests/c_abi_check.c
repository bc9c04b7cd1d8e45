/* A plain C consumer of libarea: includes the public header, links the
 * shared library and calls the host-side entry points (no GPU needed).
 * Exit code 0 when every check holds; the failing check's number otherwise. */
#include <stdio.h>
#include <string.h>

#include "area.h"

int main(void) {
  if (strncmp(area_version(), "libarea", 7) != 0) return 1;
  if (area_status_string(AREA_EINVAL) == NULL) return 2;

  /* plan sizing for a 256 x 256 grid, w = 64 */
  area_plan_cfg cfg = {1, 256, 256, 64, 4, 512, 0.4f, 0ull};
  size_t nb = 0;
  if (area_window_plan_bytes(&cfg, &nb) != AREA_OK || nb == 0 || nb % 256 != 0) return 3;
  /* merge workspace: a header of 1 + 4 * B * H counters (4 * 97 bytes for
   * 24 heads, rounded up to 512) plus one fp32 row per overlapped token and
   * head; 64-token windows tile 256 exactly (no overlap), 80-token windows
   * (starts 0, 58, 117, 176) overlap on 64 positions per axis, so on
   * 64 * 256 + 192 * 64 = 28672 tokens */
  size_t ws = 0;
  if (area_window_attn_ws_bytes(&cfg, 24, 128, &ws) != AREA_OK || ws != 512) return 4;
  area_plan_cfg cfg80 = {1, 256, 256, 80, 4, 512, 0.4f, 0ull};
  if (area_window_attn_ws_bytes(&cfg80, 24, 128, &ws) != AREA_OK ||
      ws != (size_t)512 + (size_t)24 * 28672 * 128 * 4)
    return 4;
  /* staging area of the global-KV rows: K and V, [B][H][nw][G][D] bf16 each,
   * nw = 4 final windows per base window = 4 * 16 at w = 64 */
  size_t sb = 0;
  if (area_window_attn_stage_bytes(&cfg, 24, 128, &sb) != AREA_OK ||
      sb != (size_t)2 * 24 * 64 * 512 * 128 * 2)
    return 13;

  /* the printed pooling ramp at a 256 x 256 grid */
  const int want[8] = {4, 4, 4, 4, 2, 2, 2, 2};
  int ramp[8];
  if (area_pool_ramp(4, 2, 8, 256, 256, ramp) != AREA_OK) return 5;
  for (int i = 0; i < 8; ++i)
    if (ramp[i] != want[i]) return 6;

  /* noise-level switch over a 28-step flow-matching sampler (shift 3) */
  float sig[28];
  for (int i = 0; i < 28; ++i) {
    const double t = 1.0 - i / 28.0;
    sig[i] = (float)(3.0 * t / (1.0 + 2.0 * t));
  }
  int n1 = -1;
  if (area_phase_switch(sig, 28, 0.89f, &n1) != AREA_OK || n1 != 8) return 7;
  int kind[28], param[28];
  if (area_schedule(sig, 28, 0.89f, 4, 2, 256, 64, 256, 256, kind, param) != AREA_OK) return 8;
  if (kind[7] != AREA_PHASE_COARSE || kind[8] != AREA_PHASE_WINDOW) return 9;
  if (param[8] != 256 || param[27] != 64) return 10;

  /* argument validation answers before any device work */
  if (area_pool_kv(NULL, NULL, NULL, NULL, 1, 1, 4, 4, 8, 2, AREA_POOL_MEAN, AREA_DTYPE_BF16, 0) !=
      AREA_EINVAL)
    return 11;
  size_t bws = 0;
  if (area_bridge_select_ws_bytes(1, 24, 384, 384, 128, &bws) != AREA_OK ||
      bws != (size_t)24 * 128 * (1 + 144) * 4)
    return 12;
  printf("%s: C-ABI host checks passed\n", area_version());
  return 0;
}
