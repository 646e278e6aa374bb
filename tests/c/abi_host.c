/* A plain C (C11) user of the C ABI: host-only plan, plan info, workspace size
   and error reporting.  No GPU is needed.  Prints one line of results; exit code
   0 on success. */
#include <stdio.h>
#include <string.h>

#include "tileshare.h"
#include "tileshare_ops.h"

int main(void) {
  const int grid[3] = {1, 48, 48}, win[3] = {1, 16, 16}, stride[3] = {1, 12, 12};
  ts_plan_t plan = NULL;
  if (ts_plan_create_host_registers(grid, win, stride, TS_BLEND_LINEAR_RAMP, 2, &plan) != TS_OK) return 1;
  ts_plan_desc d;
  memset(&d, 0, sizeof d);
  if (ts_plan_info(plan, &d) != TS_OK) return 2;
  ts_model_desc m;
  memset(&m, 0, sizeof m);
  m.d = 512;
  m.heads = 8;
  m.mlp = 2048;
  m.dtype = TS_BF16;
  m.eps_ln = 1e-6f;
  m.eps_qk = 1e-6f;
  m.rope_base = 10000.0f;
  m.rope_dims[0] = 0;
  m.rope_dims[1] = 32;
  m.rope_dims[2] = 32;
  m.block = TS_BLOCK_RMS_SWIGLU;
  size_t ws = 0;
  if (ts_workspace_size(plan, &m, 8, 2, &ws) != TS_OK) return 3;
  /* a bad argument is refused with a status and a reason, nothing aborts */
  const ts_status bad = ts_workspace_size(plan, &m, 4, 5, &ws);
  const char* why = ts_last_error();
  printf("T=%d U=%d Nw=%d N=%d R=%d nnz=%d max_cover=%d device=%d ws=%zu bad=%d reason=%s status=%s\n", d.T, d.U,
         d.Nw, d.N, d.R, d.nnz, d.max_cover, d.device, ws, (int)bad, why ? why : "", ts_status_string(bad));
  ts_plan_destroy(plan);
  return bad == TS_ERR_INVALID_ARG ? 0 : 4;
}
