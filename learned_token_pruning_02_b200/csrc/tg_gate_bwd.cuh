// Gate-network parameter gradients (tg_gate_mlp_bwd): workspace plan and launcher.
#pragma once

#include "tg_internal.cuh"

namespace tg {

// Workspace layout for M kept rows: u [M, dg] fp32 at 0; the row tiles' column sums of u and of
// ds' GELU(z) at off_part; with more than one row split, the splits' dW1 blocks at off_w.
struct GateBwdPlan {
  int n_tiles = 0;         // 64-row tiles
  int splits = 1;          // row splits of the dW1 accumulation
  int rows_per_split = 0;
  int64_t off_part = 0, off_w = 0, bytes = 0;
};

GateBwdPlan gate_bwd_plan(int64_t M, int d, int dg, int sms);

// Device address, on the current device, of the library's fixed scratch array for
// tg_gate_mlp_bwd_noalloc (TG_GATE_NOALLOC_SCRATCH_BYTES); looked up once per device.
tg_status gate_bwd_fixed_scratch(void** ptr);

tg_status launch_gate_bwd(tg_dtype dt, const void* H, int64_t M, int d, const void* W1, const float* b1,
                          const void* w2, float inv_t, int dg, const float* dscore, float* dW1, float* db1,
                          float* dw2, float* db2, void* ws, const GateBwdPlan& p, cudaStream_t st);

}  // namespace tg
