// Gate-network parameter gradients (tg_gate_mlp_bwd): workspace plan and launcher.
#pragma once

#include "tg_internal.cuh"

namespace tg {

// Workspace layouts for M kept rows; the workspace query has no dtype, so `bytes` covers both.
// CUDA-core kernels: u [M, dg] fp32 at 0; the row tiles' column sums of u and of ds' GELU(z) at
// off_part; with more than one row split, the splits' dW1 blocks at off_w.
// Tensor-core kernels (bf16, tc set): u^T [dg, tc_Mp] bf16 at 0; the 256-row block sums of u, of
// ds' GELU(z) and of ds' at tc_off_part; at tc_off_big the split partials of z [tc_ks][dg][tc_Mp]
// fp32, and after they are consumed, with more than one split of the kept rows, the splits' dW1
// blocks.
struct GateBwdPlan {
  int n_tiles = 0;         // 64-row tiles
  int splits = 1;          // row splits of the dW1 accumulation
  int rows_per_split = 0;
  int64_t off_part = 0, off_w = 0;
  bool tc = false;         // the shape suits the tensor-core kernels
  int tc_Mp = 0;           // kept rows rounded up to 128
  int tc_ks = 1;           // splits of the first product's K (columns of d)
  int tc_ublocks = 0;      // 256-row blocks of the u pass
  int tc_nchunk = 0;       // 64-row chunks of the kept rows
  int tc_cps = 0;          // chunks per split
  int tc_splits = 1;
  int64_t tc_off_part = 0, tc_off_big = 0, tc_bytes = 0;
  int64_t bytes = 0;
};

GateBwdPlan gate_bwd_plan(int64_t M, int d, int dg, int sms);

// Tensor-core kernels (csrc/tg_gate_bwd_tc.cu): the shapes they take (dg and d multiples of
// 128), their part of the plan, and their launcher.
bool gate_bwd_tc_shape(int64_t M, int d, int dg);
void gate_bwd_tc_plan(GateBwdPlan& p, int64_t M, int d, int dg, int sms);
tg_status launch_gate_bwd_tc(const void* H, int64_t M, int d, const void* W1, const float* b1, const void* w2,
                             float inv_t, int dg, const float* dscore, float* dW1, float* db1, float* dw2, float* db2,
                             void* ws, const GateBwdPlan& p, int32_t* dev_status, cudaStream_t st);

// Device address, on the current device, of the library's fixed scratch array for
// tg_gate_mlp_bwd_noalloc (TG_GATE_NOALLOC_SCRATCH_BYTES); looked up once per device.
tg_status gate_bwd_fixed_scratch(void** ptr);

tg_status launch_gate_bwd(tg_dtype dt, const void* H, int64_t M, int d, const void* W1, const float* b1,
                          const void* w2, float inv_t, int dg, const float* dscore, float* dW1, float* db1,
                          float* dw2, float* db2, void* ws, const GateBwdPlan& p, int32_t* dev_status, cudaStream_t st);

}  // namespace tg
