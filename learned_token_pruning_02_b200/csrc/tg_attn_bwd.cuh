// Declarations of the gated-attention backward, shared by its kernels and the C ABI.
#pragma once

#include "tg_internal.cuh"

namespace tg {

// Function-attribute slots of the backward's kernels (after the forward path's slots):
// CUDA-core (f32) D 64, 128, then tensor-core (bf16) D 64, 128.
enum { ATTR_BWD = ATTR_SLOTS, ATTR_ALL = ATTR_BWD + 4 };

// Gradients of the gated attention (normalised form): dQ, dK, dV (f32) and optionally d log g,
// d score (f32), from the forward's inputs, O and lse and the upstream dO.
struct AttnBwdArgs {
  tg_dtype dt;
  const void* Q;
  const void* K;
  const void* V;
  const void* O;
  const void* dO;
  const float* logg;
  const float* head_gain;
  const int32_t* pos;
  const float* lse;
  int Hq, Hkv, D;
  float scale;
  float* dQ;
  float* dK;
  float* dV;
  float* dlogg;
  float* dscore;
  int32_t* dev_status;
  int64_t m_tot;
};
tg_status launch_attn_bwd(const AttnBwdArgs& a, const AttnSeq* seqs, int nseq, cudaStream_t st);
// bf16 on the tensor cores (tcgen05); called by launch_attn_bwd
tg_status launch_attn_bwd_tc(const AttnBwdArgs& a, const AttnSeq* seqs, int nseq, cudaStream_t st);

}  // namespace tg
