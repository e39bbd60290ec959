// Internal declarations shared by the CUDA translation units of libtokengate.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tokengate.h"

namespace tg {

constexpr int kMaxSeqPerLaunch = 64;  // per-sequence descriptors travel as kernel params

// ----------------------------------------------------------------------------- error text
void set_error(const char* fmt, ...);
tg_status fail(tg_status st, const char* fmt, ...);
tg_status cuda_status(cudaError_t e, const char* what);

// Checks that the current device is a B200-class part (compute capability 10.x) once per
// device; returns TG_ERR_UNSUPPORTED otherwise.
tg_status check_device();
int device_sm_count();

// Limit of the test-only wait probe of the tensor-core kernels on this thread (0 = off; set by
// tg_set_test_wait_probe). A kernel given a non-zero limit waits that long on a barrier that
// nothing signals, records TG_DEV_TIMEOUT and skips all of its work.
uint64_t wait_probe_ns();

// Function attributes (shared-memory size, carveout) apply per device. True until
// mark_attrs_set(slot) is called on the current device; slots name the launchers.
// Template kernels take one slot per instantiation (score: dg 64/128/256; attention: D 64/128
// times the normalised / unnormalised form; projection: 128- and 256-row tiles).
enum {
  ATTR_SCORE64 = 0, ATTR_SCORE128, ATTR_SCORE256,
  ATTR_SELECT, ATTR_GATHER,
  ATTR_ATTN64, ATTR_ATTN64_UN, ATTR_ATTN128, ATTR_ATTN128_UN,
  ATTR_QKV, ATTR_GATE_TC, ATTR_QKV2, ATTR_SLOTS
};
bool attrs_needed(int slot);
void mark_attrs_set(int slot);

// Launch attribute for programmatic dependent launch (the tensor-core chain kernels start
// their prologue while the previous kernel drains; each waits on griddepcontrol.wait before
// its first global memory access). TG_DISABLE_PDL=1 in the environment turns it off.
// kernel ids for the launch-chaining mask
// (default: every bit but PDL_GATE, whose four short kernels measured slower chained than in
// plain stream order, 23.6 against 20.7 us per call replayed from a CUDA graph at 2176 x 2048)
enum { PDL_SCORE = 1, PDL_SELECT = 2, PDL_GATHER = 4, PDL_ATTN = 8, PDL_QKV = 16, PDL_BWD = 32, PDL_GATE = 64 };
bool pdl_enabled(int kernel_id);
inline cudaLaunchAttribute pdl_attribute(int kernel_id) {
  cudaLaunchAttribute a;
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = pdl_enabled(kernel_id) ? 1 : 0;
  return a;
}

// Gate value of a score and its logarithm: g = sigmoid(s), log g = log-sigmoid(s), computed
// stably for either sign of s (TokenGate paper page, Figure 1(c): the keys' gate values come
// from the selector's scores). Used wherever the chain needs g or log g, so every kernel that
// derives them gets bit-identical values.
__device__ __forceinline__ void gate_from_score(float s, float* g, float* lg) {
  const float e = expf(-fabsf(s));
  *g = s >= 0.f ? 1.f / (1.f + e) : e / (1.f + e);
  *lg = s >= 0.f ? -log1pf(e) : s - log1pf(e);
}

// ----------------------------------------------------------------------------- launchers
// Each returns TG_OK or TG_ERR_CUDA (argument checks happen in the C-ABI layer).

// inv_t = 1 / temperature multiplies the score (exactly 1 for the plain score).
tg_status launch_score_simt(tg_dtype dt, const void* H, int64_t ldh, int64_t n_tok, int d,
                            const void* W1, const float* b1, const void* w2, float b2, float inv_t, int dg,
                            float* score, cudaStream_t st);

tg_status launch_score_tc(const void* H, int64_t ldh, int64_t n_tok, int d, const void* W1,
                          const float* b1, const void* w2, float b2, float inv_t, int dg, float* score,
                          int32_t* dev_status, cudaStream_t st);

struct SelSeq {
  int32_t start;    // packed row of the sequence's first token
  int32_t n_ctx;    // context tokens N - q
  int32_t q;        // question-tail tokens
  int32_t kc;       // context tokens to keep, min(max(k,0), n_ctx)
  int32_t out_off;  // first output row (cu_kept[b])
  int32_t b;        // sequence index in the whole batch
  int32_t tail;     // index written for the first question-tail token (normally start + n_ctx)
  int32_t wbase;    // index written for context position 0 (normally start)
};

// With pos != nullptr (the chained prefill) every kept row also gets pos, g and log g, the
// values the gather writes (the question tail with g = 1 under TG_QUESTION_GATE_ONE).
// With idxmap != nullptr a kept context position p writes idxmap[start + p] instead of
// start + p, and with kept_score != nullptr each kept context row also gets its score (the
// split selection across devices: candidates, then their merge).
tg_status launch_select(const float* score, const SelSeq* seqs, int nseq, int n_ctx_max,
                        int32_t* kept_idx, int32_t* cu_kept_dev, int32_t* dev_status,
                        cudaStream_t st, int32_t* pos = nullptr, float* g = nullptr,
                        float* logg = nullptr, uint32_t flags = 0, const int32_t* idxmap = nullptr,
                        float* kept_score = nullptr);

// The many-sequence form of the select (csrc/tg_select_stream.cu): the same outputs as
// launch_select without its optional ones, from four kernels over all SMs and a workspace of
// select_stream_workspace(seqs, nseq) bytes (256-byte aligned). Any number of sequences.
int64_t select_stream_workspace(const SelSeq* seqs, int nseq);
tg_status launch_select_stream(const float* score, const SelSeq* seqs, int nseq, int32_t* kept_idx,
                               int32_t* cu_kept_dev, int32_t* dev_status, void* ws, cudaStream_t st);

struct GatherSeq {
  int32_t start;    // packed row of the sequence's first token
  int32_t n;        // tokens N
  int32_t q;        // question-tail tokens
  int32_t out_off;  // cu_kept[b]
  int32_t m;        // kept rows M_b
};

// after_kernel_reads_nothing: the previous kernel in the stream does not produce anything
// this gather reads (inside the chained prefill, attention runs between select and gather), so
// the gather starts its copies at once and waits for that kernel only before it exits.
tg_status launch_gather(tg_dtype dt, const void* H, int64_t ldh, int d, const float* score,
                        const int32_t* kept_idx, const GatherSeq* seqs, int nseq, int m_chunk,
                        uint32_t flags, void* H_kept, int32_t* pos, float* g, float* logg,
                        int32_t* dev_status, cudaStream_t st, bool after_kernel_reads_nothing = false);

struct AttnSeq {
  int32_t off;  // cu_kept[b]
  int32_t m;    // kept rows M_b
};

struct AttnArgs {
  tg_dtype dt;
  const void* Q;
  const void* K;
  const void* V;
  const float* logg;
  const float* head_gain;
  const int32_t* pos;
  int Hq, Hkv, D;
  float scale;
  uint32_t flags;
  void* O;
  float* lse;
  int32_t* dev_status;
  int64_t m_tot;
  // Q, K and V are inputs of the whole chain (the chained prefill): the kernel may load them
  // before it waits on the previous kernel.
  bool qkv_ready = false;
};

// Q/K/V = H_kept W^T with rotary embedding of Q and K at pos (bf16, tensor cores).
tg_status launch_qkv_rope(const void* Hk, int64_t M, int d, const void* W, const int32_t* pos, int Hq, int Hkv,
                          int D, float theta, void* Q, void* K, void* V, int32_t* dev_status, cudaStream_t st);

tg_status launch_attn_simt(const AttnArgs& a, const AttnSeq* seqs, int nseq, cudaStream_t st);
tg_status launch_attn_tc(const AttnArgs& a, const AttnSeq* seqs, int nseq, cudaStream_t st);

}  // namespace tg
