// Token-gated causal attention on the CUDA cores (fp32 arithmetic), used for float32
// tensors where the 1e-4 tolerance rules out reduced-precision tensor-core math.
//
// TokenGate paper page (thelatestinai.com), Figure 1(c): each attention weight is multiplied
// by its key's gate value g_j; with the row renormalised that is log g_j added to the logit
// (aitualizate.com article: the score becomes a bias on the attention logits, with a
// per-head gain). Causal on original positions; grouped KV heads (kv = h / (Hq/Hkv)).
//
// One warp per (query row, head); lanes split the head dimension; keys are visited in
// index order with an online (running max) softmax in base 2.
#include <math.h>

#include "tg_internal.cuh"

namespace tg {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int WARPS = 8;

struct AttnParams {
  AttnSeq s[kMaxSeqPerLaunch];
  int groups[kMaxSeqPerLaunch + 1];  // prefix sums of ceil(m / WARPS) row groups
  int nseq;
};

__device__ __forceinline__ float ldf(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ldf(const __nv_bfloat16* p, int64_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ void stf(float* p, int64_t i, float v) { p[i] = v; }
__device__ __forceinline__ void stf(__nv_bfloat16* p, int64_t i, float v) { p[i] = __float2bfloat16_rn(v); }

template <typename T, int D>
__global__ void __launch_bounds__(WARPS * 32)
    attn_simt_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
                     const float* __restrict__ logg, const float* __restrict__ gain, const int32_t* __restrict__ pos,
                     int Hq, int Hkv, float scale, uint32_t flags, T* __restrict__ O, float* __restrict__ lse,
                     int64_t m_tot, int32_t* __restrict__ dev_status, const __grid_constant__ AttnParams p) {
  constexpr int EPL = D / 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int h = blockIdx.y;
  const int grp = blockIdx.x;
  int b = 0;
  while (b + 1 < p.nseq && grp >= p.groups[b + 1]) ++b;
  const AttnSeq sq = p.s[b];
  const int li = (grp - p.groups[b]) * WARPS + w;
  if (li >= sq.m) return;
  const int64_t i = sq.off + li;
  const int kv = h / (Hq / Hkv);
  const bool unnorm = (flags & TG_ATTN_UNNORMALISED) != 0;
  const float gain2 = (gain ? gain[h] : 1.f) * kLog2e;
  const float qs = scale * kLog2e;
  float qv[EPL], acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    qv[e] = ldf(Q, (i * Hq + h) * D + lane * EPL + e) * qs;
    acc[e] = 0.f;
  }
  const int32_t pos_i = pos[i];
  if (h == 0 && lane == 0 && li > 0 && pos[i - 1] >= pos_i && dev_status) atomicOr(dev_status, TG_DEV_POS_NOT_ASCENDING);
  float m = -INFINITY, l = 0.f;
  for (int64_t j = sq.off; j <= i; ++j) {
    if (pos[j] > pos_i) continue;
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) dot = fmaf(qv[e], ldf(K, (j * Hkv + kv) * D + lane * EPL + e), dot);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    const float lgj = logg ? logg[j] : 0.f;
    const float b2 = lgj == -INFINITY ? -INFINITY : gain2 * lgj;  // gain * log2(g_j); g = 0 closes the key
    const float s2 = unnorm ? dot : dot + b2;
    if (s2 == -INFINITY) continue;
    const float mn = fmaxf(m, s2);
    const float corr = exp2f(m - mn);
    const float pe = exp2f(s2 - mn);
    const float wv = unnorm ? pe * exp2f(b2) : pe;
    l = l * corr + pe;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = fmaf(wv, ldf(V, (j * Hkv + kv) * D + lane * EPL + e), acc[e] * corr);
    m = mn;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) stf(O, (i * Hq + h) * D + lane * EPL + e, acc[e] * inv);
  if (lse && lane == 0) lse[(int64_t)h * m_tot + i] = (m + log2f(l)) * kLn2;
}

template <typename T>
tg_status launch_t(const AttnArgs& a, const AttnSeq* seqs, int nseq, cudaStream_t st) {
  AttnParams p = {};
  p.nseq = nseq;
  p.groups[0] = 0;
  for (int i = 0; i < nseq; ++i) {
    p.s[i] = seqs[i];
    p.groups[i + 1] = p.groups[i] + (seqs[i].m + WARPS - 1) / WARPS;
  }
  if (p.groups[nseq] == 0) return TG_OK;
  dim3 grid((unsigned)p.groups[nseq], (unsigned)a.Hq);
  const T* q = static_cast<const T*>(a.Q);
  const T* k = static_cast<const T*>(a.K);
  const T* v = static_cast<const T*>(a.V);
  T* o = static_cast<T*>(a.O);
  if (a.D == 64)
    attn_simt_kernel<T, 64><<<grid, WARPS * 32, 0, st>>>(q, k, v, a.logg, a.head_gain, a.pos, a.Hq, a.Hkv, a.scale,
                                                         a.flags, o, a.lse, a.m_tot, a.dev_status, p);
  else
    attn_simt_kernel<T, 128><<<grid, WARPS * 32, 0, st>>>(q, k, v, a.logg, a.head_gain, a.pos, a.Hq, a.Hkv, a.scale,
                                                          a.flags, o, a.lse, a.m_tot, a.dev_status, p);
  return cuda_status(cudaGetLastError(), "attn_simt launch");
}

}  // namespace

tg_status launch_attn_simt(const AttnArgs& a, const AttnSeq* seqs, int nseq, cudaStream_t st) {
  if (a.dt == TG_BF16) return launch_t<__nv_bfloat16>(a, seqs, nseq, st);
  return launch_t<float>(a, seqs, nseq, st);
}

}  // namespace tg
