// Gate-MLP score on the CUDA cores (fp32 arithmetic): score = (w2 . GELU(W1 h + b1) + b2) / temperature.
// Used for float32 inputs, where the 1e-4 tolerance rules out TF32 tensor-core math.
// TokenGate paper page (thelatestinai.com), Figure 1(b): a small scoring network scores
// every hidden state at the selection layer.
#include "tg_internal.cuh"

namespace tg {
namespace {

constexpr int TM = 32;   // tokens per block
constexpr int TK = 32;   // d-chunk staged in shared memory
constexpr int NT = 256;  // threads: 8 token groups x 32 hidden-unit lanes

__device__ __forceinline__ float ld_act(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ld_act(const __nv_bfloat16* p, int64_t i) { return __bfloat162float(p[i]); }

template <typename T, int DG>
__global__ void __launch_bounds__(NT) score_simt_kernel(const T* __restrict__ H, int64_t ldh, int n_tok, int d,
                                                        const T* __restrict__ W1, const float* __restrict__ b1,
                                                        const T* __restrict__ w2, float b2, float inv_t, float* __restrict__ score) {
  constexpr int CPT = DG / 32;  // hidden units per thread
  __shared__ float hs[TM][TK + 1];
  __shared__ float ws[DG][TK + 1];
  const int tx = threadIdx.x & 31;  // hidden-unit lane
  const int ty = threadIdx.x >> 5;  // token group (4 tokens each)
  const int64_t tok0 = (int64_t)blockIdx.x * TM;
  float acc[4][CPT];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int c = 0; c < CPT; ++c) acc[i][c] = 0.f;

  for (int k0 = 0; k0 < d; k0 += TK) {
    for (int e = threadIdx.x; e < TM * TK; e += NT) {
      int r = e / TK, c = e % TK;
      int64_t t = tok0 + r;
      hs[r][c] = (t < n_tok) ? ld_act(H, t * ldh + k0 + c) : 0.f;
    }
    for (int e = threadIdx.x; e < DG * TK; e += NT) {
      int r = e / TK, c = e % TK;
      ws[r][c] = ld_act(W1, (int64_t)r * d + k0 + c);
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], w[CPT];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = hs[ty * 4 + i][kk];
#pragma unroll
      for (int c = 0; c < CPT; ++c) w[c] = ws[tx + 32 * c][kk];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < CPT; ++c) acc[i][c] = fmaf(a[i], w[c], acc[i][c]);
    }
    __syncthreads();
  }
  // epilogue: + b1, exact-erf GELU, times w2, reduce over the hidden units
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float part = 0.f;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      int u = tx + 32 * c;
      float z = acc[i][c] + (b1 ? b1[u] : 0.f);
      float gz = 0.5f * z * (1.f + erff(z * 0.70710678118654752f));
      part = fmaf(gz, ld_act(w2, u), part);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    int64_t t = tok0 + ty * 4 + i;
    if (tx == 0 && t < n_tok) score[t] = (part + b2) * inv_t;
  }
}

template <typename T>
tg_status launch_t(const void* H, int64_t ldh, int64_t n_tok, int d, const void* W1, const float* b1,
                   const void* w2, float b2, float inv_t, int dg, float* score, cudaStream_t st) {
  dim3 grid((unsigned)((n_tok + TM - 1) / TM));
  const T* h = static_cast<const T*>(H);
  const T* w = static_cast<const T*>(W1);
  const T* v = static_cast<const T*>(w2);
  if (dg == 64) score_simt_kernel<T, 64><<<grid, NT, 0, st>>>(h, ldh, (int)n_tok, d, w, b1, v, b2, inv_t, score);
  else if (dg == 128) score_simt_kernel<T, 128><<<grid, NT, 0, st>>>(h, ldh, (int)n_tok, d, w, b1, v, b2, inv_t, score);
  else score_simt_kernel<T, 256><<<grid, NT, 0, st>>>(h, ldh, (int)n_tok, d, w, b1, v, b2, inv_t, score);
  return cuda_status(cudaGetLastError(), "score_simt launch");
}

}  // namespace

tg_status launch_score_simt(tg_dtype dt, const void* H, int64_t ldh, int64_t n_tok, int d, const void* W1,
                            const float* b1, const void* w2, float b2, float inv_t, int dg, float* score,
                            cudaStream_t st) {
  if (dt == TG_BF16) return launch_t<__nv_bfloat16>(H, ldh, n_tok, d, W1, b1, w2, b2, inv_t, dg, score, st);
  return launch_t<float>(H, ldh, n_tok, d, W1, b1, w2, b2, inv_t, dg, score, st);
}

}  // namespace tg
