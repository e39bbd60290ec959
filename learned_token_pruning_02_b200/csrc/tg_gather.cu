// Forward the kept hidden states, their original positions and gate values.
//
// TokenGate paper page (thelatestinai.com), Figure 1(b): the top-K selector forwards the
// kept hidden states together with their importance scores; aitualizate.com article,
// phase 3: layers above L receive only the kept tokens.
//
// Design (B200): a pure HBM copy. One warp moves one kept row with 16-byte vector loads
// and stores (a 2048-wide bf16 row is 4 KB = 8 x 16 B per lane), all loads of a row issued
// before its stores so each warp keeps 4 KB in flight. Lane 0 also writes pos = row index
// within its sequence, g = sigmoid(score) and log g (stable log-sigmoid). Grid-stride over
// rows with a grid of a few waves of the SM count.
#include "tg_internal.cuh"
#include "tg_sm100.cuh"

namespace tg {
namespace {

struct GatherParams {
  GatherSeq s[kMaxSeqPerLaunch];
  int nseq;
};

constexpr int WARPS = 4;
constexpr int MAXV = 8;  // 16-byte vectors per lane held in registers per pass

template <bool WAIT_LAST>
__global__ void __launch_bounds__(WARPS * 32)
    gather_kernel(const uint4* __restrict__ H, int64_t ldv, int nvec, const float* __restrict__ score,
                  const int32_t* __restrict__ kept, uint32_t flags, uint4* __restrict__ Hk, int32_t* __restrict__ pos,
                  float* __restrict__ g, float* __restrict__ logg, int32_t* __restrict__ dev_status, int m_chunk,
                  const __grid_constant__ GatherParams p) {
  const int lane = threadIdx.x & 31;
  const int row0 = p.s[0].out_off;
  sm100::griddep_launch_dependents();  // the next kernel may start its prologue
  if (!WAIT_LAST) sm100::griddep_wait();  // the kept indices of the previous kernel are visible
  for (int r = blockIdx.x * WARPS + (threadIdx.x >> 5); r < m_chunk; r += gridDim.x * WARPS) {
    const int row = row0 + r;
    int b = 0;
    while (b + 1 < p.nseq && row >= p.s[b + 1].out_off) ++b;
    const GatherSeq sq = p.s[b];
    const int32_t j = __ldcg(kept + row);
    if (j < sq.start || j >= sq.start + sq.n) {
      if (lane == 0 && dev_status) atomicOr(dev_status, TG_DEV_BAD_INDEX);
      continue;
    }
    // the score load goes out together with the row loads (one round trip, not two)
    const float s = (lane == 0 && (g || logg)) ? __ldcg(score + j) : 0.f;
    const uint4* src = H + (int64_t)j * ldv;
    uint4* dst = Hk + (int64_t)row * nvec;
    for (int v0 = 0; v0 < nvec; v0 += 32 * MAXV) {
      uint4 buf[MAXV];
#pragma unroll
      for (int u = 0; u < MAXV; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < nvec) buf[u] = __ldcs(src + v);
      }
#pragma unroll
      for (int u = 0; u < MAXV; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < nvec) __stcs(dst + v, buf[u]);
      }
    }
    if (lane == 0) {
      if (pos) pos[row] = j - sq.start;
      if (g || logg) {
        float gv, lg;
        if ((flags & TG_QUESTION_GATE_ONE) && (row - sq.out_off) >= sq.m - sq.q) {
          gv = 1.f;
          lg = 0.f;
        } else {
          gate_from_score(s, &gv, &lg);
        }
        if (g) g[row] = gv;
        if (logg) logg[row] = lg;
      }
    }
  }
  // the kernel before this one only ends after it: the gather completes after it too, so stream
  // order past the gather still means past both
  if (WAIT_LAST) sm100::griddep_wait();
}

}  // namespace

tg_status launch_gather(tg_dtype dt, const void* H, int64_t ldh, int d, const float* score, const int32_t* kept_idx,
                        const GatherSeq* seqs, int nseq, int m_chunk, uint32_t flags, void* H_kept, int32_t* pos,
                        float* g, float* logg, int32_t* dev_status, cudaStream_t st,
                        bool after_kernel_reads_nothing) {
  GatherParams p = {};
  for (int i = 0; i < nseq; ++i) p.s[i] = seqs[i];
  p.nseq = nseq;
  const int es = dt == TG_BF16 ? 2 : 4;
  const int nvec = d * es / 16;
  const int64_t ldv = ldh * es / 16;
  if (attrs_needed(ATTR_GATHER)) {  // the carveout of the other chain kernels: no reconfiguration between them
    for (auto k : {gather_kernel<false>, gather_kernel<true>}) {
      cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                                           (int)cudaSharedmemCarveoutMaxShared);
      if (e != cudaSuccess) return cuda_status(e, "gather: cudaFuncSetAttribute");
    }
    mark_attrs_set(ATTR_GATHER);
  }
  int blocks = (m_chunk + WARPS - 1) / WARPS;
  const int cap = device_sm_count() * 16;
  if (blocks > cap) blocks = cap;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(WARPS * 32);
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attribute(PDL_GATHER)};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, after_kernel_reads_nothing ? gather_kernel<true> : gather_kernel<false>,
                                        static_cast<const uint4*>(H), ldv, nvec, score, kept_idx,
                                        flags, static_cast<uint4*>(H_kept), pos, g, logg, dev_status, m_chunk, p),
                     "gather launch");
}

}  // namespace tg
