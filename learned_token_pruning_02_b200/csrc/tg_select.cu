// Exact, deterministic top-K over each sequence's context with the question tail kept.
//
// aitualizate.com TokenGate article, phase 2: a top-K selector keeps the K tokens with the
// highest gate score, and only the document part of the prompt may be pruned. TokenGate
// paper page (thelatestinai.com), Figure 1(a)-(b).
//
// Design (B200): one thread-block cluster per sequence (1-8 CTAs of 1024 threads). Every
// thread holds up to R order-preserving 32-bit keys in registers, so the scores are read
// from HBM exactly once. An MSB-first radix select (11 + 11 + 10 bit digits) finds the
// K-th largest key T: each CTA builds a shared-memory histogram of the keys that still
// match the prefix, the cluster barrier publishes them, and every CTA sums the cluster's
// histograms through distributed shared memory (DSMEM) and scans them itself. Then keys
// > T are kept, and keys == T are kept in index order until K is reached (lower index
// wins ties). An ascending compaction uses warp ballots and block-wide scans; CTA offsets
// come from the cluster's counts over DSMEM. Cluster barriers are hardware barriers, so
// nothing spins. No workspace: the per-sequence descriptors travel as kernel parameters.
#include <cooperative_groups.h>

#include "tg_internal.cuh"

namespace cg = cooperative_groups;

namespace tg {
namespace {

constexpr int NT = 1024;

struct SelParams {
  SelSeq s[kMaxSeqPerLaunch];
  int C;  // CTAs per cluster (= per sequence)
};

// float -> uint32 whose unsigned order is the score order. NaN -> 0 (below -inf, whose key
// is 0x007fffff); -0 -> the key of +0.
__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inclusive block-wide scan of one int per thread (1024 threads); returns the inclusive
// value and writes the block total to *total.
__device__ __forceinline__ int block_scan_incl(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_sums[w] = v;
  __syncthreads();
  if (w == 0) {
    int s = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += n;
    }
    warp_sums[lane] = s;  // inclusive over warps
  }
  __syncthreads();
  int res = v + (w > 0 ? warp_sums[w - 1] : 0);
  if (total) *total = warp_sums[31];
  __syncthreads();
  return res;
}

template <int R>
__global__ void __launch_bounds__(NT, 1)
    select_kernel(const float* __restrict__ score, int32_t* __restrict__ kept, int32_t* __restrict__ cu_kept_dev,
                  int32_t* __restrict__ dev_status, const __grid_constant__ SelParams p) {
  cg::cluster_group cluster = cg::this_cluster();
  const int C = p.C;
  const int rank = (int)cluster.block_rank();
  const SelSeq sq = p.s[blockIdx.x / C];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;

  __shared__ uint32_t hist[3][2048];
  __shared__ int tab_a[32 * R];
  __shared__ int tab_b[32 * R];
  __shared__ int warp_sums[32];
  __shared__ int cta_cnt[2];  // keys > T, keys == T in this CTA
  __shared__ uint32_t s_digit;
  __shared__ int s_above;

  // outputs that do not depend on the selection
  if (rank == 0 && tid == 0 && cu_kept_dev) {
    if (sq.b == 0) cu_kept_dev[0] = 0;
    cu_kept_dev[sq.b + 1] = sq.out_off + sq.kc + sq.q;
  }
  for (int j = rank * NT + tid; j < sq.q; j += C * NT)
    kept[sq.out_off + sq.kc + j] = sq.start + sq.n_ctx + j;
  if (sq.kc == 0) return;  // whole cluster takes this branch: no barrier is pending
  if (sq.kc == sq.n_ctx) {
    for (int j = rank * NT + tid; j < sq.n_ctx; j += C * NT) kept[sq.out_off + j] = sq.start + j;
    return;
  }

  // load this CTA's slice of keys once
  const int base = rank * (NT * R);
  uint32_t key[R];
  uint32_t valid = 0;
  bool saw_nan = false;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    int idx = base + i * NT + tid;
    key[i] = 0u;
    if (idx < sq.n_ctx) {
      key[i] = order_key(__ldg(score + sq.start + idx));
      valid |= 1u << i;
      saw_nan |= (key[i] == 0u);
    }
  }
  if (saw_nan && dev_status) atomicOr(dev_status, TG_DEV_NAN_SCORE);
  for (int e = tid; e < 3 * 2048; e += NT) (&hist[0][0])[e] = 0u;
  __syncthreads();

  uint32_t prefix = 0u, pmask = 0u;
  int need = sq.kc;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nb = pass == 2 ? 1024 : 2048;
    const uint32_t dmask = (uint32_t)nb - 1u;
    uint32_t* h = hist[pass];
#pragma unroll
    for (int i = 0; i < R; ++i)
      if (((valid >> i) & 1u) && (key[i] & pmask) == prefix) atomicAdd(&h[(key[i] >> shift) & dmask], 1u);
    cluster.sync();
    // this thread owns bins in descending order: positions bpt*tid .. bpt*tid+bpt-1
    const int bpt = nb / NT;
    int c0 = 0, c1 = 0;
    const int hi = nb - 1 - bpt * tid;
    for (int r = 0; r < C; ++r) {
      const uint32_t* rh = (r == rank) ? h : cluster.map_shared_rank(h, r);
      c0 += (int)rh[hi];
      if (bpt == 2) c1 += (int)rh[hi - 1];
    }
    const int tsum = c0 + c1;
    const int incl = block_scan_incl(tsum, warp_sums, nullptr);
    const int excl = incl - tsum;
    if (excl < need && need <= incl) {
      if (excl + c0 >= need) {
        s_digit = (uint32_t)hi;
        s_above = excl;
      } else {
        s_digit = (uint32_t)(hi - 1);
        s_above = excl + c0;
      }
    }
    __syncthreads();
    prefix |= s_digit << shift;
    pmask |= dmask << shift;
    need -= s_above;
    __syncthreads();
  }
  const uint32_t T = prefix;  // the K-th largest key; `need` keys equal to T are kept

  uint32_t gtm = 0u, eqm = 0u;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if ((valid >> i) & 1u) {
      if (key[i] > T) gtm |= 1u << i;
      else if (key[i] == T) eqm |= 1u << i;
    }
  }
  // per (row i, warp) counts in index order: element index = base + i*NT + w*32 + lane
#pragma unroll
  for (int i = 0; i < R; ++i) {
    uint32_t bg = __ballot_sync(0xffffffffu, (gtm >> i) & 1u);
    uint32_t be = __ballot_sync(0xffffffffu, (eqm >> i) & 1u);
    if (lane == 0) {
      tab_a[i * 32 + w] = __popc(bg);
      tab_b[i * 32 + w] = __popc(be);
    }
  }
  __syncthreads();
  int gt_tot = 0, eq_tot = 0;
  const int va = tid < 32 * R ? tab_a[tid] : 0;
  const int vb = tid < 32 * R ? tab_b[tid] : 0;
  block_scan_incl(va, warp_sums, &gt_tot);
  const int eq_incl = block_scan_incl(vb, warp_sums, &eq_tot);
  if (tid == 0) {
    cta_cnt[0] = gt_tot;
    cta_cnt[1] = eq_tot;
  }
  __syncthreads();
  if (tid < 32 * R) tab_b[tid] = eq_incl - vb;  // exclusive offsets of equal keys
  cluster.sync();
  int eq_before = 0, sel_before = 0;
  for (int r = 0; r < rank; ++r) {
    const int* rc = cluster.map_shared_rank(cta_cnt, r);
    const int g_r = rc[0], e_r = rc[1];
    int take = need - eq_before;
    take = take < 0 ? 0 : (take > e_r ? e_r : take);
    sel_before += g_r + take;
    eq_before += e_r;
  }
  __syncthreads();
  // selection mask: equal keys are kept while their global rank among equals is < need
  uint32_t selm = gtm;
  const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    uint32_t be = __ballot_sync(0xffffffffu, (eqm >> i) & 1u);
    int rank_eq = eq_before + tab_b[i * 32 + w] + __popc(be & lt);
    if (((eqm >> i) & 1u) && rank_eq < need) selm |= 1u << i;
  }
#pragma unroll
  for (int i = 0; i < R; ++i) {
    uint32_t bs = __ballot_sync(0xffffffffu, (selm >> i) & 1u);
    if (lane == 0) tab_a[i * 32 + w] = __popc(bs);
  }
  __syncthreads();
  const int vs = tid < 32 * R ? tab_a[tid] : 0;
  const int s_incl = block_scan_incl(vs, warp_sums, nullptr);
  if (tid < 32 * R) tab_a[tid] = s_incl - vs;
  __syncthreads();
  bool overflow = false;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    uint32_t bs = __ballot_sync(0xffffffffu, (selm >> i) & 1u);
    if ((selm >> i) & 1u) {
      const int o = sel_before + tab_a[i * 32 + w] + __popc(bs & lt);  // rank among kept context tokens
      if (o < sq.kc) kept[sq.out_off + o] = sq.start + base + i * NT + tid;
      else overflow = true;  // cannot happen for a correct threshold; never write past the slot
    }
  }
  if (overflow && dev_status) atomicOr(dev_status, TG_DEV_BAD_INDEX);
  cluster.sync();  // no CTA leaves while a peer may still read its counters
}

template <int R>
tg_status launch_r(const float* score, const SelParams& p, int nseq, int32_t* kept, int32_t* cu_kept_dev,
                   int32_t* dev_status, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nseq * p.C));
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, select_kernel<R>, score, kept, cu_kept_dev, dev_status, p),
                     "select launch");
}

}  // namespace

tg_status launch_select(const float* score, const SelSeq* seqs, int nseq, int n_ctx_max, int32_t* kept_idx,
                        int32_t* cu_kept_dev, int32_t* dev_status, cudaStream_t st) {
  SelParams p = {};
  for (int i = 0; i < nseq; ++i) p.s[i] = seqs[i];
  // Spread a sequence over up to 8 SMs (one cluster) so its scores stream in parallel, with
  // at least 4 keys per thread; R keys per thread are held in registers.
  int C = (int)((n_ctx_max + 4 * NT - 1) / (4 * NT));
  C = C < 1 ? 1 : (C > 8 ? 8 : C);
  int R = 1;
  while (R < 32 && (int64_t)NT * R * C < n_ctx_max) R *= 2;
  if ((int64_t)NT * R * C < n_ctx_max)
    return fail(TG_ERR_UNSUPPORTED, "context of %d tokens exceeds the select capacity", n_ctx_max);
  p.C = C;
  switch (R) {
    case 1: return launch_r<1>(score, p, nseq, kept_idx, cu_kept_dev, dev_status, st);
    case 2: return launch_r<2>(score, p, nseq, kept_idx, cu_kept_dev, dev_status, st);
    case 4: return launch_r<4>(score, p, nseq, kept_idx, cu_kept_dev, dev_status, st);
    case 8: return launch_r<8>(score, p, nseq, kept_idx, cu_kept_dev, dev_status, st);
    case 16: return launch_r<16>(score, p, nseq, kept_idx, cu_kept_dev, dev_status, st);
    default: return launch_r<32>(score, p, nseq, kept_idx, cu_kept_dev, dev_status, st);
  }
}

}  // namespace tg
