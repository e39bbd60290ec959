// Exact, deterministic top-K over each sequence's context with the question tail kept.
//
// aitualizate.com TokenGate article, phase 2: a top-K selector keeps the K tokens with the
// highest gate score, and only the document part of the prompt may be pruned. TokenGate
// paper page (thelatestinai.com), Figure 1(a)-(b).
//
// Design (B200): one thread-block cluster of 1-8 CTAs (1024 threads each, up to 8192 keys
// per CTA below 64K keys, at most 32768) per sequence. The scores are read from HBM exactly
// once (loads batched 8 deep per thread) into order-preserving 32-bit keys in shared
// memory. An MSB-first radix select with 8-bit digits (4 passes, 256 bins) finds the K-th
// largest key T. Pass 0 (sign + 7 exponent bits) sees scores crowded into a few bins, so
// lanes with the same bin are merged with match.any before one shared atomic; later passes
// only count keys that still match the prefix. After a hardware cluster barrier 64 threads
// of every CTA sum the cluster's 256-bin histograms with 16-byte distributed-shared-memory
// loads and pick the digit. Keys > T are kept, and keys == T in index order until K is
// reached (lower index wins ties). An ascending compaction uses warp ballots and
// block-wide scans. No workspace: the per-sequence descriptors travel as kernel
// parameters; nothing spins.
#include <cooperative_groups.h>

#include "tg_internal.cuh"
#include "tg_sm100.cuh"

namespace cg = cooperative_groups;

namespace tg {
namespace {

constexpr int NT = 1024;
constexpr int MAX_ROWS = 32;  // keys per thread: 32 x 1024 = 32768 keys per CTA
constexpr int NB = 256;  // bins per pass (8-bit digits)

struct SelParams {
  SelSeq s[kMaxSeqPerLaunch];
  int C;     // CTAs per cluster (= per sequence)
  int rows;  // keys per thread (elements per CTA = rows * NT)
};

// float -> uint32 whose unsigned order is the score order. NaN -> 0 (below -inf, whose key
// is 0x007fffff); -0 -> the key of +0.
__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inclusive block-wide scan of one int per thread; optionally returns the block total.
__device__ __forceinline__ int block_scan_incl(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  if (lane == 31) warp_sums[w] = v;
  __syncthreads();
  if (w == 0) {
    int s = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s;
  }
  __syncthreads();
  const int res = v + (w > 0 ? warp_sums[w - 1] : 0);
  if (total) *total = warp_sums[31];
  __syncthreads();
  return res;
}

// Exclusive scan, in place, of n <= 1024 ints in shared memory; returns the total.
__device__ __forceinline__ int block_scan_excl(int* a, int n, int* warp_sums) {
  const int v = threadIdx.x < n ? a[threadIdx.x] : 0;
  int total = 0;
  const int incl = block_scan_incl(v, warp_sums, &total);
  if (threadIdx.x < n) a[threadIdx.x] = incl - v;
  __syncthreads();
  return total;
}

// Finds, over the cluster's 256-bin histograms h (ascending digit order), the digit whose
// bin holds the need-th largest key; writes it and the count of keys in higher bins.
// Threads 0..63 each own 4 bins (descending) and read them from every CTA with one 16-byte
// load per CTA.
__device__ __forceinline__ void find_digit(const uint32_t* h, int need, cg::cluster_group& cluster, int C, int rank,
                                           int* warp_sums, uint32_t* s_digit, int* s_above) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  int cnt[4] = {0, 0, 0, 0};
  if (tid < NB / 4) {
    const int lo = NB - 4 * (tid + 1);  // bins lo..lo+3; this thread's order is lo+3, lo+2, lo+1, lo
    uint4 part[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const uint32_t* rh = (r < C && r != rank) ? cluster.map_shared_rank(h, r) : h;
      part[r] = r < C ? *reinterpret_cast<const uint4*>(rh + lo) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      cnt[0] += (int)part[r].w;
      cnt[1] += (int)part[r].z;
      cnt[2] += (int)part[r].y;
      cnt[3] += (int)part[r].x;
    }
  }
  // inclusive scan over threads 0..63 (two warps) of their 4-bin totals
  const int local = cnt[0] + cnt[1] + cnt[2] + cnt[3];
  int incl = local;
  if (w < 2) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sums[w] = incl;
  }
  __syncthreads();
  if (w == 1) incl += warp_sums[0];
  const int excl = incl - local;
  if (tid < NB / 4 && excl < need && need <= incl) {
    int run = excl;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (run + cnt[e] >= need) {
        *s_digit = (uint32_t)(NB - 1 - (4 * tid + e));
        *s_above = run;
        break;
      }
      run += cnt[e];
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(NT, 1)
    select_kernel(const float* __restrict__ score, int32_t* __restrict__ kept, int32_t* __restrict__ cu_kept_dev,
                  int32_t* __restrict__ dev_status, const __grid_constant__ SelParams p) {
  cg::cluster_group cluster = cg::this_cluster();
  const int C = p.C, R = p.rows;
  const int rank = (int)cluster.block_rank();
  const SelSeq sq = p.s[blockIdx.x / C];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;

  extern __shared__ uint32_t keys[];  // [R][NT]
  __shared__ __align__(16) uint32_t hist[4][NB];  // one per pass (read by the cluster)
  __shared__ int tab_a[32 * MAX_ROWS];
  __shared__ int tab_b[32 * MAX_ROWS];
  __shared__ int warp_sums[32];
  __shared__ int cta_tot[2];  // keys > T, keys == T in this CTA
  __shared__ uint32_t s_digit;
  __shared__ int s_above;

  sm100::griddep_launch_dependents();  // the next kernel may start its prologue
  sm100::griddep_wait();  // the scores of the previous kernel are visible from here on, and no
                          // kernel before it still reads kept or cu_kept
  if (rank == 0 && tid == 0 && cu_kept_dev) {
    if (sq.b == 0) cu_kept_dev[0] = 0;
    cu_kept_dev[sq.b + 1] = sq.out_off + sq.kc + sq.q;
  }
  for (int j = rank * NT + tid; j < sq.q; j += C * NT) kept[sq.out_off + sq.kc + j] = sq.start + sq.n_ctx + j;
  if (sq.kc == 0) return;  // the whole cluster takes this branch: no barrier is pending
  if (sq.kc == sq.n_ctx) {
    for (int j = rank * NT + tid; j < sq.n_ctx; j += C * NT) kept[sq.out_off + j] = sq.start + j;
    return;
  }

  for (int e = tid; e < 4 * NB; e += NT) (&hist[0][0])[e] = 0u;

  // ---- load this CTA's slice once, 8 loads in flight per thread: element = base + i*NT + tid
  const int base = rank * (NT * R);
  const int nvalid = sq.n_ctx - base - tid;  // key i of this thread exists iff i * NT < nvalid
  bool saw_nan = false;
#pragma unroll 1
  for (int i0 = 0; i0 < R; i0 += 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u;
      v[u] = (i < R && i * NT < nvalid) ? __ldg(score + sq.start + base + i * NT + tid) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u;
      if (i < R) {
        const bool ok = i * NT < nvalid;
        const uint32_t k = ok ? order_key(v[u]) : 0u;
        saw_nan |= ok && k == 0u;
        keys[i * NT + tid] = k;
      }
    }
  }
  if (saw_nan && dev_status) atomicOr(dev_status, TG_DEV_NAN_SCORE);
  __syncthreads();

  // ---- pass 0: sign + 7 exponent bits; lanes with equal bins merged before the atomic
  for (int i = 0; i < R; ++i) {
    const bool ok = i * NT < nvalid;
    const uint32_t act = __ballot_sync(0xffffffffu, ok);
    if (ok) {
      const uint32_t d = keys[i * NT + tid] >> 24;
      const uint32_t grp = __match_any_sync(act, d);
      if (lane == __ffs(grp) - 1) atomicAdd(&hist[0][d], (uint32_t)__popc(grp));
    }
  }
  if (C > 1) cluster.sync();
  else __syncthreads();
  int need = sq.kc;
  find_digit(hist[0], need, cluster, C, rank, warp_sums, &s_digit, &s_above);
  uint32_t prefix = s_digit;  // key >> 24
  need -= s_above;
  __syncthreads();
  // ---- passes 1-3: the next byte of the keys that still match the prefix
#pragma unroll 1
  for (int pass = 1; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = 0; i < R; ++i) {
      if (i * NT >= nvalid) break;
      const uint32_t k = keys[i * NT + tid];
      if ((k >> (shift + 8)) == prefix) atomicAdd(&hist[pass][(k >> shift) & (NB - 1)], 1u);
    }
    if (C > 1) cluster.sync();
    else __syncthreads();
    find_digit(hist[pass], need, cluster, C, rank, warp_sums, &s_digit, &s_above);
    prefix = (prefix << 8) | s_digit;
    need -= s_above;
    __syncthreads();
  }
  const uint32_t T = prefix;  // the K-th largest key; `need` keys equal to T are kept

  // ---- compaction in index order: per (row i, warp) counts, element = base + i*NT + w*32 + lane
  const uint32_t lt = (1u << lane) - 1u;
  for (int i = 0; i < R; ++i) {
    const uint32_t k = keys[i * NT + tid];
    const bool v = i * NT < nvalid;
    const uint32_t bg = __ballot_sync(0xffffffffu, v && k > T);
    const uint32_t be = __ballot_sync(0xffffffffu, v && k == T);
    if (lane == 0) {
      tab_a[i * 32 + w] = __popc(bg);
      tab_b[i * 32 + w] = __popc(be);
    }
  }
  __syncthreads();
  const int gt_tot = block_scan_excl(tab_a, 32 * R, warp_sums);  // exclusive offsets of keys > T
  const int eq_tot = block_scan_excl(tab_b, 32 * R, warp_sums);  // exclusive offsets of keys == T
  if (tid == 0) {
    cta_tot[0] = gt_tot;
    cta_tot[1] = eq_tot;
  }
  // Keys before this CTA in index order: gt_before keys > T and eq_before keys == T.
  int eq_before = 0, gt_before = 0;
  if (C > 1) {
    cluster.sync();
    for (int r = 0; r < rank; ++r) {
      const int* rc = cluster.map_shared_rank(cta_tot, r);
      gt_before += rc[0];
      eq_before += rc[1];
    }
  }
  // A kept key's output slot is the number of kept keys before it: GT(p) + min(EQ(p), need),
  // where GT(p) and EQ(p) count the keys > T and == T before position p (equal keys are kept
  // in index order while their rank is below `need`).
  bool overflow = false;
  for (int i = 0; i < R; ++i) {
    const uint32_t k = keys[i * NT + tid];
    const bool v = i * NT < nvalid;
    const bool gt = v && k > T, eq = v && k == T;
    const uint32_t bg = __ballot_sync(0xffffffffu, gt);
    const uint32_t be = __ballot_sync(0xffffffffu, eq);
    const int GT = gt_before + tab_a[i * 32 + w] + __popc(bg & lt);
    const int EQ = eq_before + tab_b[i * 32 + w] + __popc(be & lt);
    if (gt || (eq && EQ < need)) {
      const int o = GT + (EQ < need ? EQ : need);  // rank among kept context tokens
      if (o < sq.kc) kept[sq.out_off + o] = sq.start + base + i * NT + tid;
      else overflow = true;  // cannot happen for a correct threshold; never write past the slot
    }
  }
  if (overflow && dev_status) atomicOr(dev_status, TG_DEV_BAD_INDEX);
  if (C > 1) cluster.sync();  // no CTA leaves while a peer may still read its shared memory
}

}  // namespace

tg_status launch_select(const float* score, const SelSeq* seqs, int nseq, int n_ctx_max, int32_t* kept_idx,
                        int32_t* cu_kept_dev, int32_t* dev_status, cudaStream_t st) {
  SelParams p = {};
  for (int i = 0; i < nseq; ++i) p.s[i] = seqs[i];
  const int per_cta = NT * MAX_ROWS;
  // about 8192 keys per CTA (up to 8 CTAs): the passes are instruction-bound, so a sequence
  // is spread over several SMs rather than one
  int C = (n_ctx_max + 8 * NT - 1) / (8 * NT);
  C = C < 1 ? 1 : (C > 8 ? 8 : C);
  if ((int64_t)C * per_cta < n_ctx_max)
    return fail(TG_ERR_UNSUPPORTED, "context of %d tokens exceeds the select capacity", n_ctx_max);
  int rows = (n_ctx_max + NT * C - 1) / (NT * C);
  if (rows < 1) rows = 1;
  p.C = C;
  p.rows = rows;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, per_cta * 4);
    if (e != cudaSuccess) return cuda_status(e, "select: cudaFuncSetAttribute");
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nseq * C));
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = (size_t)rows * NT * 4;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute(PDL_SELECT);
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cuda_status(cudaLaunchKernelEx(&cfg, select_kernel, score, kept_idx, cu_kept_dev, dev_status, p),
                     "select launch");
}

}  // namespace tg
