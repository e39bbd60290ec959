// Exact, deterministic top-K over each sequence's context with the question tail kept.
//
// aitualizate.com TokenGate article, phase 2: a top-K selector keeps the K tokens with the
// highest gate score, and only the document part of the prompt may be pruned. TokenGate
// paper page (thelatestinai.com), Figure 1(a)-(b).
//
// Design (B200): one CTA of 1024 threads per sequence while its context fits in shared
// memory (32768 keys = 128 KB), otherwise one thread-block cluster of up to 8 CTAs. The
// scores are read from HBM exactly once and turned into order-preserving 32-bit keys held in
// shared memory. An MSB-first radix select with 4-bit digits (8 passes) finds the K-th
// largest key T without any atomics: every thread counts its keys per digit in four
// registers of packed 8-bit counters, warps reduce the 16 counts with redux.sync, and warp
// 0 sums the warps (and, in a cluster, the CTAs over distributed shared memory after a
// hardware cluster barrier) and picks the digit. Keys > T are kept, and keys == T in index
// order until K is reached (lower index wins ties). An ascending compaction uses warp
// ballots and one block-wide scan per class. No workspace: the per-sequence descriptors
// travel as kernel parameters; nothing spins.
#include <cooperative_groups.h>

#include "tg_internal.cuh"

namespace cg = cooperative_groups;

namespace tg {
namespace {

constexpr int NT = 1024;
constexpr int MAX_ROWS = 32;  // keys per thread: 32 x 1024 = 32768 keys per CTA

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

// Exclusive scan, in place, of n <= 1024 ints in shared memory; returns the total.
__device__ __forceinline__ int block_scan_excl(int* a, int n, int* warp_sums) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int v = threadIdx.x < n ? a[threadIdx.x] : 0;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[w] = x;
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
  const int total = warp_sums[31];
  if (threadIdx.x < n) a[threadIdx.x] = x - v + (w > 0 ? warp_sums[w - 1] : 0);
  __syncthreads();
  return total;
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
  __shared__ int wcnt[32][16];        // per-warp digit counts
  __shared__ int cta_cnt[8][16];      // per-pass digit counts of this CTA (read by the cluster)
  __shared__ int tab_a[32 * MAX_ROWS];
  __shared__ int tab_b[32 * MAX_ROWS];
  __shared__ int warp_sums[32];
  __shared__ int cta_tot[2];  // keys > T, keys == T in this CTA
  __shared__ uint32_t s_digit;
  __shared__ int s_above;

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

  // ---- load this CTA's slice once: element e = base + i * NT + tid, i < R
  const int base = rank * (NT * R);
  bool saw_nan = false;
  for (int i = 0; i < R; ++i) {
    const int idx = base + i * NT + tid;
    uint32_t k = 0u;
    if (idx < sq.n_ctx) {
      k = order_key(__ldg(score + sq.start + idx));
      saw_nan |= (k == 0u);
    }
    keys[i * NT + tid] = k;
  }
  if (saw_nan && dev_status) atomicOr(dev_status, TG_DEV_NAN_SCORE);
  const int nvalid = sq.n_ctx - base - tid;  // key i of this thread exists iff i * NT < nvalid
  __syncthreads();

  // ---- radix select, 4-bit digits, most significant first
  uint32_t prefix = 0u, pmask = 0u;
  int need = sq.kc;
#pragma unroll 1
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 28 - 4 * pass;
    uint32_t c0 = 0, c1 = 0, c2 = 0, c3 = 0;  // 16 packed 8-bit counters (<= 32 keys each)
    for (int i = 0; i < R; ++i) {
      if (i * NT >= nvalid) break;
      const uint32_t k = keys[i * NT + tid];
      if ((k & pmask) == prefix) {
        const uint32_t d = (k >> shift) & 15u;
        const uint32_t inc = 1u << ((d & 3u) * 8u);
        const uint32_t q = d >> 2;
        c0 += q == 0 ? inc : 0u;
        c1 += q == 1 ? inc : 0u;
        c2 += q == 2 ? inc : 0u;
        c3 += q == 3 ? inc : 0u;
      }
    }
    int mine = 0;  // lane d (< 16) keeps the warp's count of digit d
#pragma unroll
    for (int d = 0; d < 16; ++d) {
      const uint32_t word = d < 4 ? c0 : (d < 8 ? c1 : (d < 12 ? c2 : c3));
      const int v = (int)((word >> ((d & 3) * 8)) & 0xffu);
      const int sum = (int)__reduce_add_sync(0xffffffffu, (unsigned)v);
      if (lane == d) mine = sum;
    }
    if (lane < 16) wcnt[w][lane] = mine;
    __syncthreads();
    if (w == 0 && lane < 16) {
      int tot = 0;
#pragma unroll 8
      for (int x = 0; x < 32; ++x) tot += wcnt[x][lane];
      cta_cnt[pass][lane] = tot;
    }
    if (C > 1) cluster.sync();
    else __syncthreads();
    if (w == 0) {
      // lane l holds the cluster-wide count of digit 15 - l (descending order)
      int c = 0;
      if (lane < 16) {
        int part[8];
#pragma unroll
        for (int r = 0; r < 8; ++r)
          part[r] = r < C ? (r == rank ? cta_cnt[pass][15 - lane]
                                       : cluster.map_shared_rank(&cta_cnt[pass][0], r)[15 - lane])
                          : 0;
#pragma unroll
        for (int r = 0; r < 8; ++r) c += part[r];
      }
      int incl = c;
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int excl = incl - c;
      if (lane < 16 && excl < need && need <= incl) {
        s_digit = (uint32_t)(15 - lane);
        s_above = excl;
      }
    }
    __syncthreads();
    prefix |= s_digit << shift;
    pmask |= 15u << shift;
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
  const int gt_tot = block_scan_excl(tab_a, 32 * R, warp_sums);
  const int eq_tot = block_scan_excl(tab_b, 32 * R, warp_sums);  // exclusive offsets of equal keys
  if (tid == 0) {
    cta_tot[0] = gt_tot;
    cta_tot[1] = eq_tot;
  }
  int eq_before = 0, sel_before = 0;
  if (C > 1) {
    cluster.sync();
    for (int r = 0; r < rank; ++r) {
      const int* rc = cluster.map_shared_rank(cta_tot, r);
      const int g_r = rc[0], e_r = rc[1];
      int take = need - eq_before;
      take = take < 0 ? 0 : (take > e_r ? e_r : take);
      sel_before += g_r + take;
      eq_before += e_r;
    }
  }
  // selected: key > T, or key == T with global rank among equal keys < need
  for (int i = 0; i < R; ++i) {
    const uint32_t k = keys[i * NT + tid];
    const bool v = i * NT < nvalid;
    const bool eq = v && k == T;
    const uint32_t be = __ballot_sync(0xffffffffu, eq);
    const bool sel = (v && k > T) || (eq && eq_before + tab_b[i * 32 + w] + __popc(be & lt) < need);
    const uint32_t bs = __ballot_sync(0xffffffffu, sel);
    if (lane == 0) tab_a[i * 32 + w] = __popc(bs);
  }
  __syncthreads();
  block_scan_excl(tab_a, 32 * R, warp_sums);
  bool overflow = false;
  for (int i = 0; i < R; ++i) {
    const uint32_t k = keys[i * NT + tid];
    const bool v = i * NT < nvalid;
    const bool eq = v && k == T;
    const uint32_t be = __ballot_sync(0xffffffffu, eq);
    const bool sel = (v && k > T) || (eq && eq_before + tab_b[i * 32 + w] + __popc(be & lt) < need);
    const uint32_t bs = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const int o = sel_before + tab_a[i * 32 + w] + __popc(bs & lt);  // rank among kept context tokens
      if (o < sq.kc) kept[sq.out_off + o] = sq.start + base + i * NT + tid;
      else overflow = true;  // cannot happen for a correct threshold; never write past the slot
    }
  }
  if (overflow && dev_status) atomicOr(dev_status, TG_DEV_BAD_INDEX);
  if (C > 1) cluster.sync();  // no CTA leaves while a peer may still read its counters
}

}  // namespace

tg_status launch_select(const float* score, const SelSeq* seqs, int nseq, int n_ctx_max, int32_t* kept_idx,
                        int32_t* cu_kept_dev, int32_t* dev_status, cudaStream_t st) {
  SelParams p = {};
  for (int i = 0; i < nseq; ++i) p.s[i] = seqs[i];
  const int per_cta = NT * MAX_ROWS;
  int C = (n_ctx_max + per_cta - 1) / per_cta;
  if (C < 1) C = 1;
  if (C > 8) return fail(TG_ERR_UNSUPPORTED, "context of %d tokens exceeds the select capacity", n_ctx_max);
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
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, select_kernel, score, kept_idx, cu_kept_dev, dev_status, p),
                     "select launch");
}

}  // namespace tg
