// Exact, deterministic top-K over each sequence's context with the question tail kept.
//
// aitualizate.com TokenGate article, phase 2: a top-K selector keeps the K tokens with the
// highest gate score, and only the document part of the prompt may be pruned. TokenGate
// paper page (thelatestinai.com), Figure 1(a)-(b).
//
// Design (B200): one thread-block cluster of 1-8 CTAs (1024 threads each, up to 8192 keys
// per CTA below 64K keys, at most 32768) per sequence. The scores are read from HBM exactly
// once (loads batched 8 deep per thread) into order-preserving 32-bit keys in shared
// memory. The K-th largest key T comes from an MSB-first radix select whose cost is a few
// round trips between the CTAs, so the rounds are arranged to need as few as possible:
//   1. Every CTA histograms the top 12 bits (sign, exponent, 3 mantissa bits) of its keys
//      and pushes its 64 run totals (runs of 64 bins) into every CTA before a cluster
//      barrier. One warp per CTA then picks the run holding the K-th largest key from local
//      data and the bin within it with one parallel read of that run from every CTA.
//   2. Each CTA compacts its keys of that bin (a few hundred for the score distributions
//      of a gate network) into a local list; after a second barrier every CTA pulls all the
//      lists into registers and resolves the remaining 20 bits itself with 10-bit passes
//      (CTA barriers only), so no result has to travel back. Should the bin hold more keys
//      than the lists can take, 8-bit passes over all keys narrow it first.
//   3. Keys > T are kept, and keys == T in index order until K is reached (lower index
//      wins ties). A CTA's output offset is the kept count of the CTAs before it, taken from
//      the pulled lists and the per-CTA counts of keys above the bin; an ascending
//      compaction uses warp ballots and one block-wide scan.
// Two cluster barriers, plus one whose wait is deferred to the kernel's end so no CTA
// leaves while a peer may still read its list. No workspace: the per-sequence descriptors
// travel as kernel parameters; nothing spins.
#include <cooperative_groups.h>

#include "tg_internal.cuh"
#include "tg_sm100.cuh"

namespace cg = cooperative_groups;

namespace tg {
namespace {

constexpr int NT = 1024;
constexpr int MAX_ROWS = 32;   // keys per thread: 32 x 1024 = 32768 keys per CTA
constexpr int NRUN = 64;       // first pass: 12-bit digit = run * 64 + bin
constexpr int NB0 = NRUN * 64;
constexpr int NB = 256;        // bins of the narrowing passes over all keys (8-bit digits)
constexpr int NBL = 1024;      // bins of the candidate passes (10-bit digits)
constexpr int MAXC = 4096;     // candidates of a cluster, resolved in registers
constexpr int CPT = MAXC / NT;  // candidates per thread

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

__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// The score bits of a key (the inverse of order_key): exact for every score except -0, which
// comes back as +0 (the same gate value), and NaN, whose key 0 carries no bits (the caller
// reads NaN scores from memory instead).
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}

// Inclusive block-wide scan of one value per thread; optionally returns the block total.
template <typename V>
__device__ __forceinline__ V block_scan_incl(V v, V* warp_sums, V* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const V y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  if (lane == 31) warp_sums[w] = v;
  __syncthreads();
  if (w == 0) {
    V s = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const V y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s;
  }
  __syncthreads();
  const V res = v + (w > 0 ? warp_sums[w - 1] : V(0));
  if (total) *total = warp_sums[31];
  __syncthreads();
  return res;
}

// Exclusive scan, in place, of n <= 1024 values in shared memory; returns the total.
template <typename V>
__device__ __forceinline__ V block_scan_excl(V* a, int n, V* warp_sums) {
  const V v = threadIdx.x < n ? a[threadIdx.x] : V(0);
  V total = 0;
  const V incl = block_scan_incl<V>(v, warp_sums, &total);
  if (threadIdx.x < n) a[threadIdx.x] = incl - v;
  __syncthreads();
  return total;
}

template <typename P>
__device__ __forceinline__ P* on_rank(P* p, cg::cluster_group& cluster, int r, int rank) {
  return r == rank ? p : cluster.map_shared_rank(p, r);
}

__device__ __forceinline__ void cluster_or_cta_sync(cg::cluster_group& cluster, int C) {
  if (C > 1) cluster.sync();
  else __syncthreads();
}

// Within one warp: lane l holds the total t of a group of bins (groups in descending digit
// order by lane). Returns the lane whose group holds the need-th largest key and, in
// *excl_out, the count of keys in the groups before it.
__device__ __forceinline__ int warp_pick(int t, int need, int* excl_out) {
  const int incl = warp_incl_scan(t);
  const int excl = incl - t;
  const int src = __ffs(__ballot_sync(0xffffffffu, excl < need && need <= incl)) - 1;
  *excl_out = __shfl_sync(0xffffffffu, excl, src);
  return src;
}

// One warp finds, in a local NBL-bin histogram h, the digit whose bin holds the need-th
// largest key: first the 32-bin group (lane l sums bins [NBL-32(l+1), NBL-32l), reading in
// a lane-rotated order so the 32 lanes hit 32 banks), then the bin within that group.
__device__ __forceinline__ void warp_find_local(const uint32_t* h, int need, uint32_t* digit, int* above) {
  const int lane = threadIdx.x & 31;
  int t = 0;
  const int g0 = NBL - 32 * (lane + 1);
#pragma unroll 8
  for (int j = 0; j < 32; ++j) t += (int)h[g0 + ((j + lane) & 31)];
  int ex;
  const int g = warp_pick(t, need, &ex);  // lane g's group: bins NBL-32(g+1) .. NBL-32g-1
  const int bin = NBL - 32 * g - 1 - lane;  // lane l examines the l-th highest bin of the group
  int ex2;
  const int l2 = warp_pick((int)h[bin], need - ex, &ex2);
  if (lane == 0) {
    *digit = (uint32_t)(NBL - 32 * g - 1 - l2);
    *above = ex + ex2;
  }
}

__device__ __forceinline__ void cluster_arrive_relaxed(int C) {
  if (C > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive(int C) {
  if (C > 1) asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait(int C) {
  if (C > 1) asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Narrowing passes over all keys (8-bit digits), run only while the keys of the threshold bin
// outnumber the candidate lists. Kept out of line: the common path never executes it.
__device__ __noinline__ void narrow(const uint32_t* keys, int R, int nvalid, cg::cluster_group& cluster, int C,
                                    int rank, uint32_t* hist, int* s_cnt, uint32_t* s_digit, int* s_above,
                                    int* s_my_above, uint32_t* prefix_io, int* shift_io, int* need_io, int* ctot_io) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  uint32_t prefix = *prefix_io;
  int shift = *shift_io, need = *need_io, ctot = *ctot_io;
  for (int pass = 0; ctot > MAXC && shift > 0; ++pass) {
    const int db = shift < 8 ? shift : 8;
    shift -= db;
    uint32_t* hp = hist + pass * NB;
    for (int i = 0; i < R && i * NT < nvalid; ++i) {
      const uint32_t k = keys[i * NT + tid];
      if ((k >> (shift + db)) == prefix) atomicAdd(&hp[(k >> shift) & ((1u << db) - 1u)], 1u);
    }
    cluster_or_cta_sync(cluster, C);
    if (w == 0) {
      // lane l owns bins 255-8l .. 248-8l, read from every CTA in parallel
      const int b0 = NB - 8 * (lane + 1);
      int t[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (r < C) {
          const uint4* q = reinterpret_cast<const uint4*>(on_rank(hp, cluster, r, rank) + b0);
          const uint4 a = q[0], b = q[1];
          t[0] += (int)a.x, t[1] += (int)a.y, t[2] += (int)a.z, t[3] += (int)a.w;
          t[4] += (int)b.x, t[5] += (int)b.y, t[6] += (int)b.z, t[7] += (int)b.w;
        }
      }
      int ex;
      const int src = warp_pick(t[0] + t[1] + t[2] + t[3] + t[4] + t[5] + t[6] + t[7], need, &ex);
      int d = 0, run = ex;
      if (lane == src) {
        for (int j = 7; j >= 0; --j) {
          if (run + t[j] >= need) {
            d = b0 + j;
            break;
          }
          run += t[j];
        }
      }
      d = __shfl_sync(0xffffffffu, d, src);
      run = __shfl_sync(0xffffffffu, run, src);
      if (lane < C) s_cnt[lane] = (int)on_rank(hp, cluster, lane, rank)[d];
      int m = 0;
      for (int j = 0; j < 8; ++j)
        if (b0 + j > d) m += (int)hp[b0 + j];
      m = __reduce_add_sync(0xffffffffu, m);
      if (lane == 0) {
        *s_digit = (uint32_t)d;
        *s_above = run;
        *s_my_above += m;
      }
    }
    __syncthreads();
    prefix = (prefix << db) | *s_digit;
    need -= *s_above;
    ctot = 0;
    for (int r = 0; r < C; ++r) ctot += s_cnt[r];
    __syncthreads();  // the shared results are rewritten by the next pass
  }
  *prefix_io = prefix;
  *shift_io = shift;
  *need_io = need;
  *ctot_io = ctot;
}

__global__ void __launch_bounds__(NT, 1)
    select_kernel(const float* __restrict__ score, int32_t* __restrict__ kept, int32_t* __restrict__ cu_kept_dev,
                  int32_t* __restrict__ dev_status, int32_t* __restrict__ pos, float* __restrict__ gate,
                  float* __restrict__ logg, uint32_t flags, const int32_t* __restrict__ idxmap,
                  float* __restrict__ kept_score, const __grid_constant__ SelParams p) {
  cg::cluster_group cluster = cg::this_cluster();
  const int C = p.C, R = p.rows;
  const int rank = (int)cluster.block_rank();
  const SelSeq sq = p.s[blockIdx.x / C];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const uint32_t lt = (1u << lane) - 1u;

  extern __shared__ uint32_t dyn[];
  uint32_t* keys = dyn;           // [R][NT]
  uint32_t* cand = dyn + R * NT;  // [MAXC] this CTA's keys in the threshold bin
  __shared__ __align__(16) uint32_t hist0[NB0];
  __shared__ __align__(16) uint32_t runs[8][NRUN];  // run totals of every CTA, pushed by each
  __shared__ __align__(16) uint32_t hist[3][NB];
  __shared__ uint32_t histl[2][NBL];
  __shared__ uint32_t tab[32 * MAX_ROWS];  // per (row, warp): keys > T << 16 | keys == T
  __shared__ int warp_sums[32];
  __shared__ int above_all[8];  // keys of CTA r above the threshold bin, pushed by CTA r
  __shared__ int s_cnt[8];      // keys of CTA r in the threshold bin
  __shared__ uint32_t s_digit;
  __shared__ int s_above, s_my_above, s_ccount, s_gt, s_eq;

  sm100::griddep_launch_dependents();  // the next kernel may start its prologue
  sm100::griddep_wait();  // the scores of the previous kernel are visible from here on, and no
                          // kernel before it still reads kept or cu_kept
  if (rank == 0 && tid == 0 && cu_kept_dev) {
    if (sq.b == 0) cu_kept_dev[0] = 0;
    cu_kept_dev[sq.b + 1] = sq.out_off + sq.kc + sq.q;
  }
  // output row `row` keeps the token at `ip` within the sequence (tail: a question token);
  // key is its order key when the caller holds it (0: read the score from memory)
  auto emit = [&](int row, int ip, bool tail, uint32_t key) {
    kept[row] = tail ? sq.tail + (ip - sq.n_ctx) : (idxmap ? __ldcg(idxmap + sq.start + ip) : sq.wbase + ip);
    if (kept_score && !tail) kept_score[row] = key ? key_score(key) : __ldcg(score + sq.start + ip);
    if (pos) {
      float gv = 1.f, lg = 0.f;
      if (!(tail && (flags & TG_QUESTION_GATE_ONE)))
        gate_from_score(key ? key_score(key) : __ldcg(score + sq.start + ip), &gv, &lg);
      pos[row] = ip;
      gate[row] = gv;
      logg[row] = lg;
    }
  };
  for (int j = rank * NT + tid; j < sq.q; j += C * NT) emit(sq.out_off + sq.kc + j, sq.n_ctx + j, true, 0u);
  if (sq.kc == 0) return;  // the whole cluster takes this branch: no barrier is pending
  if (sq.kc == sq.n_ctx) {  // every context token is kept; NaN scores are still reported
    bool nan = false;
    for (int j = rank * NT + tid; j < sq.n_ctx; j += C * NT) {
      const float v = __ldcg(score + sq.start + j);
      nan |= v != v;
      emit(sq.out_off + j, j, false, 0u);
    }
    if (nan && dev_status) atomicOr(dev_status, TG_DEV_NAN_SCORE);
    return;
  }

  // peers may touch this CTA's shared memory only once it runs: the wait for this arrival
  // comes right before the first push into a peer
  cluster_arrive_relaxed(C);
#pragma unroll 1
  for (int e = tid; e < NB0; e += NT) hist0[e] = 0u;
  if (tid < 3 * NB) (&hist[0][0])[tid] = 0u;
  histl[0][tid] = 0u;
  histl[1][tid] = 0u;
  if (tid == 0) {
    s_ccount = 0;
    s_gt = 0;
    s_eq = 0;
  }

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

  // ---- round 1: 12-bit histogram; run totals go to every CTA of the cluster
#pragma unroll 1
  for (int i = 0; i < R && i * NT < nvalid; ++i) atomicAdd(&hist0[keys[i * NT + tid] >> 20], 1u);
  __syncthreads();
  {
    uint32_t c4 = hist0[4 * tid] + hist0[4 * tid + 1] + hist0[4 * tid + 2] + hist0[4 * tid + 3];
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) c4 += __shfl_xor_sync(0xffffffffu, c4, o);
    cluster_wait(C);  // every CTA of the cluster is running
    if ((tid & 15) == 0)
      for (int r = 0; r < C; ++r) *on_rank(&runs[rank][tid >> 4], cluster, r, rank) = c4;
  }
  cluster_or_cta_sync(cluster, C);
  int need = sq.kc;
  if (w == 0) {
    // the run: lane l owns runs 63-2l and 62-2l, summed over the CTAs from local copies
    const int rh = NRUN - 1 - 2 * lane;
    int t0 = 0, t1 = 0;
    for (int r = 0; r < C; ++r) {
      t0 += (int)runs[r][rh];
      t1 += (int)runs[r][rh - 1];
    }
    int ex;
    const int src = warp_pick(t0 + t1, need, &ex);
    const int t0s = __shfl_sync(0xffffffffu, t0, src);
    const bool upper = ex + t0s >= need;
    const int run = NRUN - 1 - 2 * src - (upper ? 0 : 1);
    const int above_run = upper ? ex : ex + t0s;
    int m = (rh > run ? (int)runs[rank][rh] : 0) + (rh - 1 > run ? (int)runs[rank][rh - 1] : 0);
    // the bin: lane l owns bins 63-2l and 62-2l of the run; one parallel read from every CTA
    const int bh = 63 - 2 * lane;
    uint32_t hi[8], lo[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if (r < C) {
        const uint2 x = *reinterpret_cast<const uint2*>(on_rank(hist0, cluster, r, rank) + run * 64 + bh - 1);
        hi[r] = x.y;
        lo[r] = x.x;
      } else {
        hi[r] = lo[r] = 0u;
      }
    }
    int f0 = 0, f1 = 0;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      f0 += (int)hi[r];
      f1 += (int)lo[r];
    }
    const int need2 = need - above_run;
    int ex2;
    const int src2 = warp_pick(f0 + f1, need2, &ex2);
    const int f0s = __shfl_sync(0xffffffffu, f0, src2);
    const bool upper2 = ex2 + f0s >= need2;
    const int bin = 63 - 2 * src2 - (upper2 ? 0 : 1);
    if (lane == src2) {
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < C) s_cnt[r] = (int)(upper2 ? hi[r] : lo[r]);
    }
    m += (bh > bin ? (int)hist0[run * 64 + bh] : 0) + (bh - 1 > bin ? (int)hist0[run * 64 + bh - 1] : 0);
    m = __reduce_add_sync(0xffffffffu, m);
    if (lane == 0) {
      s_digit = (uint32_t)(run * 64 + bin);
      s_above = above_run + (upper2 ? ex2 : ex2 + f0s);
      s_my_above = m;
    }
  }
  __syncthreads();
  uint32_t prefix = s_digit;  // key >> shift
  int shift = 20;
  need -= s_above;
  int ctot = 0;
  for (int r = 0; r < C; ++r) ctot += s_cnt[r];

  // ---- narrowing passes over all keys, only while the bin is too full for the lists
  if (ctot > MAXC)
    narrow(keys, R, nvalid, cluster, C, rank, &hist[0][0], s_cnt, &s_digit, &s_above, &s_my_above, &prefix, &shift,
           &need, &ctot);

  // ---- this CTA's count above the bin goes to every CTA; its keys in the bin to a local list
  if (tid < C) *on_rank(&above_all[rank], cluster, tid, rank) = s_my_above;
  if (shift > 0) {
#pragma unroll 1
    for (int i = 0; i < R; ++i) {  // warp-uniform trip count: the ballot needs every lane
      const bool v = i * NT < nvalid;
      const uint32_t k = v ? keys[i * NT + tid] : 0u;
      const bool c = v && (k >> shift) == prefix;
      const uint32_t b = __ballot_sync(0xffffffffu, c);
      if (b) {
        int pos = 0;
        if (lane == 0) pos = atomicAdd(&s_ccount, __popc(b));
        pos = __shfl_sync(0xffffffffu, pos, 0);
        if (c) cand[pos + __popc(b & lt)] = k;
      }
    }
  }
  cluster_or_cta_sync(cluster, C);

  // ---- every CTA pulls the lists (grouped by CTA) and resolves T among them
  int my_off = 0;
  for (int r = 0; r < rank; ++r) my_off += s_cnt[r];
  uint32_t T = prefix;
  int gt_before = 0, eq_before = 0;
  for (int r = 0; r < rank; ++r) gt_before += above_all[r];
  if (shift > 0) {
    uint32_t ck[CPT];
    bool cv[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int c = tid + j * NT;
      cv[j] = c < ctot;
      ck[j] = 0u;
      if (cv[j]) {
        int r = 0, off = 0;
        while (c >= off + s_cnt[r]) off += s_cnt[r++];
        ck[j] = on_rank(cand, cluster, r, rank)[c - off];
      }
    }
    cluster_arrive(C);  // this CTA is done reading its peers' lists
    int sl = shift;
    for (int pass = 0; sl > 0; ++pass) {  // at most two passes (sl <= 20)
      const int db = sl < 10 ? sl : 10;
      sl -= db;
      uint32_t* hl = histl[pass];
#pragma unroll
      for (int j = 0; j < CPT; ++j)
        if (cv[j] && (ck[j] >> (sl + db)) == T) atomicAdd(&hl[(ck[j] >> sl) & ((1u << db) - 1u)], 1u);
      __syncthreads();
      if (w == 0) warp_find_local(hl, need, &s_digit, &s_above);
      __syncthreads();
      T = (T << db) | s_digit;
      need -= s_above;
    }
    // kept keys of the CTAs before this one that sit in the threshold bin
    int g = 0, e = 0;
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int c = tid + j * NT;
      g += (cv[j] && c < my_off && ck[j] > T) ? 1 : 0;
      e += (cv[j] && c < my_off && ck[j] == T) ? 1 : 0;
    }
    g = __reduce_add_sync(0xffffffffu, g);
    e = __reduce_add_sync(0xffffffffu, e);
    if (lane == 0 && (g | e)) {
      atomicAdd(&s_gt, g);
      atomicAdd(&s_eq, e);
    }
    __syncthreads();
    gt_before += s_gt;
    eq_before = s_eq;
  } else {
    cluster_arrive(C);
    eq_before = my_off;  // the narrowing resolved every bit: the whole bin equals T
  }

  // ---- compaction in index order: per (row i, warp) counts, element = base + i*NT + w*32 + lane
#pragma unroll 1
  for (int i = 0; i < R; ++i) {
    const uint32_t k = keys[i * NT + tid];
    const bool v = i * NT < nvalid;
    const uint32_t bg = __ballot_sync(0xffffffffu, v && k > T);
    const uint32_t be = __ballot_sync(0xffffffffu, v && k == T);
    if (lane == 0) tab[i * 32 + w] = (uint32_t)__popc(bg) << 16 | (uint32_t)__popc(be);
  }
  __syncthreads();
  // exclusive offsets of keys > T (high half) and == T (low half); a CTA holds at most 32768
  // keys, so the low half never carries into the high half
  block_scan_excl<uint32_t>(tab, 32 * R, reinterpret_cast<uint32_t*>(warp_sums));
  // A kept key's output slot is the number of kept keys before it: GT(p) + min(EQ(p), need),
  // where GT(p) and EQ(p) count the keys > T and == T before position p (equal keys are kept
  // in index order while their rank is below `need`).
  bool overflow = false;
#pragma unroll 1
  for (int i = 0; i < R; ++i) {
    const uint32_t k = keys[i * NT + tid];
    const bool v = i * NT < nvalid;
    const bool gt = v && k > T, eq = v && k == T;
    const uint32_t bg = __ballot_sync(0xffffffffu, gt);
    const uint32_t be = __ballot_sync(0xffffffffu, eq);
    const int GT = gt_before + (int)(tab[i * 32 + w] >> 16) + __popc(bg & lt);
    const int EQ = eq_before + (int)(tab[i * 32 + w] & 0xffffu) + __popc(be & lt);
    if (gt || (eq && EQ < need)) {
      const int o = GT + (EQ < need ? EQ : need);  // rank among kept context tokens
      if (o < sq.kc) emit(sq.out_off + o, base + i * NT + tid, false, k);
      else overflow = true;  // cannot happen for a correct threshold; never write past the slot
    }
  }
  if (overflow && dev_status) atomicOr(dev_status, TG_DEV_BAD_INDEX);
  cluster_wait(C);  // no CTA leaves while a peer may still read its list
}

}  // namespace

tg_status launch_select(const float* score, const SelSeq* seqs, int nseq, int n_ctx_max, int32_t* kept_idx,
                        int32_t* cu_kept_dev, int32_t* dev_status, cudaStream_t st, int32_t* pos, float* g,
                        float* logg, uint32_t flags, const int32_t* idxmap, float* kept_score) {
  SelParams p = {};
  for (int i = 0; i < nseq; ++i) p.s[i] = seqs[i];
  const int per_cta = NT * MAX_ROWS;
  // CTAs per sequence: enough to hold the keys, otherwise as many as fill the GPU once across
  // this launch's sequences (a sequence's time is a chain of dependent phases, so spreading it
  // over more SMs pays only while SMs would otherwise idle), at most one per 4096 keys and 8.
  // Measured: one 32K sequence 18.4 us with 8 CTAs against 20.5 with 4; 64 sequences of 128K
  // 76 us with 4 CTAs each against 117 with 8.
  const int c_min = (n_ctx_max + per_cta - 1) / per_cta;
  const int c_keys = (n_ctx_max + 4 * NT - 1) / (4 * NT);
  int c_fill = device_sm_count() / (nseq > 0 ? nseq : 1);
  c_fill = c_fill < 1 ? 1 : c_fill;
  int C = c_fill < c_keys ? c_fill : c_keys;
  C = C < c_min ? c_min : C;
  C = C < 1 ? 1 : (C > 8 ? 8 : C);
  if ((int64_t)C * per_cta < n_ctx_max)
    return fail(TG_ERR_UNSUPPORTED, "context of %d tokens exceeds the select capacity", n_ctx_max);
  int rows = (n_ctx_max + NT * C - 1) / (NT * C);
  if (rows < 1) rows = 1;
  p.C = C;
  p.rows = rows;
  if (attrs_needed(ATTR_SELECT)) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (per_cta + MAXC) * 4);
    if (e != cudaSuccess) return cuda_status(e, "select: cudaFuncSetAttribute");
    e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return cuda_status(e, "select: cudaFuncSetAttribute");
    mark_attrs_set(ATTR_SELECT);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nseq * C));
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = (size_t)(rows * NT + MAXC) * 4;  // keys, then the candidate buffer
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute(PDL_SELECT);
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cuda_status(cudaLaunchKernelEx(&cfg, select_kernel, score, kept_idx, cu_kept_dev, dev_status, pos, g, logg,
                                        flags, idxmap, kept_score, p),
                     "select launch");
}

}  // namespace tg
