// Exact top-K for many long sequences at once, as a stream over all SMs (the many-sequence
// counterpart of tg_select.cu, same results bit for bit).
//
// aitualizate.com TokenGate article, phase 2: a top-K selector keeps the K tokens with the highest
// gate score, and only the document part of the prompt may be pruned. TokenGate paper page
// (thelatestinai.com), Figure 1(a)-(b).
//
// The cluster select gives each sequence one thread-block cluster and keeps its keys in shared
// memory; with many long sequences that is a few waves of 1024-thread CTAs bound by instruction
// issue and barriers. Here the work is cut into chunks of 8192 keys of one sequence, and four
// kernels run in stream order (the scores are read from HBM once; the later passes find them in
// L2):
//   1. select_hist_kernel (one CTA of 256 threads per chunk): order keys, a 12-bit histogram in
//      shared memory, added to the sequence's global histogram with integer atomics (exact, so the
//      totals do not depend on their order). The sequence's last CTA to finish (a counter behind
//      a fence, no waiting) finds the bin b1 that holds the K-th largest key.
//   2. select_cand_kernel (one CTA per chunk): counts its keys above bin b1 and appends its keys
//      in the bin, with their positions, to the sequence's candidate list (one slot reservation
//      per CTA).
//   3. select_resolve_kernel (one CTA per sequence): two 10-bit radix passes over the candidates
//      give the K-th largest key T and the number of keys equal to T to keep; each chunk then
//      gets its output offset and its quota of keys equal to T (lowest positions first, chunk
//      by chunk). This CTA also writes the question tail and cu_kept.
//   4. select_compact_kernel (one CTA per chunk): keys > T, and keys == T within the chunk's
//      quota in position order, go to the chunk's output rows in ascending position order. Each
//      thread holds 32 consecutive positions, so one block scan of per-thread counts places them.
// Only integer counts decide anything, so the result is deterministic; the candidate list's order
// (set by atomics) does not matter, because T is found by value and the placement by counts.
#include "tg_internal.cuh"
#include "tg_sm100.cuh"

namespace tg {
namespace {

constexpr int SNT = 128;               // threads per chunk CTA
constexpr int SROWS = 32;              // keys per thread
constexpr int CH = SNT * SROWS;        // keys per chunk
constexpr int NB12 = 4096;             // first-level bins (top 12 bits of the order key)
constexpr int NB10 = 1024;             // bins of the two candidate passes
constexpr int BPT = NB12 / SNT;        // first-level bins per thread in the bin search
constexpr int MAX_CHUNKS_SEQ = (TG_MAX_CTX + CH - 1) / CH;
constexpr int RNT = 1024;              // threads of the resolve CTA
constexpr int RCPT = 4;                // candidates a resolve thread keeps in registers

enum : uint32_t { MODE_SELECT = 0, MODE_ALL = 1, MODE_NONE = 2 };

struct StreamSeq {
  int32_t start;    // packed row of the sequence's first token
  int32_t n_ctx;    // context tokens N - q
  int32_t q;        // question-tail tokens
  int32_t kc;       // context tokens kept
  int32_t out_off;  // first output row
  int32_t b;        // sequence index in the batch
  int32_t chunk0;   // first chunk of this sequence in the launch
  int32_t nch;      // chunks (0 unless some context is kept)
  int64_t cand_off; // first candidate slot of this sequence (n_ctx slots)
  uint32_t mode;
};

struct StreamParams {
  StreamSeq s[kMaxSeqPerLaunch];
  int nseq;
};

// Per-sequence words in the workspace (after the histograms).
enum { SI_CAND = 0, SI_B1 = 1, SI_NEED = 2, SI_T = 3, SI_DONE = 4, SI_WORDS = 8 };
// Per-chunk words.
enum { CI_GT = 0, CI_OUT = 1, CI_EQ = 2, CI_WORDS = 4 };

__device__ __forceinline__ uint32_t order_key(float x) {  // as in the cluster select
  uint32_t u = __float_as_uint(x);
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The sequence of chunk c (the launch holds at most kMaxSeqPerLaunch sequences).
__device__ __forceinline__ int seq_of_chunk(const StreamParams& p, int c) {
  int s = 0;
  while (s + 1 < p.nseq && c >= p.s[s + 1].chunk0) ++s;
  return s;
}

// Loads the chunk's keys into registers, thread-major: thread t holds positions t * SROWS + i of
// the chunk (i = 0..SROWS-1), so the chunk's order is the threads' order and then i. Whole
// 128-byte runs load as eight 16-byte vectors when their address is 16-byte aligned; the ragged
// end and unaligned runs load word by word. Keys past the context are 0 and not
// valid (nvalid_out: this thread's valid keys). Returns whether a NaN score was seen.
__device__ __forceinline__ bool load_chunk(const float* __restrict__ score, const StreamSeq& sq, int chunk_in_seq,
                                           uint32_t (&k)[SROWS], int* nvalid_out) {
  const int base = chunk_in_seq * CH + (int)threadIdx.x * SROWS;
  const int nvalid = max(0, min(SROWS, sq.n_ctx - base));
  const float* src = score + sq.start + base;
  if (nvalid == SROWS && (reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
    const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
    for (int j = 0; j < SROWS / 4; ++j) {
      const float4 v = __ldg(s4 + j);
      k[4 * j] = __float_as_uint(v.x);
      k[4 * j + 1] = __float_as_uint(v.y);
      k[4 * j + 2] = __float_as_uint(v.z);
      k[4 * j + 3] = __float_as_uint(v.w);
    }
  } else {
#pragma unroll
    for (int i = 0; i < SROWS; ++i) k[i] = i < nvalid ? __float_as_uint(__ldg(src + i)) : 0u;
  }
  bool nan = false;
#pragma unroll
  for (int i = 0; i < SROWS; ++i) {
    const bool ok = i < nvalid;
    k[i] = ok ? order_key(__uint_as_float(k[i])) : 0u;
    nan |= ok && k[i] == 0u;
  }
  *nvalid_out = nvalid;
  return nan;
}

// Exclusive scan of one int per thread over the block (warp shuffles, then the warp totals).
template <int NT>
__device__ __forceinline__ int block_excl_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    int t = lane < NT / 32 ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < NT / 32) warp_tot[lane] = t;  // inclusive
  }
  __syncthreads();
  const int excl = x - v + (w > 0 ? warp_tot[w - 1] : 0);
  if (total) *total = warp_tot[NT / 32 - 1];
  __syncthreads();
  return excl;
}

// ------------------------------------------------------------------ 1. histograms
__global__ void __launch_bounds__(SNT, 8) select_hist_kernel(const float* __restrict__ score,
                                                             const __grid_constant__ StreamParams p,
                                                             uint32_t* __restrict__ ghist, uint32_t* __restrict__ sinfo,
                                                             int32_t* __restrict__ dev_status) {
  __shared__ uint32_t h[NB12];
  const int c = blockIdx.x, s = seq_of_chunk(p, c);
  const StreamSeq& sq = p.s[s];
  if (sq.mode != MODE_SELECT) return;  // the whole CTA
  for (int j = threadIdx.x; j < NB12; j += SNT) h[j] = 0u;
  uint32_t k[SROWS];
  int nvalid;
  const bool nan = load_chunk(score, sq, c - sq.chunk0, k, &nvalid);
  __syncthreads();
#pragma unroll
  for (int i = 0; i < SROWS; ++i)
    if (i < nvalid) atomicAdd(&h[k[i] >> 20], 1u);
  const int any_nan = __syncthreads_or(nan);
  uint32_t* gh = ghist + (int64_t)s * NB12;
  for (int j = threadIdx.x; j < NB12; j += SNT)
    if (h[j]) atomicAdd(&gh[j], h[j]);
  if (any_nan && threadIdx.x == 0 && dev_status) atomicOr(dev_status, TG_DEV_NAN_SCORE);
  // The sequence's last CTA to finish finds the bin b1 of the kc-th largest key once for all
  // (no CTA waits: the others have already added their counts when it sees the final count).
  __shared__ int s_last, warp_tot[32];
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&sinfo[s * SI_WORDS + SI_DONE], 1u) == (uint32_t)(sq.nch - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // thread t holds bins [NB12 - BPT (t + 1), NB12 - BPT t), read high to low, so a scan in
  // thread order runs over the bins from the top
  const int tid = threadIdx.x, top = NB12 - BPT * tid;
  const uint4* hs = reinterpret_cast<const uint4*>(gh + top - BPT);
  uint32_t hb[BPT];
#pragma unroll
  for (int q = 0; q < BPT / 4; ++q) {
    const uint4 v = __ldcg(hs + q);  // bins top - BPT + 4 q .. + 3
    hb[BPT - 1 - 4 * q] = v.x;
    hb[BPT - 2 - 4 * q] = v.y;
    hb[BPT - 3 - 4 * q] = v.z;
    hb[BPT - 4 - 4 * q] = v.w;
  }
  int sum = 0;
#pragma unroll
  for (int j = 0; j < BPT; ++j) sum += (int)hb[j];
  const int excl = block_excl_scan<SNT>(sum, warp_tot, nullptr);
  if (excl < sq.kc && sq.kc <= excl + sum) {
    int acc = excl;
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      if (acc < sq.kc && sq.kc <= acc + (int)hb[j]) {
        sinfo[s * SI_WORDS + SI_B1] = (uint32_t)(top - 1 - j);
        sinfo[s * SI_WORDS + SI_NEED] = (uint32_t)(sq.kc - acc);
      }
      acc += (int)hb[j];
    }
  }
}

// ------------------------------------------------------------------ 2. threshold bin, candidates
__global__ void __launch_bounds__(SNT, 8) select_cand_kernel(const float* __restrict__ score,
                                                             const __grid_constant__ StreamParams p,
                                                             uint32_t* __restrict__ sinfo, uint32_t* __restrict__ cinfo,
                                                             uint2* __restrict__ cand) {
  __shared__ int warp_tot[32];
  const int c = blockIdx.x, s = seq_of_chunk(p, c);
  const StreamSeq& sq = p.s[s];
  if (sq.mode != MODE_SELECT) return;
  const int tid = threadIdx.x;
  uint32_t k[SROWS];
  int nvalid;
  load_chunk(score, sq, c - sq.chunk0, k, &nvalid);
  const uint32_t b1 = __ldcg(sinfo + s * SI_WORDS + SI_B1);  // from the histogram pass
  const int base = (c - sq.chunk0) * CH + tid * SROWS;  // this thread's first position
  // the chunk's keys above the bin, and its candidates: one slot reservation per CTA, each thread
  // writing its candidates after those of the threads before it
  int gt = 0, nc = 0;
#pragma unroll
  for (int i = 0; i < SROWS; ++i) {
    const bool ok = i < nvalid;
    const uint32_t bin = k[i] >> 20;
    gt += (ok && bin > b1) ? 1 : 0;
    nc += (ok && bin == b1) ? 1 : 0;
  }
  __shared__ uint32_t s_at;
  int total;
  const int cexcl = block_excl_scan<SNT>(nc, warp_tot, &total);
  if (tid == 0) s_at = total ? atomicAdd(&sinfo[s * SI_WORDS + SI_CAND], (uint32_t)total) : 0u;
  int gtotal;
  block_excl_scan<SNT>(gt, warp_tot, &gtotal);  // its barriers also publish s_at
  if (tid == 0) cinfo[(int64_t)c * CI_WORDS + CI_GT] = (uint32_t)gtotal;
  if (nc) {
    uint2* dst = cand + sq.cand_off + s_at + cexcl;
    int run = 0;
#pragma unroll
    for (int i = 0; i < SROWS; ++i)
      if (i < nvalid && (k[i] >> 20) == b1) dst[run++] = make_uint2(k[i], (uint32_t)(base + i));
  }
}

// ------------------------------------------------------------------ 3. T, per-chunk offsets, tail
__global__ void __launch_bounds__(RNT) select_resolve_kernel(const __grid_constant__ StreamParams p,
                                                             uint32_t* __restrict__ sinfo, uint32_t* __restrict__ cinfo,
                                                             const uint2* __restrict__ cand, int32_t* __restrict__ kept,
                                                             int32_t* __restrict__ cu_kept_dev,
                                                             int32_t* __restrict__ dev_status) {
  __shared__ uint32_t h[NB10];
  __shared__ int warp_tot[32];
  __shared__ uint32_t s_digit;
  __shared__ int s_need;
  __shared__ int gtc[MAX_CHUNKS_SEQ], eqc[MAX_CHUNKS_SEQ], gtb[MAX_CHUNKS_SEQ];
  const int s = blockIdx.x, tid = threadIdx.x;
  const StreamSeq& sq = p.s[s];
  for (int j = tid; j < sq.q; j += RNT) kept[sq.out_off + sq.kc + j] = sq.start + sq.n_ctx + j;
  if (tid == 0 && cu_kept_dev) {
    if (sq.b == 0) cu_kept_dev[0] = 0;
    cu_kept_dev[sq.b + 1] = sq.out_off + sq.kc + sq.q;
  }
  if (sq.mode == MODE_NONE) return;
  if (sq.mode == MODE_ALL) {  // every context token is kept: chunk c starts at row c CH
    for (int c = tid; c < sq.nch; c += RNT) cinfo[(int64_t)(sq.chunk0 + c) * CI_WORDS + CI_OUT] = (uint32_t)(c * CH);
    return;
  }
  const uint32_t* si = sinfo + s * SI_WORDS;
  const int ncand = (int)__ldcg(si + SI_CAND);
  uint32_t T = __ldcg(si + SI_B1);
  int need = (int)__ldcg(si + SI_NEED);
  const uint2* cs = cand + sq.cand_off;
  // the first RCPT * RNT candidates stay in registers; any beyond them are read again per pass
  uint2 rc[RCPT];
#pragma unroll
  for (int j = 0; j < RCPT; ++j) rc[j] = tid + j * RNT < ncand ? __ldcg(&cs[tid + j * RNT]) : make_uint2(0u, 0u);
  // the remaining 20 bits: two 10-bit passes over the candidates (all of them lie in bin T)
#pragma unroll 1
  for (int shift = 10; shift >= 0; shift -= 10) {
    h[tid] = 0u;  // RNT == NB10
    __syncthreads();
#pragma unroll
    for (int j = 0; j < RCPT; ++j)
      if (tid + j * RNT < ncand && (rc[j].x >> (shift + 10)) == T) atomicAdd(&h[(rc[j].x >> shift) & (NB10 - 1)], 1u);
    for (int i = tid + RCPT * RNT; i < ncand; i += RNT) {
      const uint32_t key = __ldcg(&cs[i].x);
      if ((key >> (shift + 10)) == T) atomicAdd(&h[(key >> shift) & (NB10 - 1)], 1u);
    }
    __syncthreads();
    const int v = (int)h[NB10 - 1 - tid];  // thread t holds digit NB10 - 1 - t: a scan from the top
    const int excl = block_excl_scan<RNT>(v, warp_tot, nullptr);
    if (excl < need && need <= excl + v) {
      s_digit = (uint32_t)(NB10 - 1 - tid);
      s_need = need - excl;
    }
    __syncthreads();
    T = (T << 10) | s_digit;
    need = s_need;
    __syncthreads();
  }
  // T is the kc-th largest key; `need` keys equal to T are kept, the lowest positions first
  for (int c = tid; c < sq.nch; c += RNT) {
    gtc[c] = 0;
    eqc[c] = 0;
    gtb[c] = (int)__ldcg(cinfo + (int64_t)(sq.chunk0 + c) * CI_WORDS + CI_GT);
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < RCPT; ++j) {
    if (tid + j * RNT >= ncand) continue;
    if (rc[j].x > T) atomicAdd(&gtc[rc[j].y / CH], 1);
    else if (rc[j].x == T) atomicAdd(&eqc[rc[j].y / CH], 1);
  }
  for (int i = tid + RCPT * RNT; i < ncand; i += RNT) {
    const uint2 e = __ldcg(&cs[i]);
    if (e.x > T) atomicAdd(&gtc[e.y / CH], 1);
    else if (e.x == T) atomicAdd(&eqc[e.y / CH], 1);
  }
  __syncthreads();
  if (tid == 0) {
    int out = 0, eq_rem = need;
    for (int c = 0; c < sq.nch; ++c) {
      uint32_t* ci = cinfo + (int64_t)(sq.chunk0 + c) * CI_WORDS;
      const int ek = eqc[c] < eq_rem ? eqc[c] : eq_rem;
      eq_rem -= ek;
      ci[CI_OUT] = (uint32_t)out;
      ci[CI_EQ] = (uint32_t)ek;
      out += gtb[c] + gtc[c] + ek;
    }
    if ((out != sq.kc || eq_rem != 0) && dev_status) atomicOr(dev_status, TG_DEV_BAD_INDEX);
    sinfo[s * SI_WORDS + SI_T] = T;
  }
}

// ------------------------------------------------------------------ 4. ordered compaction
__global__ void __launch_bounds__(SNT, 8) select_compact_kernel(const float* __restrict__ score,
                                                             const __grid_constant__ StreamParams p,
                                                             const uint32_t* __restrict__ sinfo,
                                                             const uint32_t* __restrict__ cinfo, int32_t* __restrict__ kept,
                                                             int32_t* __restrict__ dev_status) {
  __shared__ int warp_tot[32];
  const int c = blockIdx.x, s = seq_of_chunk(p, c);
  const StreamSeq& sq = p.s[s];
  const int tid = threadIdx.x;
  uint32_t k[SROWS];
  int nvalid;
  const bool nan = load_chunk(score, sq, c - sq.chunk0, k, &nvalid);
  const int base = (c - sq.chunk0) * CH + tid * SROWS;  // this thread's first position
  const int out0 = sq.out_off + (int)__ldcg(cinfo + (int64_t)c * CI_WORDS + CI_OUT);
  if (sq.mode == MODE_ALL) {  // every key is kept, in position order; NaN scores are still reported
#pragma unroll
    for (int i = 0; i < SROWS; ++i)
      if (i < nvalid) kept[out0 + tid * SROWS + i] = sq.start + base + i;
    if (__syncthreads_or(nan) && tid == 0 && dev_status) atomicOr(dev_status, TG_DEV_NAN_SCORE);
    return;
  }
  const uint32_t T = __ldcg(sinfo + s * SI_WORDS + SI_T);
  const int eq_keep = (int)__ldcg(cinfo + (int64_t)c * CI_WORDS + CI_EQ);
  uint32_t mg = 0u, me = 0u;  // bit i: key i of this thread is > T / == T
#pragma unroll
  for (int i = 0; i < SROWS; ++i) {
    const bool ok = i < nvalid;
    mg |= (ok && k[i] > T) ? (1u << i) : 0u;
    me |= (ok && k[i] == T) ? (1u << i) : 0u;
  }
  // the keys > T and == T before this thread (a chunk holds 4096 keys: no carry between halves)
  const int before = block_excl_scan<SNT>((__popc(mg) << 16) | __popc(me), warp_tot, nullptr);
  int GT = before >> 16, EQ = before & 0xffff;
  bool overflow = false;
  uint32_t m = mg | me;
  while (m) {  // this thread's candidates for output, in position order
    const int i = __ffs(m) - 1;
    m &= m - 1;
    const bool gt = (mg >> i) & 1u;
    const int eq_before = EQ + __popc(me & ((1u << i) - 1u));
    const int gt_before = GT + __popc(mg & ((1u << i) - 1u));
    if (gt || eq_before < eq_keep) {
      const int o = gt_before + (eq_before < eq_keep ? eq_before : eq_keep);
      if (out0 + o < sq.out_off + sq.kc) kept[out0 + o] = sq.start + base + i;
      else overflow = true;  // cannot happen for a correct threshold; never write past the slot
    }
  }
  if (overflow && dev_status) atomicOr(dev_status, TG_DEV_BAD_INDEX);
}

}  // namespace

namespace {

int64_t al256s(int64_t x) { return (x + 255) & ~int64_t(255); }

// Workspace layout (reused by every batch of kMaxSeqPerLaunch sequences): the histograms, the
// per-sequence words (both cleared before each batch), the per-chunk words, the candidates.
struct StreamLayout {
  int64_t off_sinfo, off_cinfo, off_cand, bytes;
};

StreamLayout stream_layout(int64_t max_chunks, int64_t max_cand) {
  StreamLayout L;
  L.off_sinfo = al256s((int64_t)kMaxSeqPerLaunch * NB12 * 4);
  L.off_cinfo = L.off_sinfo + al256s((int64_t)kMaxSeqPerLaunch * SI_WORDS * 4);
  L.off_cand = L.off_cinfo + al256s((max_chunks > 0 ? max_chunks : 1) * CI_WORDS * 4);
  L.bytes = L.off_cand + al256s((max_cand > 0 ? max_cand : 1) * 8);
  return L;
}

int chunks_of(const SelSeq& d) { return (d.kc > 0 && d.n_ctx > 0) ? (d.n_ctx + CH - 1) / CH : 0; }

void batch_extent(const SelSeq* seqs, int nseq, int64_t* max_chunks, int64_t* max_cand) {
  *max_chunks = 0;
  *max_cand = 0;
  for (int b0 = 0; b0 < nseq; b0 += kMaxSeqPerLaunch) {
    int64_t ch = 0, cd = 0;
    for (int i = b0; i < nseq && i < b0 + kMaxSeqPerLaunch; ++i) {
      ch += chunks_of(seqs[i]);
      if (seqs[i].kc > 0 && seqs[i].kc < seqs[i].n_ctx) cd += seqs[i].n_ctx;
    }
    *max_chunks = ch > *max_chunks ? ch : *max_chunks;
    *max_cand = cd > *max_cand ? cd : *max_cand;
  }
}

}  // namespace

int64_t select_stream_workspace(const SelSeq* seqs, int nseq) {
  int64_t mc, md;
  batch_extent(seqs, nseq, &mc, &md);
  return stream_layout(mc, md).bytes;
}

tg_status launch_select_stream(const float* score, const SelSeq* seqs, int nseq, int32_t* kept, int32_t* cu_kept_dev,
                               int32_t* dev_status, void* ws, cudaStream_t st) {
  int64_t mc, md;
  batch_extent(seqs, nseq, &mc, &md);
  const StreamLayout L = stream_layout(mc, md);
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* ghist = reinterpret_cast<uint32_t*>(base);
  uint32_t* sinfo = reinterpret_cast<uint32_t*>(base + L.off_sinfo);
  uint32_t* cinfo = reinterpret_cast<uint32_t*>(base + L.off_cinfo);
  uint2* cand = reinterpret_cast<uint2*>(base + L.off_cand);
  for (int b0 = 0; b0 < nseq; b0 += kMaxSeqPerLaunch) {
    const int nb = nseq - b0 < kMaxSeqPerLaunch ? nseq - b0 : kMaxSeqPerLaunch;
    StreamParams p = {};
    p.nseq = nb;
    int chunks = 0;
    int64_t cand_off = 0;
    for (int i = 0; i < nb; ++i) {
      const SelSeq& d = seqs[b0 + i];
      StreamSeq& q = p.s[i];
      q.start = d.start;
      q.n_ctx = d.n_ctx;
      q.q = d.q;
      q.kc = d.kc;
      q.out_off = d.out_off;
      q.b = d.b;
      q.chunk0 = chunks;
      q.nch = chunks_of(d);
      q.mode = q.nch == 0 ? MODE_NONE : (d.kc == d.n_ctx ? MODE_ALL : MODE_SELECT);
      q.cand_off = cand_off;
      if (q.mode == MODE_SELECT) cand_off += d.n_ctx;
      chunks += q.nch;
    }
    cudaError_t e = cudaMemsetAsync(base, 0, (size_t)(L.off_sinfo + (int64_t)kMaxSeqPerLaunch * SI_WORDS * 4), st);
    if (e != cudaSuccess) return cuda_status(e, "select (stream): clearing the histograms");
    if (chunks > 0) {
      select_hist_kernel<<<chunks, SNT, 0, st>>>(score, p, ghist, sinfo, dev_status);
      select_cand_kernel<<<chunks, SNT, 0, st>>>(score, p, sinfo, cinfo, cand);
    }
    select_resolve_kernel<<<nb, RNT, 0, st>>>(p, sinfo, cinfo, cand, kept, cu_kept_dev, dev_status);
    if (chunks > 0) select_compact_kernel<<<chunks, SNT, 0, st>>>(score, p, sinfo, cinfo, kept, dev_status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_status(e, "select (stream) launch");
  }
  return TG_OK;
}

}  // namespace tg
