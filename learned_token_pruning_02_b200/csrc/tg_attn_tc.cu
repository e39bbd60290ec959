// Token-gated causal attention over the kept tokens on the 5th-generation tensor cores.
//
// TokenGate paper page (thelatestinai.com), Figure 1(c): each attention weight is multiplied
// by its key's gate value g_j; with the row renormalised this is log g_j added to the logit
// (aitualizate.com article: the score acts as a bias on the attention logits, with a
// per-head gain). Causal on original positions, grouped KV heads (kv = h / (Hq/Hkv)).
//
// Design (B200, bf16 in, fp32 softmax and accumulation). A persistent grid, one CTA per SM (a CTA
// holds all 512 TMEM columns), walks work items (sequence, 128-row query tile, query head) from a
// list ordered by causal key range, longest first; CTA i takes items i, 2G-1-i, 2G+i, ... so each
// long item is paired with a short one. The key tiles of an item are split into two interleaved
// chains (even and odd tiles), each with its own softmax warpgroup, TMEM score buffer and TMEM
// output accumulator, so one group's exponentials overlap the other group's matrix products:
//   * warp 0: TMA loads each item's Q (as soon as the previous item's last S product has read
//     the old one) and the key tiles K_j (128 keys) into a 3-deep ring that runs across items;
//     warp 2 loads V_j into the stage of chain j % 2; warp 3 stages each tile's per-key bias
//     gain*log2(e)*log g_j in shared memory (a key with g = 0 is closed whatever the gain).
//   * warp 1: tcgen05.mma, issued by one elected lane while the whole warp runs the schedule
//     (its loop counters and operand descriptors stay warp-uniform, so issuing a product takes
//     few instructions on a scheduler it shares with two softmax warps). S_j = Q K_j^T
//     (M=128, N=128, K=D) into the chain's TMEM S buffer; O_c += P_j V_j with P_j read from
//     TMEM (A operand in tensor memory) and V_j from
//     shared memory (N-contiguous operand), in two halves of 64 keys so the first half enters the
//     tensor core while the softmax computes the second. S_{j+2} is issued right after PV_j: the
//     MMAs of one thread execute in issue order, so it overwrites P_j only after PV_j read it.
//   * warps 4-7 (chain 0) and 8-11 (chain 1): one query row per thread. The thread loads its
//     whole S row from TMEM into registers, forms scale*log2(e)*S + bias in pairs (causal mask
//     on the diagonal tile only), takes the row max with three-input max, and writes
//     P = 2^(x - m) back as packed bf16 into the same TMEM columns. The running max is only
//     moved (and O rescaled in TMEM, before the exponentials) when it grows by more than 8 (a
//     factor 256), which keeps every P <= 256 and the result exact after normalisation.
//   * Both warpgroups merge the two chains (max, sum, O), each writing half of the head
//     dimension of O (bf16); chain 0 also writes the LSE. The next item's Q load and first S
//     products overlap the merge; its first PV products wait until the merge has read O.
//   * The loader/issuer warpgroup gives registers to the softmax warpgroups (setmaxnreg).
//   * The unnormalised variant multiplies P by g_j^gain before the PV product and sums the
//     unbiased weights.
//   * Every wait is bounded (about 2 s); on a timeout the CTA sets TG_DEV_TIMEOUT, drains
//     its copies and MMAs, frees TMEM and returns.
#include "tg_internal.cuh"
#include "tg_sm100.cuh"

namespace tg {
namespace {

using namespace sm100;

constexpr int BQ = 128;
constexpr int BKV = 128;
constexpr int NTHREADS = 384;  // warp 0: Q/K loads, 1: MMA, 2: V loads, 3: key bias, 4-11: softmax
constexpr int KS = 3;           // K ring depth
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleSlack = 8.f;  // log2 units the running max may lag behind

struct ATParams {
  int off[kMaxSeqPerLaunch];
  int m[kMaxSeqPerLaunch];
  int nt[kMaxSeqPerLaunch];
  int nseq;
  int tmax;
  int n_items;  // (sequence, query tile, head) work items of the launch
};

template <int D>
struct ACfg {
  static constexpr int TILE_BYTES = BQ * D * 2;  // one 128 x D bf16 tile
  static constexpr int NBOX = D / 64;            // 64-column boxes per tile
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = TILE_BYTES;               // KS stages
  static constexpr int V_OFF = TILE_BYTES * (1 + KS);    // 2 stages (one per chain)
  static constexpr int TAIL_OFF = TILE_BYTES * (3 + KS);
  static constexpr int TAIL = 8192;  // barriers (256 B), bias and gate multipliers (2 KB), chain max/sum (4 KB)
  static constexpr int SMEM = 1024 + TAIL_OFF + TAIL;
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BQ, BKV, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BQ, D, true);
  static constexpr uint32_t TMEM_COLS = 512;  // S_c at [128c, 128c+128), O_c at [256 + Dc, 256 + D(c+1))
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}


// Work item w of the longest-first list: query tile t of sequence b, query head h. Items are
// ordered by the length of their causal key range (tile index) descending, sequences in order
// within one length, heads innermost.
struct Item {
  int b, t, h;
};

__device__ __forceinline__ Item decode_item(int w, int Hq, const ATParams& p) {
  Item it{0, 0, w % Hq};
  int r = w / Hq;
  for (int tt = p.tmax - 1; tt >= 0; --tt) {
    int cnt = 0;
    for (int s = 0; s < p.nseq; ++s) cnt += p.nt[s] > tt;
    if (r < cnt) {
      it.t = tt;
      for (int s = 0; s < p.nseq; ++s)
        if (p.nt[s] > tt) {
          if (r == 0) {
            it.b = s;
            break;
          }
          --r;
        }
      break;
    }
    r -= cnt;
  }
  return it;
}

// The k-th item of this CTA: a back-and-forth walk over the longest-first list (CTA i takes
// items i, 2G-1-i, 2G+i, 4G-1-i, ...), which pairs each CTA's long items with short ones.
__device__ __forceinline__ int item_of(int k, int G) {
  return (k & 1) ? (k + 1) * G - 1 - (int)blockIdx.x : k * G + (int)blockIdx.x;
}

template <int D, bool UNNORM>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const float* __restrict__ logg,
                   const float* __restrict__ gain, const int32_t* __restrict__ pos, __nv_bfloat16* __restrict__ O,
                   float* __restrict__ lse, int64_t m_tot, int Hq, int Hkv, float qk_scale, uint32_t flags,
                   int32_t* __restrict__ dev_status, int qkv_ready, uint64_t probe_ns,
                   const __grid_constant__ ATParams p) {
  using C = ACfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tail = smem + C::TAIL_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(tail);
  uint64_t* qfull = bars + 0;
  uint64_t* kfull = bars + 1;    // [KS]
  uint64_t* kempty = bars + 4;   // [KS]
  uint64_t* vfull = bars + 7;    // [2] per chain
  uint64_t* vempty = bars + 9;   // [2]
  uint64_t* bfull = bars + 11;   // [2]
  uint64_t* sfull = bars + 13;   // [2]
  uint64_t* pready = bars + 15;  // [2]
  uint64_t* pvdone = bars + 17;  // [2]
  uint64_t* mlready = bars + 19;
  uint64_t* drain = bars + 20;
  uint64_t* probe = bars + 21;   // test hook: a barrier nothing signals
  uint64_t* qempty = bars + 22;  // the item's last S product read Q: the next Q may load
  uint64_t* oempty = bars + 23;  // the item's merge read both O accumulators: the next PV may write
  uint64_t* phalf = bars + 26;   // [2] the first 64 keys of the chain's P are in TMEM
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 24);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* bias_s = reinterpret_cast<float*>(tail + 256);  // [2][128]
  float* gmul_s = bias_s + 2 * BKV;                      // [2][128]
  float* ml_s = gmul_s + 2 * BKV;                        // [2 items][2 chains][max, sum][128]

  const int G = gridDim.x, n_items = p.n_items;
  const int grp = Hq / Hkv;
  constexpr bool unnorm = UNNORM;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&vfull[s], 1);
      mbar_init(&vempty[s], 1);
      mbar_init(&bfull[s], 32);
      mbar_init(&sfull[s], 1);
      mbar_init(&pready[s], 128);
      mbar_init(&phalf[s], 128);
      mbar_init(&pvdone[s], 1);
    }
    mbar_init(mlready, 256);
    mbar_init(oempty, 256);
    mbar_init(drain, 1);
    *abort = 0;
    fence_barrier_init();
    wait_probe(probe, probe_ns, abort, dev_status);  // no-op unless a test asked for it
    // With qkv_ready (the chained prefill, where Q, K and V are inputs of the whole chain and the
    // previous kernel only produces log g and pos), the first item's Q and key tiles go out before
    // the wait on that kernel; otherwise anything may come from it and the wait is first.
    if (!qkv_ready) griddep_wait();  // inputs written by the previous kernel are visible from here on
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    const Item it = decode_item(item_of(0, G), Hq, p);
    const int off = p.off[it.b], nt = it.t + 1, kvh = it.h / grp;
    if (!*abort) {
      mbar_arrive_expect_tx(qfull, C::TILE_BYTES);
      for (int bx = 0; bx < C::NBOX; ++bx)
        tma_load_2d(smem + C::Q_OFF + bx * (BQ * 128), &tmQ, it.h * D + bx * 64, off + it.t * BQ, qfull);
      for (int j = 0; j < KS && j < nt; ++j) {
        uint8_t* kb = smem + C::K_OFF + j * C::TILE_BYTES;
        mbar_arrive_expect_tx(&kfull[j], C::TILE_BYTES);
        for (int bx = 0; bx < C::NBOX; ++bx)
          tma_load_2d(kb + bx * (BKV * 128), &tmK, kvh * D + bx * 64, off + j * BKV, &kfull[j]);
      }
    }
    if (qkv_ready) griddep_wait();  // log g and pos of the previous kernel are visible from here on
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_launch_dependents();  // the next kernel may start its prologue
  griddep_wait();               // (a no-op once thread 0's wait has returned)
  const uint32_t tmem = *tmem_slot;
  const bool skip = *abort;  // only the test probe sets it this early: nothing was issued

  // Register split: the loader / issuer warpgroup (warps 0-3) gives registers to the two softmax
  // warpgroups, which hold a whole 128-key row per thread. 128 x 64 + 256 x 216 = 63488 does not
  // exceed the launch's 384 x 168 = 64512, and the 13312 registers released cover the 12288 taken.
  if (warp < 4) {
  regs_dec<64>();
  if (skip) {
  } else if (warp == 0) {  // ------------------------------------------ Q and K producer
    if (lane == 0) {
      int jk = 0;         // key tiles issued so far (ring position)
      int q_issued = 1;   // Q tiles issued so far
      bool ok = true;
      for (int k = 0, w = item_of(0, G); ok && w < n_items; w = item_of(++k, G)) {
        const Item it = decode_item(w, Hq, p);
        const int off = p.off[it.b], nt = it.t + 1, kvh = it.h / grp;
        int j0 = 0;
        if (k == 0) {
          j0 = KS < nt ? KS : nt;  // loaded before the CTA-wide sync
          jk = j0;
        } else {
          if (!mbar_wait(qempty, (k - 1) & 1, abort, dev_status)) break;
          mbar_arrive_expect_tx(qfull, C::TILE_BYTES);
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_2d(smem + C::Q_OFF + bx * (BQ * 128), &tmQ, it.h * D + bx * 64, off + it.t * BQ, qfull);
          ++q_issued;
        }
        for (int j = j0; j < nt; ++j, ++jk) {
          const int s = jk % KS;
          if (!mbar_wait(&kempty[s], ((jk / KS) & 1) ^ 1u, abort, dev_status)) {
            ok = false;
            break;
          }
          uint8_t* kb = smem + C::K_OFF + s * C::TILE_BYTES;
          mbar_arrive_expect_tx(&kfull[s], C::TILE_BYTES);
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_2d(kb + bx * (BKV * 128), &tmK, kvh * D + bx * 64, off + j * BKV, &kfull[s]);
        }
      }
      if (*abort) {  // let the copies in flight land before the CTA can leave
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(qfull, (q_issued - 1) & 1) && globaltimer_ns() - t0 < 1000000000ull) {
        }
        for (int jj = jk - KS < 0 ? 0 : jk - KS; jj < jk; ++jj) {
          const uint64_t t1 = globaltimer_ns();
          while (!mbar_try_wait(&kfull[jj % KS], (jj / KS) & 1) && globaltimer_ns() - t1 < 1000000000ull) {
          }
        }
      }
    }
  } else if (warp == 2) {  // ------------------------------------------------- V producer
    if (lane == 0) {
      int vc[2] = {0, 0};  // V tiles issued per chain
      bool ok = true;
      for (int k = 0, w = item_of(0, G); ok && w < n_items; w = item_of(++k, G)) {
        const Item it = decode_item(w, Hq, p);
        const int off = p.off[it.b], nt = it.t + 1, kvh = it.h / grp;
        for (int j = 0; j < nt; ++j) {
          const int c = j & 1;
          if (!mbar_wait(&vempty[c], (vc[c] & 1) ^ 1u, abort, dev_status)) {
            ok = false;
            break;
          }
          uint8_t* vb = smem + C::V_OFF + c * C::TILE_BYTES;
          mbar_arrive_expect_tx(&vfull[c], C::TILE_BYTES);
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_2d(vb + bx * (BKV * 128), &tmV, kvh * D + bx * 64, off + j * BKV, &vfull[c]);
          ++vc[c];
        }
      }
      if (*abort) {
        for (int c = 0; c < 2; ++c) {
          const uint64_t t1 = globaltimer_ns();
          while (vc[c] > 0 && !mbar_try_wait(&vfull[c], (vc[c] - 1) & 1) && globaltimer_ns() - t1 < 1000000000ull) {
          }
        }
      }
    }
  } else if (warp == 3) {  // ---------------------------------------------- key-bias stager
    // Per-key bias of key tile j (log2 domain), 4 keys per lane, staged in the chain's slot as
    // soon as the chain's previous softmax has read it; the log g loads go out first.
    int bc[2] = {0, 0};  // tiles staged per chain
    bool ok = true;
    for (int k = 0, w = item_of(0, G); ok && w < n_items; w = item_of(++k, G)) {
      const Item it = decode_item(w, Hq, p);
      const int off = p.off[it.b], m = p.m[it.b], nt = it.t + 1;
      const float gain2 = (gain ? gain[it.h] : 1.f) * kLog2e;
      for (int j = 0; j < nt; ++j) {
        const int c = j & 1;
        float bv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kl = j * BKV + lane * 4 + e;
          const float lg = (logg && kl < m) ? logg[off + kl] : 0.f;
          bv[e] = lg == -INFINITY ? -INFINITY : gain2 * lg;  // g = 0 closes the key whatever the gain
        }
        if (bc[c] > 0 && !__all_sync(0xffffffffu, mbar_wait(&pready[c], (bc[c] - 1) & 1, abort, dev_status))) {
          ok = false;
          break;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          bias_s[c * BKV + lane * 4 + e] = unnorm ? 0.f : bv[e];
          gmul_s[c * BKV + lane * 4 + e] = unnorm ? ex2(bv[e]) : 1.f;
        }
        mbar_arrive(&bfull[c]);
        ++bc[c];
      }
    }
  } else if (warp == 1) {  // ------------------------------------------------ MMA issuer
    {
      const bool leader = elect_one();
      const uint32_t qa = smem_u32(smem + C::Q_OFF);
      int jk = 0;           // key tiles consumed (ring position)
      int pc[2] = {0, 0};  // PV products issued per chain
      // Per item, a fixed schedule with blocking (suspending) waits: S_0, S_1, then PV_j
      // followed by S_{j+2} for j = 0, 1, ... The chains alternate, so this is the order the
      // products become ready in, and a waiting issuer sleeps instead of taking issue slots from
      // the softmax warps that share its scheduler. PV_j needs P_j and V_j; S_{j+2} needs
      // K_{j+2} and overwrites the TMEM columns PV_j reads P_j from, which is safe without
      // waiting for PV_j to complete: the MMAs one thread issues execute in issue order, so
      // S_{j+2} writes only after PV_j has read its operand, and the tensor pipe never drains
      // between them. The next item's first S products follow the last PV products the same
      // way; its first PV products wait until the merge of the item before has read O.
      auto issue_s = [&](int c) -> bool {
        const int ks = jk % KS;
        if (!__all_sync(0xffffffffu, mbar_wait(&kfull[ks], (jk / KS) & 1, abort, dev_status))) return false;
        tc_fence_after();
        const uint32_t ka = smem_u32(smem + C::K_OFF + ks * C::TILE_BYTES);
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t o = (kk >> 2) * (BQ * 128) + (kk & 3) * 32;
            mma_ss(tmem + c * BKV, sdesc_sw128(qa + o, 16, 1024), sdesc_sw128(ka + o, 16, 1024), C::IDESC_QK, kk > 0);
          }
          mma_commit(&sfull[c]);
          mma_commit(&kempty[ks]);
        }
        __syncwarp();
        ++jk;
        return true;
      };
      bool ok = true;
      for (int k = 0, w = item_of(0, G); ok && w < n_items; w = item_of(++k, G)) {
        const Item it = decode_item(w, Hq, p);
        const int nt = it.t + 1;
        ok = __all_sync(0xffffffffu, mbar_wait(qfull, k & 1, abort, dev_status));
        for (int j = 0; ok && j < 2 && j < nt; ++j) ok = issue_s(j);
        if (ok && nt <= 2 && leader) mma_commit(qempty);  // every S product of the item is issued
        for (int j = 0; ok && j < nt; ++j) {
          const int c = j & 1;
          if (!__all_sync(0xffffffffu, mbar_wait(&phalf[c], pc[c] & 1, abort, dev_status) &&
                                           mbar_wait(&vfull[c], pc[c] & 1, abort, dev_status) &&
                                           (j != 0 || k == 0 || mbar_wait(oempty, (k - 1) & 1, abort, dev_status)))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t va = smem_u32(smem + C::V_OFF + c * C::TILE_BYTES);
          if (leader) {
#pragma unroll
            for (int kk = 0; kk < BKV / 32; ++kk)  // keys 0-63: their P is in TMEM
              mma_ts(tmem + 256 + c * D, tmem + c * BKV + kk * 8, sdesc_sw128(va + kk * 2048, BKV * 128, 1024),
                     C::IDESC_PV, (j >= 2 || kk > 0) ? 1u : 0u);
          }
          __syncwarp();
          if (!__all_sync(0xffffffffu, mbar_wait(&pready[c], pc[c] & 1, abort, dev_status))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (leader) {
#pragma unroll
            for (int kk = BKV / 32; kk < BKV / 16; ++kk)  // keys 64-127
              mma_ts(tmem + 256 + c * D, tmem + c * BKV + kk * 8, sdesc_sw128(va + kk * 2048, BKV * 128, 1024),
                     C::IDESC_PV, 1u);
            mma_commit(&pvdone[c]);
            mma_commit(&vempty[c]);
          }
          __syncwarp();
          ++pc[c];
          if (j + 2 < nt) {
            ok = issue_s(c);
            if (ok && j + 3 == nt && leader) mma_commit(qempty);  // that was the item's last S product
          }
        }
      }
      if (leader) {
        mma_commit(drain);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < 1000000000ull) {
        }
      }
      __syncwarp();
    }
  }
  } else if (!skip) {  // ----------------------------------------------------- softmax warpgroups
    regs_inc<216>();
    const int c = (warp - 4) >> 2;  // chain: 0 = warps 4-7 (even tiles), 1 = warps 8-11 (odd tiles)
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;  // query row in the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const uint32_t tS = tmem + lane_base + c * BKV;
    const uint32_t tO = tmem + lane_base + 256 + c * D;
    int cnt[2] = {0, 0};  // tiles through each chain so far (this thread tracks both)
    bool ok = true;
    for (int k = 0, w = item_of(0, G); ok && w < n_items; w = item_of(++k, G)) {
      const Item it = decode_item(w, Hq, p);
      const int t = it.t, h = it.h, off = p.off[it.b], m = p.m[it.b];
      const int nt = t + 1;
      const int n0 = (nt + 1) >> 1, n1 = nt >> 1;  // key tiles in chain 0 (even) and chain 1 (odd)
      const int il = t * BQ + r;                   // row within the sequence
      const bool valid = il < m;
      if (c == 0 && h == 0 && valid && il > 0 && dev_status && pos && pos[off + il - 1] >= pos[off + il])
        atomicOr(dev_status, TG_DEV_POS_NOT_ASCENDING);
      float m_run = -INFINITY, l_run = 0.f;
      const int n_mine = c == 0 ? n0 : n1;
      for (int u = 0; u < n_mine; ++u) {
        const int j = 2 * u + c;
        const int nc = cnt[c] + u;  // this tile's use count of the chain's buffers
        // warp-uniform waits: the tcgen05.ld/st below are warp-collective
        if (!__all_sync(0xffffffffu, mbar_wait(&bfull[c], nc & 1, abort, dev_status) &&
                                         mbar_wait(&sfull[c], nc & 1, abort, dev_status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[BKV];  // the whole S row of this thread, then the logits
#pragma unroll
        for (int ch = 0; ch < BKV / 32; ++ch)
          tmem_ld32(tS + ch * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[ch * 32]));
        tmem_wait_ld();
        float* x = reinterpret_cast<float*>(sr);
        const float4* bs4 = reinterpret_cast<const float4*>(bias_s + c * BKV);
        const float2 qs2 = make_float2(qk_scale, qk_scale);
        // log2-domain logits scale*log2(e)*S + bias in pairs; causal mask on the diagonal tile only
#pragma unroll
        for (int q = 0; q < BKV / 4; ++q) {
          const float4 bb = bs4[q];
          const float2 v0 = __ffma2_rn(make_float2(x[4 * q], x[4 * q + 1]), qs2, make_float2(bb.x, bb.y));
          const float2 v1 = __ffma2_rn(make_float2(x[4 * q + 2], x[4 * q + 3]), qs2, make_float2(bb.z, bb.w));
          x[4 * q] = v0.x;
          x[4 * q + 1] = v0.y;
          x[4 * q + 2] = v1.x;
          x[4 * q + 3] = v1.y;
        }
        if (j == t) {
#pragma unroll
          for (int col = 0; col < BKV; ++col)
            if (col > r) x[col] = -INFINITY;
        }
        // row max with three-input max, four independent chains
        float ma = -INFINITY, mbx = -INFINITY, mc = -INFINITY, md = -INFINITY;
#pragma unroll
        for (int q = 0; q < BKV / 8; ++q) {
          ma = max3(ma, x[8 * q], x[8 * q + 1]);
          mbx = max3(mbx, x[8 * q + 2], x[8 * q + 3]);
          mc = max3(mc, x[8 * q + 4], x[8 * q + 5]);
          md = max3(md, x[8 * q + 6], x[8 * q + 7]);
        }
        const float mx = max3(ma, mbx, fmaxf(mc, md));
        const float m_cand = fmaxf(m_run, mx);
        // lazy rescale: move the running max only when it grows by more than the slack
        const bool resc = __any_sync(0xffffffffu, m_cand > m_run + kRescaleSlack);
        float alpha = 1.f;
        if (resc) {
          alpha = m_run == -INFINITY ? 0.f : ex2(m_run - m_cand);  // 0 on the chain's first tile
          m_run = m_cand;
        }
        if (resc && u > 0) {  // rescale the chain's O once its previous PV product has landed
          if (!__all_sync(0xffffffffu, mbar_wait(&pvdone[c], (nc - 1) & 1, abort, dev_status))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tO + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tO + c0, o);
          }
          tmem_wait_st();
        }
        const float mb = m_run == -INFINITY ? 0.f : m_run;
        const float2 nm2 = make_float2(-mb, -mb);
        // P = 2^(x - m) as packed bf16 into the first half of the same TMEM columns, 32 columns
        // (64 keys) at a time so the first store overlaps the second half's arithmetic
        float2 sa = make_float2(0.f, 0.f), sb = make_float2(0.f, 0.f);
        uint32_t pk[BKV / 2];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
          for (int q = h2 * (BKV / 4); q < (h2 + 1) * (BKV / 4); ++q) {
            const float2 d = __fadd2_rn(make_float2(x[2 * q], x[2 * q + 1]), nm2);
            float2 pr;
            if constexpr (UNNORM) {
              pr = make_float2(ex2(d.x), ex2(d.y));
              const float2 gg = *reinterpret_cast<const float2*>(gmul_s + c * BKV + 2 * q);
              if (q & 1) sb = __fadd2_rn(sb, pr); else sa = __fadd2_rn(sa, pr);
              pr = __fmul2_rn(pr, gg);
            } else {
              pr = make_float2(ex2(d.x), ex2(d.y));
              if (q & 1) sb = __fadd2_rn(sb, pr); else sa = __fadd2_rn(sa, pr);
            }
            pk[q] = pack_bf16(pr.x, pr.y);
          }
          tmem_st32(tS + h2 * 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[h2 * 32]));
          if (h2 == 0) {  // the first 64 keys' P may go into the tensor core already
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&phalf[c]);
          }
        }
        const float2 s2 = __fadd2_rn(sa, sb);
        const float sum = s2.x + s2.y;
        tmem_wait_st();
        l_run = l_run * alpha + sum;
        tc_fence_before();
        mbar_arrive(&pready[c]);
      }
      if (!ok) break;
      cnt[0] += n0;
      cnt[1] += n1;
      // Merge the two chains: both warpgroups publish their (max, sum), then each writes half of
      // the head dimension of O from both accumulators; chain 0 also writes the LSE. The (max,
      // sum) slots alternate between items, so a warpgroup that runs ahead into the next item
      // never overwrites values the other one still reads.
      float* mlb = ml_s + (k & 1) * 4 * BKV;
      mlb[c * 2 * BKV + r] = m_run;
      mlb[c * 2 * BKV + BKV + r] = l_run;
      mbar_arrive(mlready);
      if (!__all_sync(0xffffffffu, mbar_wait(mlready, k & 1, abort, dev_status) &&
                                       mbar_wait(&pvdone[0], (cnt[0] - 1) & 1, abort, dev_status) &&
                                       (n1 == 0 || mbar_wait(&pvdone[1], (cnt[1] - 1) & 1, abort, dev_status)))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float m0 = mlb[r], l0 = mlb[BKV + r];
      const float m1 = mlb[2 * BKV + r], l1 = mlb[3 * BKV + r];
      const float mfin = fmaxf(m0, m1);
      const float mz = mfin == -INFINITY ? 0.f : mfin;
      const float f0 = ex2(m0 - mz), f1 = n1 > 0 ? ex2(m1 - mz) : 0.f;
      const float lt = l0 * f0 + l1 * f1;
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const float s0 = f0 * inv, s1 = f1 * inv;
      __nv_bfloat16* orow = O + ((int64_t)(off + il) * Hq + h) * D;
      const uint32_t tO0 = tmem + lane_base + 256, tO1 = tmem + lane_base + 256 + D;
#pragma unroll 1
      for (int c0 = c * (D / 2); c0 < (c + 1) * (D / 2); c0 += 32) {
        uint32_t o0[32], o1[32];
        tmem_ld32(tO0 + c0, o0);
        if (n1 > 0) tmem_ld32(tO1 + c0, o1);
        tmem_wait_ld();
        uint32_t pkd[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float a0 = __uint_as_float(o0[2 * e]) * s0, a1 = __uint_as_float(o0[2 * e + 1]) * s0;
          if (n1 > 0) {
            a0 = fmaf(__uint_as_float(o1[2 * e]), s1, a0);
            a1 = fmaf(__uint_as_float(o1[2 * e + 1]), s1, a1);
          }
          pkd[e] = pack_bf16(a0, a1);
        }
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pkd[4 * v], pkd[4 * v + 1], pkd[4 * v + 2], pkd[4 * v + 3]);
        }
      }
      if (c == 0 && valid && lse) lse[(int64_t)h * m_tot + off + il] = (mz + __log2f(lt)) * kLn2;
      tc_fence_before();
      mbar_arrive(oempty);  // both accumulators are read: the next item's PV products may overwrite them
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int D>
tg_status launch_d(const AttnArgs& a, const AttnSeq* seqs, int nseq, cudaStream_t st) {
  using C = ACfg<D>;
  ATParams p = {};
  p.nseq = nseq;
  int units = 0, tmax = 0;
  for (int i = 0; i < nseq; ++i) {
    p.off[i] = seqs[i].off;
    p.m[i] = seqs[i].m;
    p.nt[i] = (seqs[i].m + BQ - 1) / BQ;
    units += p.nt[i];
    tmax = p.nt[i] > tmax ? p.nt[i] : tmax;
  }
  p.tmax = tmax;
  if (units == 0) return TG_OK;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_bf16_2d(&tq, a.Q, (uint64_t)a.m_tot, (uint64_t)a.Hq * D, (uint64_t)a.Hq * D, BQ, 64) ||
      !make_tmap_bf16_2d(&tk, a.K, (uint64_t)a.m_tot, (uint64_t)a.Hkv * D, (uint64_t)a.Hkv * D, BKV, 64) ||
      !make_tmap_bf16_2d(&tv, a.V, (uint64_t)a.m_tot, (uint64_t)a.Hkv * D, (uint64_t)a.Hkv * D, BKV, 64))
    return fail(TG_ERR_CUDA, "tg_gated_attn_fwd: building the TMA tensor maps failed");
  const bool un = (a.flags & TG_ATTN_UNNORMALISED) != 0;
  auto kern = un ? attn_tc_kernel<D, true> : attn_tc_kernel<D, false>;
  const int slot = D == 64 ? (un ? ATTR_ATTN64_UN : ATTR_ATTN64) : (un ? ATTR_ATTN128_UN : ATTR_ATTN128);
  if (attrs_needed(slot)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return cuda_status(e, "tg_gated_attn_fwd: cudaFuncSetAttribute");
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return cuda_status(e, "tg_gated_attn_fwd: cudaFuncSetAttribute");
    mark_attrs_set(slot);
  }
  // persistent: one CTA per SM (the kernel holds all of an SM's TMEM), each walking its items
  p.n_items = units * a.Hq;
  const int sms = device_sm_count();
  const int grid = p.n_items < sms ? p.n_items : sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(NTHREADS);
  cfg.dynamicSmemBytes = (size_t)C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attribute(PDL_ATTN)};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, a.logg, a.head_gain, a.pos,
                                        static_cast<__nv_bfloat16*>(a.O), a.lse, a.m_tot, a.Hq, a.Hkv,
                                        a.scale * kLog2e, a.flags, a.dev_status, a.qkv_ready ? 1 : 0,
                                        wait_probe_ns(), p),
                     "tg_gated_attn_fwd: attn_tc launch");
}

}  // namespace

tg_status launch_attn_tc(const AttnArgs& a, const AttnSeq* seqs, int nseq, cudaStream_t st) {
  if (a.D == 64) return launch_d<64>(a, seqs, nseq, st);
  return launch_d<128>(a, seqs, nseq, st);
}

}  // namespace tg
