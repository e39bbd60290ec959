// Gradients of the token-gated causal attention on the 5th-generation tensor cores (bf16 in,
// fp32 softmax arithmetic and accumulation).
//
// TokenGate paper page (thelatestinai.com), Figure 1(c): the gated attention is what lets the
// top-K selector train end to end; aitualizate.com article ("Cómo consigue entrenar una
// selección top-K"): the score enters the attention logits as a bias, so its gradient is that
// of an additive logit bias. Per sequence, query head h and KV head h / (Hq / Hkv), with
// S = scale Q K^T + gain_h log g^T (causal), P = exp(S - lse), Dv_i = rowsum(dO_i * O_i):
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - Dv),  dQ = scale dS K,  dK = scale dS^T Q,
//   d log g_j = sum_h gain_h sum_i dS_ij,  d score_j = d log g_j * -expm1(log g_j).
//
// Four launches per group of sequences; no workspace, no atomics, deterministic results:
//   1. bwd_prep_kernel: Dv of every (row, query head), written into element 0 of that row's dQ
//      vector. Only the dQ kernel (launch 4) overwrites it, after reading it.
//   2. attn_bwd_dkdv_tc: per (128-key tile, KV head) one CTA, or a cluster of two CTAs when
//      the KV group has an even number G of query heads (each CTA takes every other head);
//      every CTA walks the query tiles at or after its key tile. Per step (query tile, head):
//        S^T = K Q^T and dP^T = V dO^T (M = 128 keys, N = 128 queries, both operands K-major as
//        stored) take turns in one 128-column TMEM region: dP^T_n is issued as soon as the two
//        epilogue warpgroups (one key row per thread, 64 queries each) hold S^T_n in registers,
//        and S^T_{n+1} as soon as they hold dP^T_n. They write P^T and dS^T as packed bf16 into
//        TMEM regions of their own; dV += P^T dO and dK += dS^T Q take that A operand from TMEM
//        and dO, Q from shared memory as N-contiguous (MN-major) B operands.
//      A cluster's two partial dK, dV (and d log g) are added in rank order: each CTA owns half
//      of the columns, the other CTA bulk-copies its staged partial of them into the owner's
//      shared memory, and the owner stores the sums; rank 0 stores the KV head's d log g
//      partial in element 1 of the dQ vector (key row, query head kvh).
//   3. bwd_dlogg_kernel: d log g = the sum of those partials over the KV heads, in order, and
//      d score.
//   4. attn_bwd_dq_tc: per (128-query tile, head), walking the key tiles up to the diagonal:
//      S = Q K^T (two TMEM buffers, so S_{j+1} is formed while the epilogue works on tile j),
//      dP = dO V^T, dS written as bf16 into dP's columns, dQ += dS K (K as an MN-major B).
// Work items are ordered by the length of their chain, longest first, so the hardware's
// in-order dispatch of CTAs balances the causal triangle.
// Masks use the kept-row index on the diagonal tile (positions ascend inside a sequence; a
// violation is flagged by the pre-pass), the same rule as the forward. Key rows past the
// sequence get a -inf bias and query rows past it lse = +inf, so their weights are exactly 0.
// Every wait is bounded (about 2 s); on a timeout the CTA sets TG_DEV_TIMEOUT, drains its
// copies and products, frees TMEM and returns without writing results.
#include "tg_attn_bwd.cuh"
#include "tg_sm100.cuh"

namespace tg {
namespace {

using namespace sm100;

constexpr int BT = 128;        // rows of every tile (keys or queries)
constexpr int NTHREADS = 384;  // warp 0: TMA, 1: MMA + TMEM, 2: idle, 3: vector stager, 4-11: epilogue
constexpr int MAXC = 2;        // CTAs per cluster of the dK/dV kernel
constexpr float kLog2e = 1.4426950408889634f;
constexpr int SMEM_LIMIT = 227 * 1024;

struct TcParams {
  int off[kMaxSeqPerLaunch];
  int m[kMaxSeqPerLaunch];
  int nt[kMaxSeqPerLaunch];  // ceil(m / 128)
  int nseq;
  int tmax;
  int C;  // CTAs per cluster of the dK/dV kernel
};

__device__ __forceinline__ float key_bias(float gain2, float lg) { return lg == -INFINITY ? -INFINITY : gain2 * lg; }
__device__ __forceinline__ float lse_or_inf(float l) { return l == -INFINITY ? INFINITY : l; }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Entries (sequence, L) with 1 <= L <= nt[b] whose length is at least L
__device__ __forceinline__ int count_ge(int L, const TcParams& p) {
  int c = 0;
  for (int s = 0; s < p.nseq; ++s) c += max(0, p.nt[s] - L + 1);
  return c;
}

// The w-th entry of the list of every (sequence b, chain length L), 1 <= L <= nt[b], ordered
// by L descending and by sequence within one L.
__device__ __forceinline__ void decode_len(int w, const TcParams& p, int& b, int& L) {
  int lo = 1, hi = p.tmax;  // the largest L with count_ge(L) > w
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (count_ge(mid, p) > w) lo = mid; else hi = mid - 1;
  }
  L = lo;
  int r = w - count_ge(L + 1, p);
  b = 0;
  for (int s = 0; s < p.nseq; ++s)
    if (p.nt[s] >= L) {
      if (r == 0) {
        b = s;
        return;
      }
      --r;
    }
}

__device__ __forceinline__ uint32_t mapa_rank(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ int ld_cluster_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// Barrier over the first `nthreads` threads arriving at named barrier `id`, returning whether
// any of them passed a nonzero `pred`.
__device__ __forceinline__ int bar_red_or(int id, int nthreads, int pred) {
  int r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.s32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n selp.s32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"(pred), "r"(id), "r"(nthreads)
      : "memory");
  return r;
}

// Bounded wait for copies still in flight after an abort (the CTA may not exit before they land).
__device__ __forceinline__ void settle(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity) && globaltimer_ns() - t0 < 1000000000ull) {
  }
}

// ------------------------------------------------------------------ 1. Dv = rowsum(dO * O)
// Vectors (row, query head) of rows [r0, r1) are contiguous D-element runs of O and dO. A warp
// takes 4 * 32 / (D / 8) consecutive ones: each lane loads 16 bytes of a vector per load, all
// eight loads (four of dO, four of O) in flight before the first use; the D / 8 lanes of a
// vector add their parts with shuffles and the first writes Dv to dQ[row, h, 0]. The lanes that
// write a head-0 vector also check that positions ascend inside each sequence.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ O,
                                                       const __nv_bfloat16* __restrict__ dO,
                                                       const int32_t* __restrict__ pos, float* __restrict__ dQ,
                                                       int r0, int r1, int Hq, int32_t* __restrict__ dev_status,
                                                       const __grid_constant__ TcParams p) {
  constexpr int LPV = D / 8;     // lanes per vector (16 bytes each)
  constexpr int VPL = 32 / LPV;  // vectors per load instruction of the warp
  constexpr int NL = 4;          // loads per tensor per lane
  griddep_wait();  // O and dO come from earlier work on the stream
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t v_end = (int64_t)r1 * Hq;
  const int64_t vw = (int64_t)r0 * Hq + ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * (VPL * NL);
  uint4 a[NL], o[NL];
#pragma unroll
  for (int j = 0; j < NL; ++j) {
    const int64_t v = vw + j * VPL + lane / LPV;
    const int64_t e = v * D + (lane % LPV) * 8;
    a[j] = v < v_end ? *reinterpret_cast<const uint4*>(dO + e) : make_uint4(0, 0, 0, 0);
    o[j] = v < v_end ? *reinterpret_cast<const uint4*>(O + e) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int j = 0; j < NL; ++j) {
    const uint32_t* aw = reinterpret_cast<const uint32_t*>(&a[j]);
    const uint32_t* ow = reinterpret_cast<const uint32_t*>(&o[j]);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&aw[i]));
      const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ow[i]));
      s = fmaf(x.x, y.x, fmaf(x.y, y.y, s));
    }
#pragma unroll
    for (int m = LPV / 2; m > 0; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
    const int64_t v = vw + j * VPL + lane / LPV;
    if (lane % LPV == 0 && v < v_end) {
      dQ[v * D] = s;
      const int64_t row = v / Hq;
      if (v % Hq == 0 && dev_status) {
        bool start = false;
        for (int i = 0; i < p.nseq; ++i) start |= p.off[i] == row;
        if (!start && pos[row - 1] >= pos[row]) atomicOr(dev_status, TG_DEV_POS_NOT_ASCENDING);
      }
    }
  }
}

// ------------------------------------------------------------------ 2. dK, dV (and d log g partials)
template <int D>
struct KCfg {
  static constexpr int TILE = BT * D * 2;  // one 128 x D bf16 tile (D / 64 boxes of 128 rows x 128 bytes)
  static constexpr int NBOX = D / 64;
  static constexpr int K_OFF = 0, V_OFF = TILE;
  static constexpr int Q_OFF = 2 * TILE;  // stage s: Q at Q_OFF + 2 s TILE, dO right after it
  static constexpr int TAIL_OFF = 6 * TILE;
  static constexpr int TAIL = 256 + 4 * BT * 4 + 2 * BT * 4;  // barriers, [2 stages][-lse2, -Dv][128], dl [2][128]
  static constexpr int SMEM = 1024 + TAIL_OFF + TAIL;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(BT, BT, false);
  static constexpr uint32_t IDESC_G = idesc_bf16_f32(BT, D, true);
  // TMEM columns: region A [0, 128) holds S^T_n and then dP^T_n, P^T [128, 192) and dS^T
  // [192, 256) (bf16, 32 columns per query half), dV [256, 256 + D), dK [256 + D, 256 + 2D)
  static constexpr uint32_t T_P = 128, T_DS = 192, T_DV = 256, T_DK = 256 + D;
  static_assert(SMEM <= SMEM_LIMIT, "shared memory budget");
  static_assert(4 * TILE >= 2 * BT * D * 4, "the Q / dO stages hold the fp32 dK, dV partials at the end");
};

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_bwd_dkdv_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                     const float* __restrict__ logg, const float* __restrict__ gain, const float* __restrict__ lse,
                     float* __restrict__ dQ, float* __restrict__ dK, float* __restrict__ dV, int64_t m_tot, int Hq,
                     int Hkv, float qk_scale2, float scale, int want_dl, int32_t* __restrict__ dev_status,
                     uint64_t probe_ns, const __grid_constant__ TcParams p) {
  using C = KCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* tail = smem + C::TAIL_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(tail);
  uint64_t* kvfull = bars + 0;
  uint64_t* qfull = bars + 1;    // [2] Q and dO of a stage landed
  uint64_t* qempty = bars + 3;   // [2] the stage's last product (dK) read them
  uint64_t* vfull = bars + 5;    // [2] the stage's per-query vectors are staged
  uint64_t* vempty = bars + 7;   // [2] both epilogue warpgroups read them
  uint64_t* sfull = bars + 9;    // S^T landed in region A
  uint64_t* dpfull = bars + 10;  // dP^T landed in region A
  uint64_t* pready = bars + 11;  // [2] a warpgroup's half of P^T is in TMEM
  uint64_t* dsready = bars + 13; // [2] a warpgroup's half of dS^T is in TMEM
  uint64_t* accdone = bars + 15;
  uint64_t* drain = bars + 16;
  uint64_t* probe = bars + 17;   // test hook: a barrier nothing signals
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
  uint64_t* xbar = bars + 19;    // the peer's partials of this CTA's columns landed
  uint64_t* sfree = bars + 20;   // the epilogue holds S^T in registers: dP^T may overwrite region A
  uint64_t* afree = bars + 21;   // the epilogue holds dP^T in registers: the next S^T may overwrite A
  uint64_t* pfree = bars + 22;   // dV read P^T: the next P^T may overwrite it
  uint64_t* dsfree = bars + 23;  // dK read dS^T: the next dS^T may overwrite it
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* vec_s = reinterpret_cast<float*>(tail + 256);  // [2 stages][-lse * log2(e), -Dv][128]
  float* dl_s = vec_s + 4 * BT;                         // [2 warpgroups][128]

  const int G = Hq / Hkv, Cn = p.C;
  const int rank = (int)(blockIdx.x % (unsigned)Cn);
  const int kvh = (int)((blockIdx.x / (unsigned)Cn) % (unsigned)Hkv);
  int b, L;
  decode_len((int)(blockIdx.x / (unsigned)(Cn * Hkv)), p, b, L);
  const int off = p.off[b], m = p.m[b];
  const int kt = p.nt[b] - L;                 // this key tile; query tiles kt .. nt-1 see it
  const int nh = G / Cn;                      // query heads kvh G + rank + i C, i < nh
  const int N = nh * L;                       // steps (head, query tile)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(kvfull, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qempty[s], 1);
      mbar_init(&vfull[s], 32);
      mbar_init(&vempty[s], 256);
      mbar_init(&pready[s], 128);
      mbar_init(&dsready[s], 128);
    }
    mbar_init(sfull, 1);
    mbar_init(dpfull, 1);
    mbar_init(accdone, 1);
    mbar_init(drain, 1);
    mbar_init(xbar, 1);
    mbar_init(sfree, 256);
    mbar_init(afree, 256);
    mbar_init(pfree, 1);
    mbar_init(dsfree, 1);
    *abort = 0;
    fence_barrier_init();
    wait_probe(probe, probe_ns, abort, dev_status);  // no-op unless a test asked for it
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmdO);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // The pre-pass waited for all earlier work on the stream, and this grid starts only after every
  // pre-pass block has done so: Q, K, V, dO, lse and log g may be read at once, and the outputs
  // written. Only the per-query stager reads what the pre-pass writes (Dv), after its wait.
  griddep_launch_dependents();  // the next kernel may start its prologue
  const uint32_t tmem = *tmem_slot;
  const bool skip = *abort;  // only the test probe sets it this early: nothing was issued
  bool done = false;         // this epilogue thread's accumulators are final
  float dl = 0.f;            // this thread's d log g partial (its key row, its query half)

  // The loader / issuer warpgroup gives registers to the epilogue warpgroups:
  // 128 x 64 + 256 x 216 = 63488 <= the launch's 384 x 168 = 64512.
  if (warp < 4) {
    regs_dec<64>();
    if (skip) {
    } else if (warp == 0) {  // -------------------------------------------------- TMA producer
      if (lane == 0) {
        int issued = 0;
        mbar_arrive_expect_tx(kvfull, 2 * C::TILE);
        for (int bx = 0; bx < C::NBOX; ++bx) {
          tma_load_2d(smem + C::K_OFF + bx * (BT * 128), &tmK, kvh * D + bx * 64, off + kt * BT, kvfull);
          tma_load_2d(smem + C::V_OFF + bx * (BT * 128), &tmV, kvh * D + bx * 64, off + kt * BT, kvfull);
        }
        for (int n = 0; n < N; ++n) {
          const int s = n & 1;
          if (n >= 2 && !mbar_wait(&qempty[s], ((n >> 1) - 1) & 1, abort, dev_status)) break;
          const int h = kvh * G + rank + (n / L) * Cn, qt = kt + n % L;
          uint8_t* qb = smem + C::Q_OFF + s * 2 * C::TILE;
          mbar_arrive_expect_tx(&qfull[s], 2 * C::TILE);
          for (int bx = 0; bx < C::NBOX; ++bx) {
            tma_load_2d(qb + bx * (BT * 128), &tmQ, h * D + bx * 64, off + qt * BT, &qfull[s]);
            tma_load_2d(qb + C::TILE + bx * (BT * 128), &tmdO, h * D + bx * 64, off + qt * BT, &qfull[s]);
          }
          ++issued;
        }
        if (*abort) {  // let the copies in flight land before the CTA can leave
          settle(kvfull, 0);
          for (int n = issued - 2 < 0 ? 0 : issued - 2; n < issued; ++n) settle(&qfull[n & 1], (n >> 1) & 1);
        }
      }
    } else if (warp == 1) {  // ------------------------------------------------- MMA issuer
      {
        const bool leader = elect_one();
        const uint32_t ka = smem_u32(smem + C::K_OFF), va = smem_u32(smem + C::V_OFF);
        auto qa = [&](int n) { return smem_u32(smem + C::Q_OFF + (n & 1) * 2 * C::TILE); };
        auto issue_ss = [&](uint32_t d, uint32_t a, uint32_t bq) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t o = (kk >> 2) * (BT * 128) + (kk & 3) * 32;
            if (leader) mma_ss(d, sdesc_sw128(a + o, 16, 1024), sdesc_sw128(bq + o, 16, 1024), C::IDESC_S, kk > 0);
          }
        };
        // Program per step n: dP^T_n into region A once the epilogue holds S^T_n, dV_n once P^T_n
        // is in TMEM, S^T_{n+1} into A once the epilogue holds dP^T_n, dK_n once dS^T_n is in TMEM.
        bool ok = __all_sync(0xffffffffu, mbar_wait(kvfull, 0, abort, dev_status)) && __all_sync(0xffffffffu, mbar_wait(&qfull[0], 0, abort, dev_status));
        if (ok) {
          tc_fence_after();
          issue_ss(tmem + 0, ka, qa(0));  // S^T_0 = K Q_0^T
          if (leader) mma_commit(sfull);
        }
        for (int n = 0; ok && n < N; ++n) {
          const uint32_t ph = n & 1;
          const uint32_t q_a = qa(n), do_a = q_a + C::TILE;
          if (!__all_sync(0xffffffffu, mbar_wait(sfree, ph, abort, dev_status))) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_ss(tmem + 0, va, do_a);  // dP^T_n = V dO_n^T
          if (leader) mma_commit(dpfull);
          // dV += P^T dO in the two query halves, each as soon as its P^T is in TMEM
          for (int c = 0; c < 2; ++c) {
            if (!__all_sync(0xffffffffu, mbar_wait(&pready[c], ph, abort, dev_status))) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const int kk = 4 * c + k4;
              if (leader) mma_ts(tmem + C::T_DV, tmem + C::T_P + c * 32 + k4 * 8, sdesc_sw128(do_a + kk * 2048, BT * 128, 1024),
                     C::IDESC_G, (n > 0 || kk > 0) ? 1u : 0u);
            }
          }
          if (!ok) break;
          if (leader) mma_commit(pfree);
          if (n + 1 < N) {  // S^T_{n+1} = K Q_{n+1}^T into region A
            if (!__all_sync(0xffffffffu, mbar_wait(afree, ph, abort, dev_status)) ||
                !__all_sync(0xffffffffu, mbar_wait(&qfull[(n + 1) & 1], ((n + 1) >> 1) & 1, abort, dev_status))) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_ss(tmem + 0, ka, qa(n + 1));
            if (leader) mma_commit(sfull);
          }
          for (int c = 0; c < 2; ++c) {  // dK += dS^T Q
            if (!__all_sync(0xffffffffu, mbar_wait(&dsready[c], ph, abort, dev_status))) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const int kk = 4 * c + k4;
              if (leader) mma_ts(tmem + C::T_DK, tmem + C::T_DS + c * 32 + k4 * 8, sdesc_sw128(q_a + kk * 2048, BT * 128, 1024),
                     C::IDESC_G, (n > 0 || kk > 0) ? 1u : 0u);
            }
          }
          if (!ok) break;
          if (leader) mma_commit(dsfree);
          if (leader) mma_commit(&qempty[n & 1]);  // the stage's Q and dO are no longer read
        }
        if (ok && leader) mma_commit(accdone);
        if (leader) mma_commit(drain);
        if (leader) settle(drain, 0);
        __syncwarp();
      }
    } else if (warp == 3) {  // ----------------------------------- per-query vectors stager
      // -lse * log2(e) (-inf for rows past the sequence, whose lse reads as +inf) and -Dv of
      // the step's 128 queries, 4 per lane, into the stage's slots.
      griddep_wait();  // Dv of the pre-pass is visible from here on
      for (int n = 0; n < N; ++n) {
        const int s = n & 1;
        const int h = kvh * G + rank + (n / L) * Cn, qt = kt + n % L;
        float nl[4], nd[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int q = qt * BT + lane * 4 + e;
          const bool v = q < m;
          nl[e] = v ? -lse_or_inf(lse[(int64_t)h * m_tot + off + q]) * kLog2e : -INFINITY;
          nd[e] = v ? -dQ[((int64_t)(off + q) * Hq + h) * D] : 0.f;
        }
        if (n >= 2 && !__all_sync(0xffffffffu, mbar_wait(&vempty[s], ((n >> 1) - 1) & 1, abort, dev_status))) break;
        *reinterpret_cast<float4*>(vec_s + s * 2 * BT + lane * 4) = make_float4(nl[0], nl[1], nl[2], nl[3]);
        *reinterpret_cast<float4*>(vec_s + s * 2 * BT + BT + lane * 4) = make_float4(nd[0], nd[1], nd[2], nd[3]);
        mbar_arrive(&vfull[s]);
      }
    }
  } else if (!skip) {  // ------------------------------------------------------ epilogue
    regs_inc<216>();
    const int c = (warp - 4) >> 2;  // query half: 0 = queries 0-63 (warps 4-7), 1 = 64-127 (warps 8-11)
    const int q4 = warp & 3;
    const int kr = q4 * 32 + lane;  // key row in the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const uint32_t tA = tmem + lane_base + c * 64;  // this half of region A (S^T, then dP^T)
    const uint32_t tPo = tmem + lane_base + C::T_P + c * 32, tDSo = tmem + lane_base + C::T_DS + c * 32;
    const int kl = kt * BT + kr;
    const bool kvalid = kl < m;
    const float lgk = (logg && kvalid) ? __ldcg(logg + off + kl) : 0.f;
    const float2 qs2 = make_float2(qk_scale2, qk_scale2);
    float racc = 0.f, gh = 1.f, bias2 = 0.f;
    bool ok = true;
    for (int n = 0; n < N; ++n) {
      const int s = n & 1;
      const int qt = kt + n % L;
      if (n % L == 0) {  // a new query head
        dl = fmaf(gh, racc, dl);
        racc = 0.f;
        gh = gain ? __ldcg(gain + kvh * G + rank + (n / L) * Cn) : 1.f;
        bias2 = kvalid ? key_bias(gh * kLog2e, lgk) : -INFINITY;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&vfull[s], (n >> 1) & 1, abort, dev_status) &&
                                       mbar_wait(sfull, n & 1, abort, dev_status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t xr[64];
      tmem_ld32(tA, *reinterpret_cast<uint32_t(*)[32]>(&xr[0]));
      tmem_ld32(tA + 32, *reinterpret_cast<uint32_t(*)[32]>(&xr[32]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(sfree);  // region A may receive dP^T_n
      float* x = reinterpret_cast<float*>(xr);
      const float4* nl4 = reinterpret_cast<const float4*>(vec_s + s * 2 * BT + c * 64);
      const float2 bb = make_float2(bias2, bias2);
      uint32_t pk[32];
      // P^T = 2^(scale log2(e) S^T + bias - lse log2(e)); on the diagonal tile query < key is masked
      // (a separate loop, so the other tiles carry no mask arithmetic)
      if (qt == kt) {
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float4 l4 = nl4[q];
          float2 v0 = __fadd2_rn(__ffma2_rn(make_float2(x[4 * q], x[4 * q + 1]), qs2, bb), make_float2(l4.x, l4.y));
          float2 v1 = __fadd2_rn(__ffma2_rn(make_float2(x[4 * q + 2], x[4 * q + 3]), qs2, bb), make_float2(l4.z, l4.w));
          const int q0 = c * 64 + 4 * q;
          if (q0 < kr) v0.x = -INFINITY;
          if (q0 + 1 < kr) v0.y = -INFINITY;
          if (q0 + 2 < kr) v1.x = -INFINITY;
          if (q0 + 3 < kr) v1.y = -INFINITY;
          x[4 * q] = ex2(v0.x);
          x[4 * q + 1] = ex2(v0.y);
          x[4 * q + 2] = ex2(v1.x);
          x[4 * q + 3] = ex2(v1.y);
          pk[2 * q] = pack_bf16(x[4 * q], x[4 * q + 1]);
          pk[2 * q + 1] = pack_bf16(x[4 * q + 2], x[4 * q + 3]);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float4 l4 = nl4[q];
          const float2 v0 = __fadd2_rn(__ffma2_rn(make_float2(x[4 * q], x[4 * q + 1]), qs2, bb), make_float2(l4.x, l4.y));
          const float2 v1 =
              __fadd2_rn(__ffma2_rn(make_float2(x[4 * q + 2], x[4 * q + 3]), qs2, bb), make_float2(l4.z, l4.w));
          x[4 * q] = ex2(v0.x);
          x[4 * q + 1] = ex2(v0.y);
          x[4 * q + 2] = ex2(v1.x);
          x[4 * q + 3] = ex2(v1.y);
          pk[2 * q] = pack_bf16(x[4 * q], x[4 * q + 1]);
          pk[2 * q + 1] = pack_bf16(x[4 * q + 2], x[4 * q + 3]);
        }
      }
      if (n > 0 && !__all_sync(0xffffffffu, mbar_wait(pfree, (n - 1) & 1, abort, dev_status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_st32(tPo, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&pready[c]);
      if (!__all_sync(0xffffffffu, mbar_wait(dpfull, n & 1, abort, dev_status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t yr[64];
      tmem_ld32(tA, *reinterpret_cast<uint32_t(*)[32]>(&yr[0]));
      tmem_ld32(tA + 32, *reinterpret_cast<uint32_t(*)[32]>(&yr[32]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(afree);  // region A may receive S^T_{n+1}
      const float* y = reinterpret_cast<const float*>(yr);
      const float4* nd4 = reinterpret_cast<const float4*>(vec_s + s * 2 * BT + BT + c * 64);
      float2 ra = make_float2(0.f, 0.f), rb = make_float2(0.f, 0.f);
      // dS^T = P^T * (dP^T - Dv), with the fp32 P^T
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const float4 d4 = nd4[q];
        const float2 s0 = __fmul2_rn(make_float2(x[4 * q], x[4 * q + 1]),
                                     __fadd2_rn(make_float2(y[4 * q], y[4 * q + 1]), make_float2(d4.x, d4.y)));
        const float2 s1 = __fmul2_rn(make_float2(x[4 * q + 2], x[4 * q + 3]),
                                     __fadd2_rn(make_float2(y[4 * q + 2], y[4 * q + 3]), make_float2(d4.z, d4.w)));
        ra = __fadd2_rn(ra, s0);
        rb = __fadd2_rn(rb, s1);
        pk[2 * q] = pack_bf16(s0.x, s0.y);
        pk[2 * q + 1] = pack_bf16(s1.x, s1.y);
      }
      mbar_arrive(&vempty[s]);
      if (n > 0 && !__all_sync(0xffffffffu, mbar_wait(dsfree, (n - 1) & 1, abort, dev_status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_st32(tDSo, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&dsready[c]);
      racc += (ra.x + ra.y) + (rb.x + rb.y);
    }
    dl = fmaf(gh, racc, dl);
    done = ok && __all_sync(0xffffffffu, mbar_wait(accdone, 0, abort, dev_status));
    dl_s[c * BT + kr] = dl;
    fence_proxy_async_smem();  // a bulk copy may read dl_s

    // ---------------------------------------------------------- cluster reduction of dK, dV
    // With C = 2, rank r owns the columns [r D/2, (r + 1) D/2) of dK and dV: those of its
    // epilogue warpgroup r. Each warpgroup stages its half of dV and dK (fp32, [tensor][128
    // rows][D/2], 16-byte slots of a row permuted by row % 8) in the freed Q / dO stages. After
    // barrier 1 (every CTA of the pair has finished its products and copies and armed its receive
    // barrier) the other warpgroup bulk-copies its stage into the owner's freed K / V tiles, and
    // rank 1 its d log g partials into rank 0's freed per-query vector slots. The owner adds the
    // two partials in rank order and stores the sums with consecutive threads on consecutive 16
    // bytes of a row; rank 0 does the same for d log g. Barrier 2 keeps every CTA alive until the
    // copies that read its shared memory have landed. With C = 1 every column is owned. Every CTA
    // reaches both barriers (all waits above are bounded); a CTA that could not finish publishes
    // a nonzero flag and then its peer neither copies nor writes results. The other warps take
    // part in the same CTA and cluster barriers below the role branches.
    const int bad = __syncthreads_or(!done);  // also publishes dl_s
    constexpr int H4 = D / 8;   // 16-byte slots of a half row
    constexpr int LH4 = D == 128 ? 4 : 3;
    constexpr uint32_t STAGE_BYTES = 2 * BT * (D / 2) * 4;
    float* stage = reinterpret_cast<float*>(smem + C::Q_OFF) + c * (2 * BT * (D / 2));
    const float* rx = reinterpret_cast<const float*>(smem + C::K_OFF);  // the peer's stage of this half
    const float* dl_rx = vec_s;                                         // rank 0: rank 1's dl_s
    const int tw = threadIdx.x & 127;  // thread index in the warpgroup
    const int64_t ostride = (int64_t)Hkv * D;
    const int64_t obase = ((int64_t)(off + kt * BT) * Hkv + kvh) * D + c * (D / 2);  // row 0 of the tile, this half
    const bool owner = Cn == 1 || c == rank;
    if (!bad) {
      tc_fence_after();
#pragma unroll
      for (int t = 0; t < 2; ++t) {
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t v[16];
          tmem_ld16(tmem + lane_base + (t ? C::T_DK : C::T_DV) + c * (D / 2) + ch * 16, v);
          tmem_wait_ld();
          float* row = stage + (t * BT + kr) * (D / 2);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            *reinterpret_cast<float4*>(row + (((ch * 4 + i) ^ (kr & 7)) << 2)) =
                make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]), __uint_as_float(v[4 * i + 2]),
                            __uint_as_float(v[4 * i + 3]));
        }
      }
      if (!owner) fence_proxy_async_smem();  // the stage is read by a bulk copy
      if (Cn == 2 && owner && tw == 0)
        mbar_arrive_expect_tx(xbar, STAGE_BYTES + (rank == 0 && want_dl ? 2 * BT * 4 : 0));
    }
    tc_fence_before();
    __syncwarp();
    cluster_sync_all();
    tc_fence_after();
    int any_bad = 0;
    for (int q = 0; q < Cn; ++q) any_bad |= ld_cluster_s32(mapa_rank(smem_u32(const_cast<int*>(abort)), (uint32_t)q));
    if (!any_bad && !owner && tw == 0) {
      const uint32_t peer = (uint32_t)(1 - rank);
      const uint32_t pbar = mapa_rank(smem_u32(xbar), peer);
      bulk_copy_to_cluster(mapa_rank(smem_u32(rx), peer), smem_u32(stage), STAGE_BYTES, pbar);
      if (rank == 1 && want_dl) bulk_copy_to_cluster(mapa_rank(smem_u32(dl_rx), peer), smem_u32(dl_s), 2 * BT * 4, pbar);
      bulk_commit_group();
    }
    if (!any_bad && owner && (Cn == 1 || __all_sync(0xffffffffu, mbar_wait(xbar, 0, abort, dev_status)))) {
      if (Cn == 1) named_bar_sync(1 + c, 128);  // the warpgroup's stage is complete
#pragma unroll 4
      for (int i = tw; i < 2 * BT * H4; i += 128) {
        const int t = i >> (7 + LH4), r = (i >> LH4) & (BT - 1), x = i & (H4 - 1);
        if (kt * BT + r >= m) continue;
        const int o = (t * BT + r) * (D / 2) + ((x ^ (r & 7)) << 2);
        float4 a = *reinterpret_cast<const float4*>(stage + o);
        if (Cn == 2) {
          const float4 pp = *reinterpret_cast<const float4*>(rx + o);
          a = rank == 0 ? make_float4(a.x + pp.x, a.y + pp.y, a.z + pp.z, a.w + pp.w)
                        : make_float4(pp.x + a.x, pp.y + a.y, pp.z + a.z, pp.w + a.w);
        }
        const float f = t ? scale : 1.f;
        *reinterpret_cast<float4*>((t ? dK : dV) + obase + r * ostride + x * 4) =
            make_float4(a.x * f, a.y * f, a.z * f, a.w * f);
      }
      if (want_dl && rank == 0 && c == 0 && kvalid) {
        float sdl = dl_s[kr] + dl_s[BT + kr];
        if (Cn == 2) sdl += dl_rx[kr] + dl_rx[BT + kr];
        dQ[((int64_t)(off + kl) * Hq + kvh) * D + 1] = sdl;
      }
    }
    tc_fence_before();
    __syncwarp();
    cluster_sync_all();  // the copies that read this CTA's shared memory have landed
  }
  if (warp < 4 || skip) {  // the same barriers for the loader / issuer warps (and all warps on skip)
    const int bad = __syncthreads_or(skip ? 1 : 0);
    if (threadIdx.x == 0) *abort = bad ? 1 : 0;
    tc_fence_before();
    __syncwarp();
    cluster_sync_all();
    __syncwarp();
    cluster_sync_all();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ 3. d log g and d score
__global__ void __launch_bounds__(256) bwd_dlogg_kernel(const float* __restrict__ dQ, const float* __restrict__ logg,
                                                        float* __restrict__ dlogg, float* __restrict__ dscore, int r0,
                                                        int r1, int Hq, int Hkv, int D) {
  griddep_launch_dependents();  // the dQ kernel may start its prologue
  griddep_wait();               // the dK/dV kernel's partials are visible from here on
  const int64_t row = r0 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= r1) return;
  float s = 0.f;
  for (int kvh = 0; kvh < Hkv; ++kvh) s += dQ[(row * Hq + kvh) * D + 1];
  if (dlogg) dlogg[row] = s;
  if (dscore) dscore[row] = s * -expm1f(logg[row]);
}

// ------------------------------------------------------------------ 4. dQ
template <int D>
struct QCfg {
  static constexpr int TILE = BT * D * 2;
  static constexpr int NBOX = D / 64;
  static constexpr int KSL = 3;  // K ring: K_j is read by S_j and, a step later, by dQ_j
  static constexpr int Q_OFF = 0, DO_OFF = TILE, K_OFF = 2 * TILE, V_OFF = (2 + KSL) * TILE;
  static constexpr int TAIL_OFF = (4 + KSL) * TILE;
  static constexpr int TAIL = 256 + 2 * BT * 4;  // barriers, key bias [2][128]
  static constexpr int SMEM = 1024 + TAIL_OFF + TAIL;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(BT, BT, false);
  static constexpr uint32_t IDESC_G = idesc_bf16_f32(BT, D, true);
  // TMEM columns: S buffers [0, 128) and [128, 256), dP [256, 384), dQ [384, 384 + D)
  static constexpr uint32_t T_DP = 256, T_DQ = 384;
  static_assert(SMEM <= SMEM_LIMIT, "shared memory budget");
  static_assert(2 * TILE == BT * D * 4, "the Q and dO tiles hold the fp32 dQ tile at the end");
};

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_bwd_dq_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                   const float* __restrict__ logg, const float* __restrict__ gain, const float* __restrict__ lse,
                   float* __restrict__ dQ, int64_t m_tot, int Hq, int Hkv, float qk_scale2, float scale,
                   int32_t* __restrict__ dev_status, uint64_t probe_ns, const __grid_constant__ TcParams p) {
  using C = QCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* tail = smem + C::TAIL_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(tail);
  uint64_t* qfull = bars + 0;
  uint64_t* kfull = bars + 1;    // [3]
  uint64_t* kempty = bars + 4;   // [3]
  uint64_t* vfull = bars + 7;    // [2]
  uint64_t* vempty = bars + 9;   // [2]
  uint64_t* sfull = bars + 11;   // [2] per S buffer
  uint64_t* dpfull = bars + 13;
  uint64_t* dsready = bars + 14; // [2] per epilogue warpgroup
  uint64_t* bfull = bars + 16;   // [2] key bias slots
  uint64_t* bempty = bars + 18;  // [2]
  uint64_t* accdone = bars + 20;
  uint64_t* drain = bars + 21;
  uint64_t* probe = bars + 22;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 23);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* bias_s = reinterpret_cast<float*>(tail + 256);  // [2][128]

  const int G = Hq / Hkv;
  const int h = (int)(blockIdx.x % (unsigned)Hq), kvh = h / G;
  int b, L;
  decode_len((int)(blockIdx.x / (unsigned)Hq), p, b, L);
  const int off = p.off[b], m = p.m[b];
  const int qt = L - 1;  // this query tile; key tiles 0 .. qt
  const int N = L;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    for (int s = 0; s < C::KSL; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&vfull[s], 1);
      mbar_init(&vempty[s], 1);
      mbar_init(&sfull[s], 1);
      mbar_init(&dsready[s], 128);
      mbar_init(&bfull[s], 32);
      mbar_init(&bempty[s], 256);
    }
    mbar_init(dpfull, 1);
    mbar_init(accdone, 1);
    mbar_init(drain, 1);
    *abort = 0;
    fence_barrier_init();
    wait_probe(probe, probe_ns, abort, dev_status);
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmdO);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // The tiles (Q, dO, K, V) and the per-key bias are inputs of the call, complete before the
  // pre-pass passed its wait; only the epilogue reads (Dv) and writes (dQ) memory that the
  // kernels before this one write, after its wait.
  griddep_launch_dependents();
  const uint32_t tmem = *tmem_slot;
  const bool skip = *abort;

  // The loader / issuer warpgroup gives registers to the epilogue warpgroups:
  // 128 x 80 + 256 x 208 = 63488 <= the launch's 384 x 168 = 64512.
  if (warp < 4) {
    regs_dec<80>();
    if (skip) {
    } else if (warp == 0) {  // -------------------------------------------------- TMA producer
      if (lane == 0) {
        int nk = 0, nv = 0;
        mbar_arrive_expect_tx(qfull, 2 * C::TILE);
        for (int bx = 0; bx < C::NBOX; ++bx) {
          tma_load_2d(smem + C::Q_OFF + bx * (BT * 128), &tmQ, h * D + bx * 64, off + qt * BT, qfull);
          tma_load_2d(smem + C::DO_OFF + bx * (BT * 128), &tmdO, h * D + bx * 64, off + qt * BT, qfull);
        }
        for (int j = 0; j < N; ++j) {  // K_j and V_j in the order the products need them
          const int ks = j % C::KSL;
          if (j >= C::KSL && !mbar_wait(&kempty[ks], ((j / C::KSL) - 1) & 1, abort, dev_status)) break;
          mbar_arrive_expect_tx(&kfull[ks], C::TILE);
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_2d(smem + C::K_OFF + ks * C::TILE + bx * (BT * 128), &tmK, kvh * D + bx * 64, off + j * BT,
                        &kfull[ks]);
          ++nk;
          const int vs = j & 1;
          if (j >= 2 && !mbar_wait(&vempty[vs], ((j >> 1) - 1) & 1, abort, dev_status)) break;
          mbar_arrive_expect_tx(&vfull[vs], C::TILE);
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_2d(smem + C::V_OFF + vs * C::TILE + bx * (BT * 128), &tmV, kvh * D + bx * 64, off + j * BT,
                        &vfull[vs]);
          ++nv;
        }
        if (*abort) {
          settle(qfull, 0);
          for (int j = nk - C::KSL < 0 ? 0 : nk - C::KSL; j < nk; ++j) settle(&kfull[j % C::KSL], (j / C::KSL) & 1);
          for (int j = nv - 2 < 0 ? 0 : nv - 2; j < nv; ++j) settle(&vfull[j & 1], (j >> 1) & 1);
        }
      }
    } else if (warp == 1) {  // ------------------------------------------------- MMA issuer
      {
        const bool leader = elect_one();
        const uint32_t qa = smem_u32(smem + C::Q_OFF), doa = smem_u32(smem + C::DO_OFF);
        auto ka = [&](int j) { return smem_u32(smem + C::K_OFF + (j % C::KSL) * C::TILE); };
        auto issue_ss = [&](uint32_t d, uint32_t a, uint32_t bk) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t o = (kk >> 2) * (BT * 128) + (kk & 3) * 32;
            if (leader) mma_ss(d, sdesc_sw128(a + o, 16, 1024), sdesc_sw128(bk + o, 16, 1024), C::IDESC_S, kk > 0);
          }
        };
        auto issue_s = [&](int j) -> bool {  // S_j = Q K_j^T into buffer j % 2
          if (!__all_sync(0xffffffffu, mbar_wait(&kfull[j % C::KSL], (j / C::KSL) & 1, abort, dev_status))) return false;
          tc_fence_after();
          issue_ss(tmem + (j & 1) * 128, qa, ka(j));
          if (leader) mma_commit(&sfull[j & 1]);
          return true;
        };
        auto issue_dp = [&](int j) -> bool {  // dP_j = dO V_j^T
          if (!__all_sync(0xffffffffu, mbar_wait(&vfull[j & 1], (j >> 1) & 1, abort, dev_status))) return false;
          tc_fence_after();
          issue_ss(tmem + C::T_DP, doa, smem_u32(smem + C::V_OFF + (j & 1) * C::TILE));
          if (leader) mma_commit(dpfull);
          if (leader) mma_commit(&vempty[j & 1]);
          return true;
        };
        bool ok = __all_sync(0xffffffffu, mbar_wait(qfull, 0, abort, dev_status));
        ok = ok && issue_s(0) && issue_dp(0) && (N < 2 || issue_s(1));
        for (int j = 0; ok && j < N; ++j) {
          const uint32_t k_a = ka(j);
          for (int c = 0; c < 2; ++c) {  // dQ += dS K_j, each key half as soon as its dS is in TMEM
            if (!__all_sync(0xffffffffu, mbar_wait(&dsready[c], j & 1, abort, dev_status))) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const int kk = 4 * c + k4;
              if (leader) mma_ts(tmem + C::T_DQ, tmem + C::T_DP + c * 64 + k4 * 8, sdesc_sw128(k_a + kk * 2048, BT * 128, 1024),
                     C::IDESC_G, (j > 0 || kk > 0) ? 1u : 0u);
            }
          }
          if (!ok) break;
          if (leader) mma_commit(&kempty[j % C::KSL]);
          // dP_{j+1} overwrites dS_j only after dQ_j read it; S_{j+2} reuses S_j's buffer, which
          // the epilogue finished reading before it wrote dS_j
          if (j + 1 < N) ok = issue_dp(j + 1);
          if (ok && j + 2 < N) ok = issue_s(j + 2);
        }
        if (ok && leader) mma_commit(accdone);
        if (leader) mma_commit(drain);
        if (leader) settle(drain, 0);
        __syncwarp();
      }
    } else if (warp == 3) {  // ------------------------------------------- key bias stager
      const float gain2 = (gain ? __ldcg(gain + h) : 1.f) * kLog2e;
      for (int j = 0; j < N; ++j) {
        const int bs = j & 1;
        float bv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kl = j * BT + lane * 4 + e;
          bv[e] = kl < m ? (logg ? key_bias(gain2, __ldcg(logg + off + kl)) : 0.f) : -INFINITY;
        }
        if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bempty[bs], ((j >> 1) - 1) & 1, abort, dev_status))) break;
        *reinterpret_cast<float4*>(bias_s + bs * BT + lane * 4) = make_float4(bv[0], bv[1], bv[2], bv[3]);
        mbar_arrive(&bfull[bs]);
      }
    }
  } else if (!skip) {  // ------------------------------------------------------ epilogue
    regs_inc<208>();
    const int c = (warp - 4) >> 2;  // key half: 0 = keys 0-63 (warps 4-7), 1 = 64-127 (warps 8-11)
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;  // query row in the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const uint32_t tP = tmem + lane_base + C::T_DP + c * 64;
    const int il = qt * BT + r;
    const bool valid = il < m;
    const float nlse2 = valid ? -lse_or_inf(__ldcg(lse + (int64_t)h * m_tot + off + il)) * kLog2e : -INFINITY;
    griddep_wait();  // Dv, and the d log g partials in dQ, are final from here on
    const float ndv = valid ? -dQ[((int64_t)(off + il) * Hq + h) * D] : 0.f;  // read before any dQ write below
    const float2 qs2 = make_float2(qk_scale2, qk_scale2), nl2 = make_float2(nlse2, nlse2), nd2 = make_float2(ndv, ndv);
    bool ok = true;
    for (int j = 0; j < N; ++j) {
      const int bs = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bfull[bs], (j >> 1) & 1, abort, dev_status) &&
                                       mbar_wait(&sfull[j & 1], (j >> 1) & 1, abort, dev_status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tmem + lane_base + (j & 1) * 128 + c * 64;
      uint32_t xr[64];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&xr[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&xr[32]));
      tmem_wait_ld();
      float* x = reinterpret_cast<float*>(xr);
      const float4* bb4 = reinterpret_cast<const float4*>(bias_s + bs * BT + c * 64);
      // P = 2^(scale log2(e) S + bias - lse log2(e)); on the diagonal tile key > query is masked
      // (a separate loop, so the other tiles carry no mask arithmetic)
      if (j == qt) {
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float4 b4 = bb4[q];
          float2 v0 = __fadd2_rn(__ffma2_rn(make_float2(x[4 * q], x[4 * q + 1]), qs2, make_float2(b4.x, b4.y)), nl2);
          float2 v1 = __fadd2_rn(__ffma2_rn(make_float2(x[4 * q + 2], x[4 * q + 3]), qs2, make_float2(b4.z, b4.w)), nl2);
          const int k0 = c * 64 + 4 * q;
          if (k0 > r) v0.x = -INFINITY;
          if (k0 + 1 > r) v0.y = -INFINITY;
          if (k0 + 2 > r) v1.x = -INFINITY;
          if (k0 + 3 > r) v1.y = -INFINITY;
          x[4 * q] = ex2(v0.x);
          x[4 * q + 1] = ex2(v0.y);
          x[4 * q + 2] = ex2(v1.x);
          x[4 * q + 3] = ex2(v1.y);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float4 b4 = bb4[q];
          const float2 v0 =
              __fadd2_rn(__ffma2_rn(make_float2(x[4 * q], x[4 * q + 1]), qs2, make_float2(b4.x, b4.y)), nl2);
          const float2 v1 =
              __fadd2_rn(__ffma2_rn(make_float2(x[4 * q + 2], x[4 * q + 3]), qs2, make_float2(b4.z, b4.w)), nl2);
          x[4 * q] = ex2(v0.x);
          x[4 * q + 1] = ex2(v0.y);
          x[4 * q + 2] = ex2(v1.x);
          x[4 * q + 3] = ex2(v1.y);
        }
      }
      mbar_arrive(&bempty[bs]);
      if (!__all_sync(0xffffffffu, mbar_wait(dpfull, j & 1, abort, dev_status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t yr[64];
      tmem_ld32(tP, *reinterpret_cast<uint32_t(*)[32]>(&yr[0]));
      tmem_ld32(tP + 32, *reinterpret_cast<uint32_t(*)[32]>(&yr[32]));
      tmem_wait_ld();
      const float* y = reinterpret_cast<const float*>(yr);
      uint32_t pk[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const float2 d = __fadd2_rn(make_float2(y[2 * q], y[2 * q + 1]), nd2);
        const float2 ds = __fmul2_rn(make_float2(x[2 * q], x[2 * q + 1]), d);
        pk[q] = pack_bf16(ds.x, ds.y);
      }
      tmem_st32(tP, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&dsready[c]);
    }
    ok = ok && __all_sync(0xffffffffu, mbar_wait(accdone, 0, abort, dev_status));
    if (ok) {
      tc_fence_after();
      // the dQ tile (fp32) into the Q and dO tiles' space, then coalesced row stores
      float* stg = reinterpret_cast<float*>(smem + C::Q_OFF);
#pragma unroll 1
      for (int col0 = c * (D / 2); col0 < (c + 1) * (D / 2); col0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + C::T_DQ + col0, v);
        tmem_wait_ld();
        float4* rowp = reinterpret_cast<float4*>(stg + r * D);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          rowp[((col0 >> 2) + i) ^ (r & 7)] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                                          __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
      }
    }
    // both warpgroups: every Dv read above is done and the staged tile is complete
    const bool all_ok = bar_red_or(1, 256, !ok) == 0;
    if (all_ok) {
      constexpr int D4 = D / 4;
      const float* stg = reinterpret_cast<const float*>(smem + C::Q_OFF);
      for (int idx = threadIdx.x - 128; idx < BT * D4; idx += 256) {
        const int row = idx / D4, c4 = idx % D4;
        const int i2 = qt * BT + row;
        if (i2 >= m) continue;
        const float4 v = *reinterpret_cast<const float4*>(stg + row * D + ((c4 ^ (row & 7)) << 2));
        *reinterpret_cast<float4*>(dQ + ((int64_t)(off + i2) * Hq + h) * D + c4 * 4) =
            make_float4(v.x * scale, v.y * scale, v.z * scale, v.w * scale);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int D>
tg_status launch_tc_d(const AttnBwdArgs& a, const AttnSeq* seqs, int nseq, cudaStream_t st) {
  using KC = KCfg<D>;
  using QC = QCfg<D>;
  TcParams p = {};
  p.nseq = nseq;
  int units = 0, tmax = 0;
  for (int i = 0; i < nseq; ++i) {
    p.off[i] = seqs[i].off;
    p.m[i] = seqs[i].m;
    p.nt[i] = (seqs[i].m + BT - 1) / BT;
    units += p.nt[i];
    tmax = p.nt[i] > tmax ? p.nt[i] : tmax;
  }
  p.tmax = tmax;
  if (units == 0) return TG_OK;
  const int r0 = seqs[0].off, r1 = seqs[nseq - 1].off + seqs[nseq - 1].m;
  const int G = a.Hq / a.Hkv;
  p.C = G % MAXC == 0 ? MAXC : 1;  // an even number of query heads per KV head: two CTAs split them

  CUtensorMap tq, tk, tv, tdo;
  if (!make_tmap_bf16_2d(&tq, a.Q, (uint64_t)a.m_tot, (uint64_t)a.Hq * D, (uint64_t)a.Hq * D, BT, 64) ||
      !make_tmap_bf16_2d(&tdo, a.dO, (uint64_t)a.m_tot, (uint64_t)a.Hq * D, (uint64_t)a.Hq * D, BT, 64) ||
      !make_tmap_bf16_2d(&tk, a.K, (uint64_t)a.m_tot, (uint64_t)a.Hkv * D, (uint64_t)a.Hkv * D, BT, 64) ||
      !make_tmap_bf16_2d(&tv, a.V, (uint64_t)a.m_tot, (uint64_t)a.Hkv * D, (uint64_t)a.Hkv * D, BT, 64))
    return fail(TG_ERR_CUDA, "tg_gated_attn_bwd: building the TMA tensor maps failed");

  auto kdkdv = attn_bwd_dkdv_tc<D>;
  auto kdq = attn_bwd_dq_tc<D>;
  const int slot = ATTR_BWD + 2 + (D == 128 ? 1 : 0);
  if (attrs_needed(slot)) {
    cudaError_t e = cudaFuncSetAttribute(kdkdv, cudaFuncAttributeMaxDynamicSharedMemorySize, KC::SMEM);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kdq, cudaFuncAttributeMaxDynamicSharedMemorySize, QC::SMEM);
    if (e != cudaSuccess) return cuda_status(e, "tg_gated_attn_bwd: cudaFuncSetAttribute");
    mark_attrs_set(slot);
  }
  const __nv_bfloat16* O = static_cast<const __nv_bfloat16*>(a.O);
  const __nv_bfloat16* dO = static_cast<const __nv_bfloat16*>(a.dO);
  const uint64_t probe = wait_probe_ns();
  const float qk2 = a.scale * kLog2e;

  // Every launch may start early (programmatic dependent launch): each kernel waits on the
  // previous one before it touches memory that kernel or earlier work writes.
  cudaLaunchAttribute pdl[1] = {pdl_attribute(PDL_BWD)};
  // 1. Dv into dQ[., ., 0]: warps of 4 * 32 / (D / 8) vectors
  const int64_t nvec = (int64_t)(r1 - r0) * a.Hq, per_block = 8 * 4 * (32 / (D / 8));
  cudaLaunchConfig_t cp = {};
  cp.gridDim = dim3((unsigned)((nvec + per_block - 1) / per_block));
  cp.blockDim = dim3(256);
  cp.stream = st;
  cp.attrs = pdl;
  cp.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cp, bwd_prep_kernel<D>, O, dO, a.pos, a.dQ, r0, r1, a.Hq, a.dev_status, p);
  if (e != cudaSuccess) return cuda_status(e, "tg_gated_attn_bwd: prep launch");

  // 2. dK, dV: clusters of C CTAs over the query heads of one (key tile, KV head)
  const int want_dl = (a.dlogg || a.dscore) ? 1 : 0;
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(units * a.Hkv * p.C));
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = (size_t)KC::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)p.C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl[0];
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, kdkdv, tq, tk, tv, tdo, a.logg, a.head_gain, a.lse, a.dQ, a.dK, a.dV, a.m_tot, a.Hq,
                           a.Hkv, qk2, a.scale, want_dl, a.dev_status, probe, p);
    if (e != cudaSuccess) return cuda_status(e, "tg_gated_attn_bwd: dK/dV launch");
  }

  // 3. d log g, d score
  if (want_dl) {
    cudaLaunchConfig_t cl = {};
    cl.gridDim = dim3((unsigned)((r1 - r0 + 255) / 256));
    cl.blockDim = dim3(256);
    cl.stream = st;
    cl.attrs = pdl;
    cl.numAttrs = 1;
    e = cudaLaunchKernelEx(&cl, bwd_dlogg_kernel, (const float*)a.dQ, a.logg, a.dlogg, a.dscore, r0, r1, a.Hq, a.Hkv, D);
    if (e != cudaSuccess) return cuda_status(e, "tg_gated_attn_bwd: d log g launch");
  }

  // 4. dQ: one CTA per (query tile, head), longest chains first
  {
    cudaLaunchConfig_t cq = {};
    cq.gridDim = dim3((unsigned)(units * a.Hq));
    cq.blockDim = dim3(NTHREADS);
    cq.dynamicSmemBytes = (size_t)QC::SMEM;
    cq.stream = st;
    cq.attrs = pdl;
    cq.numAttrs = 1;
    e = cudaLaunchKernelEx(&cq, kdq, tq, tk, tv, tdo, a.logg, a.head_gain, a.lse, a.dQ, a.m_tot, a.Hq, a.Hkv, qk2,
                           a.scale, a.dev_status, probe, p);
  }
  return cuda_status(e, "tg_gated_attn_bwd: dQ launch");
}

}  // namespace

tg_status launch_attn_bwd_tc(const AttnBwdArgs& a, const AttnSeq* seqs, int nseq, cudaStream_t st) {
  return a.D == 64 ? launch_tc_d<64>(a, seqs, nseq, st) : launch_tc_d<128>(a, seqs, nseq, st);
}

}  // namespace tg
