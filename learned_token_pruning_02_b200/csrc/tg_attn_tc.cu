// Token-gated causal attention over the kept tokens on the 5th-generation tensor cores.
//
// TokenGate paper page (thelatestinai.com), Figure 1(c): each attention weight is multiplied
// by its key's gate value g_j; with the row renormalised this is log g_j added to the logit
// (aitualizate.com article: the score acts as a bias on the attention logits, with a
// per-head gain). Causal on original positions, grouped KV heads (kv = h / (Hq/Hkv)).
//
// Design (B200, bf16 in, fp32 softmax and accumulation), one CTA per (sequence, 128-row
// query tile, query head), launched longest causal row-range first so the block scheduler
// packs the triangle like a longest-processing-time list schedule:
//   * warp 0: TMA loads the Q tile once and K_j, V_j tiles (128 keys) into a 2-stage ring
//     (128-byte swizzle; K and V have separate "full" barriers so S_j can start early).
//   * warp 1 (one thread): tcgen05.mma. S_j = Q K_j^T (M=128, N=128, K=D) into one of two
//     TMEM S buffers, then O += P_j V_j with P_j read straight from TMEM (A operand in
//     tensor memory) and V_j from shared memory (N-contiguous operand). The issue order
//     S_0, S_1, PV_0, S_2, PV_1, ... overlaps each softmax with the next QK^T.
//   * warps 2-5: online softmax, one query row per thread: log2-domain logits
//     scale*log2e*S + gain*log2e*log g_j (staged in shared memory per key tile), causal mask
//     on the diagonal tile, running max/sum, O rescale in TMEM when the max moves, and P
//     written back as packed bf16 into the S buffer it came from. The epilogue normalises
//     O, writes it as bf16 and the row's log-sum-exp.
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
constexpr int NTHREADS = 192;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct ATParams {
  int off[kMaxSeqPerLaunch];
  int m[kMaxSeqPerLaunch];
  int nt[kMaxSeqPerLaunch];
  int nseq;
  int tmax;
};

template <int D>
struct ACfg {
  static constexpr int TILE_BYTES = BQ * D * 2;  // one 128 x D bf16 tile
  static constexpr int NBOX = D / 64;            // 64-column boxes per tile
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = TILE_BYTES;  // + stage * 2 * TILE_BYTES
  static constexpr int V_OFF = 2 * TILE_BYTES;
  static constexpr int STAGES = 2;
  static constexpr int TAIL_OFF = TILE_BYTES * (1 + 2 * STAGES);
  static constexpr int TAIL = 4096;
  static constexpr int SMEM = 1024 + TAIL_OFF + TAIL;
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BQ, BKV, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BQ, D, true);
  static constexpr uint32_t TMEM_COLS = 512;  // S0 [0,128), S1 [128,256), O [256, 256+D)
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const float* __restrict__ logg,
                   const float* __restrict__ gain, const int32_t* __restrict__ pos, __nv_bfloat16* __restrict__ O,
                   float* __restrict__ lse, int64_t m_tot, int Hq, int Hkv, float qk_scale, uint32_t flags,
                   int32_t* __restrict__ dev_status, const __grid_constant__ ATParams p) {
  using C = ACfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tail = smem + C::TAIL_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(tail);
  uint64_t* qfull = bars + 0;
  uint64_t* kfull = bars + 1;   // [2]
  uint64_t* vfull = bars + 3;   // [2]
  uint64_t* empty = bars + 5;   // [2]
  uint64_t* sfull = bars + 7;   // [2]
  uint64_t* pready = bars + 9;  // [2]
  uint64_t* pvdone = bars + 11;
  uint64_t* drain = bars + 12;
  uint64_t* bfull = bars + 13;  // [2] key-tile bias staged by the producer warp
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* bias_s = reinterpret_cast<float*>(tail + 256);  // [2][128]
  float* gmul_s = bias_s + 2 * BKV;                      // [2][128]

  // ---- which (sequence, query tile, head) this CTA owns: longest row-ranges first
  const int h = blockIdx.x % Hq;
  int w = blockIdx.x / Hq;
  int t = 0, b = 0;
  for (int tt = p.tmax - 1; tt >= 0; --tt) {
    int cnt = 0;
    for (int s = 0; s < p.nseq; ++s) cnt += p.nt[s] > tt;
    if (w < cnt) {
      t = tt;
      for (int s = 0; s < p.nseq; ++s)
        if (p.nt[s] > tt) {
          if (w == 0) {
            b = s;
            break;
          }
          --w;
        }
      break;
    }
    w -= cnt;
  }
  const int off = p.off[b], m = p.m[b];
  const int nt = t + 1;  // key tiles 0..t (causal)
  const int kvh = h / (Hq / Hkv);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&vfull[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sfull[s], 1);
      mbar_init(&pready[s], 128);
      mbar_init(&bfull[s], 32);
    }
    mbar_init(pvdone, 1);
    mbar_init(drain, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + 256;

  const bool unnorm = (flags & TG_ATTN_UNNORMALISED) != 0;
  const float gain2 = (gain ? gain[h] : 1.f) * kLog2e;
  if (warp == 0) {  // ------------------------------------------------ TMA producer warp
    int issued = 0;
    if (lane == 0) {
      mbar_arrive_expect_tx(qfull, C::TILE_BYTES);
      for (int bx = 0; bx < C::NBOX; ++bx)
        tma_load_2d(smem + C::Q_OFF + bx * (BQ * 128), &tmQ, h * D + bx * 64, off + t * BQ, qfull);
    }
    for (int j = 0; j < nt; ++j) {
      const int s = j & 1;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&empty[s], ((j >> 1) & 1) ^ 1u, abort, dev_status);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (lane == 0) {
        uint8_t* kb = smem + C::K_OFF + s * 2 * C::TILE_BYTES;
        uint8_t* vb = smem + C::V_OFF + s * 2 * C::TILE_BYTES;
        mbar_arrive_expect_tx(&kfull[s], C::TILE_BYTES);
        for (int bx = 0; bx < C::NBOX; ++bx)
          tma_load_2d(kb + bx * (BKV * 128), &tmK, kvh * D + bx * 64, off + j * BKV, &kfull[s]);
        mbar_arrive_expect_tx(&vfull[s], C::TILE_BYTES);
        for (int bx = 0; bx < C::NBOX; ++bx)
          tma_load_2d(vb + bx * (BKV * 128), &tmV, kvh * D + bx * 64, off + j * BKV, &vfull[s]);
      }
      ++issued;
      // per-key bias of this key tile (log2 domain), 4 keys per lane; the stage's slot is free
      // because PV of the tile that used it last has completed (empty barrier above)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = lane * 4 + e;
        const int kl = j * BKV + c;
        const float bv = (logg && kl < m) ? gain2 * logg[off + kl] : 0.f;
        bias_s[s * BKV + c] = unnorm ? 0.f : bv;
        gmul_s[s * BKV + c] = unnorm ? ex2(bv) : 1.f;
      }
      mbar_arrive(&bfull[s]);
    }
    if (lane == 0 && *abort) {  // let the copies in flight land before the CTA can leave
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(qfull, 0) && globaltimer_ns() - t0 < 1000000000ull) {
      }
      for (int j = issued - 2 < 0 ? 0 : issued - 2; j < issued; ++j) {
        const uint32_t ph = (j >> 1) & 1;
        const uint64_t t1 = globaltimer_ns();
        while (!(mbar_try_wait(&kfull[j & 1], ph) && mbar_try_wait(&vfull[j & 1], ph)) &&
               globaltimer_ns() - t1 < 1000000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ------------------------------------------------ MMA issuer
      const uint32_t qa = smem_u32(smem + C::Q_OFF);
      bool ok = mbar_wait(qfull, 0, abort, dev_status);
      for (int j = 0; ok && j <= nt; ++j) {
        if (j < nt) {
          const int sb = j & 1;
          if (j >= 2 && !mbar_wait(pvdone, (j - 2) & 1, abort, dev_status)) break;
          if (!mbar_wait(&kfull[sb], (j >> 1) & 1, abort, dev_status)) break;
          tc_fence_after();
          const uint32_t ka = smem_u32(smem + C::K_OFF + sb * 2 * C::TILE_BYTES);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t o = (kk >> 2) * (BQ * 128) + (kk & 3) * 32;
            mma_ss(tS + sb * BKV, sdesc_sw128(qa + o, 16, 1024), sdesc_sw128(ka + o, 16, 1024), C::IDESC_QK, kk > 0);
          }
          mma_commit(&sfull[sb]);
        }
        if (j >= 1) {
          const int jj = j - 1, pb = jj & 1;
          if (!mbar_wait(&pready[pb], (jj >> 1) & 1, abort, dev_status)) break;
          if (!mbar_wait(&vfull[pb], (jj >> 1) & 1, abort, dev_status)) break;
          tc_fence_after();
          const uint32_t va = smem_u32(smem + C::V_OFF + pb * 2 * C::TILE_BYTES);
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk)
            mma_ts(tO, tS + pb * BKV + kk * 8, sdesc_sw128(va + kk * 2048, BKV * 128, 1024), C::IDESC_PV,
                   (jj > 0 || kk > 0) ? 1u : 0u);
          mma_commit(pvdone);
          mma_commit(&empty[pb]);
        }
      }
      mma_commit(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < 1000000000ull) {
      }
    }
  } else {  // ------------------------------------------------------------ softmax warps 2..5
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;  // query row in the tile == TMEM lane
    const int il = t * BQ + r;     // row within the sequence
    const bool valid = il < m;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    if (h == 0 && valid && il > 0 && dev_status && pos[off + il - 1] >= pos[off + il])
      atomicOr(dev_status, TG_DEV_POS_NOT_ASCENDING);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int sb = j & 1;
      // warp-uniform waits: the tcgen05.ld/st below are warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&bfull[sb], (j >> 1) & 1, abort, dev_status) &&
                                       mbar_wait(&sfull[sb], (j >> 1) & 1, abort, dev_status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[BKV];
#pragma unroll
      for (int c = 0; c < BKV / 32; ++c)
        tmem_ld32(tS + lane_base + sb * BKV + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_wait_ld();
      const float* bs = bias_s + sb * BKV;
      const bool diag = (j == t);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < BKV; ++c) {
        float x = fmaf(__uint_as_float(sr[c]), qk_scale, bs[c]);
        if (diag && c > r) x = -INFINITY;
        sr[c] = __float_as_uint(x);
        mx = fmaxf(mx, x);
      }
      const float m_new = fmaxf(m_run, mx);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;  // a row whose keys are all -inf stays finite
      const float alpha = ex2(m_run - m_use);
      float sum = 0.f;
      uint32_t pk[BKV / 2];
      const float* gm = gmul_s + sb * BKV;
#pragma unroll
      for (int c = 0; c < BKV; c += 2) {
        const float p0 = ex2(__uint_as_float(sr[c]) - m_use);
        const float p1 = ex2(__uint_as_float(sr[c + 1]) - m_use);
        sum += p0 + p1;
        pk[c / 2] = unnorm ? pack_bf16(p0 * gm[c], p1 * gm[c + 1]) : pack_bf16(p0, p1);
      }
      l_run = l_run * alpha + sum;
      m_run = m_new;
      if (j > 0) {
        if (!__all_sync(0xffffffffu, mbar_wait(pvdone, (j - 1) & 1, abort, dev_status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {  // rescale the running O in TMEM
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tO + lane_base + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tO + lane_base + c0, o);
          }
          tmem_wait_st();
        }
      }
      tmem_st32(tS + lane_base + sb * BKV, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
      tmem_st32(tS + lane_base + sb * BKV + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&pready[sb]);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(pvdone, (nt - 1) & 1, abort, dev_status))) {
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      __nv_bfloat16* orow = O + ((int64_t)(off + il) * Hq + h) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tO + lane_base + c0, o);
        tmem_wait_ld();
        uint32_t pkd[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pkd[e] = pack_bf16(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pkd[4 * v], pkd[4 * v + 1], pkd[4 * v + 2], pkd[4 * v + 3]);
        }
      }
      if (valid && lse) lse[(int64_t)h * m_tot + off + il] = (m_run + __log2f(l_run)) * kLn2;
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
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return cuda_status(e, "tg_gated_attn_fwd: cudaFuncSetAttribute");
    attr_set = true;
  }
  const int grid = units * a.Hq;
  attn_tc_kernel<D><<<grid, NTHREADS, C::SMEM, st>>>(tq, tk, tv, a.logg, a.head_gain, a.pos,
                                                     static_cast<__nv_bfloat16*>(a.O), a.lse, a.m_tot, a.Hq, a.Hkv,
                                                     a.scale * kLog2e, a.flags, a.dev_status, p);
  return cuda_status(cudaGetLastError(), "tg_gated_attn_fwd: attn_tc launch");
}

}  // namespace

tg_status launch_attn_tc(const AttnArgs& a, const AttnSeq* seqs, int nseq, cudaStream_t st) {
  if (a.D == 64) return launch_d<64>(a, seqs, nseq, st);
  return launch_d<128>(a, seqs, nseq, st);
}

}  // namespace tg
