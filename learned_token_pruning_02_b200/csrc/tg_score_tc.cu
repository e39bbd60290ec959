// Gate-MLP score on the 5th-generation tensor cores: score = w2 . GELU(W1 h + b1) + b2.
//
// TokenGate paper page (thelatestinai.com), Figure 1(b): a small scoring network scores
// every hidden state at the selection layer; aitualizate.com article, phase 2.
//
// Design (B200, bf16 in, fp32 accumulate). The whole hidden width dg (<= 256) is one UMMA N,
// so the [n_tok, dg] activation lives only in TMEM and H is read from HBM exactly once.
// W1 (dg x d) is re-read from L2 by every CTA, so each CTA multiplies one W1 slice into TWO
// 128-token tiles (a 256-token pair) to halve the W1 bytes per flop, and each CTA starts its
// K loop at a different slice so the CTAs do not all hit the same L2 lines at once:
//   * warp 0 (one thread): TMA loads, per 64-wide K slice, H rows of both tiles and the W1
//     slice into a ring of shared-memory stages (128-byte swizzle).
//   * warp 1 (one thread): tcgen05.mma M=128, N=dg, K=16 for both tiles into two fp32 TMEM
//     accumulators (2 x dg columns); releases stages with tcgen05.commit; owns TMEM.
//   * warps 2-17: epilogue. Four warps cover the 128 TMEM lanes; four such groups split the
//     work into (tile, half of the dg columns). Each thread reduces + b1 -> exact-erf GELU
//     -> * w2 over its 128 columns in registers; the two halves meet in shared memory.
//   * Persistent over tile pairs; every wait is bounded (about 2 s); on a timeout the kernel
//     sets its abort flag, drains outstanding copies and MMAs, frees TMEM and returns.
#include "tg_internal.cuh"
#include "tg_sm100.cuh"

namespace tg {
namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int NEPI = 16;                      // epilogue warps
constexpr int NTHREADS = 32 * (2 + NEPI);     // 576

template <int DG>
struct Cfg {
  static constexpr int A_BYTES = BM * BK * 2;  // one 128 x 64 slice of H
  static constexpr int B_BYTES = DG * BK * 2;  // one dg x 64 slice of W1
  static constexpr int STAGE = 2 * A_BYTES + B_BYTES;
  static constexpr int STAGES = DG == 256 ? 3 : (DG == 128 ? 4 : 5);
  static constexpr int TMEM_COLS = 2 * DG;
  static constexpr int TAIL = 1024;  // barriers, flags
  static constexpr int SMEM = 1024 + STAGES * STAGE + TAIL + 2 * DG * 4 + 2 * BM * 4;
  static constexpr uint32_t IDESC = idesc_bf16_f32(BM, DG, false);
};

template <int DG>
__global__ void __launch_bounds__(NTHREADS, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW,
                    const float* __restrict__ b1, const __nv_bfloat16* __restrict__ w2, float b2,
                    float* __restrict__ score, int n_tok, int nk, int n_pairs, int32_t* __restrict__ dev_status) {
  using C = Cfg<DG>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tail = smem + C::STAGES * C::STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accf = empty + C::STAGES;
  uint64_t* acce = accf + 1;
  uint64_t* half_ready = acce + 1;  // [2] one per tile of the pair
  uint64_t* drain = half_ready + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* b1s = reinterpret_cast<float*>(tail + C::TAIL);
  float* w2s = b1s + DG;
  float* part = w2s + DG;  // [2][BM] partial sums of the upper column half

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb0 = (int)(((long)blockIdx.x * nk) / gridDim.x);  // first K slice of this CTA
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    mbar_init(acce, NEPI);
    mbar_init(&half_ready[0], 128);
    mbar_init(&half_ready[1], 128);
    mbar_init(drain, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmH);
    prefetch_tmap(&tmW);
  }
  if (warp >= 2) {
    for (int u = threadIdx.x - 64; u < DG; u += 32 * NEPI) {
      b1s[u] = b1 ? b1[u] : 0.f;
      w2s[u] = __bfloat162float(w2[u]);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {  // ---------------------------------------------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      for (int pr = blockIdx.x; pr < n_pairs && !*abort; pr += gridDim.x) {
        for (int i = 0; i < nk; ++i) {
          const int kb = (i + kb0) % nk;  // CTAs start at different W1 slices (spreads L2 hot spots)
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort, dev_status)) break;
          uint8_t* st = smem + stage * C::STAGE;
          mbar_arrive_expect_tx(&full[stage], C::STAGE);
          tma_load_2d(st, &tmH, kb * BK, (2 * pr) * BM, &full[stage]);
          tma_load_2d(st + C::A_BYTES, &tmH, kb * BK, (2 * pr + 1) * BM, &full[stage]);
          tma_load_2d(st + 2 * C::A_BYTES, &tmW, kb * BK, 0, &full[stage]);
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort) {  // drain the copies still in flight before the CTA can leave
        for (long n = issued - C::STAGES < 0 ? 0 : issued - C::STAGES; n < issued; ++n) {
          const int s2 = (int)(n % C::STAGES);
          const uint32_t ph = (uint32_t)((n / C::STAGES) & 1);
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&full[s2], ph) && globaltimer_ns() - t0 < 1000000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int pr = blockIdx.x; pr < n_pairs && !*abort; pr += gridDim.x, ++it) {
        if (!mbar_wait(acce, (it & 1) ^ 1u, abort, dev_status)) break;
        tc_fence_after();
        bool ok = true;
        for (int i = 0; i < nk; ++i) {
          if (!mbar_wait(&full[stage], phase, abort, dev_status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * C::STAGE);
          const uint32_t a1 = a0 + C::A_BYTES;
          const uint32_t b0 = a0 + 2 * C::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t bd = sdesc_sw128(b0 + 32 * k, 16, 1024);
            mma_ss(tmem, sdesc_sw128(a0 + 32 * k, 16, 1024), bd, C::IDESC, (i | k) != 0);
            mma_ss(tmem + DG, sdesc_sw128(a1 + 32 * k, 16, 1024), bd, C::IDESC, (i | k) != 0);
          }
          mma_commit(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(accf);
      }
      // every MMA issued above completes before TMEM can be released
      mma_commit(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < 1000000000ull) {
      }
    }
  } else {  // ------------------------------------------- epilogue: warps 2..17
    const int grp = (warp - 2) >> 2;  // 0..3
    const int tile = grp >> 1, half = grp & 1;
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;
    const int c_lo = half * (DG / 2);
    int it = 0;
    for (int pr = blockIdx.x; pr < n_pairs; pr += gridDim.x, ++it) {
      // warp-uniform: the tcgen05.ld below is warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(accf, it & 1, abort, dev_status))) break;
      tc_fence_after();
      float s = 0.f;
      const uint32_t base = tmem + ((uint32_t)(q * 32) << 16) + tile * DG + c_lo;
#pragma unroll 1
      for (int c0 = 0; c0 < DG / 2; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(base + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float z = __uint_as_float(v[j]) + b1s[c_lo + c0 + j];
          const float gz = 0.5f * z * (1.f + erff(z * 0.70710678118654752f));
          s = fmaf(gz, w2s[c_lo + c0 + j], s);
        }
      }
      tc_fence_before();
      bool ok = true;
      if (half == 1) {
        part[tile * BM + row] = s;
        mbar_arrive(&half_ready[tile]);
      } else {
        ok = __all_sync(0xffffffffu, mbar_wait(&half_ready[tile], it & 1, abort, dev_status));
        const long r = (long)(2 * pr + tile) * BM + row;
        if (ok && r < n_tok) score[r] = (s + part[tile * BM + row]) + b2;
      }
      // the accumulators (and the partial sums) are released only once this pair is fully
      // consumed, so neither can be overwritten early
      __syncwarp();
      if (lane == 0) mbar_arrive(acce);
      if (!ok) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int DG>
tg_status launch_dg(const void* H, int64_t ldh, int64_t n_tok, int d, const void* W1, const float* b1, const void* w2,
                    float b2, float* score, cudaStream_t st) {
  using C = Cfg<DG>;
  CUtensorMap tmH, tmW;
  if (!make_tmap_bf16_2d(&tmH, H, (uint64_t)n_tok, (uint64_t)d, (uint64_t)ldh, BM, BK) ||
      !make_tmap_bf16_2d(&tmW, W1, (uint64_t)DG, (uint64_t)d, (uint64_t)d, DG, BK))
    return fail(TG_ERR_CUDA, "tg_score: building the TMA tensor maps failed");
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<DG>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return cuda_status(e, "tg_score: cudaFuncSetAttribute");
    attr_set = true;
  }
  const int n_tiles = (int)((n_tok + BM - 1) / BM);
  const int n_pairs = (n_tiles + 1) / 2;
  int grid = device_sm_count();
  if (grid > n_pairs) grid = n_pairs;
  score_tc_kernel<DG><<<grid, NTHREADS, C::SMEM, st>>>(tmH, tmW, b1, static_cast<const __nv_bfloat16*>(w2), b2, score,
                                                      (int)n_tok, d / BK, n_pairs, nullptr);
  return cuda_status(cudaGetLastError(), "tg_score: score_tc launch");
}

}  // namespace

tg_status launch_score_tc(const void* H, int64_t ldh, int64_t n_tok, int d, const void* W1, const float* b1,
                          const void* w2, float b2, int dg, float* score, cudaStream_t st) {
  if (dg == 64) return launch_dg<64>(H, ldh, n_tok, d, W1, b1, w2, b2, score, st);
  if (dg == 128) return launch_dg<128>(H, ldh, n_tok, d, W1, b1, w2, b2, score, st);
  return launch_dg<256>(H, ldh, n_tok, d, W1, b1, w2, b2, score, st);
}

}  // namespace tg
