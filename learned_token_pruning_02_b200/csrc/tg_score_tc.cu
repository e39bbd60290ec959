// Gate-MLP score on the 5th-generation tensor cores: score = w2 . GELU(W1 h + b1) + b2.
//
// TokenGate paper page (thelatestinai.com), Figure 1(b): a small scoring network scores
// every hidden state at the selection layer; aitualizate.com article, phase 2.
//
// Design (B200, bf16 in, fp32 accumulate), 2-SM tensor-core tiles:
//   * A cluster of two CTAs on two SMs computes a 256-token tile with one tcgen05.mma
//     M=256, N=dg (the whole hidden width), K=16 stream. Each CTA holds its 128 rows of H
//     and HALF of the current W1 slice (dg/2 rows) in its own shared memory, so every SM
//     pulls only half of W1 per tile from L2, and the [n_tok, dg] activation lives only in
//     TMEM (each CTA keeps its 128 rows x dg columns).
//   * Warp 0 of each CTA streams 64-wide K slices of its H rows and W1 half with TMA
//     (128-byte swizzle) into a 6-deep ring; the bytes of both CTAs are counted on the even
//     CTA's barrier. Each CTA starts its K loop at a different slice, which spreads the W1
//     reads over L2.
//   * One thread of the even CTA issues the pair's MMAs into a double-buffered TMEM
//     accumulator and releases ring stages and accumulators in both CTAs with a
//     multicast tcgen05.commit.
//   * Warps 2-9 of each CTA are the epilogue: two groups of four warps (one per TMEM lane
//     quarter) take half of the dg columns each and reduce + b1 -> exact-erf GELU -> * w2
//     in registers; the halves meet in shared memory. Thanks to the second accumulator the
//     epilogue of tile t overlaps the MMAs of tile t+1.
//   * Every wait is bounded (about 2 s); on a timeout the CTA sets its abort flag, drains
//     outstanding copies and MMAs, frees TMEM and returns.
#include "tg_internal.cuh"
#include "tg_sm100.cuh"

namespace tg {
namespace {

using namespace sm100;

constexpr int BM = 128;  // token rows per CTA (256 per pair)
constexpr int BK = 64;
constexpr int NEPI = 8;                   // epilogue warps per CTA
constexpr int NTHREADS = 32 * (2 + NEPI);  // 320

template <int DG>
struct Cfg {
  static constexpr int A_BYTES = BM * BK * 2;        // this CTA's 128 x 64 slice of H
  static constexpr int B_BYTES = (DG / 2) * BK * 2;  // this CTA's dg/2 x 64 slice of W1
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES = DG == 256 ? 6 : (DG == 128 ? 8 : 10);
  static constexpr int TMEM_COLS = 2 * DG;  // two accumulators of 128 lanes x dg
  static constexpr int TAIL = 1024;         // barriers, flags
  static constexpr int SMEM = 1024 + STAGES * STAGE + TAIL + 2 * DG * 4 + 2 * BM * 4;
  static constexpr uint32_t IDESC = idesc_bf16_f32(2 * BM, DG, false);  // M = 256 across the pair
};

template <int DG>
__global__ void __launch_bounds__(NTHREADS, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW,
                    const float* __restrict__ b1, const __nv_bfloat16* __restrict__ w2, float b2,
                    float* __restrict__ score, int n_tok, int nk, int n_tiles, int32_t* __restrict__ dev_status) {
  using C = Cfg<DG>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tail = smem + C::STAGES * C::STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);  // [STAGES] used in the even CTA
  uint64_t* empty = full + C::STAGES;                   // [STAGES] per CTA
  uint64_t* accf = empty + C::STAGES;                   // [2] per CTA
  uint64_t* acce = accf + 2;                            // [2] used in the even CTA
  uint64_t* half_ready = acce + 2;                      // [2] per CTA, one per accumulator
  uint64_t* drain = half_ready + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* b1s = reinterpret_cast<float*>(tail + C::TAIL);
  float* w2s = b1s + DG;
  float* part = w2s + DG;  // [2][BM] partial sums of the upper column half, per accumulator

  const uint32_t cr = cluster_ctarank();  // 0 = even CTA (issues the MMAs), 1 = odd
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 2 * NEPI);
      mbar_init(&half_ready[a], 128);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmH);
    prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  griddep_launch_dependents();  // the next kernel may start its prologue
  griddep_wait();               // the previous kernel's results are visible from here on
  if (warp >= 2) {
    for (int u = threadIdx.x - 64; u < DG; u += 32 * NEPI) {
      b1s[u] = b1 ? b1[u] : 0.f;
      w2s[u] = __bfloat162float(w2[u]);
    }
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised, TMEM of the pair allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int kb0 = (int)(((long)pair * nk) / npairs);  // first K slice of this pair

  if (warp == 0) {
    if (lane == 0) {  // ---------------------------------------------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      for (int tile = pair; tile < n_tiles && !*abort; tile += npairs) {
        for (int i = 0; i < nk; ++i) {
          const int kb = (i + kb0) % nk;
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort, dev_status)) break;
          uint8_t* st = smem + stage * C::STAGE;
          if (cr == 0) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE);  // both CTAs' bytes
          tma_load_2d_pair(st, &tmH, kb * BK, tile * (2 * BM) + (int)cr * BM, &full[stage]);
          tma_load_2d_pair(st + C::A_BYTES, &tmW, kb * BK, (int)cr * (DG / 2), &full[stage]);
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort && cr == 0) {  // drain the copies still in flight before the pair can leave
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
    if (lane == 0 && cr == 0) {  // ------------------------------------ MMA issuer (even CTA)
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int tile = pair; tile < n_tiles && !*abort; tile += npairs, ++it) {
        const int acc = it & 1;
        if (!mbar_wait(&acce[acc], ((it >> 1) & 1) ^ 1u, abort, dev_status)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * DG;
        bool ok = true;
        for (int i = 0; i < nk; ++i) {
          if (!mbar_wait(&full[stage], phase, abort, dev_status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * C::STAGE);
          const uint32_t b0 = a0 + C::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_ss_pair(d, sdesc_sw128(a0 + 32 * k, 16, 1024), sdesc_sw128(b0 + 32 * k, 16, 1024), C::IDESC,
                        (i | k) != 0);
          mma_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair_mc(&accf[acc], 0x3);
      }
      // every MMA issued above completes before TMEM can be released (in both CTAs)
      mma_commit_pair_mc(drain, 0x3);
    }
  } else {  // ------------------------------------------------ epilogue: warps 2..9
    const int half = (warp - 2) >> 2;  // which half of the dg columns
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;
    const int c_lo = half * (DG / 2);
    int it = 0;
    for (int tile = pair; tile < n_tiles; tile += npairs, ++it) {
      const int acc = it & 1;
      // warp-uniform: the tcgen05.ld below is warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&accf[acc], (it >> 1) & 1, abort, dev_status))) break;
      tc_fence_after();
      float s = 0.f;
      const uint32_t base = tmem + ((uint32_t)(q * 32) << 16) + acc * DG + c_lo;
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
        part[acc * BM + row] = s;
        mbar_arrive(&half_ready[acc]);
      } else {
        ok = __all_sync(0xffffffffu, mbar_wait(&half_ready[acc], (it >> 1) & 1, abort, dev_status));
        const long r = (long)tile * (2 * BM) + (long)cr * BM + row;
        if (ok && r < n_tok) score[r] = (s + part[acc * BM + row]) + b2;
      }
      // the accumulator (and this buffer's partial sums) is released only once fully consumed
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(&acce[acc], 0);
      if (!ok) break;
    }
  }

  // both CTAs wait until every MMA of the pair has completed before TMEM is released
  if (warp == 1) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < 1000000000ull) {
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still signal its barriers
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, C::TMEM_COLS);
}

template <int DG>
tg_status launch_dg(const void* H, int64_t ldh, int64_t n_tok, int d, const void* W1, const float* b1, const void* w2,
                    float b2, float* score, cudaStream_t st) {
  using C = Cfg<DG>;
  CUtensorMap tmH, tmW;
  if (!make_tmap_bf16_2d(&tmH, H, (uint64_t)n_tok, (uint64_t)d, (uint64_t)ldh, BM, BK) ||
      !make_tmap_bf16_2d(&tmW, W1, (uint64_t)DG, (uint64_t)d, (uint64_t)d, DG / 2, BK))
    return fail(TG_ERR_CUDA, "tg_score: building the TMA tensor maps failed");
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<DG>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return cuda_status(e, "tg_score: cudaFuncSetAttribute");
    attr_set = true;
  }
  const int n_tiles = (int)((n_tok + 2 * BM - 1) / (2 * BM));
  int pairs = device_sm_count() / 2;
  if (pairs > n_tiles) pairs = n_tiles;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  cfg.blockDim = dim3(NTHREADS);
  cfg.dynamicSmemBytes = (size_t)C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute(PDL_SCORE);
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cuda_status(cudaLaunchKernelEx(&cfg, score_tc_kernel<DG>, tmH, tmW, b1,
                                        static_cast<const __nv_bfloat16*>(w2), b2, score, (int)n_tok, d / BK,
                                        n_tiles, (int32_t*)nullptr),
                     "tg_score: score_tc launch");
}

}  // namespace

tg_status launch_score_tc(const void* H, int64_t ldh, int64_t n_tok, int d, const void* W1, const float* b1,
                          const void* w2, float b2, int dg, float* score, cudaStream_t st) {
  if (dg == 64) return launch_dg<64>(H, ldh, n_tok, d, W1, b1, w2, b2, score, st);
  if (dg == 128) return launch_dg<128>(H, ldh, n_tok, d, W1, b1, w2, b2, score, st);
  return launch_dg<256>(H, ldh, n_tok, d, W1, b1, w2, b2, score, st);
}

}  // namespace tg
