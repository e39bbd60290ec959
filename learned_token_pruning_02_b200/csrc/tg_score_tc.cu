// Gate-MLP score on the 5th-generation tensor cores: score = w2 . GELU(W1 h + b1) + b2.
//
// TokenGate paper page (thelatestinai.com), Figure 1(b): a small scoring network scores
// every hidden state at the selection layer; aitualizate.com article, phase 2.
//
// Design (B200, bf16 in, fp32 accumulate):
//   * One CTA per SM, persistent over 128-token tiles. The whole hidden width dg (<= 256)
//     is one UMMA N, so a tile is one 128 x dg accumulator in TMEM (fp32) and H is read
//     from HBM exactly once. Two accumulators (2 x dg TMEM columns) let the epilogue of
//     tile t overlap the MMAs of tile t+1.
//   * Warp 0 streams 64-wide K slices of H (128 x 64) and W1 (dg x 64) with TMA into a ring
//     of shared-memory stages in the 128-byte swizzle layout; W1 stays L2-resident.
//   * Warp 1 (one thread) issues tcgen05.mma (M=128, N=dg, K=16) and releases each stage
//     with tcgen05.commit; it also owns the TMEM allocation.
//   * Warps 2-5 are the epilogue: each thread owns one token row, reads its dg fp32 values
//     with tcgen05.ld, and reduces + b1 -> exact-erf GELU -> * w2 -> sum in registers, so
//     the [n_tok, dg] hidden activation never leaves the SM. Only 4 bytes per token are
//     written.
//   * Every wait is bounded (about 2 s); on a timeout the kernel sets TG_DEV_TIMEOUT,
//     drains its outstanding copies and MMAs, frees TMEM and returns.
#include "tg_internal.cuh"
#include "tg_sm100.cuh"

namespace tg {
namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int NTHREADS = 224;  // warp 0: H loads, 1: MMA, 2-5: epilogue, 6: W1 loads

template <int DG>
struct Cfg {
  static constexpr int A_BYTES = BM * BK * 2;  // one 128 x 64 slice of H
  static constexpr int B_BYTES = DG * BK * 2;  // one dg x 64 slice of W1
  // H streams from HBM through a deep ring (about 2 us of latency cover at full rate);
  // W1 comes from L2 through a shallow one.
  static constexpr int SA = DG == 64 ? 10 : 8;
  static constexpr int SB = DG == 256 ? 2 : (DG == 128 ? 3 : 4);
  static constexpr int RING = SA * A_BYTES + SB * B_BYTES;
  static constexpr int TMEM_COLS = 2 * DG;
  static constexpr int TAIL = 2048;  // barriers, flags
  static constexpr int SMEM = 1024 + RING + TAIL + 2 * DG * 4;
  static constexpr uint32_t IDESC = idesc_bf16_f32(BM, DG, false);
};

template <int DG>
__global__ void __launch_bounds__(NTHREADS, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW,
                    const float* __restrict__ b1, const __nv_bfloat16* __restrict__ w2, float b2,
                    float* __restrict__ score, int n_tok, int nk, int n_tiles, int32_t* __restrict__ dev_status) {
  using C = Cfg<DG>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ringA = smem;
  uint8_t* ringB = smem + C::SA * C::A_BYTES;
  uint8_t* tail = smem + C::RING;
  uint64_t* afull = reinterpret_cast<uint64_t*>(tail);
  uint64_t* aempty = afull + C::SA;
  uint64_t* bfull = aempty + C::SA;
  uint64_t* bempty = bfull + C::SB;
  uint64_t* accf = bempty + C::SB;
  uint64_t* acce = accf + 2;
  uint64_t* drain = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* b1s = reinterpret_cast<float*>(tail + C::TAIL);
  float* w2s = b1s + DG;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::SA; ++s) {
      mbar_init(&afull[s], 1);
      mbar_init(&aempty[s], 1);
    }
    for (int s = 0; s < C::SB; ++s) {
      mbar_init(&bfull[s], 1);
      mbar_init(&bempty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 4);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmH);
    prefetch_tmap(&tmW);
  }
  if (warp >= 2 && warp <= 5) {
    for (int u = threadIdx.x - 64; u < DG; u += 128) {
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

  if (warp == 0 || warp == 6) {
    if (lane == 0) {  // TMA producers: warp 0 streams H, warp 6 streams W1
      const bool isA = warp == 0;
      const int NS = isA ? C::SA : C::SB;
      uint64_t* full = isA ? afull : bfull;
      uint64_t* empty = isA ? aempty : bempty;
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !*abort; tile += gridDim.x) {
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort, dev_status)) break;
          if (isA) {
            mbar_arrive_expect_tx(&full[stage], C::A_BYTES);
            tma_load_2d(ringA + stage * C::A_BYTES, &tmH, kb * BK, tile * BM, &full[stage]);
          } else {
            mbar_arrive_expect_tx(&full[stage], C::B_BYTES);
            tma_load_2d(ringB + stage * C::B_BYTES, &tmW, kb * BK, 0, &full[stage]);
          }
          ++issued;
          if (++stage == NS) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort) {  // drain the copies still in flight before the CTA can leave
        for (long n = issued - NS < 0 ? 0 : issued - NS; n < issued; ++n) {
          const int s2 = (int)(n % NS);
          const uint32_t ph = (uint32_t)((n / NS) & 1);
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&full[s2], ph) && globaltimer_ns() - t0 < 1000000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      int sa = 0, sb = 0;
      uint32_t pa = 0, pb = 0;
      int it = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !*abort; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        if (!mbar_wait(&acce[acc], ((it >> 1) & 1) ^ 1u, abort, dev_status)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * DG;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&afull[sa], pa, abort, dev_status) || !mbar_wait(&bfull[sb], pb, abort, dev_status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(ringA + sa * C::A_BYTES);
          const uint32_t b0 = smem_u32(ringB + sb * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_ss(d, sdesc_sw128(a0 + 32 * k, 16, 1024), sdesc_sw128(b0 + 32 * k, 16, 1024), C::IDESC,
                   (kb | k) != 0);
          mma_commit(&aempty[sa]);
          mma_commit(&bempty[sb]);
          if (++sa == C::SA) {
            sa = 0;
            pa ^= 1u;
          }
          if (++sb == C::SB) {
            sb = 0;
            pb ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&accf[acc]);
      }
      // every MMA issued above completes before TMEM can be released
      mma_commit(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < 1000000000ull) {
      }
    }
  } else {  // epilogue: warps 2..5, one token row per thread
    const int q = warp & 3;
    const int row = q * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      // warp-uniform: the tcgen05.ld below is warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&accf[acc], (it >> 1) & 1, abort, dev_status))) break;
      tc_fence_after();
      float s = 0.f;
      const uint32_t base = tmem + ((uint32_t)(q * 32) << 16) + acc * DG;
#pragma unroll 1
      for (int c0 = 0; c0 < DG; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(base + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float z = __uint_as_float(v[j]) + b1s[c0 + j];
          const float gz = 0.5f * z * (1.f + erff(z * 0.70710678118654752f));
          s = fmaf(gz, w2s[c0 + j], s);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[acc]);
      const long r = (long)tile * BM + row;
      if (r < n_tok) score[r] = s + b2;
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
  int grid = device_sm_count();
  if (grid > n_tiles) grid = n_tiles;
  score_tc_kernel<DG><<<grid, NTHREADS, C::SMEM, st>>>(tmH, tmW, b1, static_cast<const __nv_bfloat16*>(w2), b2, score,
                                                      (int)n_tok, d / BK, n_tiles, nullptr);
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
