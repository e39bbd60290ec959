// Gate-MLP score on the 5th-generation tensor cores: score = (w2 . GELU(W1 h + b1) + b2) / temperature.
//
// TokenGate paper page (thelatestinai.com), Figure 1(b): a small scoring network scores
// every hidden state at the selection layer; aitualizate.com article, phase 2.
//
// Design (B200, bf16 in, fp32 accumulate), one CTA per SM, each on its own:
//   * A CTA computes 128-token tiles with one tcgen05.mma M=128, N=dg (the whole hidden
//     width), K=16 stream; the [tokens, dg] activation lives only in TMEM. The score is a
//     pure stream of H, so the tile loop is built around keeping HBM busy: the kernel does
//     not pair SMs (a 2-SM MMA couples both SMs' load pipelines stage by stage, which was
//     measured to halve the streaming rate of H on this part).
//   * Warp 0 streams 64-wide K slices of the tile's H rows with TMA (128-byte swizzle) into
//     a 7-deep ring (112 KB in flight); warp 10 streams the matching W1 slices (dg x 64)
//     into a separate 3-deep ring. H comes from HBM and needs many bytes in flight; W1 is
//     served by L2. Each CTA starts its K loop at a different slice, which spreads the W1
//     reads over L2.
//   * One thread issues the MMAs into a double-buffered TMEM accumulator and releases ring
//     stages and accumulators with tcgen05.commit.
//   * Warps 2..2+4G-1 are the epilogue: G column groups of four warps (one per TMEM lane
//     quarter; G = 4 for dg >= 128) take dg/G columns each and reduce + b1 -> GELU -> * w2
//     in registers; the groups meet in shared memory. Thanks to the second accumulator the
//     epilogue of tile t overlaps the MMAs of tile t+1; the last tile's epilogue is exposed,
//     which is why it is spread over 16 warps and works on column pairs with packed f32x2
//     arithmetic, taking erf from Abramowitz-Stegun 7.1.28 (one reciprocal, no exponential).
//   * Every wait is bounded (about 2 s); on a timeout the CTA sets its abort flag, drains
//     outstanding copies and MMAs, frees TMEM and returns.
#include "tg_internal.cuh"
#include "tg_sm100.cuh"

namespace tg {
namespace {

using namespace sm100;

constexpr int BM = 128;  // token rows per tile
constexpr int BK = 64;

// GELU(z) = z (1 + erf(z / sqrt 2)) / 2 = z / 2 + |z| erf(|z| / sqrt 2) / 2, with erf from
// Abramowitz & Stegun, Handbook of Mathematical Functions, formula 7.1.28: for x >= 0,
// erf(x) = 1 - (1 + a1 x + a2 x^2 + a3 x^3 + a4 x^4 + a5 x^5 + a6 x^6)^-16, |error| <= 3e-7.
// The 1/sqrt 2 is folded into the coefficients (c_k = a_k 2^(-k/2)), so with P = 1 + sum c_k |z|^k,
// GELU(z) = z/2 + |z| (1/2 - P^-16 / 2): one reciprocal, four squarings, no exponential.
constexpr double kAS[6] = {0.0705230784, 0.0422820123, 0.0092705272, 0.0001520143, 0.0002765672, 0.0000430638};
constexpr float gelu_c(int k) {  // a_k / 2^(k/2), k = 1..6
  double v = kAS[k - 1];
  for (int i = 0; i < k; ++i) v *= 0.70710678118654752440;
  return (float)v;
}
constexpr float kG1 = gelu_c(1), kG2 = gelu_c(2), kG3 = gelu_c(3), kG4 = gelu_c(4), kG5 = gelu_c(5), kG6 = gelu_c(6);

// w * GELU(z) for a pair of columns, accumulated into s; hw = w / 2.
__device__ __forceinline__ float2 gelu_w_acc2(float2 z, float2 w, float2 hw, float2 s) {
  const float2 a = make_float2(fabsf(z.x), fabsf(z.y));
  float2 P = __ffma2_rn(a, make_float2(kG6, kG6), make_float2(kG5, kG5));
  P = __ffma2_rn(a, P, make_float2(kG4, kG4));
  P = __ffma2_rn(a, P, make_float2(kG3, kG3));
  P = __ffma2_rn(a, P, make_float2(kG2, kG2));
  P = __ffma2_rn(a, P, make_float2(kG1, kG1));
  P = __ffma2_rn(a, P, make_float2(1.f, 1.f));
  float2 r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r.x) : "f"(P.x));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r.y) : "f"(P.y));
  r = __fmul2_rn(r, r);
  r = __fmul2_rn(r, r);
  r = __fmul2_rn(r, r);
  r = __fmul2_rn(r, r);                                                           // P^-16
  const float2 m = __ffma2_rn(r, make_float2(-0.5f, -0.5f), make_float2(0.5f, 0.5f));  // erf / 2
  s = __ffma2_rn(hw, z, s);                                                       // + w z / 2
  return __ffma2_rn(w, __fmul2_rn(a, m), s);                                      // + w |z| erf / 2
}

template <int DG>
struct Cfg {
  static constexpr int NGRP = DG >= 128 ? 4 : 2;     // epilogue column groups
  static constexpr int NEPI = 4 * NGRP;              // epilogue warps (warps 2..2+NEPI-1)
  static constexpr int WPROD = 2 + NEPI;             // warp that streams W1
  static constexpr int NTHREADS = 32 * (3 + NEPI);
  static constexpr int CW = DG / NGRP;               // columns per group
  static constexpr int A_BYTES = BM * BK * 2;  // 128 x 64 slice of H
  static constexpr int B_BYTES = DG * BK * 2;  // dg x 64 slice of W1
  static constexpr int WS = DG == 256 ? 3 : 4;                      // W1 ring depth
  static constexpr int HS = DG == 256 ? 7 : (DG == 128 ? 9 : 11);  // H ring depth
  static constexpr int TMEM_COLS = 2 * DG;  // two accumulators of 128 lanes x dg
  static constexpr int TAIL = 1024;         // barriers, flags
  static constexpr int SMEM = 1024 + HS * A_BYTES + WS * B_BYTES + TAIL + 3 * DG * 4 + (NGRP - 1) * 2 * BM * 4;
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t IDESC = idesc_bf16_f32(BM, DG, false);
};

template <int DG>
__global__ void __launch_bounds__(Cfg<DG>::NTHREADS, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW,
                    const float* __restrict__ b1, const __nv_bfloat16* __restrict__ w2, float b2, float inv_t,
                    float* __restrict__ score, int n_tok, int nk, int n_tiles, int32_t* __restrict__ dev_status,
                    uint64_t probe_ns) {
  using C = Cfg<DG>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smem_w = smem + C::HS * C::A_BYTES;
  uint8_t* tail = smem_w + C::WS * C::B_BYTES;
  uint64_t* hfull = reinterpret_cast<uint64_t*>(tail);  // [HS]
  uint64_t* hempty = hfull + C::HS;                     // [HS]
  uint64_t* wfull = hempty + C::HS;                     // [WS]
  uint64_t* wempty = wfull + C::WS;                     // [WS]
  uint64_t* accf = wempty + C::WS;                      // [2] accumulator complete
  uint64_t* acce = accf + 2;                            // [2] accumulator consumed
  uint64_t* half_ready = acce + 2;                      // [2] partial sums of groups 1.. written
  uint64_t* drain = half_ready + 2;
  uint64_t* probe = drain + 1;  // test hook: a barrier nothing signals
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(probe + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* b1s = reinterpret_cast<float*>(tail + C::TAIL);
  float* w2s = b1s + DG;
  float* hw2s = w2s + DG;  // w2 / 2
  float* part = hw2s + DG;  // [NGRP-1][2][BM] partial sums of column groups 1.., per accumulator
  constexpr int NEPI = C::NEPI, WPROD = C::WPROD;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::HS; ++s) {
      mbar_init(&hfull[s], 1);
      mbar_init(&hempty[s], 1);
    }
    for (int s = 0; s < C::WS; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], NEPI);
      mbar_init(&half_ready[a], 128 * (C::NGRP - 1));
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_barrier_init();
    wait_probe(probe, probe_ns, abort, dev_status);  // no-op unless a test asked for it
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmH);
    prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  griddep_launch_dependents();  // the next kernel may start its prologue
  griddep_wait();               // the previous kernel's results are visible from here on
  if (warp >= 2 && warp < WPROD) {
    for (int u = threadIdx.x - 64; u < DG; u += 32 * NEPI) {
      b1s[u] = b1 ? b1[u] : 0.f;
      w2s[u] = __bfloat162float(w2[u]);
      hw2s[u] = 0.5f * w2s[u];
    }
  }
  tc_fence_before();
  __syncthreads();  // barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int kb0 = (int)(((long)blockIdx.x * nk) / gridDim.x);  // first K slice of this CTA
  const bool skip = *abort;  // only the test probe sets it this early: nothing was issued

  if (skip) {
  } else if (warp == 0 || warp == WPROD) {
    if (lane == 0) {  // ---------------------------------- TMA producers: H (warp 0), W1 (warp 10)
      const bool is_h = warp == 0;
      const int depth = is_h ? C::HS : C::WS;
      uint64_t* full = is_h ? hfull : wfull;
      uint64_t* empty = is_h ? hempty : wempty;
      const int bytes = is_h ? C::A_BYTES : C::B_BYTES;
      uint8_t* ring = is_h ? smem : smem_w;
      const CUtensorMap* tm = is_h ? &tmH : &tmW;
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !*abort; tile += gridDim.x) {
        const int y = is_h ? tile * BM : 0;
        for (int i = 0; i < nk; ++i) {
          const int kb = (i + kb0) % nk;
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort, dev_status)) break;
          mbar_arrive_expect_tx(&full[stage], bytes);
          tma_load_2d(ring + stage * bytes, tm, kb * BK, y, &full[stage]);
          ++issued;
          if (++stage == depth) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort) {  // drain the copies still in flight before the CTA can leave
        for (long n = issued - depth < 0 ? 0 : issued - depth; n < issued; ++n) {
          const int s2 = (int)(n % depth);
          const uint32_t ph = (uint32_t)((n / depth) & 1);
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&full[s2], ph) && globaltimer_ns() - t0 < 1000000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    {  // --------------------------- MMA issuer: the warp runs the schedule, one elected lane issues
      const bool leader = elect_one();
      int hs = 0, ws = 0;
      uint32_t hph = 0, wph = 0;
      int it = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !*abort; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&acce[acc], ((it >> 1) & 1) ^ 1u, abort, dev_status))) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * DG;
        bool ok = true;
        for (int i = 0; i < nk; ++i) {
          if (!__all_sync(0xffffffffu, mbar_wait(&hfull[hs], hph, abort, dev_status) &&
                                           mbar_wait(&wfull[ws], wph, abort, dev_status))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + hs * C::A_BYTES);
          const uint32_t b0 = smem_u32(smem_w + ws * C::B_BYTES);
          if (leader) {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              mma_ss(d, sdesc_sw128(a0 + 32 * k, 16, 1024), sdesc_sw128(b0 + 32 * k, 16, 1024), C::IDESC, (i | k) != 0);
            mma_commit(&hempty[hs]);
            mma_commit(&wempty[ws]);
          }
          __syncwarp();
          if (++hs == C::HS) {
            hs = 0;
            hph ^= 1u;
          }
          if (++ws == C::WS) {
            ws = 0;
            wph ^= 1u;
          }
        }
        if (!ok) break;
        if (leader) mma_commit(&accf[acc]);
      }
      if (leader) mma_commit(drain);  // every MMA issued above completes before TMEM can be released
    }
  } else if (warp < WPROD) {  // ------------------------------------ epilogue: warps 2..9
    const int grp = (warp - 2) >> 2;  // column group
    const int q = warp & 3;           // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;
    const int c_lo = grp * C::CW;
    int it = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      // warp-uniform: the tcgen05.ld below is warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&accf[acc], (it >> 1) & 1, abort, dev_status))) break;
      tc_fence_after();
      float2 s2 = make_float2(0.f, 0.f);
      const uint32_t base = tmem + ((uint32_t)(q * 32) << 16) + acc * DG + c_lo;
#pragma unroll 1
      for (int c0 = 0; c0 < C::CW; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(base + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const int c = c_lo + c0 + j;
          const float2 z = __fadd2_rn(make_float2(__uint_as_float(v[j]), __uint_as_float(v[j + 1])),
                                      *reinterpret_cast<const float2*>(b1s + c));
          s2 = gelu_w_acc2(z, *reinterpret_cast<const float2*>(w2s + c), *reinterpret_cast<const float2*>(hw2s + c), s2);
        }
      }
      float s = s2.x + s2.y;
      tc_fence_before();
      bool ok = true;
      if (grp > 0) {
        part[((grp - 1) * 2 + acc) * BM + row] = s;
        mbar_arrive(&half_ready[acc]);
      } else {
        ok = __all_sync(0xffffffffu, mbar_wait(&half_ready[acc], (it >> 1) & 1, abort, dev_status));
        const long r = (long)tile * BM + row;
#pragma unroll
        for (int g = 1; g < C::NGRP; ++g) s += part[((g - 1) * 2 + acc) * BM + row];
        if (ok && r < n_tok) score[r] = (s + b2) * inv_t;
      }
      // the accumulator (and this buffer's partial sums) is released only once fully consumed
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[acc]);
      if (!ok) break;
    }
  }

  // every MMA has completed before TMEM is released
  if (warp == 1 && !skip) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < 1000000000ull) {
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int DG>
tg_status launch_dg(const void* H, int64_t ldh, int64_t n_tok, int d, const void* W1, const float* b1, const void* w2,
                    float b2, float inv_t, float* score, int32_t* dev_status, cudaStream_t st) {
  using C = Cfg<DG>;
  CUtensorMap tmH, tmW;
  if (!make_tmap_bf16_2d(&tmH, H, (uint64_t)n_tok, (uint64_t)d, (uint64_t)ldh, BM, BK) ||
      !make_tmap_bf16_2d(&tmW, W1, (uint64_t)DG, (uint64_t)d, (uint64_t)d, DG, BK))
    return fail(TG_ERR_CUDA, "tg_score: building the TMA tensor maps failed");
  constexpr int slot = DG == 64 ? ATTR_SCORE64 : (DG == 128 ? ATTR_SCORE128 : ATTR_SCORE256);
  if (attrs_needed(slot)) {
    cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<DG>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return cuda_status(e, "tg_score: cudaFuncSetAttribute");
    // every kernel of the chain asks for the same (all-shared) carveout, so consecutive chain
    // kernels never wait for an SM to drain and reconfigure its L1 / shared-memory split
    e = cudaFuncSetAttribute(score_tc_kernel<DG>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return cuda_status(e, "tg_score: cudaFuncSetAttribute");
    mark_attrs_set(slot);
  }
  const int n_tiles = (int)((n_tok + BM - 1) / BM);
  int ctas = device_sm_count();
  if (ctas > n_tiles) ctas = n_tiles;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(C::NTHREADS);
  cfg.dynamicSmemBytes = (size_t)C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attribute(PDL_SCORE)};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, score_tc_kernel<DG>, tmH, tmW, b1,
                                        static_cast<const __nv_bfloat16*>(w2), b2, inv_t, score, (int)n_tok, d / BK,
                                        n_tiles, dev_status, wait_probe_ns()),
                     "tg_score: score_tc launch");
}

}  // namespace

tg_status launch_score_tc(const void* H, int64_t ldh, int64_t n_tok, int d, const void* W1, const float* b1,
                          const void* w2, float b2, float inv_t, int dg, float* score, int32_t* dev_status,
                          cudaStream_t st) {
  if (dg == 64) return launch_dg<64>(H, ldh, n_tok, d, W1, b1, w2, b2, inv_t, score, dev_status, st);
  if (dg == 128) return launch_dg<128>(H, ldh, n_tok, d, W1, b1, w2, b2, inv_t, score, dev_status, st);
  return launch_dg<256>(H, ldh, n_tok, d, W1, b1, w2, b2, inv_t, score, dev_status, st);
}

}  // namespace tg
