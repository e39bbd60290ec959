// Projection of the kept rows to Q, K and V, with rotary position embedding of Q and K at
// each kept token's original position, on the 5th-generation tensor cores.
//
// The layers above the selection layer process only the kept tokens (aitualizate.com
// TokenGate article, phase 3; thelatestinai.com TokenGate page, Figure 1(a)), at their
// original positions (the position ids the selector writes). The pages give no projection or
// rotary details; the reading taken: Q/K/V = H_kept W^T with one stacked W [(Hq + 2 Hkv) D, d],
// Q and K rotated with rotate-half pairing (i, i + D/2) by angle pos * theta^(-2i/D).
//
// Design (B200, bf16 in, fp32 accumulate), one CTA per SM walking 128- or 256-row x
// 256-column tiles of X = H_kept W^T:
//   * warp 0 streams 128 x 64 slices of H_kept through a 7-deep TMA ring (256 x 64 slices
//     through a 3-deep ring for 256-row tiles), the last warp streams the matching 256 x 64
//     slices of W through a 3-deep ring (all 128-byte swizzle);
//   * one elected lane of warp 1 issues tcgen05.mma M=128 N=256 K=16. With 128-row tiles the
//     two TMEM accumulators are a double buffer, so the epilogue of tile t overlaps the products
//     of tile t+1. Once 128-row tiles would take more than one round of the SMs, a tile is 256
//     rows: both accumulators take one tile, its two 128-row products read every W slice from
//     shared memory once (a third fewer operand bytes per product, and at 2176 kept rows 144
//     tiles in one round instead of 272 in two); the epilogue is no longer overlapped, so it
//     gets twice the warps (16, one set of 8 per 128-row block);
//   * warps 2-9 (2-17 for 256-row tiles) are the epilogue: per TMEM lane quarter and 128-row
//     block two warps, each owning a 128-column half of the tile (one head for D = 128, two for
//     D = 64). For a Q or K head a thread loads columns i and i + D/2 together, rotates the
//     pair, and stores bf16 rows. The angle
//     pos * theta^(-2i/D) reaches about 1e5 radians at 128K-token positions, so it is formed
//     and reduced to [-pi, pi] in double before a fast single-precision sine and cosine.
//   * Every wait is bounded (about 2 s); on a timeout the CTA sets TG_DEV_TIMEOUT, drains its
//     copies and products, frees TMEM and returns.
#include "tg_internal.cuh"
#include "tg_sm100.cuh"

namespace tg {
namespace {

using namespace sm100;

constexpr int BN = 256;  // output columns per tile
constexpr int BK = 64;
constexpr int B_BYTES = BN * BK * 2;       // 32 KB
constexpr int WS = 3;                      // W ring depth
constexpr int TAIL = 1024;
constexpr int TMEM_COLS = 2 * BN;
constexpr uint32_t IDESC = idesc_bf16_f32(128, BN, false);

// A tile is NACC x 128 kept rows by 256 columns, with NACC accumulators of 128 x 256 fp32 in TMEM.
//   NACC = 1: the two accumulators are a double buffer, so a tile's epilogue overlaps the next
//             tile's products (a 7-deep ring of 16 KB H_kept slices);
//   NACC = 2: both hold one tile, whose two 128-row products share every W slice, which cuts the
//             operand bytes per product by a third (a 3-deep ring of 32 KB H_kept slices).
template <int NACC>
struct QCfg {
  static constexpr int BM = 128 * NACC;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int AS = NACC == 1 ? 7 : 3;
  static constexpr int NSET = 2 / NACC;  // accumulator sets in TMEM
  static constexpr int NEPI = 8 * NACC;  // epilogue warps (warps 2..): 8 per 128-row block
  static constexpr int WPROD = 2 + NEPI;  // warp that streams W
  static constexpr int NTHREADS = 32 * (3 + NEPI);
  static constexpr int SMEM = 1024 + AS * A_BYTES + WS * B_BYTES + TAIL;
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

struct QKVParams {
  int M;        // kept rows
  int nk;       // d / 64
  int tiles_n;  // (Hq + 2 Hkv) D / 256
  int tiles;    // tiles_m * tiles_n
  int Hq, Hkv, D;
  int rotate;          // theta > 0
  double inv[64];      // theta^(-2i/D), i < D/2
};

template <int NACC>
__global__ void __launch_bounds__(QCfg<NACC>::NTHREADS, 1)
    qkv_rope_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                    const int32_t* __restrict__ pos, __nv_bfloat16* __restrict__ Qo, __nv_bfloat16* __restrict__ Ko,
                    __nv_bfloat16* __restrict__ Vo, int32_t* __restrict__ dev_status, uint64_t probe_ns,
                    const __grid_constant__ QKVParams p) {
  using C = QCfg<NACC>;
  constexpr int BM = C::BM, AS = C::AS, A_BYTES = C::A_BYTES, NSET = C::NSET, NEPI = C::NEPI, WPROD = C::WPROD;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smem_w = smem + AS * A_BYTES;
  uint8_t* tail = smem_w + WS * B_BYTES;
  uint64_t* afull = reinterpret_cast<uint64_t*>(tail);  // [AS]
  uint64_t* aempty = afull + AS;                        // [AS]
  uint64_t* wfull = aempty + AS;                        // [WS]
  uint64_t* wempty = wfull + WS;                        // [WS]
  uint64_t* accf = wempty + WS;                         // [NSET] accumulator set complete
  uint64_t* acce = accf + 2;                            // [NSET] accumulator set consumed
  uint64_t* drain = acce + 2;
  uint64_t* probe = drain + 1;  // test hook: a barrier nothing signals
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(probe + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < AS; ++s) {
      mbar_init(&afull[s], 1);
      mbar_init(&aempty[s], 1);
    }
    for (int s = 0; s < WS; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 1);
    }
    for (int a = 0; a < NSET; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], NEPI);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_barrier_init();
    wait_probe(probe, probe_ns, abort, dev_status);  // no-op unless a test asked for it
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  griddep_launch_dependents();  // the next kernel may start its prologue
  griddep_wait();               // the previous kernel's results are visible from here on
  tc_fence_before();
  __syncthreads();  // barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nk = p.nk;
  const bool skip = *abort;  // only the test probe sets it this early: nothing was issued

  if (skip) {
  } else if (warp == 0 || warp == WPROD) {
    if (lane == 0) {  // ------------------------------------ TMA producers: H_kept (warp 0), W (warp 10)
      const bool is_a = warp == 0;
      const int depth = is_a ? AS : WS;
      uint64_t* full = is_a ? afull : wfull;
      uint64_t* empty = is_a ? aempty : wempty;
      const int bytes = is_a ? A_BYTES : B_BYTES;
      uint8_t* ring = is_a ? smem : smem_w;
      const CUtensorMap* tm = is_a ? &tmA : &tmW;
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      for (int tile = blockIdx.x; tile < p.tiles && !*abort; tile += gridDim.x) {
        const int y = is_a ? (tile / p.tiles_n) * BM : (tile % p.tiles_n) * BN;
        for (int kb = 0; kb < nk; ++kb) {
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
    {  // -------------------------- MMA issuer: the warp runs the schedule, one elected lane issues
      const bool leader = elect_one();
      int as = 0, ws = 0;
      uint32_t aph = 0, wph = 0;
      int it = 0;
      for (int tile = blockIdx.x; tile < p.tiles && !*abort; tile += gridDim.x, ++it) {
        const int set = it % NSET;
        if (!__all_sync(0xffffffffu, mbar_wait(&acce[set], ((it / NSET) & 1) ^ 1u, abort, dev_status))) break;
        tc_fence_after();
        const uint32_t d = tmem + set * NACC * BN;
        bool ok = true;
        for (int i = 0; i < nk; ++i) {
          if (!__all_sync(0xffffffffu, mbar_wait(&afull[as], aph, abort, dev_status) &&
                                           mbar_wait(&wfull[ws], wph, abort, dev_status))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + as * A_BYTES);
          const uint32_t b0 = smem_u32(smem_w + ws * B_BYTES);
          if (leader) {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {
              const uint64_t bd = sdesc_sw128(b0 + 32 * k, 16, 1024);
#pragma unroll
              for (int a = 0; a < NACC; ++a)  // rows 128a..128a+127 of the slice start 16 KB apart
                mma_ss(d + a * BN, sdesc_sw128(a0 + a * (128 * 128) + 32 * k, 16, 1024), bd, IDESC, (i | k) != 0);
            }
            mma_commit(&aempty[as]);
            mma_commit(&wempty[ws]);
          }
          __syncwarp();
          if (++as == AS) {
            as = 0;
            aph ^= 1u;
          }
          if (++ws == WS) {
            ws = 0;
            wph ^= 1u;
          }
        }
        if (!ok) break;
        if (leader) mma_commit(&accf[set]);
        __syncwarp();
      }
      if (leader) mma_commit(drain);  // every product issued above completes before TMEM can be released
      __syncwarp();
    }
  } else if (warp < WPROD) {  // ------------------------------------ epilogue: warps 2..WPROD-1
    const int half = ((warp - 2) >> 2) & 1;  // which 128-column half of the tile
    const int ablk = (warp - 2) >> 3;        // which 128-row block of the tile
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;
    const int D = p.D;
    constexpr double kTwoPi = 6.283185307179586476925286766559;
    int it = 0;
    for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++it) {
      const int set = it % NSET;
      // warp-uniform: the tcgen05.ld below is warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&accf[set], (it / NSET) & 1, abort, dev_status))) break;
      tc_fence_after();
      {
      const int a = ablk;                // the tile's 128-row block of this warp
      const int acc = set * NACC + a;    // accumulator in TMEM
      const int gm = (tile / p.tiles_n) * BM + a * 128 + r;
      const bool valid = gm < p.M;
      const double pr = (valid && p.rotate) ? (double)pos[gm] : 0.0;  // pos may be NULL without rotation
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + acc * BN + half * 128;
      const int cbase = (tile % p.tiles_n) * BN + half * 128;  // first output column of this half
#pragma unroll 1
      for (int hh = 0; hh < 128 / D; ++hh) {
        const int gcol = cbase + hh * D;
        int head;
        __nv_bfloat16* out;
        bool rot = p.rotate != 0;
        if (gcol < p.Hq * D) {
          head = gcol / D;
          out = Qo + ((int64_t)gm * p.Hq + head) * D;
        } else if (gcol < (p.Hq + p.Hkv) * D) {
          head = (gcol - p.Hq * D) / D;
          out = Ko + ((int64_t)gm * p.Hkv + head) * D;
        } else {
          head = (gcol - (p.Hq + p.Hkv) * D) / D;
          out = Vo + ((int64_t)gm * p.Hkv + head) * D;
          rot = false;
        }
#pragma unroll 1
        for (int c0 = 0; c0 < D / 2; c0 += 32) {
          uint32_t lo[32], hi[32];
          tmem_ld32(tbase + hh * D + c0, lo);
          tmem_ld32(tbase + hh * D + D / 2 + c0, hi);
          tmem_wait_ld();
          uint32_t plo[16], phi[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            float y[2][2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float x1 = __uint_as_float(lo[j + e]), x2 = __uint_as_float(hi[j + e]);
              if (rot) {
                const double a = pr * p.inv[c0 + j + e];
                const float ar = (float)fma(-rint(a * (1.0 / kTwoPi)), kTwoPi, a);  // in [-pi, pi]
                float sn, cs;
                __sincosf(ar, &sn, &cs);
                y[0][e] = x1 * cs - x2 * sn;
                y[1][e] = x2 * cs + x1 * sn;
              } else {
                y[0][e] = x1;
                y[1][e] = x2;
              }
            }
            __nv_bfloat162 a2 = __floats2bfloat162_rn(y[0][0], y[0][1]);
            __nv_bfloat162 b2 = __floats2bfloat162_rn(y[1][0], y[1][1]);
            plo[j >> 1] = *reinterpret_cast<uint32_t*>(&a2);
            phi[j >> 1] = *reinterpret_cast<uint32_t*>(&b2);
          }
          if (valid) {
            uint4* dl = reinterpret_cast<uint4*>(out + c0);
            uint4* dh = reinterpret_cast<uint4*>(out + D / 2 + c0);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              dl[v] = make_uint4(plo[4 * v], plo[4 * v + 1], plo[4 * v + 2], plo[4 * v + 3]);
              dh[v] = make_uint4(phi[4 * v], phi[4 * v + 1], phi[4 * v + 2], phi[4 * v + 3]);
            }
          }
        }
      }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[set]);  // the accumulators may take the next tile
    }
  }

  // every product has completed before TMEM is released
  if (warp == 1 && !skip) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < 1000000000ull) {
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

template <int NACC>
tg_status launch_qkv_nacc(const void* Hk, int64_t M, int d, const void* W, const int32_t* pos, int N,
                          QKVParams& p, void* Q, void* K, void* V, int32_t* dev_status, cudaStream_t st) {
  using C = QCfg<NACC>;
  p.tiles = (int)((M + C::BM - 1) / C::BM) * p.tiles_n;
  CUtensorMap tmA, tmW;
  if (!make_tmap_bf16_2d(&tmA, Hk, (uint64_t)M, (uint64_t)d, (uint64_t)d, C::BM, BK) ||
      !make_tmap_bf16_2d(&tmW, W, (uint64_t)N, (uint64_t)d, (uint64_t)d, BN, BK))
    return fail(TG_ERR_CUDA, "tg_qkv_rope: building the TMA tensor maps failed");
  const int slot = NACC == 1 ? ATTR_QKV : ATTR_QKV2;
  if (attrs_needed(slot)) {
    cudaError_t e = cudaFuncSetAttribute(qkv_rope_kernel<NACC>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return cuda_status(e, "tg_qkv_rope: cudaFuncSetAttribute");
    mark_attrs_set(slot);
  }
  int ctas = device_sm_count();
  if (ctas > p.tiles) ctas = p.tiles;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(C::NTHREADS);
  cfg.dynamicSmemBytes = (size_t)C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attribute(PDL_QKV)};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, qkv_rope_kernel<NACC>, tmA, tmW, pos, static_cast<__nv_bfloat16*>(Q),
                                        static_cast<__nv_bfloat16*>(K), static_cast<__nv_bfloat16*>(V), dev_status,
                                        wait_probe_ns(), p),
                     "tg_qkv_rope: launch");
}

}  // namespace

tg_status launch_qkv_rope(const void* Hk, int64_t M, int d, const void* W, const int32_t* pos, int Hq, int Hkv,
                          int D, float theta, void* Q, void* K, void* V, int32_t* dev_status, cudaStream_t st) {
  const int N = (Hq + 2 * Hkv) * D;
  QKVParams p = {};
  p.M = (int)M;
  p.nk = d / BK;
  p.tiles_n = N / BN;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.D = D;
  p.rotate = theta > 0.f ? 1 : 0;
  for (int i = 0; i < D / 2; ++i) p.inv[i] = p.rotate ? pow((double)theta, -2.0 * i / D) : 0.0;
  const int64_t tiles128 = (M + 127) / 128 * p.tiles_n;
  if (tiles128 == 0) return TG_OK;
  // 256-row tiles once 128-row tiles would take more than one round of the SMs: fewer operand
  // bytes per product; below that, 128-row tiles keep more SMs busy.
  if (tiles128 > device_sm_count()) return launch_qkv_nacc<2>(Hk, M, d, W, pos, N, p, Q, K, V, dev_status, st);
  return launch_qkv_nacc<1>(Hk, M, d, W, pos, N, p, Q, K, V, dev_status, st);
}

}  // namespace tg
