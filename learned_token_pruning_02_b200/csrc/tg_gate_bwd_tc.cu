// Gradients of the gate network's parameters on the 5th-generation tensor cores (bf16 H, W1, w2).
//
// TokenGate paper page (thelatestinai.com), Figure 1(c): the gated attention lets the top-K
// selector learn end to end; aitualizate.com article, section on training the top-K selection.
// With s = (w2 . GELU(W1 h + b1) + b2) / T and the upstream d score of each kept row:
//   z = W1 h + b1,  ds' = dscore / T,  u = ds' w2 * GELU'(z),  q = ds' GELU(z)  (per row, dg values),
//   dW1 = sum_rows u h^T,  db1 = sum_rows u,  dw2 = sum_rows q,  db2 = sum_rows ds'.
//
// Four kernels, deterministic (fixed reduction orders, no atomics), caller workspace:
//   1. gate_zpart_tc: per (128 kept rows, 128 columns of dg, split of d), the split's part of
//      z = H W1^T (M = 128, N = 128, K = d / ks, both operands K-major as stored, fp32 in TMEM),
//      stored transposed in fp32. Splitting K keeps the grid near one CTA per SM with a quarter
//      (ks = 4) of the bytes per CTA that a whole-K tile would load.
//   2. gate_u_kernel (CUDA cores, all SMs): z = the partials in split order + b1, then u and q
//      (zero past M), u^T in bf16 (the next product's A operand) and the 256-row block sums of
//      u, q and ds' (fixed shuffle tree, then the warps in order).
//   3. gate_dw1_tc: per (128 rows of dg, 128 columns of d, split of the kept rows),
//      dW1 = u^T H (M = 128, N = 128, K = kept rows in chunks of 64; H is the N-contiguous B
//      operand). With more than one split each writes a partial block; the fp32 tile leaves
//      through shared memory in row-contiguous runs.
//   4. gate_reduce_tc: the splits' blocks in split order; db1, dw2 and db2 from the block sums in
//      block order.
// u is rounded to bf16 for the second product (its fp32 value feeds db1); the products accumulate
// in fp32. GELU and GELU' share one exponential (erf from Abramowitz & Stegun 7.1.26). Every wait
// is bounded; on a timeout a CTA records TG_DEV_TIMEOUT, drains its copies and products, frees
// TMEM and returns, and the reduction writes no output (given a status word).
#include <cuda_bf16.h>

#include "tg_gate_bwd.cuh"
#include "tg_sm100.cuh"

namespace tg {
namespace {

using namespace sm100;

constexpr int GT = 128;        // rows of a product tile (kept rows in pass 1, rows of dg in pass 2)
constexpr int ZN = 128;        // columns of dg per pass-1 tile
constexpr int GN = 128;        // columns of d per pass-2 tile
constexpr int KCH = 64;        // K elements per pipeline stage (one 128-byte swizzle row)
constexpr int WST = 6;         // pass-2 stages (32 KB each)
constexpr int GTHREADS = 192;  // warp 0: TMA, 1: MMA + TMEM, 2-5: epilogue (TMEM lane quarters 2, 3, 0, 1)
constexpr int MAX_SPLITS = 4;

// GELU(z) = z Phi(z) and GELU'(z) = Phi(z) + z phi(z) together, with erf from Abramowitz &
// Stegun, Handbook of Mathematical Functions, formula 7.1.26: for x >= 0,
// erf(x) = 1 - (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) e^(-x^2), t = 1 / (1 + p x), with
// |error| <= 1.5e-7. At x = |z| / sqrt 2 the factor e^(-x^2) = e^(-z^2 / 2) is the one the normal
// density phi needs too, so one exponential and one reciprocal serve both values (1/sqrt 2 is
// folded into p).
__device__ __forceinline__ void gelu_and_grad(float z, float* g, float* gp) {
  constexpr float kP = (float)(0.3275911 * 0.70710678118654752440);
  constexpr float kA1 = 0.254829592f, kA2 = -0.284496736f, kA3 = 1.421413741f, kA4 = -1.453152027f,
                  kA5 = 1.061405429f;
  const float az = fabsf(z);
  const float e = ex2(-0.72134752044448170368f * z * z);  // e^(-z^2 / 2) = 2^(-z^2 log2(e) / 2)
  float t;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t) : "f"(fmaf(kP, az, 1.f)));
  const float poly = t * fmaf(t, fmaf(t, fmaf(t, fmaf(t, kA5, kA4), kA3), kA2), kA1);
  const float tail = 0.5f * poly * e;  // 1 - Phi(|z|)
  const float Phi = z >= 0.f ? 1.f - tail : tail;
  *g = z * Phi;
  *gp = fmaf(z * 0.39894228040143268f, e, Phi);  // + z phi(z)
}

// Sums v[i] over the 32 lanes for every i (NV a power of two up to 32): afterwards v[0] of lane l
// holds the warp's sum of v[l % NV]. At the step with offset o < NV a lane keeps the half of its
// live values whose index has bit o equal to its own lane's bit o and adds the partner's values
// for that half; the offsets from NV up then add the groups of NV lanes. A fixed order throughout.
template <int NV>
__device__ __forceinline__ void lane_transpose_sum(float (&v)[NV], int lane) {
#pragma unroll
  for (int o = NV / 2; o > 0; o >>= 1) {
    const bool hi = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = hi ? v[i] : v[i + o];
      const float keep = hi ? v[i + o] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
#pragma unroll
  for (int o = NV; o < 32; o <<= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Bounded wait used only while draining after an abort (one second at most).
__device__ __forceinline__ void settle(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity) && globaltimer_ns() - t0 < 1000000000ull) {
  }
}

// The CTA's barriers and TMEM slot sit after the stages.
struct Ctl {
  uint64_t* full;
  uint64_t* empty;
  uint64_t* accdone;
  uint64_t* drain;
  uint64_t* probe;  // test hook: a barrier nothing signals
  uint32_t* tmem_slot;
  volatile int* abort;
};

template <int NS>
__device__ __forceinline__ Ctl ctl_at(uint8_t* p) {
  Ctl c;
  uint64_t* bars = reinterpret_cast<uint64_t*>(p);
  c.full = bars;
  c.empty = bars + NS;
  c.accdone = bars + 2 * NS;
  c.drain = bars + 2 * NS + 1;
  c.probe = bars + 2 * NS + 2;
  c.tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NS + 3);
  c.abort = reinterpret_cast<volatile int*>(c.tmem_slot + 1);
  return c;
}

// Thread 0: the barriers, then the test probe's wait (a no-op unless a test asked for it; it runs
// before any copy or product is issued, so a CTA that then skips its work has nothing in flight).
template <int NS>
__device__ __forceinline__ void ctl_init(const Ctl& c, uint64_t probe_ns, int32_t* dev_status) {
  for (int s = 0; s < NS; ++s) {
    mbar_init(&c.full[s], 1);
    mbar_init(&c.empty[s], 1);
  }
  mbar_init(c.accdone, 1);
  mbar_init(c.drain, 1);
  *c.abort = 0;
  fence_barrier_init();
  wait_probe(c.probe, probe_ns, c.abort, dev_status);
}

// After an abort, the producer waits (bounded) for the copies it issued that nobody consumed.
template <int NS>
__device__ __forceinline__ void drain_copies(const Ctl& c, int issued) {
  for (int k = issued - NS < 0 ? 0 : issued - NS; k < issued; ++k) settle(&c.full[k % NS], (k / NS) & 1);
}

// ------------------------------------------------------------------ 1. z partials per 128 x 128 tile
struct ZCfg {
  static constexpr int A_BYTES = GT * KCH * 2;  // 128 kept rows x 64 columns of H
  static constexpr int B_BYTES = ZN * KCH * 2;  // 128 rows of W1 x 64 columns
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int NS = 6;
  static constexpr int SMEM = 1024 + NS * STAGE + 256;
  static constexpr uint32_t IDESC = idesc_bf16_f32(GT, ZN, false);
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

// grid (Mp / 128, dg / 128, ks): split k takes the columns [k d / ks, (k + 1) d / ks) of H and W1.
// zp: [ks][dg][Mp] fp32, the split's part of z transposed (consecutive lanes store consecutive
// kept rows). Rows past M read zeros and give zero.
__global__ void __launch_bounds__(GTHREADS, 1)
    gate_zpart_tc(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW, int d, int dg,
                  int Mp, float* __restrict__ zp, int32_t* __restrict__ dev_status, uint64_t probe_ns) {
  using C = ZCfg;
  constexpr int NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const Ctl ct = ctl_at<NS>(smem + NS * C::STAGE);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, cb = blockIdx.y, ks = blockIdx.z;
  const int nk = d / (KCH * (int)gridDim.z), kc0 = ks * nk;
  if (threadIdx.x == 0) {
    ctl_init<NS>(ct, probe_ns, dev_status);
    prefetch_tmap(&tmH);
    prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(ct.tmem_slot, ZN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();  // earlier readers of the workspace are done from here on
  const uint32_t tmem = *ct.tmem_slot;
  const bool skip = *ct.abort;  // only the test probe sets it this early
  if (skip) {
  } else if (warp == 0) {  // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      int issued = 0;
      for (int k = 0; k < nk; ++k) {
        const int s = k % NS;
        if (k >= NS && !mbar_wait(&ct.empty[s], ((k / NS) - 1) & 1, ct.abort, dev_status)) break;
        uint8_t* st = smem + s * C::STAGE;
        mbar_arrive_expect_tx(&ct.full[s], C::STAGE);
        tma_load_2d(st, &tmH, (kc0 + k) * KCH, tile * GT, &ct.full[s]);
        tma_load_2d(st + C::A_BYTES, &tmW, (kc0 + k) * KCH, cb * ZN, &ct.full[s]);
        ++issued;
      }
      if (*ct.abort) drain_copies<NS>(ct, issued);
    }
  } else if (warp == 1) {  // -------------------------------------------------------- MMA
    {  // the warp runs the schedule, one elected lane issues
      const bool leader = elect_one();
      bool ok = true;
      for (int k = 0; k < nk; ++k) {
        const int s = k % NS;
        if (!__all_sync(0xffffffffu, mbar_wait(&ct.full[s], (k / NS) & 1, ct.abort, dev_status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a = smem_u32(smem + s * C::STAGE), b = a + C::A_BYTES;
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < KCH / 16; ++kk)
            mma_ss(tmem, sdesc_sw128(a + kk * 32, 16, 1024), sdesc_sw128(b + kk * 32, 16, 1024), C::IDESC,
                   (k > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&ct.empty[s]);
        }
        __syncwarp();
      }
      if (ok && leader) mma_commit(ct.accdone);
      if (leader) {
        mma_commit(ct.drain);
        settle(ct.drain, 0);
      }
      __syncwarp();
    }
  } else {  // ------------------------------------------------------ epilogue: one row per thread
    const int q4 = warp & 3, r = q4 * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    float* dst = zp + ((int64_t)ks * dg + cb * ZN) * Mp + tile * GT + r;
    if (__all_sync(0xffffffffu, mbar_wait(ct.accdone, 0, ct.abort, dev_status))) {
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < ZN; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) __stcg(dst + (int64_t)(c0 + e) * Mp, __uint_as_float(v[e]));
      }
    }
  }
  griddep_launch_dependents();  // after the stores: the u pass's blocks do not wait beside the products
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, ZN);
}

// ------------------------------------------------------------------ 1b. u, q and their column sums
// grid (ceil(Mp / 256), dg / UCOLS), 256 threads: thread t of block x is kept row 256 x + t and
// takes UCOLS = 4 columns of dg. z = the splits' partials added in split order + b1; u and q as
// above (zero past M); u^T in bf16 for every row below Mp. cs: [2 P][dg] + [P] fp32 (P =
// gridDim.x), the block's sums of u (rows [0, P)) and of q (rows [P, 2P)) over its 256 rows, then
// P more values: the block's sum of ds' (entry x, written by the blocks with y == 0). Block sums:
// the 8 values of a thread (u and q of its 4 columns) go through one lane butterfly (lane l ends
// with the warp's sum of value l % 8), ds' through a shuffle tree, then the 8 warps add in order.
// Few columns per thread keep many warps resident: the pass waits on its loads, not on issue.
constexpr int UCOLS = 4;

template <int KS>
__global__ void __launch_bounds__(256) gate_u_kernel(const float* __restrict__ zp, int M, int Mp, int dg,
                                                     const float* __restrict__ b1, const __nv_bfloat16* __restrict__ w2,
                                                     float inv_t, const float* __restrict__ dscore,
                                                     __nv_bfloat16* __restrict__ uT, float* __restrict__ cs) {
  __shared__ float red[8][2 * UCOLS + 1];
  griddep_wait();  // the z partials are complete from here on
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 256 + threadIdx.x, c0 = blockIdx.y * UCOLS, P = gridDim.x;
  const bool valid = t < M, inside = t < Mp;
  const float dsp = valid ? __ldcg(dscore + t) * inv_t : 0.f;
  float v[2 * UCOLS];  // u of the columns, then q
#pragma unroll
  for (int j = 0; j < UCOLS; ++j) {
    float z = inside ? __ldcg(zp + ((int64_t)c0 + j) * Mp + t) : 0.f;
#pragma unroll
    for (int k = 1; k < KS; ++k) z += inside ? __ldcg(zp + ((int64_t)k * dg + c0 + j) * Mp + t) : 0.f;
    v[j] = z;
  }
#pragma unroll
  for (int j = 0; j < UCOLS; ++j) {
    const int c = c0 + j;
    const float z = v[j] + (b1 ? __ldg(b1 + c) : 0.f);
    float g, gp;
    gelu_and_grad(z, &g, &gp);
    const float u = valid ? dsp * __bfloat162float(w2[c]) * gp : 0.f;
    v[j] = u;
    v[UCOLS + j] = valid ? dsp * g : 0.f;
    if (inside) uT[(int64_t)c * Mp + t] = __float2bfloat16_rn(u);
  }
  lane_transpose_sum(v, lane);
  float sd = dsp;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sd += __shfl_xor_sync(0xffffffffu, sd, o);
  if (lane < 2 * UCOLS) red[warp][lane] = v[0];
  if (lane == 0) red[warp][2 * UCOLS] = sd;
  __syncthreads();
  if (threadIdx.x < 2 * UCOLS + 1) {
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) a += red[w][threadIdx.x];
    const int j = threadIdx.x;
    if (j < UCOLS)
      cs[(int64_t)blockIdx.x * dg + c0 + j] = a;
    else if (j < 2 * UCOLS)
      cs[(int64_t)(P + blockIdx.x) * dg + c0 + j - UCOLS] = a;
    else if (blockIdx.y == 0)
      cs[(int64_t)2 * P * dg + blockIdx.x] = a;
  }
  // the next kernel's CTAs take their SMs only now: launched earlier they would sit beside this
  // grid's blocks while it runs
  griddep_launch_dependents();
}

// ------------------------------------------------------------------ 2. dW1 = u^T H, split over rows
struct WCfg {
  static constexpr int A_BYTES = GT * KCH * 2;  // 128 rows of dg x 64 kept rows (u^T)
  static constexpr int B_BOX = KCH * 64 * 2;    // 64 kept rows x 64 columns of d
  static constexpr int B_BYTES = (GN / 64) * B_BOX;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int SMEM = 1024 + WST * STAGE + 256;
  static constexpr uint32_t IDESC = idesc_bf16_f32(GT, GN, true);
  static_assert(WST * STAGE >= GT * GN * 4, "the stages hold the fp32 tile at the end");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

// grid (dg / 128, d / 256, splits); split z takes the 64-row chunks [z cps, min(nchunk, (z+1) cps)).
// out: dW1 [dg][d] (one split) or the partial blocks [splits][dg][d].
__global__ void __launch_bounds__(GTHREADS, 1)
    gate_dw1_tc(const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmHB, int d, int nchunk,
                int cps, float* __restrict__ out, int64_t out_split_stride, int32_t* __restrict__ dev_status,
                uint64_t probe_ns) {
  using C = WCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const Ctl ct = ctl_at<WST>(smem + WST * C::STAGE);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gi = blockIdx.x, nj = blockIdx.y, sp = blockIdx.z;
  const int k0 = sp * cps, nk = min(nchunk, k0 + cps) - k0;  // >= 1 by the plan
  if (threadIdx.x == 0) {
    ctl_init<WST>(ct, probe_ns, dev_status);
    prefetch_tmap(&tmU);
    prefetch_tmap(&tmHB);
  }
  if (warp == 1) {
    tmem_alloc(ct.tmem_slot, GN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();  // u^T of the previous kernel is complete from here on
  const uint32_t tmem = *ct.tmem_slot;
  const bool skip = *ct.abort;  // only the test probe sets it this early
  bool done = false;
  if (skip) {
  } else if (warp == 0) {  // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      int issued = 0;
      for (int k = 0; k < nk; ++k) {
        const int s = k % WST, kc = k0 + k;
        if (k >= WST && !mbar_wait(&ct.empty[s], ((k / WST) - 1) & 1, ct.abort, dev_status)) break;
        uint8_t* st = smem + s * C::STAGE;
        mbar_arrive_expect_tx(&ct.full[s], C::STAGE);
        tma_load_2d(st, &tmU, kc * KCH, gi * GT, &ct.full[s]);
#pragma unroll
        for (int bx = 0; bx < GN / 64; ++bx)
          tma_load_2d(st + C::A_BYTES + bx * C::B_BOX, &tmHB, nj * GN + bx * 64, kc * KCH, &ct.full[s]);
        ++issued;
      }
      if (*ct.abort) drain_copies<WST>(ct, issued);
    }
  } else if (warp == 1) {  // -------------------------------------------------------- MMA
    {  // the warp runs the schedule, one elected lane issues
      const bool leader = elect_one();
      bool ok = true;
      for (int k = 0; k < nk; ++k) {
        const int s = k % WST;
        if (!__all_sync(0xffffffffu, mbar_wait(&ct.full[s], (k / WST) & 1, ct.abort, dev_status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a = smem_u32(smem + s * C::STAGE), b = a + C::A_BYTES;
        // A: 128 rows of u^T x 64 kept rows, K-major. B: 64 kept rows x 256 columns of d as four
        // boxes of 64 columns (N-contiguous; the leading offset steps from box to box), 16 kept
        // rows (2048 bytes) per instruction.
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < KCH / 16; ++kk)
            mma_ss(tmem, sdesc_sw128(a + kk * 32, 16, 1024), sdesc_sw128(b + kk * 2048, C::B_BOX, 1024), C::IDESC,
                   (k > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&ct.empty[s]);
        }
        __syncwarp();
      }
      if (ok && leader) mma_commit(ct.accdone);
      if (leader) {
        mma_commit(ct.drain);
        settle(ct.drain, 0);
      }
      __syncwarp();
    }
  } else {  // ------------------------------------------ epilogue: the tile into shared memory
    const int q4 = warp & 3, r = q4 * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    done = __all_sync(0xffffffffu, mbar_wait(ct.accdone, 0, ct.abort, dev_status));
    if (done) {
      tc_fence_after();
      // fp32 [128][256]; the 16-byte slot x of row r sits at x ^ (r % 8) (conflict-free both ways)
      float4* row = reinterpret_cast<float4*>(smem) + r * (GN / 4);
#pragma unroll 1
      for (int cc = 0; cc < GN; cc += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + cc, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 8; ++i)
          row[((cc >> 2) + i) ^ (r & 7)] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                                       __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
      }
    }
  }
  // every thread takes part; a CTA with any epilogue warp that timed out writes nothing
  const bool all_done = __syncthreads_or(warp >= 2 && !done) == 0;
  griddep_launch_dependents();  // the products are done: the reduction's blocks may start
  if (all_done && warp >= 2) {
    const float4* stg = reinterpret_cast<const float4*>(smem);
    float* dst = out + (int64_t)sp * out_split_stride + (int64_t)gi * GT * d + (int64_t)nj * GN;
#pragma unroll 4
    for (int i = threadIdx.x - 64; i < GT * GN / 4; i += 128) {
      const int row = i / (GN / 4), x = i % (GN / 4);  // a warp stores one row of 512 bytes
      *reinterpret_cast<float4*>(dst + (int64_t)row * d + x * 4) = stg[row * (GN / 4) + (x ^ (row & 7))];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, GN);
}

// ------------------------------------------------------------------ 3. sums in a fixed order
// Threads [0, n_w / 4) with splits > 1: one float4 of dW1 each, the splits' partial blocks added
// in split order (all loads issued before the first add). The blocks after them: one warp per
// column h of dg, db1[h] and dw2[h] from the P block sums of gate_u_kernel (lane l adds rows l,
// l + 32, ... in order; a fixed shuffle tree adds the lanes); warp dg: db2 from the P sums of ds'.
// Nothing is written when the status word holds TG_DEV_TIMEOUT.
__global__ void __launch_bounds__(256) gate_reduce_tc(const float* __restrict__ wpart, int splits, int64_t n_w,
                                                      float* __restrict__ dW1, int nbw, const float* __restrict__ cs,
                                                      int P, int dg, float* __restrict__ db1, float* __restrict__ dw2,
                                                      float* __restrict__ db2, const int32_t* __restrict__ dev_status) {
  griddep_wait();
  if (dev_status && (__ldcg(dev_status) & TG_DEV_TIMEOUT)) return;  // a product gave up: write nothing
  if ((int)blockIdx.x < nbw) {
    const int64_t n4 = n_w / 4, i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n4) return;
    const float4* src = reinterpret_cast<const float4*>(wpart) + i;
    float4 v[MAX_SPLITS];
#pragma unroll
    for (int s = 0; s < MAX_SPLITS; ++s)
      if (s < splits) v[s] = __ldcg(src + s * n4);
    float4 acc = v[0];
#pragma unroll
    for (int s = 1; s < MAX_SPLITS; ++s)
      if (s < splits) {
        acc.x += v[s].x;
        acc.y += v[s].y;
        acc.z += v[s].z;
        acc.w += v[s].w;
      }
    reinterpret_cast<float4*>(dW1)[i] = acc;
    return;
  }
  const int h = ((int)blockIdx.x - nbw) * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (h > dg) return;
  float su = 0.f, sq = 0.f;
  if (h < dg) {
    for (int p = lane; p < P; p += 32) {
      su += __ldcg(cs + (int64_t)p * dg + h);
      sq += __ldcg(cs + (int64_t)(P + p) * dg + h);
    }
  } else {
    for (int p = lane; p < P; p += 32) su += __ldcg(cs + (int64_t)2 * P * dg + p);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    su += __shfl_xor_sync(0xffffffffu, su, o);
    sq += __shfl_xor_sync(0xffffffffu, sq, o);
  }
  if (lane == 0) {
    if (h < dg) {
      if (db1) db1[h] = su;
      if (dw2) dw2[h] = sq;
    } else if (db2) {
      *db2 = su;
    }
  }
}

int64_t al256(int64_t x) { return (x + 255) & ~int64_t(255); }

}  // namespace

bool gate_bwd_tc_shape(int64_t M, int d, int dg) {
  return M >= 1 && M <= INT32_MAX - 256 && dg % GT == 0 && dg >= GT && d % GN == 0 && d >= GN;
}

void gate_bwd_tc_plan(GateBwdPlan& p, int64_t M, int d, int dg, int sms) {
  p.tc = true;
  p.tc_Mp = (int)((M + GT - 1) / GT * GT);
  p.tc_nchunk = (int)((M + KCH - 1) / KCH);
  const int64_t row_tiles = p.tc_Mp / GT, z_tiles = row_tiles * (dg / ZN);
  p.tc_ks = 1;  // split the first product's K while the grid stays within one wave
  while (p.tc_ks < 8 && z_tiles * p.tc_ks * 2 <= sms && d % (KCH * p.tc_ks * 2) == 0) p.tc_ks *= 2;
  p.tc_ublocks = (p.tc_Mp + 255) / 256;
  const int tiles = (dg / GT) * (d / GN);
  int splits = (sms + tiles - 1) / tiles;
  splits = splits < 1 ? 1 : (splits > MAX_SPLITS ? MAX_SPLITS : splits);
  p.tc_cps = (p.tc_nchunk + splits - 1) / splits;
  p.tc_splits = (p.tc_nchunk + p.tc_cps - 1) / p.tc_cps;  // every split has at least one chunk
  // u^T, the block sums, then one region for the z partials and, once they are consumed, the
  // dW1 split partials (the kernels that use them run one after the other on the stream)
  p.tc_off_part = al256((int64_t)p.tc_Mp * dg * 2);
  p.tc_off_big = p.tc_off_part + al256(((int64_t)2 * p.tc_ublocks * dg + p.tc_ublocks) * 4);
  const int64_t zbytes = (int64_t)p.tc_ks * dg * p.tc_Mp * 4;
  const int64_t wbytes = p.tc_splits > 1 ? (int64_t)p.tc_splits * dg * d * 4 : 0;
  p.tc_bytes = p.tc_off_big + al256(zbytes > wbytes ? zbytes : wbytes);
}

tg_status launch_gate_bwd_tc(const void* H, int64_t M, int d, const void* W1, const float* b1, const void* w2,
                             float inv_t, int dg, const float* dscore, float* dW1, float* db1, float* dw2, float* db2,
                             void* ws, const GateBwdPlan& p, int32_t* dev_status, cudaStream_t st) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  __nv_bfloat16* uT = reinterpret_cast<__nv_bfloat16*>(base);
  float* cs = reinterpret_cast<float*>(base + p.tc_off_part);
  float* zp = reinterpret_cast<float*>(base + p.tc_off_big);
  float* wpart = p.tc_splits > 1 ? reinterpret_cast<float*>(base + p.tc_off_big) : dW1;
  CUtensorMap tH, tW, tU, tHB;
  if (!make_tmap_bf16_2d(&tH, H, (uint64_t)M, (uint64_t)d, (uint64_t)d, GT, KCH) ||
      !make_tmap_bf16_2d(&tW, W1, (uint64_t)dg, (uint64_t)d, (uint64_t)d, ZN, KCH) ||
      !make_tmap_bf16_2d(&tU, uT, (uint64_t)dg, (uint64_t)p.tc_Mp, (uint64_t)p.tc_Mp, GT, KCH) ||
      !make_tmap_bf16_2d(&tHB, H, (uint64_t)M, (uint64_t)d, (uint64_t)d, KCH, 64))
    return fail(TG_ERR_CUDA, "tg_gate_mlp_bwd: building the TMA tensor maps failed");
  if (attrs_needed(ATTR_GATE_TC)) {
    const cudaFuncAttribute a = cudaFuncAttributeMaxDynamicSharedMemorySize;
    cudaError_t e = cudaFuncSetAttribute(gate_zpart_tc, a, ZCfg::SMEM);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(gate_dw1_tc, a, WCfg::SMEM);
    if (e != cudaSuccess) return cuda_status(e, "tg_gate_mlp_bwd: cudaFuncSetAttribute");
    mark_attrs_set(ATTR_GATE_TC);
  }
  const uint64_t probe = wait_probe_ns();
  cudaLaunchAttribute pdl[1] = {pdl_attribute(PDL_GATE)};
  cudaLaunchConfig_t c = {};
  c.blockDim = dim3(GTHREADS);
  c.stream = st;
  c.attrs = pdl;
  c.numAttrs = 1;
  c.gridDim = dim3((unsigned)(p.tc_Mp / GT), (unsigned)(dg / ZN), (unsigned)p.tc_ks);
  c.dynamicSmemBytes = (size_t)ZCfg::SMEM;
  cudaError_t e = cudaLaunchKernelEx(&c, gate_zpart_tc, tH, tW, d, dg, p.tc_Mp, zp, dev_status, probe);
  if (e != cudaSuccess) return cuda_status(e, "tg_gate_mlp_bwd: z launch");
  c.gridDim = dim3((unsigned)p.tc_ublocks, (unsigned)(dg / UCOLS));
  c.blockDim = dim3(256);
  c.dynamicSmemBytes = 0;
  auto ku = p.tc_ks == 8 ? gate_u_kernel<8> : p.tc_ks == 4 ? gate_u_kernel<4> : p.tc_ks == 2 ? gate_u_kernel<2>
                                                                                               : gate_u_kernel<1>;
  e = cudaLaunchKernelEx(&c, ku, (const float*)zp, (int)M, p.tc_Mp, dg, b1, static_cast<const __nv_bfloat16*>(w2),
                         inv_t, dscore, uT, cs);
  if (e != cudaSuccess) return cuda_status(e, "tg_gate_mlp_bwd: u launch");
  c.gridDim = dim3((unsigned)(dg / GT), (unsigned)(d / GN), (unsigned)p.tc_splits);
  c.blockDim = dim3(GTHREADS);
  c.dynamicSmemBytes = (size_t)WCfg::SMEM;
  e = cudaLaunchKernelEx(&c, gate_dw1_tc, tU, tHB, d, p.tc_nchunk, p.tc_cps, wpart, (int64_t)dg * d, dev_status,
                         probe);
  if (e != cudaSuccess) return cuda_status(e, "tg_gate_mlp_bwd: dW1 launch");
  const int64_t n_w = (int64_t)dg * d;
  const int nbw = p.tc_splits > 1 ? (int)((n_w / 4 + 255) / 256) : 0;
  c.gridDim = dim3((unsigned)(nbw + (dg + 1 + 7) / 8));
  c.blockDim = dim3(256);
  c.dynamicSmemBytes = 0;
  e = cudaLaunchKernelEx(&c, gate_reduce_tc, (const float*)wpart, p.tc_splits, n_w, dW1, nbw, (const float*)cs,
                         p.tc_ublocks, dg, db1, dw2, db2, (const int32_t*)dev_status);
  return cuda_status(e, "tg_gate_mlp_bwd: reduce launch");
}

}  // namespace tg
