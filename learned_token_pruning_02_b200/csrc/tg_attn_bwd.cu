// Gradients of the token-gated causal attention: dQ, dK, dV, d log g and the score gradient.
//
// TokenGate paper page (thelatestinai.com), Figure 1(c): the gated attention is what lets the
// top-K selector train end to end; aitualizate.com article ("Cómo consigue entrenar una
// selección top-K"): the score enters as a bias on the attention logits, so the selector's
// gradient is that of an additive logit bias. For sequence b, head h, KV head h / (Hq / Hkv),
// with S = scale Q K^T + gain_h log g^T (causal on positions) and P = exp(S - lse):
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - rowsum(dO * O)),
//   dQ = scale dS K,  dK = scale dS^T Q,  d log g_j = sum_h gain_h sum_i dS_ij,
//   d score_j = d log g_j * (1 - g_j) = d log g_j * -expm1(log g_j)   (g = sigmoid(score)).
//
// Design (B200; no workspace, no atomics, so the results are deterministic). f32 tensors run
// on the CUDA cores in fp32 (the kernels below); bf16 tensors run their products on the
// tensor cores (the warp-level MMA kernels further down), with the same work split:
//   * attn_bwd_dkdv: one CTA per 32-key tile, in a cluster whose CTAs split the KV heads.
//     K and V of the tile stay in shared memory. The CTA walks the query tiles at or below
//     the diagonal for each query head of its KV group. dK and dV accumulate in registers,
//     32 keys x D over 256 threads. The per-key d log g partials of the cluster's CTAs are
//     added in rank order through distributed shared memory.
//   * attn_bwd_dq: one CTA per (32-row query tile, head), walking the key tiles up to the
//     diagonal; dQ accumulates in registers.
//   Both recompute S and dP for each tile pair from 32 x D fp32 tiles in shared memory (rows
//   padded by 4 floats so that 8 consecutive rows fall in distinct banks). Half of the
//   threads form S = Q K^T and the other half dP = dO V^T, each thread a 2 x 4 block.
//   rowsum(dO * O) is formed per query tile from dO and the forward's O.
//   Tiles are visited heaviest first (key tile 0 has the most query tiles below it; the last
//   query tile has the most keys).
#include <climits>
#include <cooperative_groups.h>
#include <math.h>

#include "tg_attn_bwd.cuh"
#include "tg_sm100.cuh"

namespace cg = cooperative_groups;

namespace tg {
namespace {

// A key whose gate value is exactly 0 (log g = -inf) is masked for every head gain (gain * -inf
// would give NaN for a zero gain), as in the forward.
__device__ __forceinline__ float key_bias(float gain, float lg) { return lg == -INFINITY ? -INFINITY : gain * lg; }
// A query row whose visible keys are all masked has lse = -inf in the forward; reading it as +inf
// makes every weight exp(s - lse) of the row 0 instead of NaN.
__device__ __forceinline__ float lse_or_inf(float l) { return l == -INFINITY ? INFINITY : l; }

constexpr int BT = 32;    // rows per tile (queries or keys)
constexpr int NT = 256;   // threads per CTA
constexpr int MAXC = 8;   // CTAs per cluster (KV heads split over them)

struct BwdParams {
  AttnSeq s[kMaxSeqPerLaunch];
  int tiles[kMaxSeqPerLaunch + 1];  // prefix sums of ceil(m / BT)
  int nseq;
  int C;  // CTAs per cluster of the dK/dV kernel
};

template <int D>
struct Smem {
  static constexpr int SD = D + 4;  // padded row stride in floats
  static constexpr int SS = BT + 1;
  static constexpr int TILE = BT * SD;
  // K, V, Q, dO tiles; S/P and dP/dS tiles; per-row and per-key vectors
  static constexpr int FLOATS = 4 * TILE + 2 * BT * SS + 6 * BT;
  static constexpr int BYTES = FLOATS * 4;
};

// rows [0, nvalid) of a 32-row f32 tile (row r at src + r * stride elements) into shared rows
// of stride SD; rows past nvalid become zeros
template <typename T, int D>
__device__ __forceinline__ void load_tile(const T* __restrict__ src, int64_t stride, int nvalid, float* dst) {
  static_assert(sizeof(T) == 4, "the CUDA-core kernels take f32 tensors");
  constexpr int SD = Smem<D>::SD, VPR = D / 4;
  for (int v = threadIdx.x; v < BT * VPR; v += NT) {
    const int r = v / VPR, c = (v % VPR) * 4;
    const float4 x = r < nvalid ? __ldg(reinterpret_cast<const float4*>(src + r * stride + c))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<float4*>(dst + r * SD + c) = x;
  }
}

__device__ __forceinline__ float ld1(const float* p) { return __ldg(p); }

// rowsum(dO * O) for the 32 rows of a query tile: warp w takes rows 4w .. 4w + 3; O is read from
// global memory (row r at O + r * stride), dO from its shared tile
template <typename T, int D>
__device__ __forceinline__ void row_dot_dO_O(const T* __restrict__ O, int64_t stride, int nvalid, const float* dOs,
                                             float* dv) {
  constexpr int SD = Smem<D>::SD;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int rr = 0; rr < BT / (NT / 32); ++rr) {
    const int r = w * (BT / (NT / 32)) + rr;
    float s = 0.f;
    if (r < nvalid) {
#pragma unroll
      for (int c = 0; c < D / 32; ++c) s = fmaf(dOs[r * SD + c * 32 + lane], ld1(O + r * stride + c * 32 + lane), s);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) dv[r] = s;
  }
}

// S = Qs Ks^T (threads 0-127) and dP = dOs Vs^T (threads 128-255) for one 32 x 32 tile pair,
// raw (unscaled, no bias), into Ss and dPs [32][33]. Thread u of a half owns queries
// {u/8, u/8 + 16} and keys {u%8 + 8c}.
template <int D>
__device__ __forceinline__ void products(const float* Qs, const float* Ks, const float* dOs, const float* Vs,
                                         float* Ss, float* dPs) {
  constexpr int SD = Smem<D>::SD, SS = Smem<D>::SS;
  const int half = threadIdx.x >> 7, u = threadIdx.x & 127;
  const int qy = u >> 3, kx = u & 7;
  const float* A = half ? dOs : Qs;
  const float* Bm = half ? Vs : Ks;
  float acc[2][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
#pragma unroll 4
  for (int d = 0; d < D; d += 4) {
    const float4 a0 = *reinterpret_cast<const float4*>(A + qy * SD + d);
    const float4 a1 = *reinterpret_cast<const float4*>(A + (qy + 16) * SD + d);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float4 b = *reinterpret_cast<const float4*>(Bm + (kx + 8 * c) * SD + d);
      acc[0][c] = fmaf(a0.x, b.x, fmaf(a0.y, b.y, fmaf(a0.z, b.z, fmaf(a0.w, b.w, acc[0][c]))));
      acc[1][c] = fmaf(a1.x, b.x, fmaf(a1.y, b.y, fmaf(a1.z, b.z, fmaf(a1.w, b.w, acc[1][c]))));
    }
  }
  float* out = half ? dPs : Ss;
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) out[(qy + 16 * a) * SS + kx + 8 * c] = acc[a][c];
}

// In place: Ss <- P = exp(scale S + bias_j - lse_i) where key j is visible to query i (same
// sequence, pos_j <= pos_i), else 0; dPs <- dS = P (dP - rowsum(dO * O)_i).
template <int D>
__device__ __forceinline__ void softmax_grad(float* Ss, float* dPs, float scale, const float* bias, const float* lse,
                                             const float* dv, const int* posq, const int* posk) {
  constexpr int SS = Smem<D>::SS;
#pragma unroll
  for (int e = 0; e < BT * BT / NT; ++e) {
    const int idx = threadIdx.x + e * NT;
    const int qi = idx >> 5, kj = idx & 31;
    const bool vis = posk[kj] <= posq[qi];  // invalid rows carry posq = INT_MIN, invalid keys posk = INT_MAX
    const float p = vis ? expf(fmaf(scale, Ss[qi * SS + kj], bias[kj] - lse[qi])) : 0.f;
    Ss[qi * SS + kj] = p;
    dPs[qi * SS + kj] = p * (dPs[qi * SS + kj] - dv[qi]);
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(NT, 2)
    attn_bwd_dkdv_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
                         const T* __restrict__ O, const T* __restrict__ dO, const float* __restrict__ logg,
                         const float* __restrict__ gain, const int32_t* __restrict__ pos,
                         const float* __restrict__ lse, float scale, int Hq, int Hkv, int64_t m_tot,
                         float* __restrict__ dK, float* __restrict__ dV, float* __restrict__ dlogg,
                         float* __restrict__ dscore, const __grid_constant__ BwdParams p) {
  using S_ = Smem<D>;
  constexpr int SD = S_::SD, SS = S_::SS, EPT = D / 32;  // float4 chunks per thread per row
  extern __shared__ __align__(16) float sm[];
  float* Ks = sm;
  float* Vs = Ks + S_::TILE;
  float* Qs = Vs + S_::TILE;
  float* dOs = Qs + S_::TILE;
  float* Ss = dOs + S_::TILE;
  float* dPs = Ss + BT * SS;
  float* bias = dPs + BT * SS;
  float* lse_s = bias + BT;
  float* dv = lse_s + BT;
  float* dl_s = dv + BT;
  int* posq = reinterpret_cast<int*>(dl_s + BT);
  int* posk = posq + BT;

  const int C = p.C;
  const int unit = blockIdx.x / C, rank = blockIdx.x % C;
  int b = 0;
  while (b + 1 < p.nseq && unit >= p.tiles[b + 1]) ++b;
  const AttnSeq sq = p.s[b];
  const int nt = p.tiles[b + 1] - p.tiles[b];
  const int t = unit - p.tiles[b];  // key tile: tile 0 has the most query tiles below it
  const int k0 = t * BT;
  const int kvalid = min(BT, sq.m - k0);
  const int G = Hq / Hkv;
  const int tid = threadIdx.x;
  const int kk = tid >> 3, l8 = tid & 7;  // update phase: key kk, dims c * 32 + l8 * 4 + 0..3

  if (tid < BT) posk[tid] = tid < kvalid ? pos[sq.off + k0 + tid] : INT_MAX;
  float dl = 0.f;
  for (int kvh = rank; kvh < Hkv; kvh += C) {
    __syncthreads();  // the previous KV head's readers are done with Ks and Vs
    load_tile<T, D>(K + ((int64_t)(sq.off + k0) * Hkv + kvh) * D, (int64_t)Hkv * D, kvalid, Ks);
    load_tile<T, D>(V + ((int64_t)(sq.off + k0) * Hkv + kvh) * D, (int64_t)Hkv * D, kvalid, Vs);
    float4 aK[EPT], aV[EPT];
#pragma unroll
    for (int c = 0; c < EPT; ++c) aK[c] = aV[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int hh = 0; hh < G; ++hh) {
      const int h = kvh * G + hh;
      const float gh = gain ? __ldg(gain + h) : 1.f;
      for (int qt = t; qt < nt; ++qt) {
        const int q0 = qt * BT;
        const int qvalid = min(BT, sq.m - q0);
        __syncthreads();  // the previous tile's readers are done with Qs, dOs, Ss, dPs, bias
        if (tid < BT) {
          bias[tid] = (logg && tid < kvalid) ? key_bias(gh, __ldg(logg + sq.off + k0 + tid)) : 0.f;
          posq[tid] = tid < qvalid ? pos[sq.off + q0 + tid] : INT_MIN;
          lse_s[tid] = tid < qvalid ? lse_or_inf(__ldg(lse + (int64_t)h * m_tot + sq.off + q0 + tid)) : 0.f;
        }
        const int64_t qrow = ((int64_t)(sq.off + q0) * Hq + h) * D;
        load_tile<T, D>(Q + qrow, (int64_t)Hq * D, qvalid, Qs);
        load_tile<T, D>(dO + qrow, (int64_t)Hq * D, qvalid, dOs);
        __syncthreads();
        row_dot_dO_O<T, D>(O + qrow, (int64_t)Hq * D, qvalid, dOs, dv);
        products<D>(Qs, Ks, dOs, Vs, Ss, dPs);
        __syncthreads();
        softmax_grad<D>(Ss, dPs, scale, bias, lse_s, dv, posq, posk);
        __syncthreads();
#pragma unroll 4
        for (int i = 0; i < BT; ++i) {
          const float pv = Ss[i * SS + kk], dsv = dPs[i * SS + kk];
#pragma unroll
          for (int c = 0; c < EPT; ++c) {
            const float4 o = *reinterpret_cast<const float4*>(dOs + i * SD + c * 32 + l8 * 4);
            const float4 q = *reinterpret_cast<const float4*>(Qs + i * SD + c * 32 + l8 * 4);
            aV[c].x = fmaf(pv, o.x, aV[c].x);
            aV[c].y = fmaf(pv, o.y, aV[c].y);
            aV[c].z = fmaf(pv, o.z, aV[c].z);
            aV[c].w = fmaf(pv, o.w, aV[c].w);
            aK[c].x = fmaf(dsv, q.x, aK[c].x);
            aK[c].y = fmaf(dsv, q.y, aK[c].y);
            aK[c].z = fmaf(dsv, q.z, aK[c].z);
            aK[c].w = fmaf(dsv, q.w, aK[c].w);
          }
          if (l8 == 0) dl = fmaf(gh, dsv, dl);
        }
      }
    }
    if (kk < kvalid) {
      const int64_t row = ((int64_t)(sq.off + k0 + kk) * Hkv + kvh) * D;
#pragma unroll
      for (int c = 0; c < EPT; ++c) {
        const float4 k4 = make_float4(scale * aK[c].x, scale * aK[c].y, scale * aK[c].z, scale * aK[c].w);
        *reinterpret_cast<float4*>(dK + row + c * 32 + l8 * 4) = k4;
        *reinterpret_cast<float4*>(dV + row + c * 32 + l8 * 4) = aV[c];
      }
    }
  }
  // d log g of the tile's keys: this CTA's KV heads, then the cluster's CTAs in rank order
  if (l8 == 0) dl_s[kk] = dl;
  if (C > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0 && tid < kvalid && (dlogg || dscore)) {
      float tot = 0.f;
      for (int r = 0; r < C; ++r) tot += cluster.map_shared_rank(dl_s, r)[tid];
      const int64_t row = sq.off + k0 + tid;
      if (dlogg) dlogg[row] = tot;
      if (dscore) dscore[row] = tot * -expm1f(__ldg(logg + row));
    }
    cluster.sync();  // no CTA leaves while rank 0 may still read its partials
  } else {
    __syncthreads();
    if (tid < kvalid && (dlogg || dscore)) {
      const float tot = dl_s[tid];
      const int64_t row = sq.off + k0 + tid;
      if (dlogg) dlogg[row] = tot;
      if (dscore) dscore[row] = tot * -expm1f(__ldg(logg + row));
    }
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(NT, 2)
    attn_bwd_dq_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
                       const T* __restrict__ O, const T* __restrict__ dO, const float* __restrict__ logg,
                       const float* __restrict__ gain, const int32_t* __restrict__ pos, const float* __restrict__ lse,
                       float scale, int Hq, int Hkv, int64_t m_tot, float* __restrict__ dQ,
                       int32_t* __restrict__ dev_status, const __grid_constant__ BwdParams p) {
  using S_ = Smem<D>;
  constexpr int SD = S_::SD, SS = S_::SS, EPT = D / 32;
  extern __shared__ __align__(16) float sm[];
  float* Ks = sm;
  float* Vs = Ks + S_::TILE;
  float* Qs = Vs + S_::TILE;
  float* dOs = Qs + S_::TILE;
  float* Ss = dOs + S_::TILE;
  float* dPs = Ss + BT * SS;
  float* bias = dPs + BT * SS;
  float* lse_s = bias + BT;
  float* dv = lse_s + BT;
  int* posq = reinterpret_cast<int*>(dv + 2 * BT);
  int* posk = posq + BT;

  const int unit = blockIdx.x, h = blockIdx.y;
  int b = 0;
  while (b + 1 < p.nseq && unit >= p.tiles[b + 1]) ++b;
  const AttnSeq sq = p.s[b];
  const int nt = p.tiles[b + 1] - p.tiles[b];
  const int t = nt - 1 - (unit - p.tiles[b]);  // query tile: the last one has the most keys
  const int q0 = t * BT;
  const int qvalid = min(BT, sq.m - q0);
  const int kvh = h / (Hq / Hkv);
  const float gh = gain ? __ldg(gain + h) : 1.f;
  const int tid = threadIdx.x;
  const int qi = tid >> 3, l8 = tid & 7;  // update phase: query row qi, dims c * 32 + l8 * 4 + 0..3

  if (tid < BT) {
    const bool ok = tid < qvalid;
    posq[tid] = ok ? pos[sq.off + q0 + tid] : INT_MIN;
    lse_s[tid] = ok ? lse_or_inf(__ldg(lse + (int64_t)h * m_tot + sq.off + q0 + tid)) : 0.f;
    // the positions must rise strictly inside a sequence (row order is the causal order)
    if (ok && h == 0 && q0 + tid > 0 && dev_status && pos[sq.off + q0 + tid - 1] >= posq[tid])
      atomicOr(dev_status, TG_DEV_POS_NOT_ASCENDING);
  }
  const int64_t qrow = ((int64_t)(sq.off + q0) * Hq + h) * D;
  load_tile<T, D>(Q + qrow, (int64_t)Hq * D, qvalid, Qs);
  load_tile<T, D>(dO + qrow, (int64_t)Hq * D, qvalid, dOs);
  __syncthreads();
  row_dot_dO_O<T, D>(O + qrow, (int64_t)Hq * D, qvalid, dOs, dv);
  float4 aQ[EPT];
#pragma unroll
  for (int c = 0; c < EPT; ++c) aQ[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int kt = 0; kt <= t; ++kt) {
    const int k0 = kt * BT;
    const int kvalid = min(BT, sq.m - k0);
    __syncthreads();  // the previous key tile's readers are done with Ks, Vs, Ss, dPs, bias
    if (tid < BT) {
      const bool ok = tid < kvalid;
      bias[tid] = (logg && ok) ? key_bias(gh, __ldg(logg + sq.off + k0 + tid)) : 0.f;
      posk[tid] = ok ? pos[sq.off + k0 + tid] : INT_MAX;
    }
    load_tile<T, D>(K + ((int64_t)(sq.off + k0) * Hkv + kvh) * D, (int64_t)Hkv * D, kvalid, Ks);
    load_tile<T, D>(V + ((int64_t)(sq.off + k0) * Hkv + kvh) * D, (int64_t)Hkv * D, kvalid, Vs);
    __syncthreads();
    products<D>(Qs, Ks, dOs, Vs, Ss, dPs);
    __syncthreads();
    softmax_grad<D>(Ss, dPs, scale, bias, lse_s, dv, posq, posk);
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < BT; ++k) {
      const float dsv = dPs[qi * SS + k];
#pragma unroll
      for (int c = 0; c < EPT; ++c) {
        const float4 kv = *reinterpret_cast<const float4*>(Ks + k * SD + c * 32 + l8 * 4);
        aQ[c].x = fmaf(dsv, kv.x, aQ[c].x);
        aQ[c].y = fmaf(dsv, kv.y, aQ[c].y);
        aQ[c].z = fmaf(dsv, kv.z, aQ[c].z);
        aQ[c].w = fmaf(dsv, kv.w, aQ[c].w);
      }
    }
  }
  if (qi < qvalid) {
    float* dst = dQ + ((int64_t)(sq.off + q0 + qi) * Hq + h) * D;
#pragma unroll
    for (int c = 0; c < EPT; ++c)
      *reinterpret_cast<float4*>(dst + c * 32 + l8 * 4) =
          make_float4(scale * aQ[c].x, scale * aQ[c].y, scale * aQ[c].z, scale * aQ[c].w);
  }
}

// ---------------------------------------------------------------- bf16: warp-level MMA kernels
//
// The bf16 path runs its five products on the tensor cores with warp-level mma.sync m16n8k16
// (bf16 in, fp32 accumulate). Fragment layouts (PTX ISA, mma.m16n8k16 with .bf16): lane l,
// g = l / 4, t = l % 4; A (16 x 16, row-major) regs {row g, cols 2t..2t+1}, {row g+8, cols
// 2t..}, {row g, cols 2t+8..}, {row g+8, cols 2t+8..}; B (16 x 8) regs {k 2t..2t+1, n g},
// {k 2t+8.., n g}; C (16 x 8) {row g, cols 2t, 2t+1}, {row g+8, cols 2t, 2t+1}. Two adjacent
// C tiles of one product therefore form the A fragment of the next product with those columns
// as its k dimension, so P and dS never leave registers. Operands are bf16 tiles in shared
// memory, rows padded by 16 bytes so the 8 row addresses of one 8 x 8 ldmatrix fall in
// distinct banks; a transposed B (k along rows of the stored tile) comes from ldmatrix.trans.
// P and dS are rounded to bf16 for the products that consume them, as the forward does with P.
//
//   attn_bwd_dkdv_mma: 64-key tile per CTA, clustered over the KV heads like the CUDA-core
//     kernel. One or two warp groups of 4 warps x 16 keys; with two, each takes every other
//     query head of the KV group. Per 32-query step: S^T = K Q^T and dP^T = V dO^T
//     (16 x 32 per warp), then P^T and dS^T in registers, then dV += P^T dO and
//     dK += dS^T Q (16 x D per warp).
//   attn_bwd_dq_mma: 64-query tile per CTA (4 warps x 16 rows) and head. Per 32-key step:
//     S = Q K^T, dP = dO V^T, dS in registers, dQ += dS K.
//   The streamed tiles (and their per-row vectors) are double-buffered with cp.async, so the
//   next step's copies fly while the current step computes.

constexpr int MT = 64;   // rows of a CTA's own tile (keys in dkdv, queries in dq)
constexpr int ST = 32;   // rows of the streamed tile (queries in dkdv, keys in dq)
constexpr int NTM = 128;  // 4 warps

template <int D>
struct MSmem {
  static constexpr int SH = D + 8;  // padded row stride in bf16 elements (16-byte pad)
  static constexpr int OWN = MT * SH, STR = ST * SH;
  // dK/dV kernel: two own tiles, two buffers of three streamed tiles (Q, dO, O), then vectors;
  // dQ kernel: two own tiles, two buffers of two streamed tiles (K, V), then vectors
  static constexpr int VEC = 6 * MT * 4;  // up to 6 vectors of 64 32-bit values
  // dK/dV kernel with NWG warp groups: each group has its own two buffers and 5 vectors of 32
  static constexpr int bytes_dkdv(int nwg) { return (2 * OWN + nwg * 6 * STR) * 2 + (nwg * 5 * ST + MT) * 4; }
  static constexpr int BYTES_DQ = (2 * OWN + 4 * STR) * 2 + VEC;
};

// 16-byte and 4-byte asynchronous copies global -> shared; a copy with ok == false reads
// nothing and writes zeros (src must still be a valid address)
__device__ __forceinline__ void cp16(void* dst, const void* src, bool ok) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sm100::smem_u32(dst)), "l"(src),
               "r"(ok ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp4(void* dst, const void* src, bool ok) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(sm100::smem_u32(dst)), "l"(src),
               "r"(ok ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
// every group but the most recent one has landed (for this thread's copies)
__device__ __forceinline__ void cp_wait_prev() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// rows [0, nvalid) of a tile of `rows` rows (row r at src + r * stride) into a padded bf16
// tile with asynchronous copies; rows past nvalid become zeros
// (lt: this thread's index among the nthr threads that share the copy)
template <int D>
__device__ __forceinline__ void cp_tile(const __nv_bfloat16* __restrict__ src, int64_t stride, int rows, int nvalid,
                                        __nv_bfloat16* dst, int lt = threadIdx.x, int nthr = NTM) {
  constexpr int VPR = D / 8, SH = D + 8;
  for (int v = lt; v < rows * VPR; v += nthr) {
    const int r = v / VPR, c = (v % VPR) * 8;
    const bool ok = r < nvalid;
    cp16(dst + r * SH + c, src + (ok ? r : 0) * stride + c, ok);
  }
}

// rowsum(dO * O) of `rows` rows, both from padded shared tiles, by the 4 warps of one group
// (wl: this warp's index in the group)
template <int D>
__device__ __forceinline__ void row_dot_smem(int rows, const __nv_bfloat16* dOs, const __nv_bfloat16* Os, float* dv,
                                             int wl) {
  constexpr int SH = D + 8;
  const int lane = threadIdx.x & 31;
  for (int r = wl; r < rows; r += NTM / 32) {
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(dOs + r * SH + c * 64 + 2 * lane));
      const float2 o = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(Os + r * SH + c * 64 + 2 * lane));
      s = fmaf(a.x, o.x, fmaf(a.y, o.y, s));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) dv[r] = s;
  }
}

__device__ __forceinline__ void ldsm4(const __nv_bfloat16* p, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(sm100::smem_u32(p)));
}

__device__ __forceinline__ void ldsm4t(const __nv_bfloat16* p, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(sm100::smem_u32(p)));
}

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // lo -> lower 16 bits (lower column)
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Lane addresses of one ldmatrix.x4 over the 16 x 16 block at (r0, c0) of a padded tile:
//   A (non-transposed) and B from a k-major stored tile (transposed load): matrices in the
//     order (r0, c0), (r0 + 8, c0), (r0, c0 + 8), (r0 + 8, c0 + 8);
//   B from an n-major stored tile (non-transposed load): (r0, c0), (r0, c0 + 8), (r0 + 8, c0),
//     (r0 + 8, c0 + 8), rows being n.
template <int SH>
__device__ __forceinline__ const __nv_bfloat16* frag_a(const __nv_bfloat16* t, int r0, int c0) {
  const int l = threadIdx.x & 31;
  return t + (r0 + (l & 7) + ((l >> 3) & 1) * 8) * SH + c0 + (l >> 4) * 8;
}
template <int SH>
__device__ __forceinline__ const __nv_bfloat16* frag_bn(const __nv_bfloat16* t, int r0, int c0) {
  const int l = threadIdx.x & 31;
  return t + (r0 + (l & 7) + (l >> 4) * 8) * SH + c0 + ((l >> 3) & 1) * 8;
}

// rowsum(dO * O) of `rows` rows: dO from its padded shared tile, O from global memory
template <int D>
__device__ __forceinline__ void row_dot_bf16(const __nv_bfloat16* __restrict__ O, int64_t stride, int rows, int nvalid,
                                             const __nv_bfloat16* dOs, float* dv) {
  constexpr int SH = MSmem<D>::SH;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int r = w; r < rows; r += NTM / 32) {
    float s = 0.f;
    if (r < nvalid) {
#pragma unroll
      for (int c = 0; c < D / 32; ++c)
        s = fmaf(__bfloat162float(dOs[r * SH + c * 32 + lane]), __bfloat162float(O[r * stride + c * 32 + lane]), s);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) dv[r] = s;
  }
}

// bar.sync on a named barrier shared by the 4 warps of one warp group
__device__ __forceinline__ void group_sync(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }

// NWG warp groups of 4 warps share the 64-key tile; group grp takes the query heads
// grp, grp + NWG, ... of the KV group, so each warp's chain of steps is G / NWG heads long.
// A group synchronises on its own named barrier (1 + grp); its dK / dV are added to group 0's
// through shared memory at the end of each KV head, in a fixed order.
template <int D, int NWG>
__global__ void __launch_bounds__(NTM * NWG, 1)
    attn_bwd_dkdv_mma(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                      const __nv_bfloat16* __restrict__ V, const __nv_bfloat16* __restrict__ O,
                      const __nv_bfloat16* __restrict__ dO, const float* __restrict__ logg,
                      const float* __restrict__ gain, const int32_t* __restrict__ pos, const float* __restrict__ lse,
                      float scale, int Hq, int Hkv, int64_t m_tot, float* __restrict__ dK, float* __restrict__ dV,
                      float* __restrict__ dlogg, float* __restrict__ dscore, const __grid_constant__ BwdParams p) {
  using S_ = MSmem<D>;
  constexpr int SH = S_::SH, NN = D / 8;  // n-tiles of 8 across the head dimension
  extern __shared__ __align__(16) unsigned char smraw[];
  const int tid = threadIdx.x, grp = tid >> 7, lt = tid & (NTM - 1);
  const int lane = tid & 31, wl = (tid >> 5) & 3, g = lane >> 2, t4 = lane & 3;
  __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(smraw);
  __nv_bfloat16* Vs = Ks + S_::OWN;
  // group grp, buffer b: Q, dO, O tiles at stream0 + (2 grp + b) 3 STR
  __nv_bfloat16* stream0 = Vs + S_::OWN;
  float* vec0 = reinterpret_cast<float*>(stream0 + NWG * 6 * S_::STR);
  float* lse_b = vec0 + grp * 5 * ST;                    // [2][ST] this group's
  int* posq_b = reinterpret_cast<int*>(lse_b + 2 * ST);  // [2][ST]
  float* dv = lse_b + 4 * ST;                            // [ST]
  float* dl_s = vec0 + NWG * 5 * ST;                     // [MT]

  const int C = p.C;
  const int unit = blockIdx.x / C, rank = blockIdx.x % C;
  int b = 0;
  while (b + 1 < p.nseq && unit >= p.tiles[b + 1]) ++b;
  const AttnSeq sq = p.s[b];
  const int t = unit - p.tiles[b];  // key tile: tile 0 has the most query steps below it
  const int k0 = t * MT;
  const int kvalid = min(MT, sq.m - k0);
  const int qs0 = k0 / ST;                    // first query step at or below the diagonal
  const int nq = (sq.m + ST - 1) / ST - qs0;  // query steps per head
  const int G = Hq / Hkv;
  const int nh = (G - grp + NWG - 1) / NWG;   // heads of this group (NWG <= G: at least 1)
  const int total = nh * nq;                  // (head, query step) pairs of this group per KV head
  const int kr0 = 16 * wl + g, kr1 = kr0 + 8;  // this thread's key rows within the tile
  const int pk0 = kr0 < kvalid ? pos[sq.off + k0 + kr0] : INT_MAX;
  const int pk1 = kr1 < kvalid ? pos[sq.off + k0 + kr1] : INT_MAX;
  const float lg0 = (logg && kr0 < kvalid) ? __ldg(logg + sq.off + k0 + kr0) : 0.f;
  const float lg1 = (logg && kr1 < kvalid) ? __ldg(logg + sq.off + k0 + kr1) : 0.f;

  // step n of this group for KV head kvh: head kvh G + grp + NWG (n / nq), query rows from
  // (qs0 + n % nq) ST
  auto issue = [&](int kvh, int n, int buf) {
    const int h = kvh * G + grp + NWG * (n / nq);
    const int q0 = (qs0 + n % nq) * ST;
    const int qvalid = min(ST, sq.m - q0);
    const int64_t qrow = ((int64_t)(sq.off + q0) * Hq + h) * D;
    __nv_bfloat16* base = stream0 + (2 * grp + buf) * 3 * S_::STR;
    cp_tile<D>(Q + qrow, (int64_t)Hq * D, ST, qvalid, base, lt, NTM);
    cp_tile<D>(dO + qrow, (int64_t)Hq * D, ST, qvalid, base + S_::STR, lt, NTM);
    cp_tile<D>(O + qrow, (int64_t)Hq * D, ST, qvalid, base + 2 * S_::STR, lt, NTM);
    if (lt < ST) {
      const bool ok = lt < qvalid;
      const int64_t row = sq.off + q0 + (ok ? lt : 0);
      cp4(lse_b + buf * ST + lt, lse + (int64_t)h * m_tot + row, ok);
      cp4(posq_b + buf * ST + lt, pos + row, ok);
    }
  };

  float dl0 = 0.f, dl1 = 0.f;
  for (int kvh = rank; kvh < Hkv; kvh += C) {
    __syncthreads();  // every group is done with the previous KV head (tiles and reduction)
    cp_tile<D>(K + ((int64_t)(sq.off + k0) * Hkv + kvh) * D, (int64_t)Hkv * D, MT, kvalid, Ks, tid, NTM * NWG);
    cp_tile<D>(V + ((int64_t)(sq.off + k0) * Hkv + kvh) * D, (int64_t)Hkv * D, MT, kvalid, Vs, tid, NTM * NWG);
    cp_commit();
    cp_wait_all();
    __syncthreads();  // K and V have landed for every thread of both groups
    issue(kvh, 0, 0);
    cp_commit();
    float aK[NN][4], aV[NN][4];
#pragma unroll
    for (int n = 0; n < NN; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) aK[n][e] = aV[n][e] = 0.f;
    for (int n = 0; n < total; ++n) {
      const int buf = n & 1;
      if (n + 1 < total) issue(kvh, n + 1, buf ^ 1);  // its buffer was released at the end of step n - 1
      cp_commit();
      cp_wait_prev();
      group_sync(1 + grp);  // step n's tiles have landed for every thread of the group
      const int h = kvh * G + grp + NWG * (n / nq);
      const float gh = gain ? __ldg(gain + h) : 1.f;
      const int qvalid = min(ST, sq.m - (qs0 + n % nq) * ST);
      const __nv_bfloat16* Qs = stream0 + (2 * grp + buf) * 3 * S_::STR;
      const __nv_bfloat16* dOs = Qs + S_::STR;
      const float* lse_s = lse_b + buf * ST;
      const int* posq = posq_b + buf * ST;
      row_dot_smem<D>(ST, dOs, dOs + S_::STR, dv, wl);
      // S^T (keys x queries) = K Q^T and dP^T = V dO^T, 16 x 32 per warp
      float sT[4][4], pT[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) sT[j][e] = pT[j][e] = 0.f;
#pragma unroll
      for (int kd = 0; kd < D / 16; ++kd) {
        uint32_t ak[4], av[4];
        ldsm4(frag_a<SH>(Ks, 16 * wl, 16 * kd), ak);
        ldsm4(frag_a<SH>(Vs, 16 * wl, 16 * kd), av);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          uint32_t bq[4], bo[4];
          ldsm4(frag_bn<SH>(Qs, 16 * np, 16 * kd), bq);
          ldsm4(frag_bn<SH>(dOs, 16 * np, 16 * kd), bo);
          mma16816(sT[2 * np], ak, bq[0], bq[1]);
          mma16816(sT[2 * np + 1], ak, bq[2], bq[3]);
          mma16816(pT[2 * np], av, bo[0], bo[1]);
          mma16816(pT[2 * np + 1], av, bo[2], bo[3]);
        }
      }
      group_sync(1 + grp);  // dv is complete
      // P^T and dS^T in place: rows kr0 / kr1 (keys), columns 8j + 2t4 + {0, 1} (queries)
      const float b0 = key_bias(gh, lg0), b1 = key_bias(gh, lg1);
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int qc = 8 * j + 2 * t4 + (e & 1);
          const bool vis = qc < qvalid && (e < 2 ? pk0 : pk1) <= posq[qc];
          const float pv = vis ? expf(fmaf(scale, sT[j][e], (e < 2 ? b0 : b1) - lse_or_inf(lse_s[qc]))) : 0.f;
          const float ds = pv * (pT[j][e] - dv[qc]);
          sT[j][e] = pv;
          pT[j][e] = ds;
          if (e < 2) dl0 = fmaf(gh, ds, dl0);
          else dl1 = fmaf(gh, ds, dl1);
        }
      // dV += P^T dO and dK += dS^T Q: k runs over the 32 queries (two steps of 16)
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const uint32_t ap[4] = {pack_bf16(sT[2 * kk][0], sT[2 * kk][1]), pack_bf16(sT[2 * kk][2], sT[2 * kk][3]),
                                pack_bf16(sT[2 * kk + 1][0], sT[2 * kk + 1][1]),
                                pack_bf16(sT[2 * kk + 1][2], sT[2 * kk + 1][3])};
        const uint32_t as[4] = {pack_bf16(pT[2 * kk][0], pT[2 * kk][1]), pack_bf16(pT[2 * kk][2], pT[2 * kk][3]),
                                pack_bf16(pT[2 * kk + 1][0], pT[2 * kk + 1][1]),
                                pack_bf16(pT[2 * kk + 1][2], pT[2 * kk + 1][3])};
#pragma unroll
        for (int u = 0; u < D / 16; ++u) {
          uint32_t bo[4], bq[4];
          ldsm4t(frag_a<SH>(dOs, 16 * kk, 16 * u), bo);
          ldsm4t(frag_a<SH>(Qs, 16 * kk, 16 * u), bq);
          mma16816(aV[2 * u], ap, bo[0], bo[1]);
          mma16816(aV[2 * u + 1], ap, bo[2], bo[3]);
          mma16816(aK[2 * u], as, bq[0], bq[1]);
          mma16816(aK[2 * u + 1], as, bq[2], bq[3]);
        }
      }
      group_sync(1 + grp);  // every read of this buffer is done: step n + 2 may refill it
    }
    // group 1's dK / dV go through shared memory (the stream buffers, now idle) into group 0's
    if (NWG > 1) {
      float* red = reinterpret_cast<float*>(stream0);  // [2][MT][D]: dK, then dV
      __syncthreads();  // both groups are done with their stream buffers
      if (grp == 1) {
#pragma unroll
        for (int n = 0; n < NN; ++n) {
          const int c = 8 * n + 2 * t4;
          *reinterpret_cast<float2*>(red + kr0 * D + c) = make_float2(aK[n][0], aK[n][1]);
          *reinterpret_cast<float2*>(red + kr1 * D + c) = make_float2(aK[n][2], aK[n][3]);
          *reinterpret_cast<float2*>(red + (MT + kr0) * D + c) = make_float2(aV[n][0], aV[n][1]);
          *reinterpret_cast<float2*>(red + (MT + kr1) * D + c) = make_float2(aV[n][2], aV[n][3]);
        }
      }
      __syncthreads();
      if (grp == 0) {
#pragma unroll
        for (int n = 0; n < NN; ++n) {
          const int c = 8 * n + 2 * t4;
          const float2 k0v = *reinterpret_cast<const float2*>(red + kr0 * D + c);
          const float2 k1v = *reinterpret_cast<const float2*>(red + kr1 * D + c);
          const float2 v0v = *reinterpret_cast<const float2*>(red + (MT + kr0) * D + c);
          const float2 v1v = *reinterpret_cast<const float2*>(red + (MT + kr1) * D + c);
          aK[n][0] += k0v.x;
          aK[n][1] += k0v.y;
          aK[n][2] += k1v.x;
          aK[n][3] += k1v.y;
          aV[n][0] += v0v.x;
          aV[n][1] += v0v.y;
          aV[n][2] += v1v.x;
          aV[n][3] += v1v.y;
        }
      }
    }
    // rows kr0 / kr1 of dK (scaled) and dV for this KV head, columns 8n + 2t4 + {0, 1}
    if (grp == 0) {
#pragma unroll
      for (int n = 0; n < NN; ++n) {
        const int c = 8 * n + 2 * t4;
        if (kr0 < kvalid) {
          const int64_t r = ((int64_t)(sq.off + k0 + kr0) * Hkv + kvh) * D + c;
          *reinterpret_cast<float2*>(dK + r) = make_float2(scale * aK[n][0], scale * aK[n][1]);
          *reinterpret_cast<float2*>(dV + r) = make_float2(aV[n][0], aV[n][1]);
        }
        if (kr1 < kvalid) {
          const int64_t r = ((int64_t)(sq.off + k0 + kr1) * Hkv + kvh) * D + c;
          *reinterpret_cast<float2*>(dK + r) = make_float2(scale * aK[n][2], scale * aK[n][3]);
          *reinterpret_cast<float2*>(dV + r) = make_float2(aV[n][2], aV[n][3]);
        }
      }
    }
  }
  // d log g: the quad holding a key row adds its columns, the groups add in order, then the
  // cluster adds its KV heads
  dl0 += __shfl_xor_sync(0xffffffffu, dl0, 1);
  dl0 += __shfl_xor_sync(0xffffffffu, dl0, 2);
  dl1 += __shfl_xor_sync(0xffffffffu, dl1, 1);
  dl1 += __shfl_xor_sync(0xffffffffu, dl1, 2);
  __syncthreads();  // dl_s may alias nothing in use, but keep the groups' writes ordered
  if (grp == 0 && t4 == 0) {
    dl_s[kr0] = dl0;
    dl_s[kr1] = dl1;
  }
  if (NWG > 1) {
    __syncthreads();
    if (grp == 1 && t4 == 0) {
      dl_s[kr0] += dl0;
      dl_s[kr1] += dl1;
    }
  }
  if (C > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0 && tid < kvalid && (dlogg || dscore)) {
      float tot = 0.f;
      for (int r = 0; r < C; ++r) tot += cluster.map_shared_rank(dl_s, r)[tid];
      const int64_t row = sq.off + k0 + tid;
      if (dlogg) dlogg[row] = tot;
      if (dscore) dscore[row] = tot * -expm1f(__ldg(logg + row));
    }
    cluster.sync();  // no CTA leaves while rank 0 may still read its partials
  } else {
    __syncthreads();
    if (tid < kvalid && (dlogg || dscore)) {
      const float tot = dl_s[tid];
      const int64_t row = sq.off + k0 + tid;
      if (dlogg) dlogg[row] = tot;
      if (dscore) dscore[row] = tot * -expm1f(__ldg(logg + row));
    }
  }
}

template <int D>
__global__ void __launch_bounds__(NTM)
    attn_bwd_dq_mma(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                    const __nv_bfloat16* __restrict__ V, const __nv_bfloat16* __restrict__ O,
                    const __nv_bfloat16* __restrict__ dO, const float* __restrict__ logg,
                    const float* __restrict__ gain, const int32_t* __restrict__ pos, const float* __restrict__ lse,
                    float scale, int Hq, int Hkv, int64_t m_tot, float* __restrict__ dQ,
                    int32_t* __restrict__ dev_status, const __grid_constant__ BwdParams p) {
  using S_ = MSmem<D>;
  constexpr int SH = S_::SH, NN = D / 8;
  extern __shared__ __align__(16) unsigned char smraw[];
  __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(smraw);
  __nv_bfloat16* dOs = Qs + S_::OWN;
  __nv_bfloat16* stream0 = dOs + S_::OWN;  // buffer b: K, V tiles at stream0 + 2 b STR
  float* lse_s = reinterpret_cast<float*>(stream0 + 4 * S_::STR);  // [MT]
  float* dv = lse_s + MT;                                          // [MT]
  int* posq = reinterpret_cast<int*>(dv + MT);                     // [MT]
  float* lgk_b = reinterpret_cast<float*>(posq + MT);              // [2][ST] log g of the keys
  int* posk_b = reinterpret_cast<int*>(lgk_b + 2 * ST);            // [2][ST]

  const int unit = blockIdx.x, h = blockIdx.y;
  int b = 0;
  while (b + 1 < p.nseq && unit >= p.tiles[b + 1]) ++b;
  const AttnSeq sq = p.s[b];
  const int nt = p.tiles[b + 1] - p.tiles[b];
  const int t = nt - 1 - (unit - p.tiles[b]);  // query tile: the last one has the most keys
  const int q0 = t * MT;
  const int qvalid = min(MT, sq.m - q0);
  const int kvh = h / (Hq / Hkv);
  const float gh = gain ? __ldg(gain + h) : 1.f;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, g = lane >> 2, t4 = lane & 3;
  const int qr0 = 16 * w + g, qr1 = qr0 + 8;  // this thread's query rows within the tile

  if (tid < MT) {
    const bool ok = tid < qvalid;
    posq[tid] = ok ? pos[sq.off + q0 + tid] : INT_MIN;
    lse_s[tid] = ok ? lse_or_inf(__ldg(lse + (int64_t)h * m_tot + sq.off + q0 + tid)) : 0.f;
    // the positions must rise strictly inside a sequence (row order is the causal order)
    if (ok && h == 0 && q0 + tid > 0 && dev_status && pos[sq.off + q0 + tid - 1] >= posq[tid])
      atomicOr(dev_status, TG_DEV_POS_NOT_ASCENDING);
  }
  // key step ks: keys from ks * ST, their K and V rows, log g and positions
  auto issue = [&](int ks, int buf) {
    const int k0 = ks * ST;
    const int kvalid = min(ST, sq.m - k0);
    __nv_bfloat16* base = stream0 + 2 * buf * S_::STR;
    cp_tile<D>(K + ((int64_t)(sq.off + k0) * Hkv + kvh) * D, (int64_t)Hkv * D, ST, kvalid, base);
    cp_tile<D>(V + ((int64_t)(sq.off + k0) * Hkv + kvh) * D, (int64_t)Hkv * D, ST, kvalid, base + S_::STR);
    if (tid < ST) {
      const bool ok = tid < kvalid;
      const int64_t row = sq.off + k0 + (ok ? tid : 0);
      cp4(lgk_b + buf * ST + tid, logg ? logg + row : reinterpret_cast<const float*>(pos + row), ok && logg);
      cp4(posk_b + buf * ST + tid, pos + row, ok);
    }
  };
  const int64_t qrow = ((int64_t)(sq.off + q0) * Hq + h) * D;
  cp_tile<D>(Q + qrow, (int64_t)Hq * D, MT, qvalid, Qs);
  cp_tile<D>(dO + qrow, (int64_t)Hq * D, MT, qvalid, dOs);
  issue(0, 0);
  cp_commit();
  float aQ[NN][4];
#pragma unroll
  for (int n = 0; n < NN; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) aQ[n][e] = 0.f;
  const int nks = (q0 + qvalid - 1) / ST + 1;  // key steps up to the tile's last row
  for (int ks = 0; ks < nks; ++ks) {
    const int buf = ks & 1;
    if (ks + 1 < nks) issue(ks + 1, buf ^ 1);  // its buffer was released at the end of step ks - 1
    cp_commit();
    cp_wait_prev();
    __syncthreads();  // step ks's tiles (and, at ks = 0, Q and dO) have landed for every thread
    if (ks == 0) row_dot_bf16<D>(O + qrow, (int64_t)Hq * D, MT, qvalid, dOs, dv);
    const int kvalid = min(ST, sq.m - ks * ST);
    const __nv_bfloat16* Ks = stream0 + 2 * buf * S_::STR;
    const __nv_bfloat16* Vs = Ks + S_::STR;
    const float* lgk = lgk_b + buf * ST;
    const int* posk = posk_b + buf * ST;
    // S = Q K^T and dP = dO V^T, 16 x 32 per warp
    float sc[4][4], dp[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[j][e] = dp[j][e] = 0.f;
#pragma unroll
    for (int kd = 0; kd < D / 16; ++kd) {
      uint32_t aq[4], ao[4];
      ldsm4(frag_a<SH>(Qs, 16 * w, 16 * kd), aq);
      ldsm4(frag_a<SH>(dOs, 16 * w, 16 * kd), ao);
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        uint32_t bk[4], bv[4];
        ldsm4(frag_bn<SH>(Ks, 16 * np, 16 * kd), bk);
        ldsm4(frag_bn<SH>(Vs, 16 * np, 16 * kd), bv);
        mma16816(sc[2 * np], aq, bk[0], bk[1]);
        mma16816(sc[2 * np + 1], aq, bk[2], bk[3]);
        mma16816(dp[2 * np], ao, bv[0], bv[1]);
        mma16816(dp[2 * np + 1], ao, bv[2], bv[3]);
      }
    }
    __syncthreads();  // dv is complete (written at ks = 0)
    // dS in place: rows qr0 / qr1 (queries), columns 8j + 2t4 + {0, 1} (keys)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qr = e < 2 ? qr0 : qr1, kc = 8 * j + 2 * t4 + (e & 1);
        const bool vis = kc < kvalid && posk[kc] <= posq[qr];
        const float pv = vis ? expf(fmaf(scale, sc[j][e], key_bias(gh, lgk[kc]) - lse_s[qr])) : 0.f;
        dp[j][e] = pv * (dp[j][e] - dv[qr]);
      }
    // dQ += dS K: k runs over the 32 keys (two steps of 16)
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      const uint32_t as[4] = {pack_bf16(dp[2 * kk][0], dp[2 * kk][1]), pack_bf16(dp[2 * kk][2], dp[2 * kk][3]),
                              pack_bf16(dp[2 * kk + 1][0], dp[2 * kk + 1][1]),
                              pack_bf16(dp[2 * kk + 1][2], dp[2 * kk + 1][3])};
#pragma unroll
      for (int u = 0; u < D / 16; ++u) {
        uint32_t bk[4];
        ldsm4t(frag_a<SH>(Ks, 16 * kk, 16 * u), bk);
        mma16816(aQ[2 * u], as, bk[0], bk[1]);
        mma16816(aQ[2 * u + 1], as, bk[2], bk[3]);
      }
    }
    __syncthreads();  // every read of this buffer is done: step ks + 2 may refill it
  }
#pragma unroll
  for (int n = 0; n < NN; ++n) {
    const int c = 8 * n + 2 * t4;
    if (qr0 < qvalid)
      *reinterpret_cast<float2*>(dQ + ((int64_t)(sq.off + q0 + qr0) * Hq + h) * D + c) =
          make_float2(scale * aQ[n][0], scale * aQ[n][1]);
    if (qr1 < qvalid)
      *reinterpret_cast<float2*>(dQ + ((int64_t)(sq.off + q0 + qr1) * Hq + h) * D + c) =
          make_float2(scale * aQ[n][2], scale * aQ[n][3]);
  }
}

template <typename T, int D>
tg_status launch_td(const AttnBwdArgs& a, const BwdParams& p0, cudaStream_t st) {
  BwdParams p = p0;
  const int units = p.tiles[p.nseq];
  constexpr int SMEM = Smem<D>::BYTES;
  auto kdkdv = attn_bwd_dkdv_kernel<T, D>;
  auto kdq = attn_bwd_dq_kernel<T, D>;
  const int slot = ATTR_BWD + (D == 128 ? 1 : 0);
  if (attrs_needed(slot)) {
    for (const void* k : {(const void*)kdkdv, (const void*)kdq}) {
      cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
      if (e != cudaSuccess) return cuda_status(e, "tg_gated_attn_bwd: cudaFuncSetAttribute");
    }
    mark_attrs_set(slot);
  }
  const T* q = static_cast<const T*>(a.Q);
  const T* k = static_cast<const T*>(a.K);
  const T* v = static_cast<const T*>(a.V);
  const T* o = static_cast<const T*>(a.O);
  const T* dO = static_cast<const T*>(a.dO);

  // dK, dV, d log g: clusters of C CTAs over the KV heads of one key tile
  p.C = a.Hkv < MAXC ? a.Hkv : MAXC;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(units * p.C));
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = (size_t)SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.C > 1 ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kdkdv, q, k, v, o, dO, a.logg, a.head_gain, a.pos, a.lse, a.scale, a.Hq,
                                     a.Hkv, a.m_tot, a.dK, a.dV, a.dlogg, a.dscore, p);
  if (e != cudaSuccess) return cuda_status(e, "tg_gated_attn_bwd: dK/dV launch");

  // dQ: one CTA per (query tile, head)
  p.C = 1;
  cudaLaunchConfig_t cq = {};
  cq.gridDim = dim3((unsigned)units, (unsigned)a.Hq);
  cq.blockDim = dim3(NT);
  cq.dynamicSmemBytes = (size_t)SMEM;
  cq.stream = st;
  e = cudaLaunchKernelEx(&cq, kdq, q, k, v, o, dO, a.logg, a.head_gain, a.pos, a.lse, a.scale, a.Hq, a.Hkv, a.m_tot,
                         a.dQ, a.dev_status, p);
  return cuda_status(e, "tg_gated_attn_bwd: dQ launch");
}

template <int D, int NWG>
tg_status launch_mma(const AttnBwdArgs& a, const BwdParams& p0, cudaStream_t st) {
  BwdParams p = p0;
  const int units = p.tiles[p.nseq];
  constexpr int SMEM_DKDV = MSmem<D>::bytes_dkdv(NWG), SMEM_DQ = MSmem<D>::BYTES_DQ;
  static_assert(SMEM_DKDV <= 227 * 1024, "shared memory budget");
  auto kdkdv = attn_bwd_dkdv_mma<D, NWG>;
  auto kdq = attn_bwd_dq_mma<D>;
  const int slot = ATTR_BWD + 2 + (D == 128 ? 2 : 0) + (NWG - 1);
  if (attrs_needed(slot)) {
    cudaError_t e = cudaFuncSetAttribute(kdkdv, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_DKDV);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kdq, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_DQ);
    if (e != cudaSuccess) return cuda_status(e, "tg_gated_attn_bwd: cudaFuncSetAttribute");
    mark_attrs_set(slot);
  }
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.Q);
  const __nv_bfloat16* k = static_cast<const __nv_bfloat16*>(a.K);
  const __nv_bfloat16* v = static_cast<const __nv_bfloat16*>(a.V);
  const __nv_bfloat16* o = static_cast<const __nv_bfloat16*>(a.O);
  const __nv_bfloat16* dO = static_cast<const __nv_bfloat16*>(a.dO);

  p.C = a.Hkv < MAXC ? a.Hkv : MAXC;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(units * p.C));
  cfg.blockDim = dim3(NTM * NWG);
  cfg.dynamicSmemBytes = (size_t)SMEM_DKDV;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.C > 1 ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kdkdv, q, k, v, o, dO, a.logg, a.head_gain, a.pos, a.lse, a.scale, a.Hq,
                                     a.Hkv, a.m_tot, a.dK, a.dV, a.dlogg, a.dscore, p);
  if (e != cudaSuccess) return cuda_status(e, "tg_gated_attn_bwd: dK/dV launch");
  p.C = 1;
  cudaLaunchConfig_t cq = {};
  cq.gridDim = dim3((unsigned)units, (unsigned)a.Hq);
  cq.blockDim = dim3(NTM);
  cq.dynamicSmemBytes = (size_t)SMEM_DQ;
  cq.stream = st;
  e = cudaLaunchKernelEx(&cq, kdq, q, k, v, o, dO, a.logg, a.head_gain, a.pos, a.lse, a.scale, a.Hq, a.Hkv, a.m_tot,
                         a.dQ, a.dev_status, p);
  return cuda_status(e, "tg_gated_attn_bwd: dQ launch");
}

}  // namespace

tg_status launch_attn_bwd(const AttnBwdArgs& a, const AttnSeq* seqs, int nseq, cudaStream_t st) {
  // bf16: tensor-core kernels on 64-row tiles; f32: CUDA-core kernels on 32-row tiles
  const int tile = a.dt == TG_BF16 ? MT : BT;
  BwdParams p = {};
  p.nseq = nseq;
  p.tiles[0] = 0;
  for (int i = 0; i < nseq; ++i) {
    p.s[i] = seqs[i];
    p.tiles[i + 1] = p.tiles[i] + (seqs[i].m + tile - 1) / tile;
  }
  if (p.tiles[nseq] == 0) return TG_OK;
  if (a.dt == TG_BF16) {
    // two warp groups share a key tile when its KV group has at least two query heads
    const bool two = a.Hq / a.Hkv >= 2;
    if (a.D == 64) return two ? launch_mma<64, 2>(a, p, st) : launch_mma<64, 1>(a, p, st);
    return two ? launch_mma<128, 2>(a, p, st) : launch_mma<128, 1>(a, p, st);
  }
  return a.D == 64 ? launch_td<float, 64>(a, p, st) : launch_td<float, 128>(a, p, st);
}

}  // namespace tg
