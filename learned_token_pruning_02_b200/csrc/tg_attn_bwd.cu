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
// on the CUDA cores in fp32 (the kernels below, whose 1e-4 tolerance needs fp32 products);
// bf16 tensors run on the 5th-generation tensor cores (tg_attn_bwd_tc.cu). The f32 split:
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

}  // namespace

tg_status launch_attn_bwd(const AttnBwdArgs& a, const AttnSeq* seqs, int nseq, cudaStream_t st) {
  // bf16: the tensor-core kernels (tg_attn_bwd_tc.cu); f32: the CUDA-core kernels above
  if (a.dt == TG_BF16) return launch_attn_bwd_tc(a, seqs, nseq, st);
  BwdParams p = {};
  p.nseq = nseq;
  p.tiles[0] = 0;
  for (int i = 0; i < nseq; ++i) {
    p.s[i] = seqs[i];
    p.tiles[i + 1] = p.tiles[i] + (seqs[i].m + BT - 1) / BT;
  }
  if (p.tiles[nseq] == 0) return TG_OK;
  return a.D == 64 ? launch_td<float, 64>(a, p, st) : launch_td<float, 128>(a, p, st);
}

}  // namespace tg
