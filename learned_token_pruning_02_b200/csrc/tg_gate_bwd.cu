// Gradients of the gate network's parameters from the score gradient of the kept rows.
//
// The last link of end-to-end selector training (TokenGate paper page, thelatestinai.com,
// Figure 1(c): the gated attention lets the top-K selector learn; aitualizate.com article,
// section on training the top-K selection). With s = (w2 . GELU(W1 h + b1) + b2) / T and the
// upstream d score of each kept row (tg_gated_attn_bwd's dscore):
//   z = W1 h + b1,  ds' = dscore / T,  u = ds' w2 * GELU'(z)  (per row, dg values),
//   dW1 = sum_rows u h^T,  db1 = sum_rows u,  dw2 = sum_rows ds' GELU(z),  db2 = sum_rows ds'.
//
// Three kernels, fp32 arithmetic on the CUDA cores, deterministic (fixed reduction orders, no
// atomics), with a caller-provided workspace; f32 operands, and bf16 shapes the tensor-core
// kernels (csrc/tg_gate_bwd_tc.cu: dg and d multiples of 128) do not take:
//   * rows:   one CTA per (64-row tile, 64-column block of dg) forms z = H W1^T + b1 in fp32
//             from bf16/f32 operands staged through shared memory (k-major, so each thread reads
//             its 4 rows and 4 columns as two 16-byte words), then u into the workspace and the
//             tile's column sums of u and ds' GELU(z).
//   * dW1:    one CTA per (64 x 64 block of dW1, row split) accumulates u^T h over its rows;
//             with more than one split each writes a partial block.
//   * reduce: sums the partial blocks, the tile column sums and ds' in a fixed order.
#include <cuda_bf16.h>

#include <atomic>

#include "tg_gate_bwd.cuh"

namespace tg {
namespace {

constexpr int TR = 64;   // rows per tile
constexpr int TC = 64;   // columns per tile
constexpr int KC = 32;   // k chunk
constexpr int NT = 256;  // 16 x 16 threads, 4 x 4 outputs each

__device__ __forceinline__ float gelu_exact(float z) { return 0.5f * z * (1.f + erff(z * 0.70710678118654752f)); }
__device__ __forceinline__ float gelu_grad(float z) {
  return 0.5f * (1.f + erff(z * 0.70710678118654752f)) + z * 0.39894228040143268f * expf(-0.5f * z * z);
}

// Eight consecutive elements of a row as fp32.
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 q = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
}

template <typename T>
__global__ void __launch_bounds__(NT) gate_bwd_rows_kernel(const T* __restrict__ H, int M, int d, const T* __restrict__ W1,
                                                           const float* __restrict__ b1, const T* __restrict__ w2,
                                                           float inv_t, int dg, const float* __restrict__ dscore,
                                                           float* __restrict__ U, float* __restrict__ part_db1,
                                                           float* __restrict__ part_dw2) {
  __shared__ __align__(16) float Hs[KC][TR];
  __shared__ __align__(16) float Ws[KC][TC];
  __shared__ float red[2][16][TC];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int r0 = blockIdx.x * TR, c0 = blockIdx.y * TC;
  const int lr = tid >> 2, lk = (tid & 3) * 8;  // loader: row (or column) lr, k offset lk
  float acc[4][4] = {};
  for (int k0 = 0; k0 < d; k0 += KC) {
    float hv[8], wv[8];
    if (r0 + lr < M) load8(H + (int64_t)(r0 + lr) * d + k0 + lk, hv);
    else
#pragma unroll
      for (int i = 0; i < 8; ++i) hv[i] = 0.f;
    load8(W1 + (int64_t)(c0 + lr) * d + k0 + lk, wv);
    __syncthreads();  // the previous chunk's readers are done
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      Hs[lk + i][lr] = hv[i];
      Ws[lk + i][lr] = wv[i];
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < KC; ++k) {
      const float4 a = *reinterpret_cast<const float4*>(&Hs[k][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&Ws[k][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
  }
  // epilogue: u = ds' w2 GELU'(z) into the workspace; column sums of u and ds' GELU(z)
  float su[4] = {0.f, 0.f, 0.f, 0.f}, sa[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + ty * 4 + i;
    const float ds = r < M ? dscore[r] * inv_t : 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = c0 + tx * 4 + j;
      const float z = acc[i][j] + (b1 ? b1[c] : 0.f);
      float w = (float)w2[c];
      const float u = ds * w * gelu_grad(z);
      if (r < M) U[(int64_t)r * dg + c] = u;
      su[j] += u;
      sa[j] += ds * gelu_exact(z);
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    red[0][ty][tx * 4 + j] = su[j];
    red[1][ty][tx * 4 + j] = sa[j];
  }
  __syncthreads();
  if (tid < 2 * TC) {
    const int which = tid / TC, c = tid % TC;
    float s = 0.f;
    for (int y = 0; y < 16; ++y) s += red[which][y][c];
    (which ? part_dw2 : part_db1)[(int64_t)blockIdx.x * dg + c0 + c] = s;
  }
}

template <typename T>
__global__ void __launch_bounds__(NT) gate_bwd_dw1_kernel(const T* __restrict__ H, int M, int d,
                                                          const float* __restrict__ U, int dg, int rows_per_split,
                                                          float* __restrict__ out) {
  __shared__ __align__(16) float Us[KC][TC];
  __shared__ __align__(16) float Hs[KC][TC];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int c0 = blockIdx.x * TC, j0 = blockIdx.y * TC, split = blockIdx.z;
  const int ra = split * rows_per_split, rb = min(M, ra + rows_per_split);
  const int lr = tid >> 3, lc = (tid & 7) * 8;  // loader: row lr of the chunk, 8 columns from lc
  float acc[4][4] = {};
  for (int k0 = ra; k0 < rb; k0 += KC) {
    float uv[8], hv[8];
    const int r = k0 + lr;
    if (r < rb) {
      load8(U + (int64_t)r * dg + c0 + lc, uv);
      load8(H + (int64_t)r * d + j0 + lc, hv);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) uv[i] = hv[i] = 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      Us[lr][lc + i] = uv[i];
      Hs[lr][lc + i] = hv[i];
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < KC; ++k) {
      const float4 a = *reinterpret_cast<const float4*>(&Us[k][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&Hs[k][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
  }
  float* o = out + (int64_t)split * dg * d;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    *reinterpret_cast<float4*>(o + (int64_t)(c0 + ty * 4 + i) * d + j0 + tx * 4) =
        make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
}

// Sums the row splits of dW1 (when there are several), the tiles' column sums and ds'.
__global__ void __launch_bounds__(NT) gate_bwd_reduce_kernel(const float* __restrict__ parts, int splits, int64_t n_w,
                                                             float* __restrict__ dW1, const float* __restrict__ part_db1,
                                                             const float* __restrict__ part_dw2, int n_tiles, int dg,
                                                             const float* __restrict__ dscore, int M, float inv_t,
                                                             float* __restrict__ db1, float* __restrict__ dw2,
                                                             float* __restrict__ db2) {
  const int64_t gid = (int64_t)blockIdx.x * NT + threadIdx.x;
  if (splits > 1)
    for (int64_t i = gid; i < n_w; i += (int64_t)gridDim.x * NT) {
      float s = 0.f;
      for (int sp = 0; sp < splits; ++sp) s += parts[(int64_t)sp * n_w + i];
      dW1[i] = s;
    }
  if (gid < dg) {
    float a = 0.f, b = 0.f;
    for (int t = 0; t < n_tiles; ++t) {
      a += part_db1[(int64_t)t * dg + gid];
      b += part_dw2[(int64_t)t * dg + gid];
    }
    if (db1) db1[gid] = a;
    if (dw2) dw2[gid] = b;
  }
  if (blockIdx.x == 0 && db2) {  // ds' summed by one block in a fixed order
    __shared__ float sred[NT];
    float s = 0.f;
    for (int r = threadIdx.x; r < M; r += NT) s += dscore[r];
    sred[threadIdx.x] = s;
    __syncthreads();
    for (int w = NT / 2; w > 0; w >>= 1) {
      if (threadIdx.x < w) sred[threadIdx.x] += sred[threadIdx.x + w];
      __syncthreads();
    }
    if (threadIdx.x == 0) *db2 = sred[0] * inv_t;
  }
}

int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }

// Scratch of tg_gate_mlp_bwd_noalloc: a fixed device array of this library, present on every GPU
// that loads it until the process exits, shared by every call of that entry point on the device.
static __device__ __align__(256) unsigned char g_gate_scratch[TG_GATE_NOALLOC_SCRATCH_BYTES];

// Device address of g_gate_scratch per device (the array's name in host code is only a host
// stand-in for the symbol, never a device address), looked up on a device's first call.
std::atomic<void*> g_gate_scratch_addr[64];

}  // namespace

tg_status gate_bwd_fixed_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e, "tg_gate_mlp_bwd_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(TG_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  void* p = g_gate_scratch_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    e = cudaGetSymbolAddress(&p, g_gate_scratch);  // the current device is `dev`
    if (e != cudaSuccess) return cuda_status(e, "tg_gate_mlp_bwd_noalloc: cudaGetSymbolAddress of the scratch");
    g_gate_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *ptr = p;
  return TG_OK;
}

GateBwdPlan gate_bwd_plan(int64_t M, int d, int dg, int sms) {
  GateBwdPlan p;
  p.n_tiles = (int)((M + TR - 1) / TR);
  const int blocks = (dg / TC) * (d / TC);
  int splits = (2 * sms + blocks - 1) / blocks;
  const int max_splits = (int)((M + 255) / 256);  // at least 256 rows per split
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  p.splits = splits;
  p.rows_per_split = (int)((M + splits - 1) / splits);
  p.off_part = align256(M * (int64_t)dg * 4);
  p.off_w = p.off_part + align256(2 * (int64_t)p.n_tiles * dg * 4);
  p.bytes = p.off_w + (splits > 1 ? align256((int64_t)splits * dg * d * 4) : 0);
  if (gate_bwd_tc_shape(M, d, dg)) {
    gate_bwd_tc_plan(p, M, d, dg, sms);
    if (p.tc_bytes > p.bytes) p.bytes = p.tc_bytes;
  }
  return p;
}

tg_status launch_gate_bwd(tg_dtype dt, const void* H, int64_t M, int d, const void* W1, const float* b1,
                          const void* w2, float inv_t, int dg, const float* dscore, float* dW1, float* db1,
                          float* dw2, float* db2, void* ws, const GateBwdPlan& p, int32_t* dev_status,
                          cudaStream_t st) {
  if (dt == TG_BF16 && p.tc)
    return launch_gate_bwd_tc(H, M, d, W1, b1, w2, inv_t, dg, dscore, dW1, db1, dw2, db2, ws, p, dev_status, st);
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* U = reinterpret_cast<float*>(base);
  float* part_db1 = reinterpret_cast<float*>(base + p.off_part);
  float* part_dw2 = part_db1 + (int64_t)p.n_tiles * dg;
  float* wpart = p.splits > 1 ? reinterpret_cast<float*>(base + p.off_w) : dW1;
  const dim3 g1((unsigned)p.n_tiles, (unsigned)(dg / TC));
  const dim3 g2((unsigned)(dg / TC), (unsigned)(d / TC), (unsigned)p.splits);
  if (dt == TG_BF16) {
    auto h = static_cast<const __nv_bfloat16*>(H);
    gate_bwd_rows_kernel<__nv_bfloat16><<<g1, NT, 0, st>>>(h, (int)M, d, static_cast<const __nv_bfloat16*>(W1), b1,
                                                            static_cast<const __nv_bfloat16*>(w2), inv_t, dg, dscore,
                                                            U, part_db1, part_dw2);
    gate_bwd_dw1_kernel<__nv_bfloat16><<<g2, NT, 0, st>>>(h, (int)M, d, U, dg, p.rows_per_split, wpart);
  } else {
    auto h = static_cast<const float*>(H);
    gate_bwd_rows_kernel<float><<<g1, NT, 0, st>>>(h, (int)M, d, static_cast<const float*>(W1), b1,
                                                   static_cast<const float*>(w2), inv_t, dg, dscore, U, part_db1,
                                                   part_dw2);
    gate_bwd_dw1_kernel<float><<<g2, NT, 0, st>>>(h, (int)M, d, U, dg, p.rows_per_split, wpart);
  }
  const int64_t n_w = (int64_t)dg * d;
  const int gr = p.splits > 1 ? (int)((n_w + NT - 1) / NT < 1184 ? (n_w + NT - 1) / NT : 1184) : 1;
  gate_bwd_reduce_kernel<<<gr < 1 ? 1 : gr, NT, 0, st>>>(reinterpret_cast<const float*>(base + p.off_w), p.splits,
                                                           n_w, dW1, part_db1, part_dw2, p.n_tiles, dg, dscore,
                                                           (int)M, inv_t, db1, dw2, db2);
  return cuda_status(cudaGetLastError(), "tg_gate_mlp_bwd: launch");
}

}  // namespace tg
