// C-ABI layer of libtokengate: argument validation, per-sequence descriptors, dispatch.
// No entry point allocates memory or synchronises the host with the device.
#include <stdarg.h>
#include <stdlib.h>
#include <stdio.h>
#include <string.h>

#include <vector>

#include "tg_attn_bwd.cuh"
#include "tg_gate_bwd.cuh"
#include "tg_internal.cuh"

namespace tg {

static thread_local char g_err[512] = "";
static thread_local uint64_t g_wait_probe_ns = 0;  // test hook of the bounded waits (0 = off)

uint64_t wait_probe_ns() { return g_wait_probe_ns; }

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

tg_status fail(tg_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

tg_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return TG_OK;
  return fail(TG_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Per-device capability cache: 0 = unknown, 1 = supported, -1 = not supported.
static int g_dev_ok[64];
static int g_dev_sms[64];

tg_status check_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(TG_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  if (g_dev_ok[dev] == 0) {
    cudaDeviceProp p;
    e = cudaGetDeviceProperties(&p, dev);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetDeviceProperties");
    g_dev_ok[dev] = (p.major == 10) ? 1 : -1;
    g_dev_sms[dev] = p.multiProcessorCount;
  }
  if (g_dev_ok[dev] < 0)
    return fail(TG_ERR_UNSUPPORTED, "libtokengate is built for sm_100a (B200); device %d is not", dev);
  return TG_OK;
}

static bool g_attr_set[ATTR_ALL][64];  // the forward path's slots, then the backward's

static int current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  return (dev >= 0 && dev < 64) ? dev : -1;
}

bool attrs_needed(int slot) {
  const int dev = current_device();
  return dev < 0 || !g_attr_set[slot][dev];
}

void mark_attrs_set(int slot) {
  const int dev = current_device();
  if (dev >= 0) g_attr_set[slot][dev] = true;
}

int device_sm_count() {
  int dev = 0;
  cudaGetDevice(&dev);
  return (dev >= 0 && dev < 64 && g_dev_sms[dev] > 0) ? g_dev_sms[dev] : 148;
}

bool pdl_enabled(int kernel_id) {
  static int mask = -1;
  if (mask < 0) {
    const char* off = getenv("TG_DISABLE_PDL");
    const char* m = getenv("TG_PDL_MASK");
    mask = (off && off[0] && off[0] != '0') ? 0 : (m ? atoi(m) : 63);
  }
  return (mask & kernel_id) != 0;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static size_t esize(tg_dtype dt) { return dt == TG_BF16 ? 2 : 4; }

static tg_status check_seqs(const tg_seqs* s, int64_t* n_tot, int64_t* m_tot) {
  if (!s) return fail(TG_ERR_INVALID_ARG, "seqs is NULL");
  if (s->B < 0) return fail(TG_ERR_INVALID_ARG, "seqs->B < 0");
  if (s->B > 0 && (!s->seqlens || !s->q_len || !s->k))
    return fail(TG_ERR_INVALID_ARG, "seqs arrays are NULL");
  int64_t n = 0, m = 0;
  for (int b = 0; b < s->B; ++b) {
    int32_t N = s->seqlens[b], q = s->q_len[b];
    if (N < 0 || q < 0 || q > N)
      return fail(TG_ERR_INVALID_ARG, "sequence %d: need 0 <= q_len (%d) <= seqlen (%d)", b, q, N);
    if (N - q > TG_MAX_CTX)
      return fail(TG_ERR_UNSUPPORTED, "sequence %d: context %d exceeds TG_MAX_CTX", b, N - q);
    int32_t kc = s->k[b] < 0 ? 0 : (s->k[b] > N - q ? N - q : s->k[b]);
    n += N;
    m += kc + q;
  }
  if (n > INT32_MAX) return fail(TG_ERR_UNSUPPORTED, "total tokens exceed int32 indexing");
  if (n_tot) *n_tot = n;
  if (m_tot) *m_tot = m;
  return TG_OK;
}

static int32_t kept_rows(const tg_seqs* s, int b) {
  int32_t N = s->seqlens[b], q = s->q_len[b];
  int32_t kc = s->k[b] < 0 ? 0 : (s->k[b] > N - q ? N - q : s->k[b]);
  return kc + q;
}

}  // namespace tg

using namespace tg;

extern "C" {

const char* tg_status_string(int32_t st) {
  switch (st) {
    case TG_OK: return "TG_OK";
    case TG_ERR_INVALID_ARG: return "TG_ERR_INVALID_ARG";
    case TG_ERR_UNSUPPORTED: return "TG_ERR_UNSUPPORTED";
    case TG_ERR_WORKSPACE: return "TG_ERR_WORKSPACE";
    case TG_ERR_CUDA: return "TG_ERR_CUDA";
    case TG_ERR_DEVICE_CHECK: return "TG_ERR_DEVICE_CHECK";
    case TG_ERR_DEVICE_TIMEOUT: return "TG_ERR_DEVICE_TIMEOUT";
    default: return "TG_ERR_UNKNOWN";
  }
}

const char* tg_last_error(void) { return g_err; }

int32_t tg_version(void) { return (1 << 16) | 3; }

tg_status tg_set_test_wait_probe(int64_t limit_ns) {
  g_err[0] = 0;
  if (limit_ns < 0) return fail(TG_ERR_INVALID_ARG, "limit_ns < 0");
  g_wait_probe_ns = (uint64_t)limit_ns;
  return TG_OK;
}

tg_status tg_kept_counts(const tg_seqs* seqs, int32_t* cu_kept_host) {
  g_err[0] = 0;
  tg_status st = check_seqs(seqs, nullptr, nullptr);
  if (st != TG_OK) return st;
  if (!cu_kept_host) return fail(TG_ERR_INVALID_ARG, "cu_kept_host is NULL");
  int64_t acc = 0;
  cu_kept_host[0] = 0;
  for (int b = 0; b < seqs->B; ++b) {
    acc += kept_rows(seqs, b);
    cu_kept_host[b + 1] = (int32_t)acc;
  }
  return TG_OK;
}

tg_status tg_score(tg_dtype dtype, const void* H, int64_t ldh, int64_t n_tok, int32_t d,
                   const void* W1, const float* b1, const void* w2, float b2, float temperature,
                   int32_t dg, float* score, int32_t* dev_status, void* stream) {
  g_err[0] = 0;
  if (!(temperature > 0.f) || temperature == INFINITY)
    return fail(TG_ERR_INVALID_ARG, "temperature must be positive and finite");
  if (dtype != TG_F32 && dtype != TG_BF16) return fail(TG_ERR_INVALID_ARG, "bad dtype %d", (int)dtype);
  if (n_tok < 0 || d <= 0 || dg <= 0 || ldh < d)
    return fail(TG_ERR_INVALID_ARG, "need n_tok >= 0, d > 0, dg > 0, ldh >= d");
  if (n_tok > INT32_MAX) return fail(TG_ERR_UNSUPPORTED, "n_tok exceeds int32 indexing");
  if (n_tok == 0) return TG_OK;
  if (!H || !W1 || !w2 || !score) return fail(TG_ERR_INVALID_ARG, "H, W1, w2 and score are required");
  if (dg != 64 && dg != 128 && dg != 256) return fail(TG_ERR_UNSUPPORTED, "dg must be 64, 128 or 256");
  if (d % 64) return fail(TG_ERR_UNSUPPORTED, "d must be a multiple of 64");
  if (!aligned16(H) || !aligned16(W1) || (ldh * esize(dtype)) % 16)
    return fail(TG_ERR_UNSUPPORTED, "H and W1 must be 16-byte aligned with 16-byte row strides");
  tg_status st = check_device();
  if (st != TG_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const float inv_t = (float)(1.0 / (double)temperature);
  if (dtype == TG_BF16) return launch_score_tc(H, ldh, n_tok, d, W1, b1, w2, b2, inv_t, dg, score, dev_status, s);
  return launch_score_simt(dtype, H, ldh, n_tok, d, W1, b1, w2, b2, inv_t, dg, score, s);
}

// The selector with optional per-row outputs pos, g and log g (the chained prefill).
// Per-sequence descriptors of the select (seqs already checked).
static std::vector<SelSeq> sel_seqs(const tg_seqs* seqs) {
  std::vector<SelSeq> d(seqs->B);
  int64_t start = 0, off = 0;
  for (int b = 0; b < seqs->B; ++b) {
    int32_t N = seqs->seqlens[b], q = seqs->q_len[b];
    int32_t m = kept_rows(seqs, b);
    d[b] = SelSeq{(int32_t)start, N - q, q, m - q, (int32_t)off, b, (int32_t)(start + N - q), (int32_t)start};
    start += N;
    off += m;
  }
  return d;
}

static tg_status select_impl(const float* score, const tg_seqs* seqs, int32_t* kept_idx, int32_t* cu_kept_dev,
                             int32_t* dev_status, void* stream, int32_t* pos, float* g, float* logg,
                             uint32_t flags) {
  int64_t n_tot = 0, m_tot = 0;
  tg_status st = check_seqs(seqs, &n_tot, &m_tot);
  if (st != TG_OK) return st;
  if (seqs->B == 0) return TG_OK;
  if ((n_tot > 0 && !score) || (m_tot > 0 && !kept_idx))
    return fail(TG_ERR_INVALID_ARG, "score and kept_idx are required");
  st = check_device();
  if (st != TG_OK) return st;
  const std::vector<SelSeq> d = sel_seqs(seqs);
  cudaStream_t s = (cudaStream_t)stream;
  for (int b0 = 0; b0 < seqs->B; b0 += kMaxSeqPerLaunch) {
    int nb = seqs->B - b0 < kMaxSeqPerLaunch ? seqs->B - b0 : kMaxSeqPerLaunch;
    int nmax = 0;
    for (int i = 0; i < nb; ++i) nmax = d[b0 + i].n_ctx > nmax ? d[b0 + i].n_ctx : nmax;
    st = launch_select(score, d.data() + b0, nb, nmax, kept_idx, cu_kept_dev, dev_status, s, pos, g, logg, flags);
    if (st != TG_OK) return st;
  }
  return TG_OK;
}

tg_status tg_topk_select(const float* score, const tg_seqs* seqs, int32_t* kept_idx,
                         int32_t* cu_kept_dev, int32_t* dev_status, void* stream) {
  g_err[0] = 0;
  return select_impl(score, seqs, kept_idx, cu_kept_dev, dev_status, stream, nullptr, nullptr, nullptr, 0);
}

size_t tg_topk_select_stream_workspace_size(const tg_seqs* seqs) {
  int64_t n_tot = 0, m_tot = 0;
  if (check_seqs(seqs, &n_tot, &m_tot) != TG_OK || seqs->B == 0) return 0;
  const std::vector<SelSeq> d = sel_seqs(seqs);
  return (size_t)select_stream_workspace(d.data(), seqs->B);
}

tg_status tg_topk_select_stream(const float* score, const tg_seqs* seqs, int32_t* kept_idx, int32_t* cu_kept_dev,
                                void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  g_err[0] = 0;
  int64_t n_tot = 0, m_tot = 0;
  tg_status st = check_seqs(seqs, &n_tot, &m_tot);
  if (st != TG_OK) return st;
  if (seqs->B == 0) return TG_OK;
  if ((n_tot > 0 && !score) || (m_tot > 0 && !kept_idx))
    return fail(TG_ERR_INVALID_ARG, "score and kept_idx are required");
  const std::vector<SelSeq> d = sel_seqs(seqs);
  const int64_t need = select_stream_workspace(d.data(), seqs->B);
  if (!ws || ws_bytes < (size_t)need || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(TG_ERR_WORKSPACE, "tg_topk_select_stream: the workspace needs %lld bytes at a 256-byte aligned address",
                (long long)need);
  st = check_device();
  if (st != TG_OK) return st;
  return launch_select_stream(score, d.data(), seqs->B, kept_idx, cu_kept_dev, dev_status, ws, (cudaStream_t)stream);
}

tg_status tg_qkv_rope(tg_dtype dtype, const void* H_kept, int64_t M, int32_t d, const void* W_qkv,
                      const int32_t* pos, int32_t Hq, int32_t Hkv, int32_t D, float rope_theta, void* Q, void* K,
                      void* V, int32_t* dev_status, void* stream) {
  g_err[0] = 0;
  if (dtype != TG_BF16) return fail(TG_ERR_UNSUPPORTED, "tg_qkv_rope runs on bf16 only");
  if (M < 0 || d <= 0 || Hq <= 0 || Hkv <= 0) return fail(TG_ERR_INVALID_ARG, "need M >= 0 and d, Hq, Hkv > 0");
  if (M > INT32_MAX) return fail(TG_ERR_UNSUPPORTED, "M too large");
  if (d % 64) return fail(TG_ERR_UNSUPPORTED, "d must be a multiple of 64");
  if (D != 64 && D != 128) return fail(TG_ERR_UNSUPPORTED, "D must be 64 or 128");
  if (((int64_t)(Hq + 2 * Hkv) * D) % 256) return fail(TG_ERR_UNSUPPORTED, "(Hq + 2 Hkv) * D must be a multiple of 256");
  if (!(rope_theta == rope_theta)) return fail(TG_ERR_INVALID_ARG, "rope_theta is NaN");
  if (M == 0) return TG_OK;
  if (!H_kept || !W_qkv || !Q || !K || !V || (rope_theta > 0.f && !pos))
    return fail(TG_ERR_INVALID_ARG, "H_kept, W_qkv, Q, K, V (and pos when rope_theta > 0) are required");
  if (!aligned16(H_kept) || !aligned16(W_qkv) || !aligned16(Q) || !aligned16(K) || !aligned16(V))
    return fail(TG_ERR_UNSUPPORTED, "H_kept, W_qkv, Q, K and V must be 16-byte aligned");
  tg_status st = check_device();
  if (st != TG_OK) return st;
  return launch_qkv_rope(H_kept, M, d, W_qkv, pos, Hq, Hkv, D, rope_theta, Q, K, V, dev_status, (cudaStream_t)stream);
}

tg_status tg_topk_candidates(const float* score, int32_t n, int32_t k, int32_t base, float* cand_score,
                             int32_t* cand_idx, int32_t* dev_status, void* stream) {
  g_err[0] = 0;
  if (n < 0 || k < 0 || base < 0) return fail(TG_ERR_INVALID_ARG, "need n, k, base >= 0");
  if (n > TG_MAX_CTX) return fail(TG_ERR_UNSUPPORTED, "block of %d tokens exceeds TG_MAX_CTX", n);
  const int32_t kc = k < n ? k : n;
  if (kc == 0) return TG_OK;
  if (!score || !cand_score || !cand_idx) return fail(TG_ERR_INVALID_ARG, "score, cand_score and cand_idx are required");
  tg_status st = check_device();
  if (st != TG_OK) return st;
  const SelSeq d{0, n, 0, kc, 0, 0, n, base};
  return launch_select(score, &d, 1, n, cand_idx, nullptr, dev_status, (cudaStream_t)stream, nullptr, nullptr,
                       nullptr, 0, nullptr, cand_score);
}

tg_status tg_topk_merge(const float* cand_score, const int32_t* cand_idx, int32_t n_cand, int32_t k,
                        int32_t q_start, int32_t q, int32_t* kept_idx, int32_t* dev_status, void* stream) {
  g_err[0] = 0;
  if (n_cand < 0 || k < 0 || q < 0 || q_start < 0) return fail(TG_ERR_INVALID_ARG, "need n_cand, k, q, q_start >= 0");
  if (n_cand > TG_MAX_CTX) return fail(TG_ERR_UNSUPPORTED, "%d candidates exceed TG_MAX_CTX", n_cand);
  const int32_t kc = k < n_cand ? k : n_cand;
  if (kc + q == 0) return TG_OK;
  if (!kept_idx || (n_cand > 0 && (!cand_score || !cand_idx)))
    return fail(TG_ERR_INVALID_ARG, "kept_idx (and cand_score, cand_idx) are required");
  tg_status st = check_device();
  if (st != TG_OK) return st;
  const SelSeq d{0, n_cand, q, kc, 0, 0, q_start, 0};
  return launch_select(cand_score, &d, 1, n_cand, kept_idx, nullptr, dev_status, (cudaStream_t)stream, nullptr,
                       nullptr, nullptr, 0, cand_idx, nullptr);
}

tg_status tg_gather(tg_dtype dtype, const void* H, int64_t ldh, int32_t d, const float* score,
                    const int32_t* kept_idx, const tg_seqs* seqs, uint32_t flags, void* H_kept,
                    int32_t* pos, float* g, float* logg, int32_t* dev_status, void* stream) {
  g_err[0] = 0;
  if (dtype != TG_F32 && dtype != TG_BF16) return fail(TG_ERR_INVALID_ARG, "bad dtype %d", (int)dtype);
  int64_t n_tot = 0, m_tot = 0;
  tg_status st = check_seqs(seqs, &n_tot, &m_tot);
  if (st != TG_OK) return st;
  if (d <= 0 || ldh < d) return fail(TG_ERR_INVALID_ARG, "need d > 0 and ldh >= d");
  if (m_tot == 0) return TG_OK;
  if (!H || !kept_idx || !H_kept || !pos || ((g || logg) && !score))
    return fail(TG_ERR_INVALID_ARG, "H, kept_idx, H_kept, pos (and score for g/logg) are required");
  if (!aligned16(H) || !aligned16(H_kept) || (ldh * esize(dtype)) % 16 || (d * esize(dtype)) % 16)
    return fail(TG_ERR_UNSUPPORTED, "H/H_kept must be 16-byte aligned with 16-byte rows");
  st = check_device();
  if (st != TG_OK) return st;
  std::vector<GatherSeq> v(seqs->B);
  int64_t start = 0, off = 0;
  for (int b = 0; b < seqs->B; ++b) {
    int32_t m = kept_rows(seqs, b);
    v[b] = GatherSeq{(int32_t)start, seqs->seqlens[b], seqs->q_len[b], (int32_t)off, m};
    start += seqs->seqlens[b];
    off += m;
  }
  cudaStream_t s = (cudaStream_t)stream;
  for (int b0 = 0; b0 < seqs->B; b0 += kMaxSeqPerLaunch) {
    int nb = seqs->B - b0 < kMaxSeqPerLaunch ? seqs->B - b0 : kMaxSeqPerLaunch;
    int m_chunk = 0;
    for (int i = 0; i < nb; ++i) m_chunk += v[b0 + i].m;
    if (m_chunk == 0) continue;
    st = launch_gather(dtype, H, ldh, d, score, kept_idx, v.data() + b0, nb, m_chunk, flags, H_kept,
                       pos, g, logg, dev_status, s);
    if (st != TG_OK) return st;
  }
  return TG_OK;
}

// qkv_ready: Q, K and V are inputs of the whole chain (the chained prefill), so the kernel may
// load them before it waits on the previous kernel.
static tg_status attn_impl(tg_dtype dtype, const void* Q, const void* K, const void* V, const float* logg,
                           const float* head_gain, const int32_t* pos, const int32_t* cu_kept_host, int32_t B,
                           int32_t Hq, int32_t Hkv, int32_t D, float softmax_scale, uint32_t flags, void* O,
                           float* lse, int32_t* dev_status, void* stream, bool qkv_ready) {
  if (dtype != TG_F32 && dtype != TG_BF16) return fail(TG_ERR_INVALID_ARG, "bad dtype %d", (int)dtype);
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0) return fail(TG_ERR_INVALID_ARG, "need B >= 0 and Hq, Hkv, D > 0");
  if (B > 0 && !cu_kept_host) return fail(TG_ERR_INVALID_ARG, "cu_kept_host is NULL");
  if (Hq % Hkv) return fail(TG_ERR_UNSUPPORTED, "Hq must be a multiple of Hkv");
  if (D != 64 && D != 128) return fail(TG_ERR_UNSUPPORTED, "D must be 64 or 128");
  if (!(softmax_scale == softmax_scale)) return fail(TG_ERR_INVALID_ARG, "softmax_scale is NaN");
  if (B == 0) return TG_OK;
  if (cu_kept_host[0] != 0) return fail(TG_ERR_INVALID_ARG, "cu_kept_host[0] must be 0");
  for (int b = 0; b < B; ++b)
    if (cu_kept_host[b + 1] < cu_kept_host[b]) return fail(TG_ERR_INVALID_ARG, "cu_kept_host not monotone");
  int64_t m_tot = cu_kept_host[B];
  if (m_tot == 0) return TG_OK;
  if (!Q || !K || !V || !pos || !O) return fail(TG_ERR_INVALID_ARG, "Q, K, V, pos and O are required");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return fail(TG_ERR_UNSUPPORTED, "Q, K, V and O must be 16-byte aligned");
  tg_status st = check_device();
  if (st != TG_OK) return st;
  AttnArgs a{dtype, Q, K, V, logg, head_gain, pos, Hq, Hkv, D, softmax_scale, flags, O, lse, dev_status, m_tot};
  a.qkv_ready = qkv_ready;
  std::vector<AttnSeq> v(B);
  for (int b = 0; b < B; ++b) v[b] = AttnSeq{cu_kept_host[b], cu_kept_host[b + 1] - cu_kept_host[b]};
  cudaStream_t s = (cudaStream_t)stream;
  for (int b0 = 0; b0 < B; b0 += kMaxSeqPerLaunch) {
    int nb = B - b0 < kMaxSeqPerLaunch ? B - b0 : kMaxSeqPerLaunch;
    st = (dtype == TG_BF16) ? launch_attn_tc(a, v.data() + b0, nb, s) : launch_attn_simt(a, v.data() + b0, nb, s);
    if (st != TG_OK) return st;
  }
  return TG_OK;
}

tg_status tg_gated_attn_fwd(tg_dtype dtype, const void* Q, const void* K, const void* V,
                            const float* logg, const float* head_gain, const int32_t* pos,
                            const int32_t* cu_kept_host, int32_t B, int32_t Hq, int32_t Hkv,
                            int32_t D, float softmax_scale, uint32_t flags, void* O,
                            float* lse, int32_t* dev_status, void* stream) {
  g_err[0] = 0;
  return attn_impl(dtype, Q, K, V, logg, head_gain, pos, cu_kept_host, B, Hq, Hkv, D, softmax_scale, flags, O, lse,
                   dev_status, stream, false);
}

tg_status tg_gated_attn_bwd(tg_dtype dtype, const void* Q, const void* K, const void* V,
                            const float* logg, const float* head_gain, const int32_t* pos,
                            const int32_t* cu_kept_host, int32_t B, int32_t Hq, int32_t Hkv,
                            int32_t D, float softmax_scale, uint32_t flags, const void* O,
                            const float* lse, const void* dO, float* dQ, float* dK, float* dV,
                            float* dlogg, float* dscore, int32_t* dev_status, void* stream) {
  g_err[0] = 0;
  if (dtype != TG_F32 && dtype != TG_BF16) return fail(TG_ERR_INVALID_ARG, "bad dtype %d", (int)dtype);
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0) return fail(TG_ERR_INVALID_ARG, "need B >= 0 and Hq, Hkv, D > 0");
  if (B > 0 && !cu_kept_host) return fail(TG_ERR_INVALID_ARG, "cu_kept_host is NULL");
  if (Hq % Hkv) return fail(TG_ERR_UNSUPPORTED, "Hq must be a multiple of Hkv");
  if (D != 64 && D != 128) return fail(TG_ERR_UNSUPPORTED, "D must be 64 or 128");
  if (flags & TG_ATTN_UNNORMALISED)
    return fail(TG_ERR_UNSUPPORTED, "the backward covers the normalised form only");
  if (!(softmax_scale == softmax_scale)) return fail(TG_ERR_INVALID_ARG, "softmax_scale is NaN");
  if (dscore && !logg) return fail(TG_ERR_INVALID_ARG, "dscore needs logg");
  if (B == 0) return TG_OK;
  if (cu_kept_host[0] != 0) return fail(TG_ERR_INVALID_ARG, "cu_kept_host[0] must be 0");
  for (int b = 0; b < B; ++b)
    if (cu_kept_host[b + 1] < cu_kept_host[b]) return fail(TG_ERR_INVALID_ARG, "cu_kept_host not monotone");
  const int64_t m_tot = cu_kept_host[B];
  if (m_tot == 0) return TG_OK;
  if (!Q || !K || !V || !pos || !O || !lse || !dO || !dQ || !dK || !dV)
    return fail(TG_ERR_INVALID_ARG, "Q, K, V, pos, O, lse, dO, dQ, dK and dV are required");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(dO) || !aligned16(dQ) || !aligned16(dK) ||
      !aligned16(dV))
    return fail(TG_ERR_UNSUPPORTED, "Q, K, V, dO, dQ, dK and dV must be 16-byte aligned");
  tg_status st = check_device();
  if (st != TG_OK) return st;
  AttnBwdArgs a{dtype, Q, K, V, O, dO, logg, head_gain, pos, lse, Hq, Hkv, D, softmax_scale,
                dQ, dK, dV, dlogg, dscore, dev_status, m_tot};
  std::vector<AttnSeq> v(B);
  for (int b = 0; b < B; ++b) v[b] = AttnSeq{cu_kept_host[b], cu_kept_host[b + 1] - cu_kept_host[b]};
  for (int b0 = 0; b0 < B; b0 += kMaxSeqPerLaunch) {
    const int nb = B - b0 < kMaxSeqPerLaunch ? B - b0 : kMaxSeqPerLaunch;
    st = launch_attn_bwd(a, v.data() + b0, nb, (cudaStream_t)stream);
    if (st != TG_OK) return st;
  }
  return TG_OK;
}

static tg_status gate_bwd_check(tg_dtype dtype, int64_t M, int32_t d, int32_t dg, float temperature) {
  if (dtype != TG_F32 && dtype != TG_BF16) return fail(TG_ERR_INVALID_ARG, "bad dtype %d", (int)dtype);
  if (M < 0 || d <= 0 || dg <= 0) return fail(TG_ERR_INVALID_ARG, "need M >= 0 and d, dg > 0");
  if (M > INT32_MAX) return fail(TG_ERR_UNSUPPORTED, "M exceeds int32 indexing");
  if (d % 64 || dg % 64) return fail(TG_ERR_UNSUPPORTED, "d and dg must be multiples of 64");
  if (!(temperature > 0.f) || temperature == INFINITY)
    return fail(TG_ERR_INVALID_ARG, "temperature must be positive and finite");
  return TG_OK;
}

size_t tg_gate_mlp_bwd_workspace_size(int64_t M, int32_t d, int32_t dg) {
  if (M <= 0 || d <= 0 || dg <= 0 || d % 64 || dg % 64) return 0;
  return (size_t)gate_bwd_plan(M, d, dg, device_sm_count()).bytes;
}

tg_status tg_gate_mlp_bwd(tg_dtype dtype, const void* H_kept, int64_t M, int32_t d, const void* W1,
                          const float* b1, const void* w2, float temperature, int32_t dg, const float* dscore,
                          float* dW1, float* db1, float* dw2, float* db2, void* ws, size_t ws_bytes,
                          int32_t* dev_status, void* stream) {
  g_err[0] = 0;
  tg_status st = gate_bwd_check(dtype, M, d, dg, temperature);
  if (st != TG_OK) return st;
  if (!dW1) return fail(TG_ERR_INVALID_ARG, "dW1 is required");
  if (M == 0) {  // no rows: every gradient is zero
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(dW1, 0, (size_t)dg * d * 4, s);
    if (e == cudaSuccess && db1) e = cudaMemsetAsync(db1, 0, (size_t)dg * 4, s);
    if (e == cudaSuccess && dw2) e = cudaMemsetAsync(dw2, 0, (size_t)dg * 4, s);
    if (e == cudaSuccess && db2) e = cudaMemsetAsync(db2, 0, 4, s);
    return cuda_status(e, "tg_gate_mlp_bwd: zeroing the gradients");
  }
  if (!H_kept || !W1 || !w2 || !dscore) return fail(TG_ERR_INVALID_ARG, "H_kept, W1, w2 and dscore are required");
  if (!aligned16(H_kept) || !aligned16(W1) || !aligned16(dW1))
    return fail(TG_ERR_UNSUPPORTED, "H_kept, W1 and dW1 must be 16-byte aligned");
  const GateBwdPlan p = gate_bwd_plan(M, d, dg, device_sm_count());
  if (!ws || ws_bytes < (size_t)p.bytes || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(TG_ERR_WORKSPACE, "the workspace needs %lld bytes at a 256-byte aligned address",
                (long long)p.bytes);
  st = check_device();
  if (st != TG_OK) return st;
  return launch_gate_bwd(dtype, H_kept, M, d, W1, b1, w2, (float)(1.0 / (double)temperature), dg, dscore, dW1, db1,
                         dw2, db2, ws, p, dev_status, (cudaStream_t)stream);
}

tg_status tg_gate_mlp_bwd_noalloc(tg_dtype dtype, const void* H_kept, int64_t M, int32_t d, const void* W1,
                                  const float* b1, const void* w2, float temperature, int32_t dg,
                                  const float* dscore, float* dW1, float* db1, float* dw2, float* db2,
                                  int32_t* dev_status, void* stream) {
  g_err[0] = 0;
  tg_status st = gate_bwd_check(dtype, M, d, dg, temperature);
  if (st != TG_OK) return st;
  if (M > 0) {
    const GateBwdPlan p = gate_bwd_plan(M, d, dg, device_sm_count());
    if (p.bytes > (int64_t)TG_GATE_NOALLOC_SCRATCH_BYTES)
      return fail(TG_ERR_UNSUPPORTED,
                  "tg_gate_mlp_bwd_noalloc: M=%lld, d=%d, dg=%d need %lld bytes of scratch, more than the fixed "
                  "%lld; use tg_gate_mlp_bwd with a workspace",
                  (long long)M, d, dg, (long long)p.bytes, (long long)TG_GATE_NOALLOC_SCRATCH_BYTES);
    if (!dW1) return fail(TG_ERR_INVALID_ARG, "dW1 is required");
    if (!H_kept || !W1 || !w2 || !dscore) return fail(TG_ERR_INVALID_ARG, "H_kept, W1, w2 and dscore are required");
    if (!aligned16(H_kept) || !aligned16(W1) || !aligned16(dW1))
      return fail(TG_ERR_UNSUPPORTED, "H_kept, W1 and dW1 must be 16-byte aligned");
    st = check_device();
    if (st != TG_OK) return st;
    void* scratch = nullptr;
    st = gate_bwd_fixed_scratch(&scratch);
    if (st != TG_OK) return st;
    return launch_gate_bwd(dtype, H_kept, M, d, W1, b1, w2, (float)(1.0 / (double)temperature), dg, dscore, dW1,
                           db1, dw2, db2, scratch, p, dev_status, (cudaStream_t)stream);
  }
  // no rows: the workspace entry point writes the zero gradients without touching any workspace
  return tg_gate_mlp_bwd(dtype, H_kept, M, d, W1, b1, w2, temperature, dg, dscore, dW1, db1, dw2, db2, nullptr, 0,
                         dev_status, stream);
}

// The row copy of the chained prefill (the selector already wrote pos, g and log g): launched
// after the attention layers, which read nothing it writes, so its first launch starts copying
// at once and waits for them only at its end.
static tg_status gather_rows(tg_dtype dtype, const void* H, int64_t ldh, int32_t d, const int32_t* kept_idx,
                             const tg_seqs* seqs, void* H_kept, int32_t* dev_status, void* stream,
                             bool after_kernel_reads_nothing) {
  if (d <= 0 || ldh < d) return fail(TG_ERR_INVALID_ARG, "need d > 0 and ldh >= d");
  if (!aligned16(H) || !aligned16(H_kept) || (ldh * esize(dtype)) % 16 || (d * esize(dtype)) % 16)
    return fail(TG_ERR_UNSUPPORTED, "H/H_kept must be 16-byte aligned with 16-byte rows");
  std::vector<GatherSeq> v(seqs->B);
  int64_t start = 0, off = 0;
  for (int b = 0; b < seqs->B; ++b) {
    const int32_t m = kept_rows(seqs, b);
    v[b] = GatherSeq{(int32_t)start, seqs->seqlens[b], seqs->q_len[b], (int32_t)off, m};
    start += seqs->seqlens[b];
    off += m;
  }
  bool first = after_kernel_reads_nothing;
  for (int b0 = 0; b0 < seqs->B; b0 += kMaxSeqPerLaunch) {
    const int nb = seqs->B - b0 < kMaxSeqPerLaunch ? seqs->B - b0 : kMaxSeqPerLaunch;
    int m_chunk = 0;
    for (int i = 0; i < nb; ++i) m_chunk += v[b0 + i].m;
    if (m_chunk == 0) continue;
    const tg_status st = launch_gather(dtype, H, ldh, d, nullptr, kept_idx, v.data() + b0, nb, m_chunk, 0, H_kept,
                                       nullptr, nullptr, nullptr, dev_status, (cudaStream_t)stream, first);
    if (st != TG_OK) return st;
    first = false;
  }
  return TG_OK;
}

tg_status tg_prefill_above_L(tg_dtype dtype, const void* H, int64_t ldh, int32_t d,
                             const void* W1, const float* b1, const void* w2, float b2,
                             float temperature, int32_t dg, const tg_seqs* seqs, int32_t n_layers,
                             const void* const* Q, const void* const* K, const void* const* V,
                             int32_t Hq, int32_t Hkv, int32_t D, float softmax_scale,
                             const float* head_gain, uint32_t flags, float* score,
                             int32_t* kept_idx, int32_t* cu_kept_dev, void* H_kept, int32_t* pos,
                             float* g, float* logg, void* const* O, float* const* lse,
                             int32_t* dev_status, void* stream) {
  g_err[0] = 0;
  int64_t n_tot = 0, m_tot = 0;
  tg_status st = check_seqs(seqs, &n_tot, &m_tot);
  if (st != TG_OK) return st;
  if (n_layers < 0) return fail(TG_ERR_INVALID_ARG, "n_layers < 0");
  if (n_layers > 0 && (!Q || !K || !V || !O)) return fail(TG_ERR_INVALID_ARG, "Q/K/V/O arrays are required");
  if (m_tot > 0 && (!score || !kept_idx || !H_kept || !pos || !g || !logg))
    return fail(TG_ERR_INVALID_ARG, "score, kept_idx, H_kept, pos, g and logg are required");
  std::vector<int32_t> cu(seqs->B + 1);
  st = tg_kept_counts(seqs, cu.data());
  if (st != TG_OK) return st;
  st = tg_score(dtype, H, ldh, n_tot, d, W1, b1, w2, b2, temperature, dg, score, dev_status, stream);
  if (st != TG_OK) return st;
  if (dtype != TG_BF16 || n_layers == 0 || m_tot == 0) {
    st = select_impl(score, seqs, kept_idx, cu_kept_dev, dev_status, stream, nullptr, nullptr, nullptr, 0);
    if (st != TG_OK) return st;
    st = tg_gather(dtype, H, ldh, d, score, kept_idx, seqs, flags, H_kept, pos, g, logg, dev_status, stream);
    if (st != TG_OK) return st;
    for (int l = 0; l < n_layers; ++l) {
      st = tg_gated_attn_fwd(dtype, Q[l], K[l], V[l], logg, head_gain, pos, cu.data(), seqs->B, Hq, Hkv, D,
                             softmax_scale, flags, O[l], lse ? lse[l] : nullptr, dev_status, stream);
      if (st != TG_OK) return st;
    }
    return TG_OK;
  }
  // bf16: the selector also writes pos, g and log g of every kept row, so the attention layers
  // follow it directly (their prologue and Q/K loads overlap it), and the copy of the kept rows
  // comes last, filling the SMs that attention's last CTAs leave idle.
  st = select_impl(score, seqs, kept_idx, cu_kept_dev, dev_status, stream, pos, g, logg, flags);
  if (st != TG_OK) return st;
  for (int l = 0; l < n_layers; ++l) {
    st = attn_impl(dtype, Q[l], K[l], V[l], logg, head_gain, pos, cu.data(), seqs->B, Hq, Hkv, D, softmax_scale,
                   flags, O[l], lse ? lse[l] : nullptr, dev_status, stream, true);
    if (st != TG_OK) return st;
  }
  return gather_rows(dtype, H, ldh, d, kept_idx, seqs, H_kept, dev_status, stream, true);
}

tg_status tg_prefill_projected(tg_dtype dtype, const void* H, int64_t ldh, int32_t d, const void* W1,
                               const float* b1, const void* w2, float b2, float temperature, int32_t dg,
                               const tg_seqs* seqs, int32_t n_layers, const void* const* W_qkv, float rope_theta,
                               int32_t Hq, int32_t Hkv, int32_t D, float softmax_scale, const float* head_gain,
                               uint32_t flags, float* score, int32_t* kept_idx, int32_t* cu_kept_dev, void* H_kept,
                               int32_t* pos, float* g, float* logg, void* const* Q, void* const* K_cache,
                               void* const* V_cache, void* const* O, float* const* lse, int32_t* dev_status,
                               void* stream) {
  g_err[0] = 0;
  if (dtype != TG_BF16) return fail(TG_ERR_UNSUPPORTED, "tg_prefill_projected runs on bf16 only");
  int64_t n_tot = 0, m_tot = 0;
  tg_status st = check_seqs(seqs, &n_tot, &m_tot);
  if (st != TG_OK) return st;
  if (n_layers < 0) return fail(TG_ERR_INVALID_ARG, "n_layers < 0");
  if (n_layers > 0 && (!W_qkv || !Q || !K_cache || !V_cache || !O))
    return fail(TG_ERR_INVALID_ARG, "W_qkv, Q, K_cache, V_cache and O arrays are required");
  if (m_tot > 0 && (!score || !kept_idx || !H_kept || !pos || !g || !logg))
    return fail(TG_ERR_INVALID_ARG, "score, kept_idx, H_kept, pos, g and logg are required");
  if (!(rope_theta == rope_theta)) return fail(TG_ERR_INVALID_ARG, "rope_theta is NaN");
  for (int l = 0; l < n_layers; ++l)
    if (!W_qkv[l] || !Q[l] || !K_cache[l] || !V_cache[l] || !O[l])
      return fail(TG_ERR_INVALID_ARG, "layer %d: W_qkv, Q, K_cache, V_cache and O are required", l);
  std::vector<int32_t> cu(seqs->B + 1);
  st = tg_kept_counts(seqs, cu.data());
  if (st != TG_OK) return st;
  st = tg_score(dtype, H, ldh, n_tot, d, W1, b1, w2, b2, temperature, dg, score, dev_status, stream);
  if (st != TG_OK) return st;
  // the selector writes pos, g and log g; the row copy follows it (the projections read H_kept)
  st = select_impl(score, seqs, kept_idx, cu_kept_dev, dev_status, stream, pos, g, logg, flags);
  if (st != TG_OK || m_tot == 0) return st;
  st = gather_rows(dtype, H, ldh, d, kept_idx, seqs, H_kept, dev_status, stream, false);
  if (st != TG_OK) return st;
  for (int l = 0; l < n_layers; ++l) {
    st = tg_qkv_rope(dtype, H_kept, m_tot, d, W_qkv[l], pos, Hq, Hkv, D, rope_theta, Q[l], K_cache[l], V_cache[l],
                     dev_status, stream);
    if (st != TG_OK) return st;
    st = attn_impl(dtype, Q[l], K_cache[l], V_cache[l], logg, head_gain, pos, cu.data(), seqs->B, Hq, Hkv, D,
                   softmax_scale, flags, O[l], lse ? lse[l] : nullptr, dev_status, stream, false);
    if (st != TG_OK) return st;
  }
  return TG_OK;
}

}  // extern "C"
