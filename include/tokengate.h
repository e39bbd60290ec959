/*
 * tokengate.h - C ABI of the TokenGate gated-prefill hot path for NVIDIA B200 (sm_100a).
 *
 * The method (TokenGate: Adapting LLMs for Fast and Memory-Efficient Prefill with Learned
 * Token Pruning): at a selection layer L a small gate MLP scores every token's hidden
 * state; a top-K selector keeps K context tokens and always keeps the question tail; the
 * kept hidden states travel upward with their gate values and original positions; every
 * layer above L runs token-gated causal attention over the kept tokens only, each
 * attention weight multiplied by its key's gate value g_j (row renormalised).
 *
 * Conventions shared by every entry point
 *   - Memory: every buffer is owned by the caller. Pointers named "device" must be CUDA
 *     device memory of the current device; "host" pointers are ordinary host memory that
 *     is read before the call returns. No entry point allocates or frees memory.
 *   - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     All GPU work is enqueued asynchronously on it; nothing synchronises the host and no
 *     device-to-host copy is made, so a chain of calls can be captured in a CUDA graph.
 *   - Layout: tokens are packed back to back ("varlen", token-major). Sequence b occupies
 *     rows [cu_seqlens[b], cu_seqlens[b+1]) of the hidden states and rows
 *     [cu_kept[b], cu_kept[b+1]) of every kept-token tensor.
 *   - Errors: argument problems are reported synchronously before anything is launched
 *     (TG_ERR_INVALID_ARG / TG_ERR_UNSUPPORTED). A failed launch returns TG_ERR_CUDA.
 *     Problems found by the kernels are OR-ed into the optional device status word
 *     (int32, TG_DEV_* bits), which the caller zeroes beforehand and reads after a sync.
 *     No kernel traps, asserts or waits without a bound. tg_last_error() describes the
 *     most recent failure on the calling thread.
 *   - dtype: TG_F32 means every floating-point tensor named "act" below is float32;
 *     TG_BF16 means bfloat16. Biases, scores, gate values, LSE are always float32.
 */
#ifndef TOKENGATE_H
#define TOKENGATE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TG_OK = 0,
  TG_ERR_INVALID_ARG = 1,   /* null pointer, negative size, inconsistent sizes */
  TG_ERR_UNSUPPORTED = 2,   /* valid but outside the supported shapes / alignment / GPU */
  TG_ERR_WORKSPACE = 3,     /* the workspace is missing, too small or misaligned */
  TG_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  TG_ERR_DEVICE_CHECK = 5,  /* reserved for callers that map TG_DEV_* bits to a status */
  TG_ERR_DEVICE_TIMEOUT = 6 /* reserved for callers that map TG_DEV_TIMEOUT to a status */
} tg_status;

typedef enum { TG_F32 = 0, TG_BF16 = 1 } tg_dtype;

/* flags */
#define TG_ATTN_UNNORMALISED (1u << 0) /* weight times g_j without renormalising the row */
#define TG_QUESTION_GATE_ONE (1u << 1) /* question-tail rows get g = 1 (log g = 0)       */

/* device status word bits */
#define TG_DEV_NAN_SCORE (1 << 0)        /* a context score was NaN (ranked below -inf) */
#define TG_DEV_POS_NOT_ASCENDING (1 << 1)/* kept positions not strictly ascending         */
#define TG_DEV_TIMEOUT (1 << 2)          /* a bounded wait inside a kernel gave up        */
#define TG_DEV_BAD_INDEX (1 << 3)        /* a kept index lay outside its own sequence     */

/* Limits. A sequence's context (N - q) may hold up to TG_MAX_CTX tokens. */
#define TG_MAX_CTX 262144

/* Per-sequence description of a packed batch. All three arrays are HOST memory of length B.
 * seqlens[b] = N_b >= 0 tokens; q_len[b] = question-tail length, 0 <= q_b <= N_b;
 * k[b] = number of context tokens to keep (values < 0 read as 0, values > N_b - q_b keep
 * the whole context). */
typedef struct {
  int32_t B;
  const int32_t* seqlens;
  const int32_t* q_len;
  const int32_t* k;
} tg_seqs;

/* Human-readable name of a status code. */
const char* tg_status_string(int32_t status);

/* Description of the most recent failed call on this thread ("" if none). */
const char* tg_last_error(void);

/* ABI version, (major << 16) | minor. 1.0: the gated-prefill path (tg_score, tg_topk_select,
 * tg_gather, tg_gated_attn_fwd, tg_prefill_above_L and the helpers). 1.1 adds tg_qkv_rope,
 * tg_topk_candidates, tg_topk_merge and tg_gated_attn_bwd. 1.2 gives tg_score a device
 * status word (its last argument before the stream) and a temperature (after b2, also in
 * tg_prefill_above_L), and adds tg_set_test_wait_probe, tg_gate_mlp_bwd and its
 * workspace query, and tg_prefill_projected. 1.3 adds tg_gate_mlp_bwd_noalloc,
 * tg_topk_select_stream and its workspace query, and gives
 * tg_gate_mlp_bwd a device status word (its last argument before the stream; a changed
 * signature, so 1.2 callers of it must be rebuilt). */
int32_t tg_version(void);

/* Test hook for the bounded waits, off by default (limit_ns = 0). With limit_ns > 0, every
 * tensor-core kernel this calling thread launches afterwards (tg_score, tg_gated_attn_fwd,
 * tg_qkv_rope, tg_gated_attn_bwd, the tensor-core kernels of tg_gate_mlp_bwd and the chain's
 * kernels, bf16) first waits, with that limit, on a barrier that
 * nothing signals, before it issues any copy or product. The wait runs out, the kernel ORs
 * TG_DEV_TIMEOUT into its status word, does none of its work (its outputs are left as they
 * were) and returns; the context stays usable. Only for tests of the timeout path; set 0 to
 * restore normal operation. limit_ns < 0 -> TG_ERR_INVALID_ARG. */
tg_status tg_set_test_wait_probe(int64_t limit_ns);

/* Kept-row offsets (host only, no GPU work). M_b = min(max(k_b, 0), N_b - q_b) + q_b: the
 * K highest-scoring context tokens plus the whole question tail (aitualizate.com TokenGate
 * article, phase 2: only the document part may be pruned, the question never is).
 * cu_kept_host: HOST int32 [B+1], written with the exclusive prefix sums of M_b. */
tg_status tg_kept_counts(const tg_seqs* seqs, int32_t* cu_kept_host);

/* Gate MLP score of every token (aitualizate.com TokenGate article, phase 2: an MLP scores
 * each token's post-attention residual state at layer L; thelatestinai.com TokenGate page,
 * Figure 1(b)):   score[i] = (w2 . GELU(W1 h_i + b1) + b2) / temperature,  GELU with the
 * exact erf. The temperature is a reading of the gate temperature that the thelatestinai.com
 * TokenGate page names in its Figure 7 caption (Eq. 7) without printing a formula: it
 * divides the score, so the gate value is g = sigmoid(s / temperature) and the
 * top-K selection (an order statistic) is the same for every temperature > 0. Pass 1 for the
 * plain score.
 *   H      device act [n_tok, d], row stride ldh elements (ldh >= d)
 *   W1     device act [dg, d] row-major (output-major, like torch.nn.Linear.weight)
 *   b1     device f32 [dg], or NULL for zero
 *   w2     device act [dg]
 *   b2     scalar
 *   temperature  > 0 and finite (else TG_ERR_INVALID_ARG)
 *   score  device f32 [n_tok] (written)
 *   dev_status device int32 [1] or NULL: a wait of the bf16 kernel that gave up sets
 *          TG_DEV_TIMEOUT (the scores of the tiles it did not finish are then unwritten)
 * Supported: dg in {64, 128, 256}; d % 64 == 0; ldh * sizeof(act) % 16 == 0; 16-byte
 * aligned H and W1. bf16 runs on the tensor cores with fp32 accumulation; f32 runs on the
 * CUDA cores in fp32. */
tg_status tg_score(tg_dtype dtype, const void* H, int64_t ldh, int64_t n_tok, int32_t d,
                   const void* W1, const float* b1, const void* w2, float b2, float temperature,
                   int32_t dg, float* score, int32_t* dev_status, void* stream);

/* Top-K over each sequence's context with the question tail always kept (aitualizate.com
 * TokenGate article, phase 2; thelatestinai.com TokenGate page, Figure 1(a)-(b)).
 * Per sequence the min(k_b, N_b - q_b) context tokens with the largest scores are kept;
 * equal scores keep the lower index; -0 equals +0; NaN ranks below -inf (and sets
 * TG_DEV_NAN_SCORE). The kept context indices, ascending, are followed by the q_b tail
 * indices. Exact and deterministic.
 *   score       device f32 [sum N_b]
 *   kept_idx    device int32 [sum M_b] (written): packed row indices into H / score
 *   cu_kept_dev device int32 [B+1] (written) or NULL
 *   dev_status  device int32 [1] or NULL
 * No workspace is needed: per-sequence descriptors travel as kernel parameters and each
 * sequence's histogram lives in the shared memory of its thread-block cluster.
 * Supported: N_b - q_b <= TG_MAX_CTX. */
tg_status tg_topk_select(const float* score, const tg_seqs* seqs, int32_t* kept_idx,
                         int32_t* cu_kept_dev, int32_t* dev_status, void* stream);

/* Workspace bytes tg_topk_select_stream needs for these sequences (0 when seqs is invalid or
 * empty). Host only. About 8 bytes per context token of the sequences that are pruned (the
 * worst case of the candidate lists) plus 1 MiB; at 64 sequences of 131072 tokens, 68 MB. */
size_t tg_topk_select_stream_workspace_size(const tg_seqs* seqs);

/* tg_topk_select for many long sequences at once: the same outputs bit for bit (kept_idx,
 * cu_kept_dev, TG_DEV_NAN_SCORE), computed as a stream over all SMs instead of one thread-block
 * cluster per sequence. The context is cut into chunks of 4096 tokens; four kernels run in
 * stream order: a 12-bit histogram of the order keys per sequence (integer atomics), the bin
 * holding the K-th largest key and the candidates in it, the exact threshold with each chunk's
 * output offset and quota of keys equal to it (lower positions first), and an ascending
 * compaction. The scores are read from HBM once; the later passes find them in L2 while the
 * batch's scores fit there. Deterministic: only integer counts decide anything.
 *   score, seqs, kept_idx, cu_kept_dev, dev_status: as for tg_topk_select
 *   ws       device workspace of at least tg_topk_select_stream_workspace_size(seqs) bytes,
 *            256-byte aligned (TG_ERR_WORKSPACE otherwise); owned by the caller, contents need
 *            no initialisation
 * Supported: N_b - q_b <= TG_MAX_CTX; any number of sequences (launched 64 at a time). */
tg_status tg_topk_select_stream(const float* score, const tg_seqs* seqs, int32_t* kept_idx,
                                int32_t* cu_kept_dev, void* ws, size_t ws_bytes,
                                int32_t* dev_status, void* stream);

/* Projection of the kept rows for a layer above L (aitualizate.com TokenGate article,
 * phase 3: those layers process only the kept tokens, at their original positions). The
 * pages give no projection or rotary details; the reading implemented:
 *   X = H_kept W_qkv^T split into Q [M, Hq, D], K [M, Hkv, D], V [M, Hkv, D];
 *   Q and K rotated at pos: for i < D/2, angle a = pos * rope_theta^(-2i/D),
 *   y[i] = x[i] cos a - x[i+D/2] sin a,  y[i+D/2] = x[i+D/2] cos a + x[i] sin a.
 *   H_kept   device bf16 [M, d] row-major (tg_gather's output)
 *   W_qkv    device bf16 [(Hq + 2 Hkv) D, d] row-major (output-major, like nn.Linear.weight)
 *   pos      device int32 [M] original positions (tg_gather's output); unused if rope_theta <= 0
 *   Q, K, V  device bf16 (written)
 * rope_theta <= 0: no rotation. bf16 only, on the tensor cores (fp32 accumulation; the angle
 * is reduced in double, so positions up to TG_MAX_CTX keep their accuracy).
 * Supported: d % 64 == 0; D in {64, 128}; (Hq + 2 Hkv) D % 256 == 0; 16-byte aligned tensors. */
tg_status tg_qkv_rope(tg_dtype dtype, const void* H_kept, int64_t M, int32_t d, const void* W_qkv,
                      const int32_t* pos, int32_t Hq, int32_t Hkv, int32_t D, float rope_theta, void* Q, void* K,
                      void* V, int32_t* dev_status, void* stream);

/* Sequence-split selection across devices, step 1 (one contiguous block of a sequence's
 * context per device; the merge below is step 2). The min(k, n) tokens of the block with the
 * largest scores, ordered by position, as candidates: cand_idx = base + position in the block
 * and cand_score = that token's score (bit for bit). Every token of the sequence's top-k that
 * lies in this block is among them. Same order and ties as tg_topk_select.
 *   score       device f32 [n]: the block's scores
 *   cand_score  device f32 [min(k, n)] (written);  cand_idx device int32 [min(k, n)] (written)
 * Supported: n <= TG_MAX_CTX. NaN scores set TG_DEV_NAN_SCORE. */
tg_status tg_topk_candidates(const float* score, int32_t n, int32_t k, int32_t base, float* cand_score,
                             int32_t* cand_idx, int32_t* dev_status, void* stream);

/* Step 2: the top-k among the candidates of all blocks, concatenated in block order (so
 * position order is index order and ties keep the lower index), followed by the q question-
 * tail indices q_start .. q_start+q-1. The result equals tg_topk_select over the whole
 * sequence. Candidates must all be real: a block with fewer than k tokens contributes fewer.
 *   kept_idx  device int32 [min(k, n_cand) + q] (written), ascending context indices first
 * Supported: n_cand <= TG_MAX_CTX. */
tg_status tg_topk_merge(const float* cand_score, const int32_t* cand_idx, int32_t n_cand, int32_t k,
                        int32_t q_start, int32_t q, int32_t* kept_idx, int32_t* dev_status, void* stream);

/* Forward the kept hidden states with their gate values and positions (thelatestinai.com
 * TokenGate page, Figure 1(b): the selector forwards the kept hidden states together with
 * their importance scores; aitualizate.com article, phase 3).
 *   H        device act [sum N_b, d], row stride ldh
 *   score    device f32 [sum N_b]
 *   kept_idx device int32 [sum M_b], packed indices as written by tg_topk_select
 *   H_kept   device act [sum M_b, d] contiguous (written; a bit-exact copy of the rows)
 *   pos      device int32 [sum M_b] (written): index of the row within its own sequence
 *   g, logg  device f32 [sum M_b] (written): g = sigmoid(score), log g as a stable
 *            log-sigmoid; with TG_QUESTION_GATE_ONE the tail rows get g = 1, log g = 0.
 *            Either may be NULL.
 * A kept index outside its sequence sets TG_DEV_BAD_INDEX and its row is left unwritten.
 * Supported: d * sizeof(act) % 16 == 0, ldh * sizeof(act) % 16 == 0, 16-byte aligned. */
tg_status tg_gather(tg_dtype dtype, const void* H, int64_t ldh, int32_t d, const float* score,
                    const int32_t* kept_idx, const tg_seqs* seqs, uint32_t flags, void* H_kept,
                    int32_t* pos, float* g, float* logg, int32_t* dev_status, void* stream);

/* Token-gated causal attention over the kept tokens (thelatestinai.com TokenGate page,
 * Figure 1(c): each attention weight is multiplied by its key's gate value g_j; read with
 * the row renormalised this is log g_j added to the logit; aitualizate.com article: the
 * score acts as a bias on the attention logits with a per-head gain). For sequence b,
 * query row i and head h (KV head h / (Hq / Hkv)):
 *   S_ij = softmax_scale * q_i . k_j + gain_h * log g_j   for pos_j <= pos_i (same sequence)
 *   O_i  = sum_j softmax_j(S_ij) v_j ;  lse_i = logsumexp_j S_ij (natural log)
 * With TG_ATTN_UNNORMALISED: O_i = sum_j softmax_j(softmax_scale q_i . k_j) g_j^gain_h v_j
 * and lse is that of the unbiased logits.
 *   Q            device act [sum M_b, Hq, D];  K, V device act [sum M_b, Hkv, D]
 *   logg         device f32 [sum M_b], or NULL for g == 1
 *   head_gain    device f32 [Hq], or NULL for gain 1
 *   pos          device int32 [sum M_b]: must be strictly ascending inside each sequence
 *                (as tg_gather writes them); otherwise TG_DEV_POS_NOT_ASCENDING is set.
 *   cu_kept_host HOST int32 [B+1] kept-row offsets (tg_kept_counts)
 *   O            device act [sum M_b, Hq, D] (written)
 *   lse          device f32 [Hq, sum M_b] (written) or NULL
 * Supported: D in {64, 128}; Hq % Hkv == 0; 16-byte aligned tensors. bf16 runs on the
 * tensor cores (fp32 softmax and accumulation); f32 runs on the CUDA cores in fp32. */
tg_status tg_gated_attn_fwd(tg_dtype dtype, const void* Q, const void* K, const void* V,
                            const float* logg, const float* head_gain, const int32_t* pos,
                            const int32_t* cu_kept_host, int32_t B, int32_t Hq, int32_t Hkv,
                            int32_t D, float softmax_scale, uint32_t flags, void* O,
                            float* lse, int32_t* dev_status, void* stream);

/* Gradients of tg_gated_attn_fwd in its normalised form (thelatestinai.com TokenGate page,
 * Figure 1(c): the gated attention lets the top-K selector train end to end; aitualizate.com
 * article: the score is a bias on the logits, so its gradient is that of an additive bias).
 * With S, P, O and lse as in the forward and the upstream gradient dO, per sequence and head:
 *   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - rowsum(dO * O)),
 *   dQ = scale dS K,  dK = scale dS^T Q  (the query heads of a KV group add into its dK, dV),
 *   dlogg_j  = sum_h gain_h sum_i dS_ij,
 *   dscore_j = dlogg_j * (1 - g_j) = dlogg_j * -expm1(logg_j)  (g = sigmoid(score)).
 * The per-head gain is treated as a constant (no gradient for it).
 *   Q, K, V, logg, head_gain, pos, cu_kept_host, B, Hq, Hkv, D, softmax_scale: as given to
 *                the forward (pos strictly ascending inside each sequence; a violation sets
 *                TG_DEV_POS_NOT_ASCENDING)
 *   O            device act [sum M_b, Hq, D]: the forward's output
 *   lse          device f32 [Hq, sum M_b]: the forward's lse (required)
 *   dO           device act [sum M_b, Hq, D]
 *   dQ           device f32 [sum M_b, Hq, D] (written)
 *   dK, dV       device f32 [sum M_b, Hkv, D] (written)
 *   dlogg        device f32 [sum M_b] (written) or NULL
 *   dscore       device f32 [sum M_b] (written) or NULL; needs logg
 *   dev_status   device int32 [1] or NULL: TG_DEV_POS_NOT_ASCENDING as above; a wait of the
 *                bf16 kernels that gave up sets TG_DEV_TIMEOUT (the gradients are then invalid)
 * f32 runs on the CUDA cores in fp32. bf16 runs its five products on the tensor cores with fp32
 * accumulation (P and dS rounded to bf16 as operands, as the forward rounds P); softmax,
 * rowsum(dO * O) and d log g are fp32. dQ also holds intermediate values until the call's last
 * kernel writes it. No workspace; results are deterministic.
 * Supported: D in {64, 128}; Hq % Hkv == 0; 16-byte aligned Q, K, V, dO, dQ, dK, dV;
 * flags without TG_ATTN_UNNORMALISED (TG_ERR_UNSUPPORTED otherwise). */
tg_status tg_gated_attn_bwd(tg_dtype dtype, const void* Q, const void* K, const void* V,
                            const float* logg, const float* head_gain, const int32_t* pos,
                            const int32_t* cu_kept_host, int32_t B, int32_t Hq, int32_t Hkv,
                            int32_t D, float softmax_scale, uint32_t flags, const void* O,
                            const float* lse, const void* dO, float* dQ, float* dK, float* dV,
                            float* dlogg, float* dscore, int32_t* dev_status, void* stream);

/* Workspace bytes tg_gate_mlp_bwd needs for M kept rows (0 when M <= 0 or the shape is
 * unsupported). Host only; depends on the current device's SM count. */
size_t tg_gate_mlp_bwd_workspace_size(int64_t M, int32_t d, int32_t dg);

/* Gradients of the gate network's parameters from the score gradient of the kept rows: the last
 * link of end-to-end selector training (thelatestinai.com TokenGate page, Figure 1(c): the
 * gated attention lets the top-K selector learn; aitualizate.com article, section on training
 * the top-K selection). With s = (w2 . GELU(W1 h + b1) + b2) / temperature (tg_score) and
 * dscore from tg_gated_attn_bwd, per kept row h: z = W1 h + b1, ds' = dscore / temperature,
 *   dw2 = sum ds' GELU(z),  db2 = sum ds',  u = ds' w2 * GELU'(z),  db1 = sum u,  dW1 = sum u h^T.
 *   H_kept   device act [M, d] contiguous (tg_gather's output; rows the top-K dropped get no
 *            gradient through the selection)
 *   W1, b1, w2, temperature, dg: as given to tg_score (b1 may be NULL)
 *   dscore   device f32 [M]
 *   dW1      device f32 [dg, d] (written, required); db1, dw2 device f32 [dg] and db2 device f32
 *            [1] (written, each may be NULL)
 *   ws       device workspace of at least tg_gate_mlp_bwd_workspace_size(M, d, dg) bytes,
 *            256-byte aligned (TG_ERR_WORKSPACE otherwise); owned by the caller, contents need
 *            no initialisation and are overwritten
 *   dev_status device int32 [1] or NULL: a wait of the bf16 tensor-core kernels that gave up
 *            ORs in TG_DEV_TIMEOUT, and their last kernel then writes none of the outputs (it also
 *            writes none when the word already holds TG_DEV_TIMEOUT); with NULL a timed-out call
 *            leaves invalid gradients. The CUDA-core kernels do not wait and never set it.
 * Arithmetic: bf16 with dg % 128 == 0 and d % 128 == 0 runs on the 5th-generation tensor cores
 * (z = H W1^T and dW1 = u^T H with fp32 accumulation; u is rounded to bf16 as the second
 * product's operand, db1, dw2 and db2 add fp32 values); every other shape, and f32, is fp32 on the
 * CUDA cores. Results are deterministic (fixed reduction orders). M = 0 writes zero gradients.
 * Supported: d % 64 == 0, dg % 64 == 0, 16-byte aligned H_kept, W1 and dW1. */
tg_status tg_gate_mlp_bwd(tg_dtype dtype, const void* H_kept, int64_t M, int32_t d, const void* W1,
                          const float* b1, const void* w2, float temperature, int32_t dg,
                          const float* dscore, float* dW1, float* db1, float* dw2, float* db2,
                          void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/* Size of the fixed device scratch array behind tg_gate_mlp_bwd_noalloc (16 MiB). */
#define TG_GATE_NOALLOC_SCRATCH_BYTES (16u << 20)

/* tg_gate_mlp_bwd for callers that cannot allocate device memory. The pages have no counterpart
 * of this entry point; it exists for callers such as a serving or training runtime that plans
 * all device memory up front and forbids allocations once it runs, a plugin hosted by a
 * framework whose allocator it cannot reach, or a latency-critical loop where cudaMalloc (which
 * may synchronise the device) is not allowed. The arguments and results are those of
 * tg_gate_mlp_bwd without ws / ws_bytes: the working memory is a fixed array of
 * TG_GATE_NOALLOC_SCRATCH_BYTES inside this library, which every GPU that loads the library
 * holds until the process exits. Nothing here calls cudaMalloc, cudaFree or any allocating
 * routine.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress
 *     with that device current); make that first call before any stream capture.
 *   - Shapes whose working memory exceeds the array (tg_gate_mlp_bwd_workspace_size(M, d, dg) >
 *     TG_GATE_NOALLOC_SCRATCH_BYTES; at d = 2048, dg = 256 that is well above 4096 kept rows)
 *     return TG_ERR_UNSUPPORTED before anything is launched.
 *   - Every call on a device shares the one array, which keeps the last call's contents; no part
 *     of it needs clearing (each call writes every byte it reads). Calls whose GPU work overlaps
 *     (different streams, or a stream that does not order them) race on the array: order them. */
tg_status tg_gate_mlp_bwd_noalloc(tg_dtype dtype, const void* H_kept, int64_t M, int32_t d,
                                  const void* W1, const float* b1, const void* w2, float temperature,
                                  int32_t dg, const float* dscore, float* dW1, float* db1,
                                  float* dw2, float* db2, int32_t* dev_status, void* stream);

/* The whole gated path above layer L (aitualizate.com TokenGate article, phases 2-3;
 * thelatestinai.com TokenGate page, Figure 1(a)): the results of tg_score -> tg_topk_select
 * -> tg_gather -> tg_gated_attn_fwd for each of n_layers above-L layers, enqueued on one
 * stream with no host synchronisation. Q, K, V, O, lse are HOST arrays of n_layers device
 * pointers shaped as in tg_gated_attn_fwd (lse may be NULL, or hold NULL entries). The other
 * arguments and outputs are those of the single steps; score, kept_idx, H_kept, pos, g, logg
 * are all required here. Every output is bit-identical to running the single steps in that
 * order. For bf16 with n_layers >= 1 the kernels run in another order: the selector also
 * writes pos, g and log g, the attention layers follow it, and the copy of the kept rows into
 * H_kept comes last (it overlaps the attention's tail). Q, K and V must therefore not alias
 * any output of this call. */
tg_status tg_prefill_above_L(tg_dtype dtype, const void* H, int64_t ldh, int32_t d,
                             const void* W1, const float* b1, const void* w2, float b2,
                             float temperature, int32_t dg, const tg_seqs* seqs, int32_t n_layers,
                             const void* const* Q, const void* const* K, const void* const* V,
                             int32_t Hq, int32_t Hkv, int32_t D, float softmax_scale,
                             const float* head_gain, uint32_t flags, float* score,
                             int32_t* kept_idx, int32_t* cu_kept_dev, void* H_kept, int32_t* pos,
                             float* g, float* logg, void* const* O, float* const* lse,
                             int32_t* dev_status, void* stream);

/* The gated path above layer L with each layer's own projections (aitualizate.com TokenGate
 * article, phase 3: the layers above L work on the kept tokens only, at their original
 * positions, and dropped tokens leave no key/value entries behind; thelatestinai.com TokenGate
 * page, Figure 1(a)). tg_score -> tg_topk_select -> kept rows (H_kept) -> for each layer l:
 * tg_qkv_rope(H_kept, W_qkv[l], pos, rope_theta) into Q[l], K_cache[l], V_cache[l] ->
 * tg_gated_attn_fwd into O[l], lse[l]. K_cache[l] and V_cache[l] [sum M_b, Hkv, D] are the
 * layer's key/value cache, holding the kept rows only. The pages print no projection; each
 * layer here projects the same kept rows with its own matrix (the reading of tg_qkv_rope).
 *   W_qkv, Q, K_cache, V_cache, O, lse: HOST arrays of n_layers device pointers (lse may be
 *            NULL or hold NULL entries); shapes as in tg_qkv_rope and tg_gated_attn_fwd
 *   the other arguments: as in tg_prefill_above_L (score, kept_idx, H_kept, pos, g, logg
 *            required)
 * bf16 only. Every output equals running those entry points one after another. No host
 * synchronisation; the buffers of one layer must not alias another layer's or the chain's. */
tg_status tg_prefill_projected(tg_dtype dtype, const void* H, int64_t ldh, int32_t d, const void* W1,
                               const float* b1, const void* w2, float b2, float temperature, int32_t dg,
                               const tg_seqs* seqs, int32_t n_layers, const void* const* W_qkv,
                               float rope_theta, int32_t Hq, int32_t Hkv, int32_t D, float softmax_scale,
                               const float* head_gain, uint32_t flags, float* score, int32_t* kept_idx,
                               int32_t* cu_kept_dev, void* H_kept, int32_t* pos, float* g, float* logg,
                               void* const* Q, void* const* K_cache, void* const* V_cache, void* const* O,
                               float* const* lse, int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TOKENGATE_H */
