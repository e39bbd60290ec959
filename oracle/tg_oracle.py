"""Plain CPU oracle for the TokenGate gated-prefill hot path (NumPy, float64).

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or links this file:
only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` use it.
It shares no code with the CUDA path; both sides consume the same seeded input bytes.

Sources (web pages about "TokenGate: Adapting LLMs for Fast and Memory-Efficient Prefill
with Learned Token Pruning"):
  * aitualizate.com article "TokenGate acelera prefill LLM con poda inteligente de tokens",
    section "Cómo funciona TokenGate: tres fases para seleccionar los tokens" (phases 1-3)
    and the paragraph on token-gated attention ("Cómo consigue entrenar una selección top-K").
  * thelatestinai.com paper page "TokenGate: Adapting LLMs for Fast and Memory-Efficient
    Prefill with Learned Token Pruning", Figure 1 caption, panels (a)-(c).

Each function is the plain definition of the step it names, written out with library
primitives (matmul, erf, lexsort); nothing is blocked, fused or reordered. Where the pages
leave a step open, the reading taken is stated in the function's docstring:
  * gate map g = sigmoid(score), log g as a stable log-sigmoid;
  * GELU with the exact error function; biases b1 (per hidden unit) and b2 (scalar);
  * K counts the context tokens kept by top-K; the question tail is always added on top;
  * equal scores keep the lower index; -0 equals +0; NaN ranks below -inf;
  * the gate enters attention as log g_j added to the logit (= weight times g_j, then
    row renormalisation); an optional per-head gain multiplies that bias; an
    "unnormalised" variant multiplies the weight by g_j without renormalising;
  * causal mask on original positions (key allowed iff pos_j <= pos_i, same sequence);
    grouped KV heads map query head h to KV head h // (Hq / Hkv).
  * gradients of the attention (for training the selector end to end): the derivative of
    the normalised form above with the per-head gain held constant; the score gradient
    goes through log g = log-sigmoid(s).
  * above-L projections (not on the pages, which stop at "layers above L process the kept
    tokens"): Q/K/V = kept rows times one stacked projection matrix, with rotary position
    embedding on Q and K at each kept token's original position, rotate-half pairing
    (i, i + D/2) and inverse frequencies theta^(-2i/D).

Every function is pinned by tests/test_oracle_pins.py against closed forms, textbook
values, brute force and invariants. Parity is unpinned for nothing in this file.
"""
from __future__ import annotations

import numpy as np
from scipy.special import erf

LOG2E = 1.4426950408889634

# --------------------------------------------------------------------------- phase 2: score


def gelu(z):
    """GELU with the exact error function: z * Phi(z) = 0.5 z (1 + erf(z / sqrt 2))."""
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + erf(z / np.sqrt(2.0)))


def gate_scores(H, W1, b1, w2, b2, temperature=1.0):
    """One scalar importance score per token from its hidden state at layer L.

    aitualizate.com article, phase 2 (a small multilayer network gives every token its own
    score); thelatestinai.com page, Figure 1(b) (a small scoring network scores each hidden
    state). The network is d -> dg -> 1 with GELU:
        s_i = (w2 . GELU(W1 h_i + b1) + b2) / temperature
    H: [n, d]; W1: [dg, d] (output-major, like nn.Linear); b1: [dg] or None; w2: [dg];
    b2: scalar. The hidden layer is kept at full precision (no rounding between layers).
    The temperature is a reading: the thelatestinai.com page names a gate temperature in its
    Figure 7 caption (Eq. 7) but prints no formula; here it divides the score, so the gate
    value becomes sigmoid(s / temperature) and the selected set does not depend on it.
    """
    H = np.asarray(H, dtype=np.float64)
    W1 = np.asarray(W1, dtype=np.float64)
    w2 = np.asarray(w2, dtype=np.float64).reshape(-1)
    z = H @ W1.T
    if b1 is not None:
        z = z + np.asarray(b1, dtype=np.float64)[None, :]
    return (gelu(z) @ w2 + float(b2)) / float(temperature)


def gate_value(s):
    """Gate value g = sigmoid(s) and log g, the latter as a stable log-sigmoid.

    The pages forward each kept token's importance score into attention (thelatestinai.com,
    Figure 1(b)-(c), "gate value g_j") but do not print the score -> g map; sigmoid is the
    reading taken. log g = -log1p(exp(-s)) for s >= 0, s - log1p(exp(s)) otherwise, so it is
    finite for every finite s (no row can become all -inf).
    """
    s = np.asarray(s, dtype=np.float64)
    g = np.empty_like(s)
    pos = s >= 0
    e = np.exp(-np.abs(s))
    g[pos] = 1.0 / (1.0 + e[pos])
    g[~pos] = e[~pos] / (1.0 + e[~pos])
    logg = np.where(pos, -np.log1p(e), s - np.log1p(e))
    return g, logg


# --------------------------------------------------------------------------- phase 2: top-K


def kept_count(n, q, k):
    """Rows kept for one sequence: min(K, N - q) context tokens plus the q question tokens."""
    return min(max(int(k), 0), int(n) - int(q)) + int(q)


def topk_select(s, seqlens, q_len, k):
    """Top-K over the context part of each packed sequence; the question tail is always kept.

    aitualizate.com article, phase 2 (a top-K selector keeps the K tokens with the highest
    scores) and the restriction that only the document may be pruned (the question is never
    removed); thelatestinai.com page, Figure 1(a) (the gate module keeps K tokens).

    Per sequence b (packed at offset start_b): the context positions are [0, N_b - q_b),
    the question tail is [N_b - q_b, N_b). The context is fully sorted by (score
    descending, index ascending) - NaN after every number, -0 equal to +0 - and the first
    min(K_b, N_b - q_b) are kept. The result, with the tail appended, is sorted ascending.

    Returns (kept, cu_kept): kept is int64 [M_tot] of packed (global) row indices,
    cu_kept int64 [B+1].
    """
    s = np.asarray(s, dtype=np.float64)
    kept, cu = [], [0]
    start = 0
    for n, q, kb in zip(seqlens, q_len, k):
        n, q = int(n), int(q)
        n_ctx = n - q
        kc = min(max(int(kb), 0), n_ctx)
        ctx = s[start : start + n_ctx]
        is_nan = np.isnan(ctx)
        neg = np.where(is_nan, 0.0, -ctx) + 0.0  # + 0.0 turns -0 into +0
        idx = np.arange(n_ctx)
        order = np.lexsort((idx, neg, is_nan))  # primary: not-NaN first; then -s; then index
        sel = np.sort(order[:kc])
        rows = np.concatenate([sel, np.arange(n_ctx, n)]) + start
        kept.append(rows)
        cu.append(cu[-1] + rows.size)
        start += n
    kept = np.concatenate(kept) if kept else np.zeros(0, dtype=np.int64)
    return kept.astype(np.int64), np.asarray(cu, dtype=np.int64)


# --------------------------------------------------------------------------- forward kept


def gather(H, s, kept, seqlens, q_len, cu_kept, question_gate_one=False):
    """Kept hidden states with their gate values and original positions.

    thelatestinai.com page, Figure 1(b) (the kept hidden states travel on with their
    importance scores); aitualizate.com article, phase 3 (layers above L receive only
    the kept tokens). pos is each kept row's index within its own sequence (the original
    position id the causal mask uses). With ``question_gate_one`` the question-tail rows get
    g = 1, log g = 0 instead of their own gate value.

    Returns (H_kept [M, d] (same dtype/bits as H), pos int64 [M], g [M], logg [M]).
    """
    H = np.asarray(H)
    kept = np.asarray(kept, dtype=np.int64)
    starts = np.concatenate([[0], np.cumsum(seqlens)])[:-1]
    seq_of_row = np.repeat(np.arange(len(seqlens)), np.diff(np.asarray(cu_kept)))
    pos = kept - starts[seq_of_row]
    g, logg = gate_value(np.asarray(s, dtype=np.float64)[kept])
    if question_gate_one:
        for b, q in enumerate(q_len):
            hi = int(cu_kept[b + 1])
            g[hi - int(q) : hi] = 1.0
            logg[hi - int(q) : hi] = 0.0
    return H[kept], pos, g, logg


# --------------------------------------------------------------------------- phase 3: attention


def gated_attention(Q, K, V, logg, pos, cu_kept, Hq, Hkv, scale, head_gain=None,
                    unnormalised=False, rows=None):
    """Token-gated causal attention over the kept tokens, per sequence and query head.

    thelatestinai.com page, Figure 1(c): each attention weight is multiplied by the gate
    value g_j of its key. Read with the row renormalised, this equals adding log g_j to the
    logit (aitualizate.com article: the score becomes a bias on the attention logits, with a
    per-head gain). For query row i, head h, KV head h // (Hq/Hkv):
        S_ij = scale * q_i . k_j + gain_h * log g_j,   allowed iff pos_j <= pos_i
        O_i  = sum_j softmax_j(S_i) v_j,   LSE_i = logsumexp_j S_ij
    Unnormalised variant: O_i = sum_j softmax_j(scale q_i . k_j) * g_j^gain_h * v_j, and
    LSE is that of the unbiased logits.

    Q: [M, Hq, D]; K, V: [M, Hkv, D]; logg: [M] or None (g == 1); pos: [M]; cu_kept [B+1].
    rows: optional global query rows to evaluate (default: all). Returns (O [R, Hq, D],
    LSE [Hq, R]) for the R evaluated rows, float64.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    M = Q.shape[0]
    D = Q.shape[2]
    G = Hq // Hkv
    assert Hq % Hkv == 0 and K.shape[1] == Hkv
    pos = np.asarray(pos, dtype=np.int64)
    lg = np.zeros(M) if logg is None else np.asarray(logg, dtype=np.float64)
    gain = np.ones(Hq) if head_gain is None else np.asarray(head_gain, dtype=np.float64)
    rows = np.arange(M) if rows is None else np.asarray(rows, dtype=np.int64)
    cu = np.asarray(cu_kept, dtype=np.int64)
    O = np.zeros((rows.size, Hq, D))
    LSE = np.zeros((Hq, rows.size))
    seq = np.searchsorted(cu, rows, side="right") - 1
    for b in range(cu.size - 1):
        sel = np.nonzero(seq == b)[0]
        if sel.size == 0:
            continue
        lo, hi = int(cu[b]), int(cu[b + 1])
        r = rows[sel]
        allowed = pos[lo:hi][None, :] <= pos[r][:, None]
        for h in range(Hq):
            kv = h // G
            logits = scale * (Q[r, h, :] @ K[lo:hi, kv, :].T)
            bias = _key_bias(gain[h], lg[lo:hi])
            S = logits if unnormalised else logits + bias[None, :]
            S = np.where(allowed & (bias > -np.inf)[None, :], S, -np.inf)
            m = S.max(axis=1, keepdims=True)
            m = np.where(np.isfinite(m), m, 0.0)
            P = np.exp(S - m)
            l = P.sum(axis=1, keepdims=True)
            P = P / np.where(l > 0, l, 1.0)
            if unnormalised:
                O[sel, h, :] = P @ (np.exp(bias)[:, None] * V[lo:hi, kv, :])
            else:
                O[sel, h, :] = P @ V[lo:hi, kv, :]
            with np.errstate(divide="ignore"):
                LSE[h, sel] = (m + np.log(l))[:, 0]
    return O, LSE


def _key_bias(gain, lg):
    """gain * log g per key, where a key whose gate value is exactly 0 (log g = -inf) stays at
    -inf for every gain: a zero gate closes the key (Figure 1(c) multiplies its weight by 0),
    and 0 * -inf must not turn it into NaN. A query row whose visible keys are all closed has
    all-zero weights: O = 0 and LSE = -inf."""
    lg = np.asarray(lg, dtype=np.float64)
    with np.errstate(invalid="ignore"):
        return np.where(lg == -np.inf, -np.inf, gain * lg)


def gated_attention_bwd(Q, K, V, logg, pos, cu_kept, Hq, Hkv, scale, dO, head_gain=None):
    """Gradients of the (normalised) token-gated attention with respect to Q, K, V and log g.

    thelatestinai.com page, Figure 1(c): the gated attention is what lets the selector train
    end to end; aitualizate.com article, "Cómo consigue entrenar una selección top-K": the
    score is a bias on the logits, so its gradient is that of an additive logit bias. This is
    the derivative of gated_attention() written out per sequence and query head, with
    S = scale Q K^T + gain_h log g^T (masked), P = softmax rows, O = P V, and upstream dO:
        dV = P^T dO,  dP = dO V^T,  dS = P * (dP - rowsum(dP * P)),
        dQ = scale dS K,  dK = scale dS^T Q,  d log g_j = sum_h gain_h sum_i dS_ij.
    Query heads of one KV group add into that KV head's dK, dV. The per-head gain is a
    constant here (no gradient). Returns float64 (dQ [M, Hq, D], dK [M, Hkv, D],
    dV [M, Hkv, D], dlogg [M]).
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    dO = np.asarray(dO, dtype=np.float64)
    M, _, D = Q.shape
    G = Hq // Hkv
    assert Hq % Hkv == 0 and K.shape[1] == Hkv and dO.shape == Q.shape
    pos = np.asarray(pos, dtype=np.int64)
    lg = np.zeros(M) if logg is None else np.asarray(logg, dtype=np.float64)
    gain = np.ones(Hq) if head_gain is None else np.asarray(head_gain, dtype=np.float64)
    cu = np.asarray(cu_kept, dtype=np.int64)
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    dlogg = np.zeros(M)
    for b in range(cu.size - 1):
        lo, hi = int(cu[b]), int(cu[b + 1])
        if hi == lo:
            continue
        allowed = pos[lo:hi][None, :] <= pos[lo:hi][:, None]
        for h in range(Hq):
            kv = h // G
            Qh, Kh, Vh, dOh = Q[lo:hi, h, :], K[lo:hi, kv, :], V[lo:hi, kv, :], dO[lo:hi, h, :]
            bias = _key_bias(gain[h], lg[lo:hi])
            S = np.where(allowed & (bias > -np.inf)[None, :], scale * (Qh @ Kh.T) + bias[None, :], -np.inf)
            mx = S.max(axis=1, keepdims=True)
            P = np.exp(S - np.where(np.isfinite(mx), mx, 0.0))
            l = P.sum(axis=1, keepdims=True)
            P = P / np.where(l > 0, l, 1.0)
            dP = dOh @ Vh.T
            dS = P * (dP - (dP * P).sum(axis=1, keepdims=True))
            dQ[lo:hi, h, :] = scale * (dS @ Kh)
            dK[lo:hi, kv, :] += scale * (dS.T @ Qh)
            dV[lo:hi, kv, :] += P.T @ dOh
            dlogg[lo:hi] += gain[h] * dS.sum(axis=0)
    return dQ, dK, dV, dlogg


def gate_score_grad(dlogg, logg):
    """Gradient with respect to the selector's score, given the gradient with respect to log g.

    With g = sigmoid(s) (the reading of gate_value), d log g / ds = 1 - g = -expm1(log g),
    which is exact where g is close to 1. Rows whose log g was fixed to 0 (question tail with
    the gate forced to one) get zero."""
    return np.asarray(dlogg, np.float64) * -np.expm1(np.asarray(logg, np.float64))


def gelu_grad(z):
    """Derivative of the exact-erf GELU: d/dz [z Phi(z)] = Phi(z) + z phi(z), with Phi the standard
    normal CDF and phi its density."""
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * (1.0 + erf(z / np.sqrt(2.0))) + z * np.exp(-0.5 * z * z) / np.sqrt(2.0 * np.pi)


def gate_mlp_grad(H, W1, b1, w2, dscore, temperature=1.0):
    """Gradients of the gate network's parameters from the score gradient of each row.

    The last link of the end-to-end training path (thelatestinai.com page, Figure 1(c): the
    gated attention lets the top-K selector learn; aitualizate.com article, section on how the
    top-K selection is trained): with s_i = (w2 . GELU(W1 h_i + b1) + b2) / T (gate_scores) and
    upstream gradients dscore_i (tg_gated_attn_bwd's d score, for the kept rows h_i), the
    chain rule gives, per row, z = W1 h + b1, a = GELU(z), ds' = dscore / T, and
        dw2 = sum_i ds'_i a_i,   db2 = sum_i ds'_i,
        dz_i = ds'_i w2 * GELU'(z_i),   db1 = sum_i dz_i,   dW1 = sum_i dz_i h_i^T.
    H: [M, d]; W1: [dg, d]; b1: [dg] or None; w2: [dg]; dscore: [M]. float64 throughout.
    Returns (dW1 [dg, d], db1 [dg], dw2 [dg], db2 scalar).
    """
    H = np.asarray(H, dtype=np.float64)
    W1 = np.asarray(W1, dtype=np.float64)
    w2 = np.asarray(w2, dtype=np.float64).reshape(-1)
    ds = np.asarray(dscore, dtype=np.float64).reshape(-1) / float(temperature)
    z = H @ W1.T
    if b1 is not None:
        z = z + np.asarray(b1, dtype=np.float64)[None, :]
    dz = ds[:, None] * w2[None, :] * gelu_grad(z)
    return dz.T @ H, dz.sum(axis=0), gelu(z).T @ ds, float(ds.sum())


def gated_attention_weights(q, Kmat, g, scale):
    """Figure 1(c) read literally for one query row: softmax weights times g_j, renormalised.

    Used by the pins to show it equals the logit-bias form. q: [D]; Kmat: [n, D]; g: [n].
    """
    logits = scale * (np.asarray(Kmat, np.float64) @ np.asarray(q, np.float64))
    w = np.exp(logits - logits.max())
    w = w / w.sum()
    wg = w * np.asarray(g, np.float64)
    return wg / wg.sum()


# --------------------------------------------------------------------------- whole path


def prefill_above_L(H, W1, b1, w2, b2, seqlens, q_len, k, layers, Hq, Hkv, scale,
                    head_gain=None, unnormalised=False, question_gate_one=False):
    """The gated path above layer L: score -> top-K (+question tail) -> gather -> attention.

    aitualizate.com article, phases 2 and 3; thelatestinai.com page, Figure 1(a)-(c).
    ``layers`` is a list of (Q, K, V) per above-L layer, already shaped by the kept count.
    Returns a dict with every intermediate.
    """
    s = gate_scores(H, W1, b1, w2, b2)
    return prefill_from_scores(H, s, seqlens, q_len, k, layers, Hq, Hkv, scale, head_gain,
                               unnormalised, question_gate_one)


def prefill_from_scores(H, s, seqlens, q_len, k, layers, Hq, Hkv, scale, head_gain=None,
                        unnormalised=False, question_gate_one=False):
    """The same path starting from given scores (select, gather, attention)."""
    kept, cu = topk_select(s, seqlens, q_len, k)
    Hk, pos, g, logg = gather(H, s, kept, seqlens, q_len, cu, question_gate_one)
    outs = [gated_attention(Q, Kt, V, logg, pos, cu, Hq, Hkv, scale, head_gain, unnormalised)
            for (Q, Kt, V) in layers]
    return {"score": s, "kept": kept, "cu_kept": cu, "H_kept": Hk, "pos": pos, "g": g,
            "logg": logg, "attn": outs}


# --------------------------------------------------------------------------- above L: projections


def rope(x, pos, theta):
    """Rotary position embedding of x [M, H, D] at integer positions pos [M].

    Rotate-half pairing: for i < D/2 with angle a = pos * theta**(-2 i / D),
    y[i] = x[i] cos a - x[i + D/2] sin a and y[i + D/2] = x[i + D/2] cos a + x[i] sin a.
    The pages give no projection or rotary details; this is the plainest reading of "original
    position ids" for the layers above L. theta <= 0 means no rotation.
    """
    x = np.asarray(x, dtype=np.float64)
    if theta <= 0:
        return x.copy()
    D = x.shape[-1]
    half = D // 2
    inv = float(theta) ** (-2.0 * np.arange(half, dtype=np.float64) / D)
    a = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]  # [M, D/2]
    c, s = np.cos(a)[:, None, :], np.sin(a)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def qkv_rope(Hk, W, pos, Hq, Hkv, D, theta):
    """Q, K, V of the kept rows: X = Hk W^T with W [(Hq + 2 Hkv) D, d] (output-major, like
    torch.nn.Linear.weight), split into Q [M, Hq, D], K [M, Hkv, D], V [M, Hkv, D]; Q and K
    rotated by rope() at pos. float64."""
    X = np.asarray(Hk, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T
    M = X.shape[0]
    Q = X[:, : Hq * D].reshape(M, Hq, D)
    K = X[:, Hq * D: (Hq + Hkv) * D].reshape(M, Hkv, D)
    V = X[:, (Hq + Hkv) * D:].reshape(M, Hkv, D)
    return rope(Q, pos, theta), rope(K, pos, theta), V


def prefill_projected(H, W1, b1, w2, b2, seqlens, q_len, k, W_qkv, theta, Hq, Hkv, D, scale,
                      head_gain=None, temperature=1.0):
    """The gated path above layer L with each layer's own projections of the kept rows:
    score -> top-K (+question tail) -> kept rows -> per layer qkv_rope -> gated attention.

    aitualizate.com article, phase 3 (the layers above L work on the kept tokens only, at their
    original positions, and keep no key/value entries for dropped tokens); thelatestinai.com
    page, Figure 1(a). Returns the intermediates and, per layer, (Q, K, V, O, LSE); K and V of a
    layer are its key/value cache, kept rows only.
    """
    s = gate_scores(H, W1, b1, w2, b2, temperature)
    kept, cu = topk_select(s, seqlens, q_len, k)
    Hk, pos, g, logg = gather(H, s, kept, seqlens, q_len, cu)
    layers = []
    for W in W_qkv:
        Q, K, V = qkv_rope(Hk, W, pos, Hq, Hkv, D, theta)
        O, L = gated_attention(Q, K, V, logg, pos, cu, Hq, Hkv, scale, head_gain)
        layers.append((Q, K, V, O, L))
    return {"score": s, "kept": kept, "cu_kept": cu, "H_kept": Hk, "pos": pos, "g": g, "logg": logg,
            "layers": layers}
