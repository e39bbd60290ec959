"""Seeded synthetic inputs for the TokenGate gated-prefill path.

This module draws random numbers and converts storage formats (float32 <-> bfloat16 bit
patterns). It holds none of the method's arithmetic: no gate MLP, no selection, no
gather, no attention. Both the CPU oracle (through the tests) and the CUDA path consume
the exact bytes it produces, so any disagreement between them is the method's, not the
inputs'.

Every tensor is drawn from its own stream, ``numpy.random.Generator(PCG64(SeedSequence(
[workload.seed, tag])))``, so drawing one tensor never shifts another.

The workloads mirror the shapes the TokenGate pages evaluate: Qwen3-1.7B (hidden 2048,
16 query heads / 8 KV heads, head_dim 128, bf16; thelatestinai.com TokenGate page,
Table 1 "Base model Qwen3-1.7B, bf16") at the 8k-128k context lengths of the NIAH study
(Table 3) with the kept budgets of Figure 2 (K=256) and larger. The datasets themselves
(NIAH, 2WikiMultihopQA, ...) are not used: synthetic tensors of their shapes stand in.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# --------------------------------------------------------------------------- formats


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round float32 values to bfloat16 (round-to-nearest-even), returned as uint16 bits."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = a.view(np.uint32)
    nan = np.isnan(a)
    rounded = ((u.astype(np.uint64) + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    return np.where(nan, np.uint16(0x7FC0), rounded).astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16) to float32 exactly."""
    b = np.ascontiguousarray(np.asarray(b, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32)


def widen(x, dtype: str) -> np.ndarray:
    """Stored tensor (float32 array or bf16 bits) -> float64, exactly."""
    if dtype == "bf16":
        return bf16_bits_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float32).astype(np.float64)


# --------------------------------------------------------------------------- workloads


@dataclass(frozen=True)
class Workload:
    """Shapes of one synthetic gated-prefill instance (packed varlen, token-major)."""

    name: str
    seqlens: tuple
    q_len: tuple
    k: tuple
    d: int
    dg: int
    Hq: int
    Hkv: int
    D: int
    dtype: str  # "f32" or "bf16"
    n_layers: int = 1
    seed: int = 0
    score_mode: str = "mlp"  # stage-test score recipe: "mlp", "planted", "bf16_ties"
    notes: str = field(default="", compare=False)

    @property
    def B(self) -> int:
        return len(self.seqlens)

    @property
    def n_tok(self) -> int:
        return int(sum(self.seqlens))

    @property
    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.seqlens)]).astype(np.int64)

    def kept_rows(self) -> np.ndarray:
        """Rows per sequence after pruning, used only to shape the Q/K/V draws."""
        return np.array(
            [min(max(k, 0), n - q) + q for n, q, k in zip(self.seqlens, self.q_len, self.k)],
            dtype=np.int64,
        )

    @property
    def m_tot(self) -> int:
        return int(self.kept_rows().sum())


WORKLOADS = {
    "tiny_f32": Workload(
        "tiny_f32", (512,), (32,), (64,), d=256, dg=64, Hq=4, Hkv=2, D=64, dtype="f32",
        notes="N=512, q=32, K=64, d=256, gate 256->64->1, 4/2 heads, head_dim 64, fp32",
    ),
    "qwen3_8k": Workload(
        "qwen3_8k", (8192,), (64,), (1024,), d=2048, dg=256, Hq=16, Hkv=8, D=128,
        dtype="bf16", seed=1,
        notes="Qwen3-1.7B-shaped, N=8192, q=64, K=1024, bf16",
    ),
    "qwen3_32k": Workload(
        "qwen3_32k", (32768,), (128,), (2048,), d=2048, dg=256, Hq=16, Hkv=8, D=128,
        dtype="bf16", seed=2, score_mode="planted",
        notes="Qwen3-1.7B-shaped, N=32768, q=128, K=2048, bf16, planted salient spans",
    ),
    "qwen3_128k": Workload(
        "qwen3_128k", (131072,), (256,), (4096,), d=2048, dg=256, Hq=16, Hkv=8, D=128,
        dtype="bf16", n_layers=4, seed=3, score_mode="bf16_ties",
        notes="N=131072, q=256, K=4096, 4 above-L layers, bf16-quantised (tied) scores",
    ),
    "ragged4": Workload(
        "ragged4", (16384, 12000, 8192, 3000), (64, 200, 32, 128), (256, 256, 256, 256),
        d=2048, dg=256, Hq=16, Hkv=8, D=128, dtype="bf16", seed=4,
        notes="ragged batch of 4 packed sequences, K=256 each",
    ),
}


def scaled(wl: Workload, **kw) -> Workload:
    """A copy of ``wl`` with some fields replaced (used for small parity cases)."""
    from dataclasses import replace

    return replace(wl, **kw)


# --------------------------------------------------------------------------- streams

_TAGS = {
    "hidden": 1,
    "w1": 2,
    "b1": 3,
    "w2": 4,
    "b2": 5,
    "scores": 6,
    "planted": 7,
    "wq": 8,
    "wk": 9,
    "wv": 10,
    "logg": 11,
    "pos": 12,
}


def rng(wl_or_seed, tag: str, sub: int = 0) -> np.random.Generator:
    seed = wl_or_seed.seed if isinstance(wl_or_seed, Workload) else int(wl_or_seed)
    base = _TAGS[tag] if tag in _TAGS else 1000 + sub
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, base, sub])))


# --------------------------------------------------------------------------- draws


def hidden_states(wl: Workload) -> np.ndarray:
    """Hidden states at the selection layer, [n_tok, d] token-major.

    f32 workloads: iid N(0,1) float32. bf16 workloads: iid N(0,1), each row scaled to unit
    root-mean-square (x / sqrt(mean(x^2) + 1e-6), no weight), then rounded to bf16 bits.
    """
    g = rng(wl, "hidden")
    x = g.standard_normal((wl.n_tok, wl.d), dtype=np.float32)
    if wl.dtype == "f32":
        return x
    ms = np.einsum("ij,ij->i", x, x, dtype=np.float64) / wl.d
    x *= (1.0 / np.sqrt(ms + 1e-6)).astype(np.float32)[:, None]
    return f32_to_bf16_bits(x)


def xavier_uniform(g: np.random.Generator, fan_out: int, fan_in: int) -> np.ndarray:
    bound = np.sqrt(6.0 / (fan_in + fan_out))
    return g.uniform(-bound, bound, size=(fan_out, fan_in)).astype(np.float32)


def gate_weights(wl: Workload, biased: bool = False):
    """Gate MLP d -> dg (GELU) -> 1: returns (W1 [dg, d], b1 [dg] f32, w2 [dg], b2 float).

    W1 and w2 are Xavier-uniform (stored bf16 bits for bf16 workloads, float32 otherwise);
    b1 = 0 and b2 = 0 unless ``biased``, then both are U(-0.1, 0.1).
    """
    W1 = xavier_uniform(rng(wl, "w1"), wl.dg, wl.d)
    w2 = xavier_uniform(rng(wl, "w2"), 1, wl.dg)[0]
    if biased:
        b1 = rng(wl, "b1").uniform(-0.1, 0.1, size=wl.dg).astype(np.float32)
        b2 = float(np.float32(rng(wl, "b2").uniform(-0.1, 0.1)))
    else:
        b1 = np.zeros(wl.dg, dtype=np.float32)
        b2 = 0.0
    if wl.dtype == "bf16":
        return f32_to_bf16_bits(W1), b1, f32_to_bf16_bits(w2), b2
    return W1, b1, w2, b2


def stage_scores(wl: Workload) -> np.ndarray:
    """Scores fed straight to the select stage, float32 [n_tok].

    "mlp"/default: iid N(0,1). "planted": N(0,1) plus 3 on 10% of each sequence's context
    tokens, laid out as non-overlapping spans of 64 contiguous tokens at seeded positions.
    "bf16_ties": N(0,1) rounded to bf16-representable values (many exact ties).
    """
    s = rng(wl, "scores").standard_normal(wl.n_tok).astype(np.float32)
    if wl.score_mode == "planted":
        s += 3.0 * planted_mask(wl).astype(np.float32)
    elif wl.score_mode == "bf16_ties":
        s = bf16_bits_to_f32(f32_to_bf16_bits(s))
    return s.astype(np.float32)


def planted_mask(wl: Workload, span: int = 64, frac: float = 0.10) -> np.ndarray:
    """Boolean [n_tok]: 10% of each sequence's context covered by 64-token spans."""
    g = rng(wl, "planted")
    mask = np.zeros(wl.n_tok, dtype=bool)
    for b, (n, q) in enumerate(zip(wl.seqlens, wl.q_len)):
        n_ctx = n - q
        n_slots = n_ctx // span
        n_spans = int(round(frac * n_ctx / span))
        slots = np.sort(g.choice(n_slots, size=min(n_spans, n_slots), replace=False))
        start = int(wl.cu_seqlens[b])
        for sl in slots:
            mask[start + sl * span : start + (sl + 1) * span] = True
    return mask


def qkv(wl: Workload, layer: int, m_tot: int | None = None):
    """Synthetic Q [M, Hq, D], K and V [M, Hkv, D] for one above-L layer.

    bf16 workloads: iid N(0,1)/sqrt(128) rounded to bf16 bits. Each layer has its own
    seeded streams. (The tiny f32 workload instead projects the kept hidden states; see
    ``project_kept``.)
    """
    m = wl.m_tot if m_tot is None else m_tot
    sc = np.float32(1.0 / np.sqrt(128.0))
    out = []
    for i, (tag, h) in enumerate((("wq", wl.Hq), ("wk", wl.Hkv), ("wv", wl.Hkv))):
        g = rng(wl, tag, sub=100 + layer)
        x = g.standard_normal((m, h, wl.D), dtype=np.float32) * sc
        out.append(f32_to_bf16_bits(x) if wl.dtype == "bf16" else x)
    return tuple(out)


def projection_weights(wl: Workload):
    """Wq [d, Hq*D], Wk and Wv [d, Hkv*D], entries iid N(0, 1/d), float64."""
    sd = 1.0 / np.sqrt(wl.d)
    Wq = rng(wl, "wq").standard_normal((wl.d, wl.Hq * wl.D)) * sd
    Wk = rng(wl, "wk").standard_normal((wl.d, wl.Hkv * wl.D)) * sd
    Wv = rng(wl, "wv").standard_normal((wl.d, wl.Hkv * wl.D)) * sd
    return Wq, Wk, Wv


def project_kept(wl: Workload, Hk64: np.ndarray):
    """Synthetic stand-in for an above-L layer's projections: Q/K/V = H_kept @ W, then
    rounded to float32. Not part of the method (the real layer's projections and RoPE
    are outside the gated path); it only gives the tiny workload realistic Q/K/V."""
    Wq, Wk, Wv = projection_weights(wl)
    m = Hk64.shape[0]
    Q = (Hk64 @ Wq).reshape(m, wl.Hq, wl.D).astype(np.float32)
    K = (Hk64 @ Wk).reshape(m, wl.Hkv, wl.D).astype(np.float32)
    V = (Hk64 @ Wv).reshape(m, wl.Hkv, wl.D).astype(np.float32)
    return Q, K, V


def random_logg(wl: Workload, m_tot: int, layer: int = 0) -> np.ndarray:
    """Stand-alone gate log-values for attention stage tests: log of U(0.05, 1), float32."""
    g = rng(wl, "logg", sub=layer)
    return np.log(g.uniform(0.05, 1.0, size=m_tot)).astype(np.float32)
