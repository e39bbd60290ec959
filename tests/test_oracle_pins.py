"""Pins for the CPU oracle: closed forms, textbook values, brute force and invariants.

These tests tie the oracle to what the TokenGate pages and the mathematics fix, so that a
plausible mistake in it (a dropped term, a wrong sign or index, a transposed operand, a
wrong tie-break) fails at least one of them. CPU only.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import tg_inputs as ti
from oracle import tg_oracle as orc


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _num(x):
    return float(x) if not isinstance(x, str) else float(x.replace("nan", "nan"))


# ----------------------------------------------------------------------------- score


def test_gelu_matches_normal_cdf_table(golden_dir):
    fx = _load(golden_dir, "gelu_normal_cdf.json")
    for xs, phi in fx["phi"].items():
        x = float(xs)
        assert abs(orc.gelu(x) - x * phi) <= fx["tolerance_abs"], x


def test_gelu_odd_part_identity():
    # GELU(x) - GELU(-x) = x Phi(x) + x Phi(-x) = x for every x
    x = np.linspace(-6, 6, 101)
    assert np.max(np.abs(orc.gelu(x) - orc.gelu(-x) - x)) < 1e-14


def test_score_one_hot_closed_form(golden_dir):
    fx = _load(golden_dir, "score_onehot.json")
    s = orc.gate_scores(np.array(fx["H"]), np.array(fx["W1"]), np.array(fx["b1"]),
                        np.array(fx["w2"]), fx["b2"])
    np.testing.assert_allclose(s, fx["expected"], rtol=0, atol=fx["tolerance_abs"])


def _score_bruteforce(H, W1, b1, w2, b2):
    out = []
    for h in H:
        acc = 0.0
        for kk in range(len(W1)):
            z = sum(float(W1[kk][j]) * float(h[j]) for j in range(len(h))) + float(b1[kk])
            acc += float(w2[kk]) * 0.5 * z * (1.0 + math.erf(z / math.sqrt(2.0)))
        out.append(acc + b2)
    return np.array(out)


def test_score_matches_per_token_loop_nonsquare():
    g = np.random.default_rng(5)
    n, d, dg = 7, 5, 3  # d != dg so a transposed W1 cannot pass
    H = g.standard_normal((n, d))
    W1 = g.standard_normal((dg, d))
    b1 = g.uniform(-0.5, 0.5, dg)
    w2 = g.standard_normal(dg)
    b2 = 0.3
    np.testing.assert_allclose(orc.gate_scores(H, W1, b1, w2, b2),
                               _score_bruteforce(H, W1, b1, w2, b2), rtol=1e-12, atol=1e-12)


def test_score_float32_independent_evaluation():
    # an independent float32 evaluation (torch, exact-erf GELU) agrees within float32 error
    wl = ti.scaled(ti.WORKLOADS["tiny_f32"], seqlens=(64,), q_len=(8,), k=(8,))
    H = ti.hidden_states(wl)
    W1, b1, w2, b2 = ti.gate_weights(wl, biased=True)
    s64 = orc.gate_scores(H, W1, b1, w2, b2)
    t = torch.nn.functional.gelu(torch.from_numpy(H) @ torch.from_numpy(W1).T
                                 + torch.from_numpy(b1)) @ torch.from_numpy(w2) + b2
    np.testing.assert_allclose(s64, t.numpy().astype(np.float64), rtol=0,
                               atol=2e-5 * np.abs(s64).max())


# ----------------------------------------------------------------------------- gate value


def test_gate_value_special_values():
    g, lg = orc.gate_value(np.array([0.0]))
    assert g[0] == 0.5 and abs(lg[0] - math.log(0.5)) < 1e-15
    s = np.linspace(-30, 30, 241)
    g, lg = orc.gate_value(s)
    assert np.all((g > 0) & (g < 1 + 1e-15))
    np.testing.assert_allclose(g, 1.0 / (1.0 + np.exp(-s)), rtol=1e-14)
    np.testing.assert_allclose(np.exp(lg), g, rtol=1e-14)
    # log sigma(s) - log sigma(-s) = s
    _, lgm = orc.gate_value(-s)
    np.testing.assert_allclose(lg - lgm, s, rtol=0, atol=1e-12)


def test_log_gate_is_finite_and_linear_far_left():
    s = np.array([-50.0, -700.0, -1e4, 40.0, 800.0])
    _, lg = orc.gate_value(s)
    assert np.all(np.isfinite(lg))
    np.testing.assert_allclose(lg[:3], s[:3], rtol=1e-15, atol=0)
    assert lg[3] == pytest.approx(-math.exp(-40.0), rel=1e-12)
    assert lg[4] == 0.0 or abs(lg[4]) < 1e-300


# ----------------------------------------------------------------------------- select


def _parse_scores(vals):
    out = []
    for v in vals:
        out.append(float(v) if not isinstance(v, str) else float(v))
    return np.array(out, dtype=np.float32)


def test_topk_golden_ties(golden_dir):
    fx = _load(golden_dir, "topk_ties.json")
    s = _parse_scores(fx["scores"])
    assert math.copysign(1.0, s[2]) < 0  # the fixture really holds a negative zero
    for case in fx["cases"]:
        kept, cu = orc.topk_select(s, fx["seqlens"], fx["q_len"], case["k"])
        assert kept.tolist() == case["kept"], case
        assert cu.tolist() == case["cu_kept"], case


def _exhaustive_check(s, kept, seqlens, q_len, k):
    start = 0
    kept = set(int(x) for x in kept)
    for n, q, kb in zip(seqlens, q_len, k):
        n_ctx = n - q
        ctx = range(start, start + n_ctx)
        kept_ctx = [j for j in ctx if j in kept]
        drop_ctx = [i for i in ctx if i not in kept]
        assert len(kept_ctx) == min(max(kb, 0), n_ctx)
        for j in range(start + n_ctx, start + n):
            assert j in kept  # question tail always kept

        def before(a, b):  # a ranks before b
            sa, sb = s[a], s[b]
            if np.isnan(sa) or np.isnan(sb):
                return (not np.isnan(sa) and np.isnan(sb)) or (np.isnan(sa) and np.isnan(sb) and a < b)
            return sa > sb or (sa == sb and a < b)

        for j in kept_ctx:
            for i in drop_ctx:
                assert before(j, i), (j, i, s[j], s[i])
        start += n


@pytest.mark.parametrize("seed", range(6))
def test_topk_bruteforce_small_integer_ties(seed):
    g = np.random.default_rng(seed)
    B = int(g.integers(1, 4))
    seqlens = [int(g.integers(1, 40)) for _ in range(B)]
    q_len = [int(g.integers(0, n + 1)) for n in seqlens]
    k = [int(g.integers(0, 45)) for _ in range(B)]
    s = g.integers(0, 4, size=sum(seqlens)).astype(np.float32)  # heavy ties
    s[g.random(s.size) < 0.05] = np.nan
    s[g.random(s.size) < 0.05] = -0.0
    kept, cu = orc.topk_select(s, seqlens, q_len, k)
    assert np.all(np.diff(kept[cu[0]:cu[1]]) > 0)
    for b in range(B):
        seg = kept[cu[b]:cu[b + 1]]
        assert np.all(np.diff(seg) > 0)
        assert seg.size == orc.kept_count(seqlens[b], q_len[b], k[b])
    _exhaustive_check(s, kept, seqlens, q_len, k)


def test_topk_matches_full_stable_sort_by_python_sorted():
    g = np.random.default_rng(11)
    n, q, kk = 300, 20, 37
    s = np.round(g.standard_normal(n) * 4) / 4  # ties
    kept, _ = orc.topk_select(s.astype(np.float32), [n], [q], [kk])
    ranked = sorted(range(n - q), key=lambda i: (-float(np.float32(s[i])), i))
    expect = sorted(ranked[:kk]) + list(range(n - q, n))
    assert kept.tolist() == expect


def test_topk_degenerate_budgets():
    s = np.arange(10, dtype=np.float32)
    kept, cu = orc.topk_select(s, [10], [10], [5])  # question only: nothing to prune
    assert kept.tolist() == list(range(10))
    kept, cu = orc.topk_select(s, [10], [0], [3])  # no question
    assert kept.tolist() == [7, 8, 9]
    kept, cu = orc.topk_select(s, [10], [4], [-2])  # negative budget reads as 0
    assert kept.tolist() == [6, 7, 8, 9]
    kept, cu = orc.topk_select(np.zeros(0, np.float32), [], [], [])
    assert kept.size == 0 and cu.tolist() == [0]


# ----------------------------------------------------------------------------- gather


def test_gather_positions_and_rows():
    g = np.random.default_rng(2)
    seqlens, q_len, k = [12, 7, 9], [3, 0, 9], [4, 2, 1]
    H = g.standard_normal((sum(seqlens), 5)).astype(np.float32)
    s = g.standard_normal(sum(seqlens)).astype(np.float32)
    kept, cu = orc.topk_select(s, seqlens, q_len, k)
    Hk, pos, gv, lg = orc.gather(H, s, kept, seqlens, q_len, cu)
    starts = np.cumsum([0] + seqlens[:-1])
    for r, j in enumerate(kept):
        b = max(i for i in range(3) if starts[i] <= j)
        assert pos[r] == j - starts[b]
        assert np.array_equal(Hk[r].view(np.uint32), H[j].view(np.uint32))
        assert gv[r] == pytest.approx(1 / (1 + math.exp(-float(s[j]))), rel=1e-14)
    _, _, g1, l1 = orc.gather(H, s, kept, seqlens, q_len, cu, question_gate_one=True)
    for b in range(3):
        hi = cu[b + 1]
        assert np.all(g1[hi - q_len[b]:hi] == 1.0) and np.all(l1[hi - q_len[b]:hi] == 0.0)
        lo_ctx = hi - q_len[b]
        np.testing.assert_array_equal(g1[cu[b]:lo_ctx], gv[cu[b]:lo_ctx])


# ----------------------------------------------------------------------------- attention


def _attn_bruteforce(Q, K, V, logg, pos, cu, Hq, Hkv, scale, gain=None, unnorm=False):
    M, _, D = Q.shape
    G = Hq // Hkv
    O = np.zeros((M, Hq, D))
    L = np.zeros((Hq, M))
    for b in range(len(cu) - 1):
        for i in range(cu[b], cu[b + 1]):
            for h in range(Hq):
                gh = 1.0 if gain is None else gain[h]
                js = [j for j in range(cu[b], cu[b + 1]) if pos[j] <= pos[i]]
                lo = [scale * sum(Q[i, h, t] * K[j, h // G, t] for t in range(D)) for j in js]
                bias = [gh * (0.0 if logg is None else logg[j]) for j in js]
                tot = [a + c for a, c in zip(lo, bias)] if not unnorm else lo
                m = max(tot)
                w = [math.exp(x - m) for x in tot]
                z = sum(w)
                L[h, i] = m + math.log(z)
                for jj, j in enumerate(js):
                    f = w[jj] / z * (math.exp(bias[jj]) if unnorm else 1.0)
                    O[i, h, :] += f * V[j, h // G, :]
    return O, L


def test_attention_golden_two_keys(golden_dir):
    fx = _load(golden_dir, "attention_two_keys.json")
    Q, K, V = (np.array(fx[x]) for x in ("Q", "K", "V"))
    lg = np.log(np.array(fx["g"]))
    pos = np.array(fx["pos"])
    cu = [0, 2]
    tol = fx["tolerance_abs"]
    for key, kw in (("normalised", {}), ("gain2", {"head_gain": [2.0]}),
                    ("unnormalised", {"unnormalised": True})):
        O, L = orc.gated_attention(Q, K, V, lg, pos, cu, 1, 1, fx["scale"], **kw)
        np.testing.assert_allclose(O[:, 0, :], fx["expected"][key]["O"], rtol=0, atol=tol)
        np.testing.assert_allclose(L[0], fx["expected"][key]["LSE"], rtol=0, atol=tol)


@pytest.mark.parametrize("unnorm", [False, True])
def test_attention_bruteforce_gqa_ragged_gain(unnorm):
    g = np.random.default_rng(3)
    cu = [0, 5, 6, 11]
    M, Hq, Hkv, D = 11, 4, 2, 3
    Q = g.standard_normal((M, Hq, D))
    K = g.standard_normal((M, Hkv, D))
    V = g.standard_normal((M, Hkv, D))
    lg = np.log(g.uniform(0.05, 1, M))
    pos = np.array([0, 3, 4, 9, 20, 7, 1, 2, 5, 6, 8])  # ascending within each sequence
    gain = np.array([1.0, 0.5, 2.0, -1.0])
    O, L = orc.gated_attention(Q, K, V, lg, pos, cu, Hq, Hkv, 0.7, gain, unnorm)
    Ob, Lb = _attn_bruteforce(Q, K, V, lg, pos, cu, Hq, Hkv, 0.7, gain, unnorm)
    np.testing.assert_allclose(O, Ob, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(L, Lb, rtol=1e-12, atol=1e-12)
    rows = np.array([10, 0, 5, 3])
    Os, Ls = orc.gated_attention(Q, K, V, lg, pos, cu, Hq, Hkv, 0.7, gain, unnorm, rows=rows)
    np.testing.assert_allclose(Os, O[rows], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(Ls, L[:, rows], rtol=1e-13, atol=1e-13)


def test_attention_g1_all_kept_is_textbook_causal_attention():
    # g == 1 and K >= N - q keeps every token: ordinary causal attention (torch SDPA, float64)
    g = np.random.default_rng(4)
    N, q, Hq, Hkv, D = 40, 6, 4, 2, 8
    s = g.standard_normal(N).astype(np.float32)
    kept, cu = orc.topk_select(s, [N], [q], [N])
    assert kept.tolist() == list(range(N))
    Q = g.standard_normal((N, Hq, D))
    K = g.standard_normal((N, Hkv, D))
    V = g.standard_normal((N, Hkv, D))
    scale = 1 / math.sqrt(D)
    O, _ = orc.gated_attention(Q, K, V, None, np.arange(N), cu, Hq, Hkv, scale)
    tq = torch.from_numpy(Q).permute(1, 0, 2)
    tk = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
    tv = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=scale)
    np.testing.assert_allclose(O, ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)


def test_attention_invariants():
    g = np.random.default_rng(8)
    M, Hq, Hkv, D = 17, 2, 1, 4
    Q = g.standard_normal((M, Hq, D))
    K = g.standard_normal((M, Hkv, D))
    V = g.standard_normal((M, Hkv, D))
    pos = np.arange(M) * 2
    cu = [0, M]
    lg = np.log(g.uniform(0.1, 1, M))
    O1, _ = orc.gated_attention(Q, K, V, None, pos, cu, Hq, Hkv, 0.5)
    # constant g is a shift of every logit: same as g == 1
    Oc, _ = orc.gated_attention(Q, K, V, np.full(M, math.log(0.3)), pos, cu, Hq, Hkv, 0.5)
    np.testing.assert_allclose(Oc, O1, rtol=1e-12, atol=1e-12)
    # the first kept row sees only itself: O = v0 (normalised), g0 v0 (unnormalised)
    O, _ = orc.gated_attention(Q, K, V, lg, pos, cu, Hq, Hkv, 0.5)
    np.testing.assert_allclose(O[0, 0], V[0, 0], rtol=0, atol=1e-15)
    Ou, _ = orc.gated_attention(Q, K, V, lg, pos, cu, Hq, Hkv, 0.5, unnormalised=True)
    np.testing.assert_allclose(Ou[0, 1], math.exp(lg[0]) * V[0, 0], rtol=1e-14)
    # a key whose gate goes to zero is the same as removing that key
    lz = lg.copy()
    lz[5] = -1e4
    Oz, _ = orc.gated_attention(Q, K, V, lz, pos, cu, Hq, Hkv, 0.5)
    keep = np.array([i for i in range(M) if i != 5])
    Or, _ = orc.gated_attention(Q[keep], K[keep], V[keep], lg[keep], pos[keep], [0, M - 1],
                                Hq, Hkv, 0.5)
    np.testing.assert_allclose(Oz[keep], Or, rtol=1e-12, atol=1e-12)
    # logit bias == weight times g_j, renormalised (the literal reading of Figure 1(c))
    for i in (3, 16):
        w = orc.gated_attention_weights(Q[i, 0], K[: i + 1, 0], np.exp(lg[: i + 1]), 0.5)
        np.testing.assert_allclose(w @ V[: i + 1, 0], O[i, 0], rtol=1e-12, atol=1e-12)
        assert abs(w.sum() - 1.0) < 1e-12


def test_dropped_tokens_do_not_matter():
    # layers above L see only the kept tokens: perturbing dropped rows changes nothing
    wl = ti.scaled(ti.WORKLOADS["tiny_f32"], seqlens=(96, 40), q_len=(8, 4), k=(16, 9))
    H = ti.hidden_states(wl)
    s = ti.rng(wl, "scores").standard_normal(wl.n_tok).astype(np.float32)
    kept, cu = orc.topk_select(s, wl.seqlens, wl.q_len, wl.k)
    H2 = H.copy()
    dropped = np.setdiff1d(np.arange(wl.n_tok), kept)
    H2[dropped] = 1e3
    out1 = orc.prefill_from_scores(H, s, wl.seqlens, wl.q_len, wl.k, [], 4, 2, 0.125)
    out2 = orc.prefill_from_scores(H2, s, wl.seqlens, wl.q_len, wl.k, [], 4, 2, 0.125)
    assert np.array_equal(out1["H_kept"], out2["H_kept"])
    Hk64 = out1["H_kept"].astype(np.float64)
    layers = [ti.project_kept(wl, Hk64)]
    a1 = orc.prefill_from_scores(H, s, wl.seqlens, wl.q_len, wl.k, layers, 4, 2, 0.125)["attn"]
    a2 = orc.prefill_from_scores(H2, s, wl.seqlens, wl.q_len, wl.k, layers, 4, 2, 0.125)["attn"]
    assert np.array_equal(a1[0][0], a2[0][0])


def test_softmax_rows_sum_to_one():
    g = np.random.default_rng(9)
    M, D = 30, 5
    Q = g.standard_normal((M, 1, D))
    K = g.standard_normal((M, 1, D))
    lg = np.log(g.uniform(0.01, 1, M))
    # with V = identity-like one-hot columns the output rows are the weights themselves
    V = np.zeros((M, 1, M))
    V[np.arange(M), 0, np.arange(M)] = 1.0
    Qp = np.concatenate([Q, np.zeros((M, 1, M - D))], axis=2)
    Kp = np.concatenate([K, np.zeros((M, 1, M - D))], axis=2)
    O, _ = orc.gated_attention(Qp, Kp, V, lg, np.arange(M), [0, M], 1, 1, 0.3)
    P = O[:, 0, :]
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(np.triu(P, 1) == 0.0)  # causal


def test_planted_spans_are_kept_when_salient():
    wl = ti.scaled(ti.WORKLOADS["qwen3_32k"], seqlens=(4096,), q_len=(64,), k=(409,))
    s = ti.stage_scores(wl)
    m = ti.planted_mask(wl)
    kept, _ = orc.topk_select(s, wl.seqlens, wl.q_len, wl.k)
    frac = m[kept[:409]].mean()
    assert frac > 0.8  # +3 sigma offsets dominate the kept set


# ---------------------------------------------------------------- rotary embedding / QKV projection


def test_rope_hand_values_fix_pairing_and_frequencies():
    # D = 4: pairs (0, 2) and (1, 3); frequencies theta^0 = 1 and theta^(-1/2) = 0.01 for theta 1e4
    x = np.array([[[1.0, 2.0, 3.0, 4.0]]])
    y = orc.rope(x, [1], 1.0e4)[0, 0]
    c1, s1, c2, s2 = math.cos(1.0), math.sin(1.0), math.cos(0.01), math.sin(0.01)
    want = [1 * c1 - 3 * s1, 2 * c2 - 4 * s2, 3 * c1 + 1 * s1, 4 * c2 + 2 * s2]
    assert np.allclose(y, want, rtol=0, atol=1e-15)


def test_rope_identity_norm_and_relative_position():
    g = np.random.default_rng(3)
    x = g.standard_normal((5, 3, 16))
    assert np.array_equal(orc.rope(x, [0] * 5, 1.0e6), x)  # position 0 rotates nothing
    assert np.array_equal(orc.rope(x, [7] * 5, 0.0), x)    # theta <= 0: no rotation
    y = orc.rope(x, [3, 100, 4097, 65535, 131071], 1.0e6)
    n0 = x[..., :8] ** 2 + x[..., 8:] ** 2
    n1 = y[..., :8] ** 2 + y[..., 8:] ** 2
    assert np.allclose(n0, n1, rtol=1e-12)                # each pair keeps its length
    q, k = g.standard_normal((1, 1, 16)), g.standard_normal((1, 1, 16))
    for m, n, t in ((5, 2, 11), (1000, 10, 777), (0, 0, 4096)):
        d0 = np.sum(orc.rope(q, [m], 1.0e4) * orc.rope(k, [n], 1.0e4))
        d1 = np.sum(orc.rope(q, [m + t], 1.0e4) * orc.rope(k, [n + t], 1.0e4))
        assert abs(d0 - d1) < 1e-9                        # depends on m - n only


def test_qkv_rope_split_and_projection():
    g = np.random.default_rng(4)
    M, d, Hq, Hkv, D = 6, 32, 4, 2, 8
    Hk = g.standard_normal((M, d))
    W = g.standard_normal(((Hq + 2 * Hkv) * D, d))
    pos = np.array([0, 1, 2, 50, 51, 9])
    Q, K, V = orc.qkv_rope(Hk, W, pos, Hq, Hkv, D, 1.0e4)
    X = np.array([[sum(Hk[i, c] * W[o, c] for c in range(d)) for o in range(W.shape[0])] for i in range(M)])
    assert np.allclose(V, X[:, (Hq + Hkv) * D:].reshape(M, Hkv, D), atol=1e-12)  # V is not rotated
    assert np.allclose(Q[0], X[0, : Hq * D].reshape(Hq, D), atol=1e-12)          # row at position 0
    q3 = X[3, : Hq * D].reshape(1, Hq, D)
    assert np.allclose(Q[3], orc.rope(q3, [50], 1.0e4)[0], atol=1e-12)
    k4 = X[4, Hq * D: (Hq + Hkv) * D].reshape(1, Hkv, D)
    assert np.allclose(K[4], orc.rope(k4, [51], 1.0e4)[0], atol=1e-12)


# ----------------------------------------------------------------------------- attention backward


def _bwd_case(seed, lens=(5, 7), Hq=4, Hkv=2, D=8, gain=True):
    g = np.random.default_rng(seed)
    M = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    pos = np.concatenate([np.sort(g.choice(3 * n, n, replace=False)) for n in lens]).astype(np.int64)
    Q, K, V = g.standard_normal((M, Hq, D)), g.standard_normal((M, Hkv, D)), g.standard_normal((M, Hkv, D))
    logg = orc.gate_value(g.standard_normal(M) * 2)[1]
    dO = g.standard_normal((M, Hq, D))
    hg = g.uniform(0.5, 1.5, Hq) if gain else None
    return Q, K, V, logg, pos, cu, Hq, Hkv, 1.0 / math.sqrt(D), dO, hg


def _loss(Q, K, V, logg, pos, cu, Hq, Hkv, scale, dO, hg):
    O, _ = orc.gated_attention(Q, K, V, logg, pos, cu, Hq, Hkv, scale, head_gain=hg)
    return float((O * dO).sum())


def test_attention_bwd_matches_central_differences():
    # every input element perturbed on its own: a wrong sign, scale, transposition or GQA
    # accumulation in the backward shows up as an O(1) mismatch against the forward's slopes
    case = _bwd_case(1)
    Q, K, V, logg, pos, cu, Hq, Hkv, scale, dO, hg = case
    dQ, dK, dV, dl = orc.gated_attention_bwd(Q, K, V, logg, pos, cu, Hq, Hkv, scale, dO, head_gain=hg)
    eps = 1e-6
    for name, X, dX in (("Q", Q, dQ), ("K", K, dK), ("V", V, dV), ("logg", logg, dl)):
        fd = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += eps
            Xm[idx] -= eps
            args = {"Q": Q, "K": K, "V": V, "logg": logg}
            ap, am = dict(args, **{name: Xp}), dict(args, **{name: Xm})
            lp = _loss(ap["Q"], ap["K"], ap["V"], ap["logg"], pos, cu, Hq, Hkv, scale, dO, hg)
            lm = _loss(am["Q"], am["K"], am["V"], am["logg"], pos, cu, Hq, Hkv, scale, dO, hg)
            fd[idx] = (lp - lm) / (2 * eps)
        assert np.max(np.abs(fd - dX)) <= 1e-6 * max(1.0, np.max(np.abs(dX))), name


def test_attention_bwd_matches_torch_autograd():
    # torch's own differentiation of a direct torch statement of the forward (float64, CPU)
    Q, K, V, logg, pos, cu, Hq, Hkv, scale, dO, hg = _bwd_case(2, lens=(17, 1, 23), Hq=8, Hkv=2, D=16)
    tQ, tK, tV, tl = (torch.tensor(x, requires_grad=True) for x in (Q, K, V, logg))
    G = Hq // Hkv
    loss = 0.0
    for b in range(len(cu) - 1):
        lo, hi = int(cu[b]), int(cu[b + 1])
        mask = torch.tensor(pos[lo:hi][None, :] <= pos[lo:hi][:, None])
        for h in range(Hq):
            S = scale * tQ[lo:hi, h] @ tK[lo:hi, h // G].T + float(hg[h]) * tl[lo:hi][None, :]
            P = torch.softmax(S.masked_fill(~mask, float("-inf")), dim=1)
            loss = loss + (P @ tV[lo:hi, h // G] * torch.tensor(dO[lo:hi, h])).sum()
    loss.backward()
    ref = orc.gated_attention_bwd(Q, K, V, logg, pos, cu, Hq, Hkv, scale, dO, head_gain=hg)
    for got, t in zip(ref, (tQ, tK, tV, tl)):
        np.testing.assert_allclose(got, t.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_attention_bwd_invariants():
    Q, K, V, logg, pos, cu, Hq, Hkv, scale, dO, hg = _bwd_case(3, lens=(9, 12, 1), Hq=6, Hkv=3, D=4)
    dQ, dK, dV, dl = orc.gated_attention_bwd(Q, K, V, logg, pos, cu, Hq, Hkv, scale, dO, head_gain=hg)
    # each row's dS sums to zero (softmax is shift invariant), so d log g sums to zero per sequence
    for b in range(len(cu) - 1):
        assert abs(dl[cu[b]:cu[b + 1]].sum()) <= 1e-12 * max(1.0, np.abs(dl).max())
    # a constant added to log g within a sequence changes nothing, gradients included
    shifted = logg + np.where(np.arange(len(logg)) < cu[1], 3.0, -2.0)
    for a, b in zip((dQ, dK, dV, dl),
                    orc.gated_attention_bwd(Q, K, V, shifted, pos, cu, Hq, Hkv, scale, dO, head_gain=hg)):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)
    # the first row of a sequence sees only itself: P = 1, so its dQ is 0 and dV_0 gets dO_0
    first = _bwd_case(4, lens=(1,), Hq=2, Hkv=1, D=4)
    fq, fk, fv, fl = orc.gated_attention_bwd(*first[:9], first[9], head_gain=first[10])
    assert np.all(fq == 0) and np.all(fl == 0)
    np.testing.assert_allclose(fv[0, 0], first[9][0].sum(axis=0), rtol=1e-14)


def test_gate_score_grad_matches_central_differences():
    # through the gate map: d/ds of the attention loss with log g = log-sigmoid(s)
    Q, K, V, _, pos, cu, Hq, Hkv, scale, dO, hg = _bwd_case(5)
    s = np.random.default_rng(6).standard_normal(len(pos)) * 3
    logg = orc.gate_value(s)[1]
    dl = orc.gated_attention_bwd(Q, K, V, logg, pos, cu, Hq, Hkv, scale, dO, head_gain=hg)[3]
    ds = orc.gate_score_grad(dl, logg)
    eps = 1e-6
    for j in range(len(s)):
        sp, sm = s.copy(), s.copy()
        sp[j] += eps
        sm[j] -= eps
        fd = (_loss(Q, K, V, orc.gate_value(sp)[1], pos, cu, Hq, Hkv, scale, dO, hg)
              - _loss(Q, K, V, orc.gate_value(sm)[1], pos, cu, Hq, Hkv, scale, dO, hg)) / (2 * eps)
        assert abs(fd - ds[j]) <= 1e-6 * max(1.0, np.abs(ds).max()), j
    assert orc.gate_score_grad(np.array([5.0]), np.array([0.0]))[0] == 0.0


def test_attention_closed_gate_is_a_removed_key_for_every_gain():
    """A key with gate value exactly 0 (log g = -inf) contributes nothing, whatever the head's
    gain, including a gain of 0 (where gain * log g would be 0 * -inf): it equals the sequence
    with that key removed, for the biased and the unnormalised form. A query row whose visible
    keys are all closed has all-zero weights: O = 0, LSE = -inf, and zero gradients."""
    g = np.random.default_rng(21)
    M, Hq, Hkv, D = 11, 3, 1, 4
    Q, K, V = g.standard_normal((M, Hq, D)), g.standard_normal((M, Hkv, D)), g.standard_normal((M, Hkv, D))
    pos = np.arange(M) * 3
    lg = np.log(g.uniform(0.1, 1, M))
    lg[4] = -np.inf
    gain = np.array([0.0, 1.0, 2.5])
    keep = np.array([i for i in range(M) if i != 4])
    for unnorm in (False, True):
        O, L = orc.gated_attention(Q, K, V, lg, pos, [0, M], Hq, Hkv, 0.5, head_gain=gain, unnormalised=unnorm)
        Or, Lr = orc.gated_attention(Q[keep], K[keep], V[keep], lg[keep], pos[keep], [0, M - 1], Hq, Hkv, 0.5,
                                     head_gain=gain, unnormalised=unnorm)
        assert np.isfinite(O).all()
        np.testing.assert_allclose(O[keep], Or, rtol=1e-12, atol=1e-13)
        if not unnorm:  # the removed key's own row still sees the keys before it
            np.testing.assert_allclose(L[:, keep], Lr, rtol=1e-12, atol=1e-13)
    # gain 0 with open gates is plain causal attention (bias 0)
    O0, _ = orc.gated_attention(Q, K, V, lg, pos, [0, M], Hq, Hkv, 0.5, head_gain=gain)
    P0, _ = orc.gated_attention(Q[keep], K[keep], V[keep], None, pos[keep], [0, M - 1], Hq, Hkv, 0.5)
    np.testing.assert_allclose(O0[keep, 0], P0[:, 0], rtol=1e-12, atol=1e-13)
    # the first two rows with closed gates: row 0 and row 1 see only closed keys
    lz = lg.copy()
    lz[:2] = -np.inf
    O, L = orc.gated_attention(Q, K, V, lz, pos, [0, M], Hq, Hkv, 0.5, head_gain=gain)
    assert np.all(O[:2] == 0) and np.all(L[:, :2] == -np.inf)
    dO = g.standard_normal((M, Hq, D))
    dQ, dK, dV, dl = orc.gated_attention_bwd(Q, K, V, lz, pos, [0, M], Hq, Hkv, 0.5, dO, head_gain=gain)
    for t in (dQ, dK, dV, dl):
        assert np.isfinite(t).all()
    assert np.all(dQ[:2] == 0) and np.all(dl[:2] == 0)
    # away from the closed rows the gradient is that of the sequence without those keys' weight
    dQr, dKr, dVr, dlr = orc.gated_attention_bwd(Q[2:], K[2:], V[2:], lz[2:], pos[2:], [0, M - 2], Hq, Hkv, 0.5,
                                                 dO[2:], head_gain=gain)
    np.testing.assert_allclose(dQ[2:], dQr, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dK[2:], dKr, rtol=1e-10, atol=1e-12)


def test_score_temperature_golden_and_selection_invariance(golden_dir):
    """The gate temperature (a reading: it divides the score) against the hand-derived one-hot
    case, and the property that makes it a temperature: the kept set is the same for every
    temperature > 0, while g = sigmoid(s / T) flattens towards 1/2 as T grows."""
    fx = _load(golden_dir, "score_onehot.json")
    tc = fx["temperature_case"]
    s = orc.gate_scores(np.array(fx["H"]), np.array(fx["W1"]), np.array(fx["b1"]), np.array(fx["w2"]), fx["b2"],
                        temperature=tc["temperature"])
    np.testing.assert_allclose(s, tc["expected"], rtol=0, atol=tc["tolerance_abs"])
    wl = ti.scaled(ti.WORKLOADS["tiny_f32"], seqlens=(300, 77), q_len=(20, 5), k=(40, 30))
    H = ti.hidden_states(wl)
    W1, b1, w2, b2 = ti.gate_weights(wl, biased=True)
    base = orc.gate_scores(H, W1, b1, w2, b2)
    kept1, _ = orc.topk_select(base, wl.seqlens, wl.q_len, wl.k)
    spread = []
    for T in (0.05, 0.7, 3.0, 40.0):
        sT = orc.gate_scores(H, W1, b1, w2, b2, temperature=T)
        keptT, _ = orc.topk_select(sT, wl.seqlens, wl.q_len, wl.k)
        assert np.array_equal(keptT, kept1)
        g, _ = orc.gate_value(sT)
        spread.append(float(np.max(np.abs(g - 0.5))))
    assert spread == sorted(spread, reverse=True) and spread[-1] < 0.05


def test_gelu_grad_matches_central_differences():
    z = np.linspace(-7, 7, 281)
    h = 1e-6
    fd = (orc.gelu(z + h) - orc.gelu(z - h)) / (2 * h)
    np.testing.assert_allclose(orc.gelu_grad(z), fd, rtol=0, atol=1e-8)
    assert orc.gelu_grad(0.0) == 0.5  # Phi(0) + 0


def test_gate_mlp_grad_matches_central_differences_and_autograd():
    """dW1, db1, dw2, db2 of L = sum_i dscore_i s_i against central differences of gate_scores
    (every element of a small case with d != dg and a temperature) and torch autograd of a
    direct torch statement of the score network (float64)."""
    import torch
    g = np.random.default_rng(12)
    M, d, dg, T = 7, 5, 3, 1.7
    H = g.standard_normal((M, d))
    W1 = g.standard_normal((dg, d)) * 0.7
    b1 = g.standard_normal(dg) * 0.3
    w2 = g.standard_normal(dg)
    b2 = 0.2
    ds = g.standard_normal(M)
    dW1, db1, dw2, db2 = orc.gate_mlp_grad(H, W1, b1, w2, ds, temperature=T)
    loss = lambda W1_, b1_, w2_, b2_: float(ds @ orc.gate_scores(H, W1_, b1_, w2_, b2_, temperature=T))
    h = 1e-6
    for arr, grad, name in ((W1, dW1, "W1"), (b1, db1, "b1"), (w2, dw2, "w2")):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            up, dn = arr.copy(), arr.copy()
            up[idx] += h
            dn[idx] -= h
            args_up = {"W1": (up, b1, w2), "b1": (W1, up, w2), "w2": (W1, b1, up)}[name]
            args_dn = {"W1": (dn, b1, w2), "b1": (W1, dn, w2), "w2": (W1, b1, dn)}[name]
            fd[idx] = (loss(*args_up, b2) - loss(*args_dn, b2)) / (2 * h)
        np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-8, err_msg=name)
    assert abs(db2 - (loss(W1, b1, w2, b2 + h) - loss(W1, b1, w2, b2 - h)) / (2 * h)) < 1e-8
    tH = torch.tensor(H)
    tW = torch.tensor(W1, requires_grad=True)
    tb = torch.tensor(b1, requires_grad=True)
    tw = torch.tensor(w2, requires_grad=True)
    tb2 = torch.tensor(b2, dtype=torch.float64, requires_grad=True)
    s = (torch.nn.functional.gelu(tH @ tW.T + tb) @ tw + tb2) / T
    (torch.tensor(ds) * s).sum().backward()
    for t, r in ((tW, dW1), (tb, db1), (tw, dw2), (tb2, db2)):
        np.testing.assert_allclose(t.grad.numpy(), r, rtol=1e-12, atol=1e-14)


def test_prefill_projected_is_the_composition_of_its_steps():
    """The projected chain is the selection path followed, per layer, by the projection of the
    kept rows and attention over them: K/V of dropped tokens never exist (a perturbed dropped row
    changes nothing), and the layer outputs equal qkv_rope + gated_attention on the kept rows."""
    wl = ti.scaled(ti.WORKLOADS["tiny_f32"], seqlens=(80, 50), q_len=(8, 4), k=(20, 9))
    H = ti.hidden_states(wl).astype(np.float64)
    W1, b1, w2, b2 = ti.gate_weights(wl, biased=True)
    g = np.random.default_rng(2)
    Ws = [g.standard_normal(((wl.Hq + 2 * wl.Hkv) * wl.D, wl.d)) / math.sqrt(wl.d) for _ in range(2)]
    r = orc.prefill_projected(H, W1, b1, w2, b2, wl.seqlens, wl.q_len, wl.k, Ws, 1e4, wl.Hq, wl.Hkv, wl.D, 0.125)
    for W, (Q, K, V, O, L) in zip(Ws, r["layers"]):
        Q2, K2, V2 = orc.qkv_rope(H[r["kept"]], W, r["pos"], wl.Hq, wl.Hkv, wl.D, 1e4)
        np.testing.assert_array_equal(K, K2)
        O2, _ = orc.gated_attention(Q2, K2, V2, r["logg"], r["pos"], r["cu_kept"], wl.Hq, wl.Hkv, 0.125)
        np.testing.assert_allclose(O, O2, rtol=0, atol=1e-14)
    dropped = np.setdiff1d(np.arange(sum(wl.seqlens)), r["kept"])
    s = orc.gate_scores(H, W1, b1, w2, b2)
    order = np.argsort(s[dropped])[:3]  # the lowest-scoring dropped rows, pushed further down
    H2 = H.copy()
    for i in dropped[order]:
        H2[i] = H[i] * 0.5
    r2 = orc.prefill_projected(H2, W1, b1, w2, b2, wl.seqlens, wl.q_len, wl.k, Ws, 1e4, wl.Hq, wl.Hkv, wl.D, 0.125)
    if np.array_equal(r2["kept"], r["kept"]):
        for a, b in zip(r["layers"], r2["layers"]):
            np.testing.assert_array_equal(a[3], b[3])
