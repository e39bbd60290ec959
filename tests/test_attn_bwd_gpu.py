"""Gradients of the token-gated attention (tg_gated_attn_bwd) against the oracle's
gated_attention_bwd: dQ, dK, dV, d log g and d score, per tensor within the tolerance of the
dtype (max-abs-relative 1e-4 for f32, 2e-2 for bf16).

Cases cover ragged tiles and empty sequences, more KV heads than a cluster holds (16), one KV
head (no cluster), no gate (log g absent), per-head gains, 70 sequences (two launches), the
ragged kept counts of the four-sequence workload, 8, 6 and 1 query heads per KV head in bf16
(the dK/dV clusters of 8, 2 and 1 CTAs), and the Qwen3-1.7B shapes at N=32K, K=2K chained after
the library's own forward. O and lse fed to the backward come from the oracle's
forward (or from the library's forward in the chained case); the oracle recomputes everything
from Q, K, V, log g and dO."""
import math

import numpy as np
import pytest
import torch

import learned_token_pruning_02_b200 as tg
import tg_inputs as ti
from oracle import tg_oracle as orc
from tg_testutil import TOL, from_dev, max_abs_rel, to_dev

pytestmark = pytest.mark.gpu


def _make(seed, lens, Hq, Hkv, D, dtype, gain, with_logg):
    g = np.random.default_rng(seed)
    M = int(sum(lens))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    pos = np.concatenate([np.sort(g.choice(3 * n + 1, n, replace=False)) for n in lens] or [np.zeros(0)])
    pos = pos.astype(np.int32)

    def arr(*shape, s=1.0):
        x = (g.standard_normal(shape) * s).astype(np.float32)
        return ti.f32_to_bf16_bits(x) if dtype == "bf16" else x

    sc = 1.0 / math.sqrt(D)
    Q, K, V = arr(M, Hq, D, s=2.0), arr(M, Hkv, D, s=2.0), arr(M, Hkv, D)
    dO = arr(M, Hq, D)
    logg = np.log(g.uniform(0.02, 1.0, M)).astype(np.float32) if with_logg else None
    hg = g.uniform(0.5, 1.5, Hq).astype(np.float32) if gain else None
    return dict(M=M, cu=cu, pos=pos, Q=Q, K=K, V=V, dO=dO, logg=logg, hg=hg, Hq=Hq, Hkv=Hkv, D=D, dtype=dtype,
                scale=sc)


def _oracle(c):
    w = lambda a: ti.widen(a, c["dtype"])
    O, lse = orc.gated_attention(w(c["Q"]), w(c["K"]), w(c["V"]), c["logg"], c["pos"], c["cu"], c["Hq"], c["Hkv"],
                                 c["scale"], head_gain=c["hg"])
    grads = orc.gated_attention_bwd(w(c["Q"]), w(c["K"]), w(c["V"]), c["logg"], c["pos"], c["cu"], c["Hq"],
                                    c["Hkv"], c["scale"], w(c["dO"]), head_gain=c["hg"])
    return O, lse, grads


def _run(c, O, lse, st, want_dscore=True, flags=0):
    dt = c["dtype"]
    O_in = ti.f32_to_bf16_bits(O.astype(np.float32)) if dt == "bf16" else O.astype(np.float32)
    dev = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return tg.tg_gated_attn_bwd(
        to_dev(c["Q"], dt), to_dev(c["K"], dt), to_dev(c["V"], dt), dev(c["logg"]), dev(c["pos"]), c["cu"].tolist(),
        to_dev(O_in, dt), dev(lse.astype(np.float32)), to_dev(c["dO"], dt), c["scale"], head_gain=dev(c["hg"]),
        flags=flags, want_dscore=want_dscore and c["logg"] is not None, dev_status=st)


def _check(c, got, grads):
    tol = TOL[c["dtype"]]
    dQ, dK, dV, dl = grads
    for name, x, r in (("dQ", got[0], dQ), ("dK", got[1], dK), ("dV", got[2], dV), ("dlogg", got[3], dl)):
        err = max_abs_rel(from_dev(x), r)
        assert err <= tol, (name, err)
    if got[4] is not None:
        err = max_abs_rel(from_dev(got[4]), orc.gate_score_grad(dl, c["logg"]))
        assert err <= tol, ("dscore", err)


CASES = {  # name: (seed, lens, Hq, Hkv, D, dtype, gain, with_logg)
    "f32_ragged_gqa": (1, [5, 7, 40, 1, 0, 33], 4, 2, 64, "f32", True, True),
    "f32_16_kv_heads": (2, [100, 37], 16, 16, 128, "f32", False, True),
    "f32_one_kv_head_no_gate": (3, [70], 4, 1, 64, "f32", True, False),
    "f32_70_sequences": (4, list(np.random.default_rng(9).integers(0, 21, 70)), 2, 1, 64, "f32", True, True),
    "bf16_qwen3_1000_rows": (5, [1000], 16, 8, 128, "bf16", True, True),
    "bf16_four_ragged": (6, [320, 456, 288, 384], 16, 8, 128, "bf16", False, True),
    "bf16_d64": (7, [130, 64], 8, 2, 64, "bf16", True, True),
    "bf16_eight_heads_per_kv": (12, [300], 16, 2, 128, "bf16", True, True),
    "bf16_six_heads_per_kv_d64": (13, [200, 77], 12, 2, 64, "bf16", True, True),
    "bf16_no_grouping": (14, [150, 0, 129], 4, 4, 128, "bf16", False, True),
}


@pytest.mark.parametrize("name", list(CASES))
def test_attn_bwd_matches_oracle(name):
    c = _make(*CASES[name])
    O, lse, grads = _oracle(c)
    st = torch.zeros(1, device="cuda", dtype=torch.int32)
    got = _run(c, O, lse, st)
    torch.cuda.synchronize()
    _check(c, got, grads)
    assert st.item() == 0


def test_attn_bwd_deterministic():
    c = _make(*CASES["f32_ragged_gqa"])
    O, lse, _ = _oracle(c)
    st = torch.zeros(1, device="cuda", dtype=torch.int32)
    a = _run(c, O, lse, st)
    b = _run(c, O, lse, st)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_attn_bwd_after_library_forward_qwen3_32k():
    """N=32K, K=2K kept set (2176 rows), 16/8 heads, D=128, bf16: the library's forward gives
    O and lse, the backward runs on them; every element of every gradient is compared."""
    c = _make(8, [2176], 16, 8, 128, "bf16", True, True)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    Qd, Kd, Vd = to_dev(c["Q"], "bf16"), to_dev(c["K"], "bf16"), to_dev(c["V"], "bf16")
    lg, ps, hg = dev(c["logg"]), dev(c["pos"]), dev(c["hg"])
    st = torch.zeros(1, device="cuda", dtype=torch.int32)
    O, lse = tg.tg_gated_attn_fwd(Qd, Kd, Vd, lg, ps, c["cu"].tolist(), c["scale"], head_gain=hg, dev_status=st)
    got = tg.tg_gated_attn_bwd(Qd, Kd, Vd, lg, ps, c["cu"].tolist(), O, lse, to_dev(c["dO"], "bf16"), c["scale"],
                               head_gain=hg, want_dscore=True, dev_status=st)
    torch.cuda.synchronize()
    w = lambda a: ti.widen(a, "bf16")
    grads = orc.gated_attention_bwd(w(c["Q"]), w(c["K"]), w(c["V"]), c["logg"], c["pos"], c["cu"], 16, 8, c["scale"],
                                    w(c["dO"]), head_gain=c["hg"])
    _check(c, got, grads)
    assert st.item() == 0


def test_attn_bwd_flags_positions_not_ascending():
    c = _make(10, [50], 2, 1, 64, "f32", False, True)
    O, lse, _ = _oracle(c)
    c["pos"] = c["pos"].copy()
    c["pos"][20], c["pos"][21] = c["pos"][21], c["pos"][20]
    st = torch.zeros(1, device="cuda", dtype=torch.int32)
    _run(c, O, lse, st)
    torch.cuda.synchronize()
    assert st.item() & tg.TG_DEV_POS_NOT_ASCENDING


def test_attn_bwd_rejects_unsupported():
    c = _make(11, [40], 2, 1, 64, "f32", False, True)
    O, lse, _ = _oracle(c)
    st = torch.zeros(1, device="cuda", dtype=torch.int32)
    with pytest.raises(tg.TokenGateError):
        _run(c, O, lse, st, flags=tg.TG_ATTN_UNNORMALISED)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    with pytest.raises(tg.TokenGateError):
        tg.tg_gated_attn_bwd(dev(c["Q"]), dev(c["K"]), dev(c["V"]), None, dev(c["pos"]), c["cu"].tolist(),
                             dev(O.astype(np.float32)), dev(lse.astype(np.float32)), dev(c["dO"]), c["scale"],
                             want_dscore=True)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_closed_gates_forward_and_backward(dtype):
    """Keys with gate value exactly 0 (log g = -inf) are masked whatever the head gain, a gain
    of 0 included; the first rows of a sequence, whose visible keys are all closed, get O = 0,
    LSE = -inf and zero gradients. Forward and backward against the oracle, no NaN anywhere."""
    c = _make(31, [300, 77], 4, 2, 128 if dtype == "bf16" else 64, dtype, True, True)
    lg = c["logg"].copy()
    lg[[0, 1, 7, 150, 299, 300, 340]] = -np.inf
    c["logg"] = lg
    c["hg"] = np.array([0.0, 1.0, 0.7, 0.0], np.float32)
    O, lse, grads = _oracle(c)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dev = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()
    Og, Lg = tg.tg_gated_attn_fwd(to_dev(c["Q"], dtype), to_dev(c["K"], dtype), to_dev(c["V"], dtype), dev(lg),
                                  dev(c["pos"]), c["cu"].tolist(), c["scale"], head_gain=dev(c["hg"]), dev_status=st)
    torch.cuda.synchronize()
    Ogn, Lgn = from_dev(Og), from_dev(Lg)
    assert not np.isnan(Ogn).any() and not np.isnan(Lgn).any()
    assert max_abs_rel(Ogn, O) <= TOL[dtype]
    fin = np.isfinite(lse)
    assert np.array_equal(np.isfinite(Lgn), fin)
    assert max_abs_rel(Lgn[fin], lse[fin]) <= TOL[dtype]
    got = _run(c, O, lse, st)
    torch.cuda.synchronize()
    for t in got:
        if t is not None:
            assert not torch.isnan(t).any()
    _check(c, got, grads)
    assert st.item() == 0
