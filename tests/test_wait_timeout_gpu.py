"""The bounded waits of the tensor-core kernels, driven to their limit on purpose.

With the test hook tg_set_test_wait_probe(limit) every tensor-core kernel first waits on a
barrier that nothing signals. That wait runs out after `limit`, the kernel records
TG_DEV_TIMEOUT in the status word, skips its work (nothing was issued yet, so nothing is in
flight) and returns. The host reads the status after an ordinary synchronise, and the next
calls, with the hook off, must match the oracle again: the context stays usable."""
import math

import numpy as np
import pytest
import torch

import learned_token_pruning_02_b200 as tg
import tg_inputs as ti
from oracle import tg_oracle as orc
from tg_testutil import TOL, from_dev, max_abs_rel, to_dev

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

PROBE_NS = 200_000  # 0.2 ms per CTA


def _inputs():
    wl = ti.scaled(ti.WORKLOADS["qwen3_8k"], seqlens=(1500,), q_len=(20,), k=(300,))
    H = ti.hidden_states(wl)
    W1, b1, w2, b2 = ti.gate_weights(wl, biased=True)
    M = tg.tg_kept_counts(wl.seqlens, wl.q_len, wl.k)[-1]
    Q, K, V = ti.qkv(wl, 0, M)
    return wl, H, (W1, b1, w2, b2), (Q, K, V), M


def test_waits_run_out_and_the_context_stays_usable():
    wl, H, (W1, b1, w2, b2), (Q, K, V), M = _inputs()
    Hd = to_dev(H, "bf16")
    W1d, b1d, w2d = to_dev(W1, "bf16"), to_dev(b1, "f32"), to_dev(w2, "bf16")
    Qd, Kd, Vd = to_dev(Q, "bf16"), to_dev(K, "bf16"), to_dev(V, "bf16")
    pos = torch.arange(M, dtype=torch.int32, device="cuda")
    scale = 1.0 / math.sqrt(wl.D)
    sentinel = torch.full((wl.n_tok,), 123.0, device="cuda")
    O_sent = torch.full((M, wl.Hq, wl.D), 7.0, device="cuda", dtype=torch.bfloat16)
    Wqkv = to_dev(ti.f32_to_bf16_bits((np.random.default_rng(3).standard_normal(
        ((wl.Hq + 2 * wl.Hkv) * wl.D, wl.d)) / math.sqrt(wl.d)).astype(np.float32)), "bf16")
    st = [torch.zeros(1, dtype=torch.int32, device="cuda") for _ in range(4)]
    try:
        tg.tg_set_test_wait_probe(PROBE_NS)
        score = sentinel.clone()
        tg.tg_score(Hd, W1d, b1d, w2d, b2, score=score, dev_status=st[0])
        O = O_sent.clone()
        tg.tg_gated_attn_fwd(Qd, Kd, Vd, None, pos, [0, M], scale, O=O, dev_status=st[1])
        Qp, _, _ = tg.tg_qkv_rope(Hd[:M].contiguous(), Wqkv, pos, wl.Hq, wl.Hkv, wl.D, 1e6, dev_status=st[2])
        out = tg.tg_prefill_above_L(Hd, W1d, b1d, w2d, b2, wl.seqlens, wl.q_len, wl.k, [(Qd, Kd, Vd)], scale,
                                    dev_status=st[3])
        torch.cuda.synchronize()
    finally:
        tg.tg_set_test_wait_probe(0)
    for s in st:
        assert s.item() & tg.TG_DEV_TIMEOUT, s.item()
    # a kernel that gave up before issuing anything leaves its outputs as they were
    assert torch.equal(score, sentinel)
    assert torch.equal(O, O_sent)

    # hook off: the same calls match the oracle, with a clean status word
    st0 = torch.zeros(1, dtype=torch.int32, device="cuda")
    score = tg.tg_score(Hd, W1d, b1d, w2d, b2, dev_status=st0)
    O, L = tg.tg_gated_attn_fwd(Qd, Kd, Vd, None, pos, [0, M], scale, dev_status=st0)
    torch.cuda.synchronize()
    ref_s = orc.gate_scores(ti.widen(H, "bf16"), ti.widen(W1, "bf16"), b1, ti.widen(w2, "bf16"), b2)
    assert max_abs_rel(from_dev(score), ref_s) <= TOL["bf16"]
    rO, rL = orc.gated_attention(ti.widen(Q, "bf16"), ti.widen(K, "bf16"), ti.widen(V, "bf16"), None,
                                 np.arange(M), [0, M], wl.Hq, wl.Hkv, scale)
    assert max_abs_rel(from_dev(O), rO) <= TOL["bf16"]
    assert max_abs_rel(from_dev(L), rL) <= TOL["bf16"]
    assert st0.item() == 0


def test_backward_waits_run_out_and_the_context_stays_usable():
    """tg_gated_attn_bwd (bf16): with the hook on, its tensor-core kernels time out, record
    TG_DEV_TIMEOUT and write neither dK nor dV; with the hook off the same call matches the oracle."""
    g = np.random.default_rng(5)
    M, Hq, Hkv, D = 300, 4, 2, 64
    scale = 1.0 / math.sqrt(D)
    bits = lambda *shape: ti.f32_to_bf16_bits(g.standard_normal(shape).astype(np.float32))
    Q, K, V, dO = bits(M, Hq, D), bits(M, Hkv, D), bits(M, Hkv, D), bits(M, Hq, D)
    logg = np.log(g.uniform(0.05, 1.0, M)).astype(np.float32)
    pos = np.arange(M, dtype=np.int32) * 2
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    Qd, Kd, Vd, dOd = (to_dev(x, "bf16") for x in (Q, K, V, dO))
    lg, ps = dev(logg), dev(pos)
    O, lse = tg.tg_gated_attn_fwd(Qd, Kd, Vd, lg, ps, [0, M], scale)
    sent = lambda shape: torch.full(shape, 5.0, device="cuda")
    bufs = dict(dQ=sent((M, Hq, D)), dK=sent((M, Hkv, D)), dV=sent((M, Hkv, D)), dlogg=sent((M,)))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        tg.tg_set_test_wait_probe(PROBE_NS)
        tg.tg_gated_attn_bwd(Qd, Kd, Vd, lg, ps, [0, M], O, lse, dOd, scale, dev_status=st, **bufs)
        torch.cuda.synchronize()
    finally:
        tg.tg_set_test_wait_probe(0)
    assert st.item() & tg.TG_DEV_TIMEOUT, st.item()
    assert torch.equal(bufs["dK"], sent((M, Hkv, D))) and torch.equal(bufs["dV"], sent((M, Hkv, D)))

    st0 = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = tg.tg_gated_attn_bwd(Qd, Kd, Vd, lg, ps, [0, M], O, lse, dOd, scale, dev_status=st0)
    torch.cuda.synchronize()
    w = lambda a: ti.widen(a, "bf16")
    ref = orc.gated_attention_bwd(w(Q), w(K), w(V), logg, pos, [0, M], Hq, Hkv, scale, w(dO))
    for x, r in zip(got[:4], ref):
        assert max_abs_rel(from_dev(x), r) <= TOL["bf16"]
    assert st0.item() == 0


def test_gate_bwd_waits_run_out_and_the_context_stays_usable():
    """tg_gate_mlp_bwd (bf16, tensor-core shape): with the hook on, its products time out, record
    TG_DEV_TIMEOUT and the call writes none of its outputs; with the hook off it matches the oracle."""
    g = np.random.default_rng(6)
    M, d, dg = 300, 512, 128
    H = ti.f32_to_bf16_bits(g.standard_normal((M, d)).astype(np.float32))
    W1 = ti.f32_to_bf16_bits((g.standard_normal((dg, d)) / math.sqrt(d)).astype(np.float32))
    w2 = ti.f32_to_bf16_bits((g.standard_normal(dg) / math.sqrt(dg)).astype(np.float32))
    b1 = (g.standard_normal(dg) * 0.1).astype(np.float32)
    ds = (g.standard_normal(M) * 0.01).astype(np.float32)
    args = (to_dev(H, "bf16"), to_dev(W1, "bf16"), to_dev(b1, "f32"), to_dev(w2, "bf16"), to_dev(ds, "f32"))
    sent = lambda *shape: torch.full(shape, 5.0, device="cuda")
    outs = dict(dW1=sent(dg, d), db1=sent(dg), dw2=sent(dg), db2=sent(1))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        tg.tg_set_test_wait_probe(PROBE_NS)
        tg.tg_gate_mlp_bwd(*args, dev_status=st, **outs)
        torch.cuda.synchronize()
    finally:
        tg.tg_set_test_wait_probe(0)
    assert st.item() & tg.TG_DEV_TIMEOUT, st.item()
    assert torch.equal(outs["dW1"], sent(dg, d)) and torch.equal(outs["db1"], sent(dg))
    assert torch.equal(outs["dw2"], sent(dg)) and torch.equal(outs["db2"], sent(1))

    st0 = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = tg.tg_gate_mlp_bwd(*args, dev_status=st0)
    torch.cuda.synchronize()
    ref = orc.gate_mlp_grad(ti.widen(H, "bf16"), ti.widen(W1, "bf16"), b1, ti.widen(w2, "bf16"), ds)
    for x, r in zip(got, ref):
        assert max_abs_rel(from_dev(x), np.atleast_1d(r)) <= TOL["bf16"]
    assert st0.item() == 0


def test_probe_off_by_default_and_thread_local():
    """The hook is per host thread: another thread's setting does not reach this one."""
    import threading

    done = []

    def other():
        tg.tg_set_test_wait_probe(PROBE_NS)
        done.append(True)

    t = threading.Thread(target=other)
    t.start()
    t.join()
    assert done
    wl, H, (W1, b1, w2, b2), _, _ = _inputs()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = tg.tg_score(to_dev(H, "bf16"), to_dev(W1, "bf16"), to_dev(b1, "f32"), to_dev(w2, "bf16"), b2,
                    dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = orc.gate_scores(ti.widen(H, "bf16"), ti.widen(W1, "bf16"), b1, ti.widen(w2, "bf16"), b2)
    assert max_abs_rel(from_dev(s), ref) <= TOL["bf16"]
