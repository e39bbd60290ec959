"""Gradients of the gate network's parameters (tg_gate_mlp_bwd) against the oracle's
gate_mlp_grad: dW1, db1, dw2, db2 within the tolerance of the dtype (max-abs-relative 1e-4 for
f32, 2e-2 for bf16), deterministic, and the end-to-end training path: the chain's kept rows,
the attention backward's d score, then these gradients. bf16 shapes with dg % 128 == 0 and
d % 128 == 0 run on the tensor cores, the others on the CUDA cores."""
import math

import numpy as np
import pytest
import torch

import learned_token_pruning_02_b200 as tg
import tg_inputs as ti
from oracle import tg_oracle as orc
from tg_testutil import TOL, bits, from_dev, max_abs_rel, to_dev

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _check(got, ref, tol):
    for name, x, r in zip(("dW1", "db1", "dw2", "db2"), got, ref):
        err = max_abs_rel(from_dev(x), np.atleast_1d(r))
        assert err <= tol, (name, err)


# bf16 with dg % 128 == 0 and d % 128 == 0 runs the tensor-core kernels: one row, ragged tails of
# 1 and of 65 rows past a 64-row chunk, three and four dg tiles, d = 384 (three K chunks per split),
# the first product's K split 8, 4, 2 and 1 ways (65, 1000 / 2176, 4352, 10000 rows) and several
# row splits of dW1, and 100000 rows (782 row tiles, the u pass over 391 row blocks); the rest
# runs on the CUDA cores.
@pytest.mark.parametrize("dtype,M,d,dg,T", [("f32", 96, 256, 64, 1.0), ("f32", 333, 512, 128, 0.6),
                                            ("bf16", 2176, 2048, 256, 1.0), ("bf16", 1, 128, 64, 2.0),
                                            ("bf16", 4352, 2048, 256, 1.3), ("bf16", 1, 256, 128, 1.0),
                                            ("bf16", 129, 256, 128, 0.7), ("bf16", 1000, 512, 384, 1.0),
                                            ("bf16", 65, 1024, 256, 2.0), ("bf16", 200, 128, 128, 1.0),
                                            ("bf16", 10000, 256, 128, 0.9), ("bf16", 700, 384, 512, 1.0),
                                            ("bf16", 100000, 256, 128, 1.0)])
def test_gate_mlp_bwd_matches_oracle(dtype, M, d, dg, T):
    g = np.random.default_rng(M + d)

    def arr(*shape, s=1.0):
        x = (g.standard_normal(shape) * s).astype(np.float32)
        return ti.f32_to_bf16_bits(x) if dtype == "bf16" else x

    H, W1, w2 = arr(M, d), arr(dg, d, s=1 / math.sqrt(d)), arr(dg, s=1 / math.sqrt(dg))
    b1 = (g.standard_normal(dg) * 0.1).astype(np.float32)
    ds = (g.standard_normal(M) * 0.01).astype(np.float32)
    got = tg.tg_gate_mlp_bwd(to_dev(H, dtype), to_dev(W1, dtype), to_dev(b1, "f32"), to_dev(w2, dtype),
                             to_dev(ds, "f32"), temperature=T)
    again = tg.tg_gate_mlp_bwd(to_dev(H, dtype), to_dev(W1, dtype), to_dev(b1, "f32"), to_dev(w2, dtype),
                               to_dev(ds, "f32"), temperature=T)
    torch.cuda.synchronize()
    ref = orc.gate_mlp_grad(ti.widen(H, dtype), ti.widen(W1, dtype), b1, ti.widen(w2, dtype), ds, temperature=T)
    _check(got, ref, TOL[dtype])
    # db1, dw2 and db2 are fp32 sums of fp32 values on both paths (only dW1 takes u in bf16), so
    # they hold a bound far below the bf16 tolerance: this pins the GELU / GELU' evaluation (erf
    # from Abramowitz & Stegun 7.1.26 on the tensor-core path, |error| <= 1.5e-7)
    for name, x, r in zip(("db1", "dw2", "db2"), got[1:], ref[1:]):
        err = max_abs_rel(from_dev(x), np.atleast_1d(r))
        assert err <= 1e-3, (name, err)
    for a, b in zip(got, again):  # deterministic
        assert np.array_equal(bits(a), bits(b))


def test_gate_mlp_bwd_no_rows_gives_zero():
    dW1 = torch.full((64, 128), 5.0, device="cuda")
    db1, dw2, db2 = (torch.full((64,), 5.0, device="cuda"), torch.full((64,), 5.0, device="cuda"),
                     torch.full((1,), 5.0, device="cuda"))
    H = torch.zeros(0, 128, device="cuda", dtype=torch.bfloat16)
    W1 = torch.zeros(64, 128, device="cuda", dtype=torch.bfloat16)
    tg.tg_gate_mlp_bwd(H, W1, None, torch.zeros(64, device="cuda", dtype=torch.bfloat16),
                       torch.zeros(0, device="cuda"), dW1=dW1, db1=db1, dw2=dw2, db2=db2)
    torch.cuda.synchronize()
    for t in (dW1, db1, dw2, db2):
        assert torch.count_nonzero(t).item() == 0


def test_training_path_chain_to_gate_gradients():
    """Score -> select -> gather -> gated attention (forward), then the attention backward's
    d score of the kept rows -> the gate network's gradients, all on the GPU, against the oracle
    run on the GPU's own kept set (ragged four-sequence workload, one layer)."""
    wl = ti.WORKLOADS["ragged4"]
    Hn = ti.hidden_states(wl)
    W1n, b1n, w2n, b2 = ti.gate_weights(wl, biased=True)
    Q, K, V = ti.qkv(wl, 0)
    layers = [tuple(to_dev(x, "bf16") for x in (Q, K, V))]
    scale = 1.0 / math.sqrt(wl.D)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = tg.tg_prefill_above_L(to_dev(Hn, "bf16"), to_dev(W1n, "bf16"), to_dev(b1n, "f32"), to_dev(w2n, "bf16"), b2,
                                wl.seqlens, wl.q_len, wl.k, layers, scale, want_lse=True, dev_status=st)
    cu = tg.tg_kept_counts(wl.seqlens, wl.q_len, wl.k)
    dO = to_dev(ti.f32_to_bf16_bits(np.random.default_rng(4).standard_normal(Q.shape).astype(np.float32)), "bf16")
    _, _, _, _, dscore = tg.tg_gated_attn_bwd(*layers[0], out["logg"], out["pos"], cu, out["O"][0], out["lse"][0], dO,
                                              scale, want_dscore=True, dev_status=st)
    got = tg.tg_gate_mlp_bwd(out["H_kept"], to_dev(W1n, "bf16"), to_dev(b1n, "f32"), to_dev(w2n, "bf16"), dscore)
    torch.cuda.synchronize()
    assert st.item() == 0
    # oracle on the GPU's own kept set (selection is bit-exact, checked elsewhere)
    s_gpu = out["score"].cpu().numpy()
    kept, cu_o = orc.topk_select(s_gpu, wl.seqlens, wl.q_len, wl.k)
    assert np.array_equal(out["kept_idx"].cpu().numpy(), kept.astype(np.int32))
    Hk, pos, _, lg = orc.gather(Hn, s_gpu, kept, wl.seqlens, wl.q_len, cu_o)
    _, _, _, dlogg = orc.gated_attention_bwd(ti.widen(Q, "bf16"), ti.widen(K, "bf16"), ti.widen(V, "bf16"), lg, pos,
                                             cu_o, wl.Hq, wl.Hkv, scale, from_dev(dO))
    ds_ref = orc.gate_score_grad(dlogg, lg)
    assert max_abs_rel(from_dev(dscore), ds_ref) <= TOL["bf16"]
    # the gate step on the d score it was given (sums such as db2 cancel, so comparing them across
    # two d score vectors that differ within tolerance would measure the cancellation, not the step)
    ref = orc.gate_mlp_grad(ti.widen(Hk, "bf16"), ti.widen(W1n, "bf16"), b1n, ti.widen(w2n, "bf16"), from_dev(dscore))
    _check(got, ref, TOL["bf16"])
