"""The gated path with each above-L layer's own projections (tg_prefill_projected): score ->
top-K -> kept rows -> per layer Q/K/V with rotary embedding at original positions (K and V are
the layer's key/value cache of kept rows only) -> gated attention.

Every output equals the single entry points run one after another, bit for bit; against the
oracle the kept set is bit-exact (top-K on the GPU's own scores), the caches and O are within the
bf16 tolerance (O both from the GPU's own Q/K/V and end to end from the float64 projections)."""
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


def _wqkv(wl, n_layers, seed=77):
    g = np.random.default_rng(seed)
    return [ti.f32_to_bf16_bits((g.standard_normal(((wl.Hq + 2 * wl.Hkv) * wl.D, wl.d)) / math.sqrt(wl.d))
                                .astype(np.float32)) for _ in range(n_layers)]


@pytest.mark.parametrize("name,n_layers,theta,sample", [("ragged4", 2, 1.0e6, False), ("qwen3_32k", 1, 1.0e6, True),
                                                        ("qwen3_8k", 1, 0.0, False)])
def test_projected_chain(name, n_layers, theta, sample):
    wl = ti.WORKLOADS[name]
    Hn = ti.hidden_states(wl)
    W1n, b1n, w2n, b2 = ti.gate_weights(wl, biased=True)
    Wn = _wqkv(wl, n_layers)
    H, W1, b1, w2 = to_dev(Hn, "bf16"), to_dev(W1n, "bf16"), to_dev(b1n, "f32"), to_dev(w2n, "bf16")
    Wd = [to_dev(w, "bf16") for w in Wn]
    scale = 1.0 / math.sqrt(wl.D)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = tg.tg_prefill_projected(H, W1, b1, w2, b2, wl.seqlens, wl.q_len, wl.k, Wd, theta, wl.Hq, wl.Hkv, wl.D,
                                  scale, want_lse=True, dev_status=st)
    # the single entry points one after another
    s = tg.tg_score(H, W1, b1, w2, b2)
    kept, cu_dev = tg.tg_topk_select(s, wl.seqlens, wl.q_len, wl.k)
    Hk, pos, gv, lg = tg.tg_gather(H, s, kept, wl.seqlens, wl.q_len, wl.k)
    cu = tg.tg_kept_counts(wl.seqlens, wl.q_len, wl.k)
    torch.cuda.synchronize()
    assert st.item() == 0
    for key, ref in (("score", s), ("kept_idx", kept), ("cu_kept_dev", cu_dev), ("H_kept", Hk), ("pos", pos),
                     ("g", gv), ("logg", lg)):
        assert np.array_equal(bits(out[key]), bits(ref)), key
    for l in range(n_layers):
        Q, K, V = tg.tg_qkv_rope(Hk, Wd[l], pos, wl.Hq, wl.Hkv, wl.D, theta)
        O, L = tg.tg_gated_attn_fwd(Q, K, V, lg, pos, cu, scale)
        torch.cuda.synchronize()
        for key, a, b in (("Q", out["Q"][l], Q), ("K_cache", out["K_cache"][l], K), ("V_cache", out["V_cache"][l], V),
                          ("O", out["O"][l], O), ("lse", out["lse"][l], L)):
            assert np.array_equal(bits(a), bits(b)), (key, l)
    # against the oracle on the GPU's own scores
    s_np = s.cpu().numpy()
    kept_o, cu_o = orc.topk_select(s_np, wl.seqlens, wl.q_len, wl.k)
    assert np.array_equal(kept.cpu().numpy(), kept_o.astype(np.int32))
    Hk_o, pos_o, _, lg_o = orc.gather(ti.widen(Hn, "bf16"), s_np, kept_o, wl.seqlens, wl.q_len, cu_o)
    M = cu[-1]
    rows = (np.unique(np.concatenate([np.random.default_rng(3).integers(0, M, 256), np.arange(M - 128, M)]))
            if sample else None)
    for l in range(n_layers):
        Qo, Ko, Vo = orc.qkv_rope(Hk_o, ti.widen(Wn[l], "bf16"), pos_o, wl.Hq, wl.Hkv, wl.D, theta)
        for got, ref in ((out["Q"][l], Qo), (out["K_cache"][l], Ko), (out["V_cache"][l], Vo)):
            assert max_abs_rel(from_dev(got), ref) <= TOL["bf16"]
        # attention stage on the GPU's own (bf16) projections
        rO, rL = orc.gated_attention(from_dev(out["Q"][l]), from_dev(out["K_cache"][l]), from_dev(out["V_cache"][l]),
                                     lg_o, pos_o, cu_o, wl.Hq, wl.Hkv, scale, rows=rows)
        sel = slice(None) if rows is None else rows
        assert max_abs_rel(from_dev(out["O"][l])[sel], rO) <= TOL["bf16"]
        assert max_abs_rel(from_dev(out["lse"][l])[:, sel], rL) <= TOL["bf16"]
        # end to end from the float64 projections
        eO, _ = orc.gated_attention(Qo, Ko, Vo, lg_o, pos_o, cu_o, wl.Hq, wl.Hkv, scale, rows=rows)
        assert max_abs_rel(from_dev(out["O"][l])[sel], eO) <= TOL["bf16"]
