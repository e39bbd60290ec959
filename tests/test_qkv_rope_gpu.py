"""Projection of the kept rows to Q/K/V with rotary embedding at original positions
(tg_qkv_rope) against the oracle's qkv_rope, within the bf16 tolerance. Cases cover two heads
per 128-column half (D = 64), the Qwen3-1.7B shapes, positions near 128K tokens (angles of
about 1e5 radians before reduction), no rotation, and both tile heights: 128-row tiles while
they fit one round of the SMs, 256-row tiles (two accumulators sharing every W slice) beyond,
with a ragged last tile and several tiles per SM."""
import numpy as np
import pytest
import torch

import learned_token_pruning_02_b200 as tg
import tg_inputs as ti
from oracle import tg_oracle as orc
from tg_testutil import TOL, from_dev, max_abs_rel, to_dev

pytestmark = pytest.mark.gpu

CASES = [  # (M, d, Hq, Hkv, D, theta, max position)
    (300, 256, 4, 2, 64, 1.0e4, 3000),
    (1088, 2048, 16, 8, 128, 1.0e6, 8192),       # 144 tiles of 128 rows: one round of the SMs
    (256, 256, 2, 1, 128, 1.0e4, 131072),
    (200, 512, 2, 1, 128, 0.0, 1000),
    (2300, 2048, 16, 8, 128, 1.0e6, 32768),      # 256-row tiles, the last one 252 rows deep
    (4352, 1024, 16, 8, 128, 1.0e6, 131072),     # 256-row tiles, about two per SM
]


@pytest.mark.parametrize("case", CASES)
def test_qkv_rope_matches_oracle(case):
    M, d, Hq, Hkv, D, theta, pmax = case
    g = np.random.default_rng(M + d + D)
    Hk = ti.f32_to_bf16_bits((g.standard_normal((M, d)) / 2).astype(np.float32))
    W = ti.f32_to_bf16_bits((g.standard_normal(((Hq + 2 * Hkv) * D, d)) / np.sqrt(d)).astype(np.float32))
    pos = np.sort(g.choice(pmax, size=M, replace=M > pmax)).astype(np.int32)
    st = torch.zeros(1, device="cuda", dtype=torch.int32)
    Q, K, V = tg.tg_qkv_rope(to_dev(Hk, "bf16"), to_dev(W, "bf16"), torch.from_numpy(pos).cuda(), Hq, Hkv, D, theta,
                             dev_status=st)
    torch.cuda.synchronize()
    rQ, rK, rV = orc.qkv_rope(ti.widen(Hk, "bf16"), ti.widen(W, "bf16"), pos, Hq, Hkv, D, theta)
    for got, ref, name in ((Q, rQ, "Q"), (K, rK, "K"), (V, rV, "V")):
        err = max_abs_rel(from_dev(got), ref)
        assert err <= TOL["bf16"], (name, err)
    assert st.item() == 0


def test_qkv_no_rotation_without_positions():
    """rope_theta = 0 needs no positions: pos=None (a NULL pointer through the C ABI) gives the
    plain projection, equal to the oracle's and bit-identical to the same call with positions."""
    M, d, Hq, Hkv, D = 333, 256, 4, 2, 64
    g = np.random.default_rng(5)
    Hk = ti.f32_to_bf16_bits((g.standard_normal((M, d)) / 2).astype(np.float32))
    W = ti.f32_to_bf16_bits((g.standard_normal(((Hq + 2 * Hkv) * D, d)) / np.sqrt(d)).astype(np.float32))
    st = torch.zeros(1, device="cuda", dtype=torch.int32)
    Hd, Wd = to_dev(Hk, "bf16"), to_dev(W, "bf16")
    Q, K, V = tg.tg_qkv_rope(Hd, Wd, None, Hq, Hkv, D, 0.0, dev_status=st)
    Q2, K2, V2 = tg.tg_qkv_rope(Hd, Wd, torch.arange(M, dtype=torch.int32, device="cuda"), Hq, Hkv, D, 0.0)
    torch.cuda.synchronize()
    rQ, rK, rV = orc.qkv_rope(ti.widen(Hk, "bf16"), ti.widen(W, "bf16"), np.zeros(M, np.int64), Hq, Hkv, D, 0.0)
    for got, again, ref in ((Q, Q2, rQ), (K, K2, rK), (V, V2, rV)):
        assert max_abs_rel(from_dev(got), ref) <= TOL["bf16"]
        assert torch.equal(got, again)
    assert st.item() == 0
