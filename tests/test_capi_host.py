"""Host-side checks of the C ABI: the library loads, exports every declared symbol, and
rejects bad arguments synchronously (before any CUDA call). No GPU needed."""
import ctypes
import os
import re

import numpy as np
import pytest

import learned_token_pruning_02_b200 as tg
from oracle import tg_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(tg_[a-zA-Z0-9_]+)\s*\(", txt, re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(tg.LIB_PATH):
        from learned_token_pruning_02_b200 import build
        build.build()
    return tg.lib()


def test_exports_every_declared_symbol(L):
    declared = _declared_functions()
    assert len(declared) >= 9, declared
    for name in declared:
        assert hasattr(L, name), name
    assert set(tg.EXPORTS) == set(declared)


def test_status_strings_and_version(L):
    assert L.tg_status_string(0) == b"TG_OK"
    assert L.tg_status_string(1) == b"TG_ERR_INVALID_ARG"
    assert L.tg_status_string(4) == b"TG_ERR_CUDA"
    assert L.tg_status_string(99) == b"TG_ERR_UNKNOWN"
    assert L.tg_version() >> 16 == 1
    assert L.tg_version() & 0xffff >= 3  # 1.1: projection, split selection, backward; 1.2: score status;
    # 1.3: allocation-free gate gradients, status word of tg_gate_mlp_bwd
    assert L.tg_set_test_wait_probe(-1) == 1
    assert L.tg_set_test_wait_probe(0) == 0


@pytest.mark.parametrize("seed", range(5))
def test_kept_counts_match_oracle_rule(L, seed):
    g = np.random.default_rng(seed)
    B = int(g.integers(1, 9))
    seqlens = g.integers(0, 5000, B)
    q_len = np.array([g.integers(0, n + 1) for n in seqlens])
    k = g.integers(-5, 6000, B)
    cu = tg.tg_kept_counts(seqlens, q_len, k)
    expect = np.concatenate([[0], np.cumsum([orc.kept_count(n, q, kk) for n, q, kk in zip(seqlens, q_len, k)])])
    assert cu == expect.tolist()


def test_kept_counts_rejects_bad_sequences(L):
    with pytest.raises(tg.TokenGateError) as e:
        tg.tg_kept_counts([10], [11], [3])
    assert e.value.status == 1
    with pytest.raises(tg.TokenGateError) as e:
        tg.tg_kept_counts([-1], [0], [3])
    assert e.value.status == 1
    with pytest.raises(tg.TokenGateError) as e:
        tg.tg_kept_counts([tg.TG_MAX_CTX + 10], [0], [3])
    assert e.value.status == 2


def _seqs(seqlens, q, k):
    return tg.Seqs(seqlens, q, k)


def test_argument_errors_are_synchronous(L):
    V = ctypes.c_void_p
    fake = V(0x1000)  # never dereferenced: every call below fails validation first
    # tg_score: null H, bad dg, bad d, misaligned pointer
    assert L.tg_score(1, None, 64, 10, 64, fake, None, fake, 0.0, 1.0, 64, fake, None, None) == 1
    assert L.tg_score(1, fake, 64, 10, 64, fake, None, fake, 0.0, 1.0, 96, fake, None, None) == 2
    assert L.tg_score(1, fake, 96, 10, 96, fake, None, fake, 0.0, 1.0, 64, fake, None, None) == 2
    assert L.tg_score(1, V(0x1002), 64, 10, 64, fake, None, fake, 0.0, 1.0, 64, fake, None, None) == 2
    assert L.tg_score(7, fake, 64, 10, 64, fake, None, fake, 0.0, 1.0, 64, fake, None, None) == 1
    assert L.tg_score(1, fake, 32, 10, 64, fake, None, fake, 0.0, 1.0, 64, fake, None, None) == 1  # ldh < d
    assert b"dg" in L.tg_last_error() or b"ldh" in L.tg_last_error()
    for bad_t in (0.0, -1.0, float("inf"), float("nan")):  # the temperature must be positive and finite
        assert L.tg_score(1, fake, 64, 10, 64, fake, None, fake, 0.0, bad_t, 64, fake, None, None) == 1
        assert b"temperature" in L.tg_last_error()
    # n_tok == 0 is a no-op that needs no device
    assert L.tg_score(1, None, 64, 0, 64, None, None, None, 0.0, 1.0, 64, None, None, None) == 0
    # tg_topk_select: q > N, null outputs
    s = _seqs([10], [11], [2])
    assert L.tg_topk_select(fake, s.ref(), fake, None, None, None) == 1
    s = _seqs([10], [2], [2])
    assert L.tg_topk_select(None, s.ref(), fake, None, None, None) == 1
    assert L.tg_topk_select(fake, None, fake, None, None, None) == 1
    s0 = _seqs([], [], [])
    assert L.tg_topk_select(None, s0.ref(), None, None, None, None) == 0
    # tg_gather: misaligned row pitch, null outputs
    s = _seqs([10], [2], [2])
    assert L.tg_gather(1, fake, 65, 64, fake, fake, s.ref(), 0, fake, fake, None, None, None, None) == 2
    assert L.tg_gather(1, fake, 64, 64, fake, fake, s.ref(), 0, None, fake, None, None, None, None) == 1
    assert L.tg_gather(1, fake, 64, 64, None, fake, s.ref(), 0, fake, fake, fake, None, None, None) == 1
    # tg_gated_attn_fwd: Hq % Hkv, D, null cu_kept, non-monotone offsets
    cu = (ctypes.c_int32 * 2)(0, 8)
    assert L.tg_gated_attn_fwd(1, fake, fake, fake, None, None, fake, cu, 1, 6, 4, 128, 0.1, 0, fake, None, None,
                               None) == 2
    assert L.tg_gated_attn_fwd(1, fake, fake, fake, None, None, fake, cu, 1, 8, 4, 96, 0.1, 0, fake, None, None,
                               None) == 2
    assert L.tg_gated_attn_fwd(1, fake, fake, fake, None, None, fake, None, 1, 8, 4, 128, 0.1, 0, fake, None, None,
                               None) == 1
    bad = (ctypes.c_int32 * 3)(0, 8, 4)
    assert L.tg_gated_attn_fwd(1, fake, fake, fake, None, None, fake, bad, 2, 8, 4, 128, 0.1, 0, fake, None, None,
                               None) == 1
    assert L.tg_gated_attn_fwd(1, None, fake, fake, None, None, fake, cu, 1, 8, 4, 128, 0.1, 0, fake, None, None,
                               None) == 1
    assert L.tg_gated_attn_fwd(1, fake, fake, fake, None, None, fake, cu, 1, 8, 4, 128, float("nan"), 0, fake, None,
                               None, None) == 1
    # tg_prefill_above_L: missing outputs
    s = _seqs([10], [2], [2])
    arr = (V * 1)(fake.value)
    assert L.tg_prefill_above_L(1, fake, 64, 64, fake, None, fake, 0.0, 1.0, 64, s.ref(), 1, arr, arr, arr, 8, 4, 128,
                                0.1, None, 0, None, fake, None, fake, fake, fake, fake, arr, None, None, None) == 1


def test_binding_refuses_cpu_tensors(L):
    import torch
    H = torch.zeros(4, 64)
    with pytest.raises(ValueError):
        tg.tg_score(H, torch.zeros(64, 64), None, torch.zeros(64), 0.0)


def test_argument_errors_of_the_next_entry_points(L):
    """The projection, the split selection and the attention backward validate before any CUDA
    call too: each bad argument below returns its status with nothing launched."""
    V = ctypes.c_void_p
    fake = V(0x1000)
    # tg_qkv_rope: f32, d not a multiple of 64, D, (Hq + 2 Hkv) D not a multiple of 256, NaN theta
    assert L.tg_qkv_rope(0, fake, 8, 128, fake, fake, 16, 8, 128, 1e6, fake, fake, fake, None, None) == 2
    assert L.tg_qkv_rope(1, fake, 8, 96, fake, fake, 16, 8, 128, 1e6, fake, fake, fake, None, None) == 2
    assert L.tg_qkv_rope(1, fake, 8, 128, fake, fake, 16, 8, 96, 1e6, fake, fake, fake, None, None) == 2
    assert L.tg_qkv_rope(1, fake, 8, 128, fake, fake, 1, 1, 64, 1e6, fake, fake, fake, None, None) == 2
    assert L.tg_qkv_rope(1, fake, 8, 128, fake, fake, 16, 8, 128, float("nan"), fake, fake, fake, None, None) == 1
    assert L.tg_qkv_rope(1, fake, 8, 128, fake, None, 16, 8, 128, 1e6, fake, fake, fake, None, None) == 1  # no pos
    assert L.tg_qkv_rope(1, None, 0, 128, None, None, 16, 8, 128, 1e6, None, None, None, None, None) == 0  # M = 0
    # tg_topk_candidates / tg_topk_merge: negative sizes, oversize blocks, missing outputs
    assert L.tg_topk_candidates(fake, -1, 4, 0, fake, fake, None, None) == 1
    assert L.tg_topk_candidates(fake, tg.TG_MAX_CTX + 1, 4, 0, fake, fake, None, None) == 2
    assert L.tg_topk_candidates(fake, 100, 4, 0, None, fake, None, None) == 1
    assert L.tg_topk_candidates(None, 100, 0, 0, None, None, None, None) == 0  # k = 0 keeps nothing
    assert L.tg_topk_merge(fake, fake, -1, 4, 0, 0, fake, None, None) == 1
    assert L.tg_topk_merge(fake, fake, tg.TG_MAX_CTX + 1, 4, 0, 0, fake, None, None) == 2
    assert L.tg_topk_merge(fake, fake, 100, 4, 0, 0, None, None, None) == 1
    # tg_gated_attn_bwd: unnormalised form, D, Hq % Hkv, d score without log g, missing lse
    cu = (ctypes.c_int32 * 2)(0, 8)
    args = lambda **kw: [kw.get(n, d) for n, d in (
        ("dtype", 1), ("Q", fake), ("K", fake), ("V", fake), ("logg", fake), ("gain", None), ("pos", fake),
        ("cu", cu), ("B", 1), ("Hq", 8), ("Hkv", 4), ("D", 128), ("scale", 0.1), ("flags", 0), ("O", fake),
        ("lse", fake), ("dO", fake), ("dQ", fake), ("dK", fake), ("dV", fake), ("dlogg", None), ("dscore", None),
        ("st", None), ("stream", None))]
    assert L.tg_gated_attn_bwd(*args(flags=tg.TG_ATTN_UNNORMALISED)) == 2
    assert L.tg_gated_attn_bwd(*args(D=96)) == 2
    assert L.tg_gated_attn_bwd(*args(Hq=6)) == 2
    assert L.tg_gated_attn_bwd(*args(logg=None, dscore=fake)) == 1
    assert L.tg_gated_attn_bwd(*args(lse=None)) == 1
    assert L.tg_gated_attn_bwd(*args(dK=V(0x1004))) == 2  # misaligned
    assert L.tg_gated_attn_bwd(*args(scale=float("nan"))) == 1
    assert L.tg_gated_attn_bwd(*args(dtype=7)) == 1
    assert L.tg_gated_attn_bwd(*args(cu=(ctypes.c_int32 * 2)(0, 0))) == 0  # no rows: nothing to do


def test_binding_refuses_wrong_side_dtypes():
    """Scores, gates, positions, indices, status words and gradients have fixed dtypes and must
    be contiguous; the binding rejects anything else before it touches a device."""
    import torch
    f64, i64 = torch.float64, torch.int64
    Q = torch.zeros(4, 2, 64, dtype=torch.bfloat16)
    K = V = torch.zeros(4, 1, 64, dtype=torch.bfloat16)
    pos = torch.arange(4, dtype=torch.int32)
    with pytest.raises(TypeError, match="logg"):
        tg.tg_gated_attn_fwd(Q, K, V, torch.zeros(4, dtype=f64), pos, [0, 4], 0.1)
    with pytest.raises(TypeError, match="pos"):
        tg.tg_gated_attn_fwd(Q, K, V, None, pos.to(i64), [0, 4], 0.1)
    with pytest.raises(TypeError, match="score"):
        tg.tg_topk_select(torch.zeros(10, dtype=f64), (10,), (2,), (3,))
    with pytest.raises(TypeError, match="kept_idx"):
        tg.tg_gather(torch.zeros(10, 64, dtype=torch.bfloat16), torch.zeros(10), torch.zeros(5, dtype=i64),
                     (10,), (2,), (3,))
    with pytest.raises(TypeError, match="cand_idx"):
        tg.tg_topk_merge(torch.zeros(8), torch.zeros(8, dtype=i64), 4, 8, 2)
    with pytest.raises(ValueError, match="lse must be contiguous"):
        tg.tg_gated_attn_bwd(Q, K, V, None, pos, [0, 4], Q, torch.zeros(4, 2).t(), Q, 0.1)
    with pytest.raises(TypeError, match="dQ"):
        tg.tg_gated_attn_bwd(Q, K, V, None, pos, [0, 4], Q, torch.zeros(2, 4), Q, 0.1,
                             dQ=torch.zeros(4, 2, 64, dtype=torch.bfloat16))


def test_binding_refuses_mixed_element_types():
    """Operands read in the element type of H (or Q) must share its dtype: an fp32 w2 beside bf16
    H would otherwise be read as bf16 pairs of its bytes."""
    import torch
    bf, f32 = torch.bfloat16, torch.float32
    H = torch.zeros(8, 128, dtype=bf)
    W1, b1 = torch.zeros(64, 128, dtype=bf), torch.zeros(64)
    with pytest.raises(TypeError, match="w2 must have H's dtype"):
        tg.tg_score(H, W1, b1, torch.zeros(64, dtype=f32), 0.0)
    with pytest.raises(TypeError, match="W1 must have H_kept's dtype"):
        tg.tg_gate_mlp_bwd(H, W1.float(), b1, torch.zeros(64, dtype=bf), torch.zeros(8))
    with pytest.raises(TypeError, match="w2 must have H_kept's dtype"):
        tg.tg_gate_mlp_bwd_noalloc(H, W1, b1, torch.zeros(64), torch.zeros(8), torch.zeros(64, 128),
                                   torch.zeros(64), torch.zeros(64), torch.zeros(1))
    with pytest.raises(TypeError, match="W_qkv must have H_kept's dtype"):
        tg.tg_qkv_rope(H, torch.zeros(4 * 64, 128), None, 2, 1, 64, 0.0)
    with pytest.raises(TypeError, match="H_kept must have H's dtype"):
        tg.tg_gather(H, torch.zeros(8), torch.zeros(4, dtype=torch.int32), (8,), (2,), (2,),
                     H_kept=torch.zeros(4, 128))
    Q = torch.zeros(4, 2, 64, dtype=bf)
    with pytest.raises(TypeError, match="V must have Q's dtype"):
        tg.tg_gated_attn_fwd(Q, torch.zeros(4, 1, 64, dtype=bf), torch.zeros(4, 1, 64), None,
                             torch.arange(4, dtype=torch.int32), [0, 4], 0.1)


def test_binding_checks_projection_shapes():
    """tg_qkv_rope builds its TMA maps from M, d and the head counts, so a short W_qkv or a
    strided H_kept would be read wrongly on the device: the binding refuses them first."""
    import torch
    bf = torch.bfloat16
    M, d, Hq, Hkv, D = 8, 128, 2, 1, 64
    Hk = torch.zeros(M, d, dtype=bf)
    W = torch.zeros((Hq + 2 * Hkv) * D, d, dtype=bf)
    pos = torch.arange(M, dtype=torch.int32)
    with pytest.raises(ValueError, match="W_qkv has shape"):
        tg.tg_qkv_rope(Hk, W[:-1], pos, Hq, Hkv, D, 1e4)
    with pytest.raises(ValueError, match="H_kept must be contiguous"):
        tg.tg_qkv_rope(torch.zeros(M, 2 * d, dtype=bf)[:, ::2], W, pos, Hq, Hkv, D, 1e4)
    with pytest.raises(ValueError, match="W_qkv must be contiguous"):
        tg.tg_qkv_rope(Hk, torch.zeros(d, (Hq + 2 * Hkv) * D, dtype=bf).t(), pos, Hq, Hkv, D, 1e4)
    with pytest.raises(ValueError, match="pos must hold"):
        tg.tg_qkv_rope(Hk, W, pos[:M - 1], Hq, Hkv, D, 1e4)
    with pytest.raises(ValueError, match="pos must hold"):
        tg.tg_qkv_rope(Hk, W, None, Hq, Hkv, D, 1e4)
    with pytest.raises(ValueError, match="Q has shape"):
        tg.tg_qkv_rope(Hk, W, pos, Hq, Hkv, D, 1e4, Q=torch.zeros(M, Hq + 1, D, dtype=bf))
    with pytest.raises(ValueError, match="V has shape"):
        tg.tg_qkv_rope(Hk, W, pos, Hq, Hkv, D, 1e4, V=torch.zeros(M - 1, Hkv, D, dtype=bf))
    # without rotation pos is not needed: the call gets as far as the device check
    with pytest.raises(ValueError, match="CUDA tensors only"):
        tg.tg_qkv_rope(Hk, W, None, Hq, Hkv, D, 0.0)


def test_binding_checks_backward_shapes():
    """tg_gated_attn_bwd indexes lse as [Hq, M] and writes dK/dV rows up to cu_kept[-1]: every
    shape that would send it out of bounds is refused before the call."""
    import torch
    bf, f32 = torch.bfloat16, torch.float32
    M, Hq, Hkv, D = 6, 4, 2, 64
    Q = torch.zeros(M, Hq, D, dtype=bf)
    K = torch.zeros(M, Hkv, D, dtype=bf)
    pos = torch.arange(M, dtype=torch.int32)
    lse = torch.zeros(Hq, M, dtype=f32)
    logg = torch.zeros(M, dtype=f32)

    def call(**kw):
        a = dict(Q=Q, K=K, V=K, logg=logg, pos=pos, cu_kept=[0, M], O=Q, lse=lse, dO=Q, softmax_scale=0.1)
        a.update(kw)
        return tg.tg_gated_attn_bwd(**a)

    with pytest.raises(ValueError, match="cu_kept"):
        call(cu_kept=[0, M - 1])
    with pytest.raises(ValueError, match="cu_kept"):
        call(cu_kept=[0, 2, M + 1])
    with pytest.raises(ValueError, match="lse has shape"):
        call(lse=torch.zeros(Hq, M - 1, dtype=f32))
    with pytest.raises(ValueError, match="pos holds"):
        call(pos=pos[:M - 1])
    with pytest.raises(ValueError, match="logg holds"):
        call(logg=logg[:M - 2])
    with pytest.raises(ValueError, match="V has shape"):
        call(V=torch.zeros(M, Hkv + 1, D, dtype=bf))
    with pytest.raises(ValueError, match="O has shape"):
        call(O=torch.zeros(M, Hq, D // 2, dtype=bf))
    with pytest.raises(ValueError, match="dO has shape"):
        call(dO=torch.zeros(M - 1, Hq, D, dtype=bf))
    with pytest.raises(ValueError, match="dK has shape"):
        call(dK=torch.zeros(M, Hq, D, dtype=f32))
    with pytest.raises(ValueError, match="dlogg has shape"):
        call(dlogg=torch.zeros(M + 1, dtype=f32))
    with pytest.raises(ValueError, match="head_gain holds"):
        call(head_gain=torch.ones(Hq - 1, dtype=f32))
    with pytest.raises(ValueError, match="CUDA tensors only"):  # well-formed: stops at the device check
        call()


def test_gate_mlp_bwd_arguments_and_workspace(L):
    """tg_gate_mlp_bwd checks its shapes, temperature and workspace before any CUDA call."""
    V = ctypes.c_void_p
    fake, ws = V(0x1000), V(0x10000)
    need = L.tg_gate_mlp_bwd_workspace_size(2176, 2048, 256)
    assert need >= 2176 * 256 * 4
    assert L.tg_gate_mlp_bwd_workspace_size(0, 2048, 256) == 0
    assert L.tg_gate_mlp_bwd_workspace_size(100, 2000, 256) == 0  # d not a multiple of 64
    args = lambda **kw: [kw.get(n, v) for n, v in (
        ("dt", 1), ("H", fake), ("M", 2176), ("d", 2048), ("W1", fake), ("b1", None), ("w2", fake), ("T", 1.0),
        ("dg", 256), ("ds", fake), ("dW1", fake), ("db1", None), ("dw2", None), ("db2", None), ("ws", ws),
        ("wsb", need), ("status", None), ("stream", None))]
    assert L.tg_gate_mlp_bwd(*args(d=2000)) == 2
    assert L.tg_gate_mlp_bwd(*args(dg=100)) == 2
    assert L.tg_gate_mlp_bwd(*args(T=0.0)) == 1
    assert L.tg_gate_mlp_bwd(*args(dt=5)) == 1
    assert L.tg_gate_mlp_bwd(*args(dW1=None)) == 1
    assert L.tg_gate_mlp_bwd(*args(ds=None)) == 1
    assert L.tg_gate_mlp_bwd(*args(H=V(0x1008))) == 2  # misaligned
    assert L.tg_gate_mlp_bwd(*args(wsb=need - 1)) == 3
    assert L.tg_gate_mlp_bwd(*args(ws=None)) == 3
    assert L.tg_gate_mlp_bwd(*args(ws=V(0x10080))) == 3  # workspace not 256-byte aligned
    assert b"workspace" in L.tg_last_error()


def test_select_stream_workspace_and_arguments(L):
    """tg_topk_select_stream sizes its workspace on the host and checks it before any CUDA call."""
    V = ctypes.c_void_p
    seqlens, q_len, k = (131072,) * 64, (256,) * 64, (4096,) * 64
    s = tg.Seqs(seqlens, q_len, k)
    need = L.tg_topk_select_stream_workspace_size(s.ref())
    ctx = sum(n - q for n, q in zip(seqlens, q_len))
    assert need >= ctx * 8  # the candidate lists' worst case
    assert need < ctx * 8 + (2 << 20)
    # sequences that keep nothing or everything need no candidate space
    assert L.tg_topk_select_stream_workspace_size(tg.Seqs((1000, 1000), (0, 0), (0, 1000)).ref()) < (2 << 20)
    assert L.tg_topk_select_stream_workspace_size(tg.Seqs((10,), (11,), (1,)).ref()) == 0  # q > N
    fake, ws = V(0x1000), V(0x100000)
    call = lambda ws=ws, wsb=need, seqs=s: L.tg_topk_select_stream(fake, seqs.ref(), fake, fake, ws, wsb, None, None)
    assert call(wsb=need - 1) == 3  # TG_ERR_WORKSPACE
    assert call(ws=None) == 3
    assert call(ws=V(0x100080)) == 3  # not 256-byte aligned
    assert b"workspace" in L.tg_last_error()
    assert call(seqs=tg.Seqs((10,), (11,), (1,))) == 1  # TG_ERR_INVALID_ARG
    assert L.tg_topk_select_stream(None, tg.Seqs((10,), (0,), (1,)).ref(), fake, fake, ws, need, None, None) == 1
