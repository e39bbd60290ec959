"""TokenGate gated-prefill hot path for B200 (sm_100a): thin Python binding of libtokengate.

Every function here marshals torch tensors into the C ABI declared in include/tokengate.h
and calls it; all computation runs in the library's CUDA kernels. There is no CPU path:
if the shared library is missing, or the tensors are not on a CUDA device, calls raise.

Build the library in-tree with ``python -m learned_token_pruning_02_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtokengate.so")

TG_F32, TG_BF16 = 0, 1
TG_ATTN_UNNORMALISED = 1 << 0
TG_QUESTION_GATE_ONE = 1 << 1
TG_DEV_NAN_SCORE = 1 << 0
TG_DEV_POS_NOT_ASCENDING = 1 << 1
TG_DEV_TIMEOUT = 1 << 2
TG_DEV_BAD_INDEX = 1 << 3
TG_MAX_CTX = 262144

EXPORTS = (
    "tg_status_string", "tg_last_error", "tg_version", "tg_kept_counts", "tg_score",
    "tg_topk_select", "tg_gather", "tg_gated_attn_fwd", "tg_prefill_above_L",
    "tg_qkv_rope",
    "tg_topk_candidates",
    "tg_topk_merge",
    "tg_gated_attn_bwd",
    "tg_set_test_wait_probe",
    "tg_gate_mlp_bwd_workspace_size",
    "tg_gate_mlp_bwd",
    "tg_prefill_projected",
    "tg_gate_mlp_bwd_noalloc",
    "tg_topk_select_stream_workspace_size",
    "tg_topk_select_stream",
)


class TokenGateError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: {msg}")
        self.status = status


class tg_seqs(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32),
        ("seqlens", ctypes.POINTER(ctypes.c_int32)),
        ("q_len", ctypes.POINTER(ctypes.c_int32)),
        ("k", ctypes.POINTER(ctypes.c_int32)),
    ]


_VP = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_F = ctypes.c_float
_U32 = ctypes.c_uint32
_SEQP = ctypes.POINTER(tg_seqs)
_lib_handle = None


def lib() -> ctypes.CDLL:
    """Load libtokengate.so (once). Raises if it has not been built."""
    global _lib_handle
    if _lib_handle is not None:
        return _lib_handle
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"libtokengate.so not found at {LIB_PATH}; build it with "
            "`python -m learned_token_pruning_02_b200.build` (no CPU fallback exists)")
    L = ctypes.CDLL(LIB_PATH)
    L.tg_status_string.restype = ctypes.c_char_p
    L.tg_status_string.argtypes = [_I32]
    L.tg_last_error.restype = ctypes.c_char_p
    L.tg_last_error.argtypes = []
    L.tg_version.restype = _I32
    L.tg_kept_counts.restype = _I32
    L.tg_kept_counts.argtypes = [_SEQP, ctypes.POINTER(_I32)]
    L.tg_score.restype = _I32
    L.tg_score.argtypes = [_I32, _VP, _I64, _I64, _I32, _VP, _VP, _VP, _F, _F, _I32, _VP, _VP, _VP]
    L.tg_gate_mlp_bwd_workspace_size.restype = ctypes.c_size_t
    L.tg_gate_mlp_bwd_workspace_size.argtypes = [_I64, _I32, _I32]
    L.tg_gate_mlp_bwd.restype = _I32
    L.tg_gate_mlp_bwd.argtypes = [_I32, _VP, _I64, _I32, _VP, _VP, _VP, _F, _I32, _VP, _VP, _VP, _VP, _VP, _VP,
                                  ctypes.c_size_t, _VP, _VP]
    L.tg_prefill_projected.restype = _I32
    L.tg_prefill_projected.argtypes = [
        _I32, _VP, _I64, _I32, _VP, _VP, _VP, _F, _F, _I32, _SEQP, _I32, ctypes.POINTER(_VP), _F,
        _I32, _I32, _I32, _F, _VP, _U32, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
        ctypes.POINTER(_VP), ctypes.POINTER(_VP), ctypes.POINTER(_VP), ctypes.POINTER(_VP), ctypes.POINTER(_VP),
        _VP, _VP]
    L.tg_gate_mlp_bwd_noalloc.restype = _I32
    L.tg_gate_mlp_bwd_noalloc.argtypes = [_I32, _VP, _I64, _I32, _VP, _VP, _VP, _F, _I32, _VP, _VP, _VP, _VP, _VP,
                                          _VP, _VP]
    L.tg_set_test_wait_probe.restype = _I32
    L.tg_set_test_wait_probe.argtypes = [_I64]
    L.tg_topk_select.restype = _I32
    L.tg_topk_select.argtypes = [_VP, _SEQP, _VP, _VP, _VP, _VP]
    L.tg_topk_select_stream_workspace_size.restype = ctypes.c_size_t
    L.tg_topk_select_stream_workspace_size.argtypes = [_SEQP]
    L.tg_topk_select_stream.restype = _I32
    L.tg_topk_select_stream.argtypes = [_VP, _SEQP, _VP, _VP, _VP, ctypes.c_size_t, _VP, _VP]
    L.tg_qkv_rope.restype = _I32
    L.tg_qkv_rope.argtypes = [_I32, _VP, _I64, _I32, _VP, _VP, _I32, _I32, _I32, _F, _VP, _VP, _VP, _VP, _VP]
    L.tg_topk_candidates.restype = _I32
    L.tg_topk_candidates.argtypes = [_VP, _I32, _I32, _I32, _VP, _VP, _VP, _VP]
    L.tg_topk_merge.restype = _I32
    L.tg_topk_merge.argtypes = [_VP, _VP, _I32, _I32, _I32, _I32, _VP, _VP, _VP]
    L.tg_gather.restype = _I32
    L.tg_gather.argtypes = [_I32, _VP, _I64, _I32, _VP, _VP, _SEQP, _U32, _VP, _VP, _VP, _VP, _VP, _VP]
    L.tg_gated_attn_fwd.restype = _I32
    L.tg_gated_attn_fwd.argtypes = [_I32, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.POINTER(_I32), _I32, _I32,
                                    _I32, _I32, _F, _U32, _VP, _VP, _VP, _VP]
    L.tg_gated_attn_bwd.restype = _I32
    L.tg_gated_attn_bwd.argtypes = [_I32, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.POINTER(_I32), _I32, _I32,
                                    _I32, _I32, _F, _U32, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]
    L.tg_prefill_above_L.restype = _I32
    L.tg_prefill_above_L.argtypes = [
        _I32, _VP, _I64, _I32, _VP, _VP, _VP, _F, _F, _I32, _SEQP, _I32,
        ctypes.POINTER(_VP), ctypes.POINTER(_VP), ctypes.POINTER(_VP),
        _I32, _I32, _I32, _F, _VP, _U32, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
        ctypes.POINTER(_VP), ctypes.POINTER(_VP), _VP, _VP]
    _lib_handle = L
    return L


def _check(fn: str, st: int):
    if st != 0:
        L = lib()
        raise TokenGateError(fn, st, f"{L.tg_status_string(st).decode()}: {L.tg_last_error().decode()}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return TG_BF16
    if t.dtype == torch.float32:
        return TG_F32
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _like(ref_name, ref, **named):
    """Operands the C ABI reads in the element type of `ref` (bf16 or fp32) must share its dtype."""
    for name, t in named.items():
        if t is not None and t.dtype != ref.dtype:
            raise TypeError(f"{name} must have {ref_name}'s dtype {ref.dtype}, got {t.dtype}")


def _want(dtype, **named):
    """Side tensors (scores, gates, positions, indices, status words, gradients) must have the
    library's fixed dtype and be contiguous: the C ABI reads them as plain arrays."""
    for name, t in named.items():
        if t is None:
            continue
        if t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def _contig(**named):
    for name, t in named.items():
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def _shape(name, t, want):
    if tuple(t.shape) != tuple(want):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(want)}")


def _len_at_least(name, t, n):
    if t is not None and t.numel() < n:
        raise ValueError(f"{name} holds {t.numel()} elements, needs at least {n}")


def _cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libtokengate works on CUDA tensors only (there is no CPU path)")


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


class Seqs:
    """Host-side sequence description (keeps the int32 arrays alive for the call)."""

    def __init__(self, seqlens, q_len, k):
        n = len(seqlens)
        assert len(q_len) == n and len(k) == n
        self._arrs = [(ctypes.c_int32 * max(n, 1))(*[int(x) for x in a]) for a in (seqlens, q_len, k)]
        self.s = tg_seqs(n, *[ctypes.cast(a, ctypes.POINTER(ctypes.c_int32)) for a in self._arrs])
        self.B = n

    def ref(self):
        return ctypes.byref(self.s)


def tg_kept_counts(seqlens, q_len, k) -> list:
    """cu_kept offsets (host list of B+1 ints)."""
    s = Seqs(seqlens, q_len, k)
    out = (ctypes.c_int32 * (s.B + 1))()
    _check("tg_kept_counts", lib().tg_kept_counts(s.ref(), out))
    return list(out)


def tg_score(H, W1, b1, w2, b2: float, score=None, dev_status=None, stream=None, temperature: float = 1.0):
    """Gate-MLP score of every token: (w2 . GELU(W1 h + b1) + b2) / temperature (float32 [n_tok])."""
    _want(torch.float32, b1=b1, score=score)
    _want(torch.int32, dev_status=dev_status)
    _like("H", H, W1=W1, w2=w2)
    _cuda(H, W1, b1, w2, score, dev_status)
    n_tok, d = H.shape
    assert H.stride(1) == 1 and W1.is_contiguous() and w2.is_contiguous()
    if score is None:
        score = torch.empty(n_tok, device=H.device, dtype=torch.float32)
    _check("tg_score", lib().tg_score(_dtype(H), _ptr(H), H.stride(0), n_tok, d, _ptr(W1), _ptr(b1), _ptr(w2),
                                      float(b2), float(temperature), W1.shape[0], _ptr(score), _ptr(dev_status),
                                      _stream(stream)))
    return score


def tg_set_test_wait_probe(limit_ns: int):
    """Test hook (off by default): with limit_ns > 0 every tensor-core kernel launched afterwards
    by this thread waits that long on a barrier nothing signals, records TG_DEV_TIMEOUT and skips
    its work. 0 restores normal operation."""
    _check("tg_set_test_wait_probe", lib().tg_set_test_wait_probe(int(limit_ns)))


def tg_topk_select(score, seqlens, q_len, k, kept_idx=None, cu_kept_dev=None, dev_status=None, stream=None):
    """Top-K context tokens per sequence plus the question tail (int32 kept_idx, cu_kept_dev)."""
    _want(torch.float32, score=score)
    _want(torch.int32, kept_idx=kept_idx, cu_kept_dev=cu_kept_dev, dev_status=dev_status)
    _cuda(score, kept_idx, cu_kept_dev, dev_status)
    s = Seqs(seqlens, q_len, k)
    cu = tg_kept_counts(seqlens, q_len, k)
    if kept_idx is None:
        kept_idx = torch.empty(cu[-1], device=score.device, dtype=torch.int32)
    if cu_kept_dev is None:
        cu_kept_dev = torch.empty(s.B + 1, device=score.device, dtype=torch.int32)
    _check("tg_topk_select", lib().tg_topk_select(_ptr(score), s.ref(), _ptr(kept_idx), _ptr(cu_kept_dev),
                                                  _ptr(dev_status), _stream(stream)))
    return kept_idx, cu_kept_dev


def tg_topk_select_stream_workspace_size(seqlens, q_len, k) -> int:
    """Workspace bytes of tg_topk_select_stream for these sequences (host only)."""
    return int(lib().tg_topk_select_stream_workspace_size(Seqs(seqlens, q_len, k).ref()))


def tg_topk_select_stream(score, seqlens, q_len, k, kept_idx=None, cu_kept_dev=None, ws=None, dev_status=None,
                          stream=None):
    """tg_topk_select for many long sequences at once (the same outputs bit for bit), from four
    kernels over all SMs. ``ws`` is a uint8 device buffer of at least
    tg_topk_select_stream_workspace_size bytes (allocated here when not given)."""
    _want(torch.float32, score=score)
    _want(torch.int32, kept_idx=kept_idx, cu_kept_dev=cu_kept_dev, dev_status=dev_status)
    _cuda(score, kept_idx, cu_kept_dev, ws, dev_status)
    s = Seqs(seqlens, q_len, k)
    cu = tg_kept_counts(seqlens, q_len, k)
    if kept_idx is None:
        kept_idx = torch.empty(cu[-1], device=score.device, dtype=torch.int32)
    if cu_kept_dev is None:
        cu_kept_dev = torch.empty(s.B + 1, device=score.device, dtype=torch.int32)
    need = lib().tg_topk_select_stream_workspace_size(s.ref())
    if ws is None:
        ws = torch.empty(max(need, 1), device=score.device, dtype=torch.uint8)
    _check("tg_topk_select_stream", lib().tg_topk_select_stream(
        _ptr(score), s.ref(), _ptr(kept_idx), _ptr(cu_kept_dev), _ptr(ws), ws.numel() * ws.element_size(),
        _ptr(dev_status), _stream(stream)))
    return kept_idx, cu_kept_dev


def tg_qkv_rope(H_kept, W_qkv, pos, Hq: int, Hkv: int, D: int, rope_theta: float, Q=None, K=None, V=None,
                dev_status=None, stream=None):
    """Q, K, V of the kept rows (bf16), Q and K rotated at their original positions: (Q, K, V)."""
    _want(torch.int32, pos=pos, dev_status=dev_status)
    _like("H_kept", H_kept, W_qkv=W_qkv, Q=Q, K=K, V=V)
    M, d = H_kept.shape
    _contig(H_kept=H_kept, W_qkv=W_qkv)
    _shape("W_qkv", W_qkv, ((Hq + 2 * Hkv) * D, d))
    if rope_theta > 0:
        if pos is None or pos.numel() < M:
            raise ValueError(f"pos must hold at least M = {M} positions when rope_theta > 0")
    dev = H_kept.device
    for name, t, h in (("Q", Q, Hq), ("K", K, Hkv), ("V", V, Hkv)):
        if t is not None:
            _shape(name, t, (M, h, D))
            _contig(**{name: t})
    _cuda(H_kept, W_qkv, pos, Q, K, V, dev_status)
    Q = torch.empty(M, Hq, D, device=dev, dtype=torch.bfloat16) if Q is None else Q
    K = torch.empty(M, Hkv, D, device=dev, dtype=torch.bfloat16) if K is None else K
    V = torch.empty(M, Hkv, D, device=dev, dtype=torch.bfloat16) if V is None else V
    _check("tg_qkv_rope", lib().tg_qkv_rope(_dtype(H_kept), _ptr(H_kept), M, d, _ptr(W_qkv), _ptr(pos), Hq, Hkv, D,
                                            float(rope_theta), _ptr(Q), _ptr(K), _ptr(V), _ptr(dev_status),
                                            _stream(stream)))
    return Q, K, V


def tg_topk_candidates(score, k: int, base: int = 0, cand_score=None, cand_idx=None, dev_status=None, stream=None):
    """Top-k of one block of a sequence's context as (cand_score, cand_idx = base + position)."""
    _want(torch.float32, score=score, cand_score=cand_score)
    _want(torch.int32, cand_idx=cand_idx, dev_status=dev_status)
    _cuda(score, cand_score, cand_idx, dev_status)
    n = score.numel()
    kc = min(int(k), n)
    if cand_score is None:
        cand_score = torch.empty(kc, device=score.device, dtype=torch.float32)
    if cand_idx is None:
        cand_idx = torch.empty(kc, device=score.device, dtype=torch.int32)
    _check("tg_topk_candidates", lib().tg_topk_candidates(_ptr(score), n, int(k), int(base), _ptr(cand_score),
                                                          _ptr(cand_idx), _ptr(dev_status), _stream(stream)))
    return cand_score, cand_idx


def tg_topk_merge(cand_score, cand_idx, k: int, q_start: int, q: int, kept_idx=None, dev_status=None, stream=None):
    """Top-k of candidates concatenated in block order, then the question tail q_start..q_start+q-1."""
    _want(torch.float32, cand_score=cand_score)
    _want(torch.int32, cand_idx=cand_idx, kept_idx=kept_idx, dev_status=dev_status)
    _cuda(cand_score, cand_idx, kept_idx, dev_status)
    n = cand_score.numel()
    m = min(int(k), n) + int(q)
    if kept_idx is None:
        kept_idx = torch.empty(m, device=cand_score.device, dtype=torch.int32)
    _check("tg_topk_merge", lib().tg_topk_merge(_ptr(cand_score), _ptr(cand_idx), n, int(k), int(q_start), int(q),
                                                _ptr(kept_idx), _ptr(dev_status), _stream(stream)))
    return kept_idx


def tg_gather(H, score, kept_idx, seqlens, q_len, k, flags=0, H_kept=None, pos=None, g=None, logg=None,
              dev_status=None, stream=None):
    """Kept rows of H with their positions and gate values: (H_kept, pos, g, logg)."""
    _want(torch.float32, score=score, g=g, logg=logg)
    _want(torch.int32, kept_idx=kept_idx, pos=pos, dev_status=dev_status)
    _like("H", H, H_kept=H_kept)
    _cuda(H, score, kept_idx, H_kept, pos, g, logg, dev_status)
    s = Seqs(seqlens, q_len, k)
    m = kept_idx.numel()
    d = H.shape[1]
    dev = H.device
    H_kept = torch.empty(m, d, device=dev, dtype=H.dtype) if H_kept is None else H_kept
    pos = torch.empty(m, device=dev, dtype=torch.int32) if pos is None else pos
    g = torch.empty(m, device=dev, dtype=torch.float32) if g is None else g
    logg = torch.empty(m, device=dev, dtype=torch.float32) if logg is None else logg
    _check("tg_gather", lib().tg_gather(_dtype(H), _ptr(H), H.stride(0), d, _ptr(score), _ptr(kept_idx), s.ref(),
                                        int(flags), _ptr(H_kept), _ptr(pos), _ptr(g), _ptr(logg), _ptr(dev_status),
                                        _stream(stream)))
    return H_kept, pos, g, logg


def tg_gated_attn_fwd(Q, K, V, logg, pos, cu_kept, softmax_scale: float, head_gain=None, flags=0, O=None,
                      lse=None, want_lse=True, dev_status=None, stream=None):
    """Token-gated causal attention over the kept tokens: (O [M, Hq, D], lse [Hq, M] or None)."""
    _want(torch.float32, logg=logg, head_gain=head_gain, lse=lse)
    _want(torch.int32, pos=pos, dev_status=dev_status)
    _like("Q", Q, K=K, V=V, O=O)
    _cuda(Q, K, V, logg, pos, head_gain, O, lse, dev_status)
    M, Hq, D = Q.shape
    Hkv = K.shape[1]
    assert Q.is_contiguous() and K.is_contiguous() and V.is_contiguous()
    cu = [int(x) for x in cu_kept]
    B = len(cu) - 1
    cu_arr = (ctypes.c_int32 * len(cu))(*cu)
    O = torch.empty_like(Q) if O is None else O
    if lse is None and want_lse:
        lse = torch.empty(Hq, M, device=Q.device, dtype=torch.float32)
    _check("tg_gated_attn_fwd", lib().tg_gated_attn_fwd(
        _dtype(Q), _ptr(Q), _ptr(K), _ptr(V), _ptr(logg), _ptr(head_gain), _ptr(pos), cu_arr, B, Hq, Hkv, D,
        float(softmax_scale), int(flags), _ptr(O), _ptr(lse), _ptr(dev_status), _stream(stream)))
    return O, lse


def tg_gated_attn_bwd(Q, K, V, logg, pos, cu_kept, O, lse, dO, softmax_scale: float, head_gain=None, flags=0,
                      want_dlogg=True, want_dscore=False, dQ=None, dK=None, dV=None, dlogg=None, dscore=None,
                      dev_status=None, stream=None):
    """Gradients of the gated attention (normalised form) from the forward's O and lse and the
    upstream dO: (dQ [M, Hq, D], dK [M, Hkv, D], dV [M, Hkv, D], dlogg [M] or None,
    dscore [M] or None), all float32."""
    _want(torch.float32, logg=logg, lse=lse, head_gain=head_gain, dQ=dQ, dK=dK, dV=dV, dlogg=dlogg, dscore=dscore)
    _want(torch.int32, pos=pos, dev_status=dev_status)
    M, Hq, D = Q.shape
    Hkv = K.shape[1]
    for name, t in (("Q", Q), ("K", K), ("V", V), ("O", O), ("dO", dO)):
        _contig(**{name: t})
        if t.dtype != Q.dtype:
            raise TypeError(f"{name} must have Q's dtype {Q.dtype}")
    cu = [int(x) for x in cu_kept]
    B = len(cu) - 1
    if B >= 0 and cu and cu[-1] != M:
        raise ValueError(f"cu_kept[-1] = {cu[-1]} must equal the row count of Q ({M})")
    _shape("K", K, (M, Hkv, D))
    _shape("V", V, (M, Hkv, D))
    _shape("O", O, (M, Hq, D))
    _shape("dO", dO, (M, Hq, D))
    if lse is not None:
        _shape("lse", lse, (Hq, M))
    _len_at_least("pos", pos, M)
    _len_at_least("logg", logg, M)
    _len_at_least("head_gain", head_gain, Hq)
    for name, t, h in (("dQ", dQ, Hq), ("dK", dK, Hkv), ("dV", dV, Hkv)):
        if t is not None:
            _shape(name, t, (M, h, D))
    for name, t in (("dlogg", dlogg), ("dscore", dscore)):
        if t is not None:
            _shape(name, t, (M,))
    _cuda(Q, K, V, logg, pos, O, lse, dO, head_gain, dQ, dK, dV, dlogg, dscore, dev_status)
    cu_arr = (ctypes.c_int32 * len(cu))(*cu)
    dev = Q.device
    f32 = torch.float32
    dQ = torch.empty(M, Hq, D, device=dev, dtype=f32) if dQ is None else dQ
    dK = torch.empty(M, Hkv, D, device=dev, dtype=f32) if dK is None else dK
    dV = torch.empty(M, Hkv, D, device=dev, dtype=f32) if dV is None else dV
    if dlogg is None and want_dlogg:
        dlogg = torch.empty(M, device=dev, dtype=f32)
    if dscore is None and want_dscore:
        dscore = torch.empty(M, device=dev, dtype=f32)
    _check("tg_gated_attn_bwd", lib().tg_gated_attn_bwd(
        _dtype(Q), _ptr(Q), _ptr(K), _ptr(V), _ptr(logg), _ptr(head_gain), _ptr(pos), cu_arr, B, Hq, Hkv, D,
        float(softmax_scale), int(flags), _ptr(O), _ptr(lse), _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dlogg),
        _ptr(dscore), _ptr(dev_status), _stream(stream)))
    return dQ, dK, dV, dlogg, dscore


def tg_gate_mlp_bwd(H_kept, W1, b1, w2, dscore, temperature: float = 1.0, dW1=None, db1=None, dw2=None, db2=None,
                    ws=None, dev_status=None, stream=None):
    """Gradients of the gate network's parameters from d score of the kept rows:
    (dW1 [dg, d], db1 [dg], dw2 [dg], db2 [1]), all float32. ``ws`` is a uint8 device buffer of
    at least tg_gate_mlp_bwd_workspace_size bytes (allocated here when not given);
    ``dev_status`` an int32 device word that a timed-out wait ORs TG_DEV_TIMEOUT into."""
    _want(torch.float32, b1=b1, dscore=dscore, dW1=dW1, db1=db1, dw2=dw2, db2=db2)
    _want(torch.int32, dev_status=dev_status)
    _like("H_kept", H_kept, W1=W1, w2=w2)
    M, d = H_kept.shape
    dg = W1.shape[0]
    _contig(H_kept=H_kept, W1=W1, w2=w2)
    _shape("W1", W1, (dg, d))
    _len_at_least("dscore", dscore, M)
    if dW1 is not None:
        _shape("dW1", dW1, (dg, d))
    for name, t in (("b1", b1), ("db1", db1), ("dw2", dw2)):
        if t is not None:
            _shape(name, t, (dg,))
    _cuda(H_kept, W1, b1, w2, dscore, dW1, db1, dw2, db2, ws, dev_status)
    dev = H_kept.device
    f32 = torch.float32
    dW1 = torch.empty(dg, d, device=dev, dtype=f32) if dW1 is None else dW1
    db1 = torch.empty(dg, device=dev, dtype=f32) if db1 is None else db1
    dw2 = torch.empty(dg, device=dev, dtype=f32) if dw2 is None else dw2
    db2 = torch.empty(1, device=dev, dtype=f32) if db2 is None else db2
    need = lib().tg_gate_mlp_bwd_workspace_size(M, d, dg)
    if ws is None:
        ws = torch.empty(max(need, 1), device=dev, dtype=torch.uint8)
    _check("tg_gate_mlp_bwd", lib().tg_gate_mlp_bwd(
        _dtype(H_kept), _ptr(H_kept), M, d, _ptr(W1), _ptr(b1), _ptr(w2), float(temperature), dg, _ptr(dscore),
        _ptr(dW1), _ptr(db1), _ptr(dw2), _ptr(db2), _ptr(ws), ws.numel() * ws.element_size(), _ptr(dev_status),
        _stream(stream)))
    return dW1, db1, dw2, db2


def tg_gate_mlp_bwd_noalloc(H_kept, W1, b1, w2, dscore, dW1, db1, dw2, db2, temperature: float = 1.0,
                            dev_status=None, stream=None):
    """tg_gate_mlp_bwd for callers that cannot allocate: the library's fixed scratch array takes
    the place of the workspace, and every output buffer is the caller's (nothing is allocated
    here either). Calls on one device share the array: do not let them overlap on the GPU."""
    _want(torch.float32, b1=b1, dscore=dscore, dW1=dW1, db1=db1, dw2=dw2, db2=db2)
    _like("H_kept", H_kept, W1=W1, w2=w2)
    M, d = H_kept.shape
    dg = W1.shape[0]
    _contig(H_kept=H_kept, W1=W1, w2=w2)
    _shape("W1", W1, (dg, d))
    _shape("dW1", dW1, (dg, d))
    _len_at_least("dscore", dscore, M)
    _want(torch.int32, dev_status=dev_status)
    _cuda(H_kept, W1, b1, w2, dscore, dW1, db1, dw2, db2, dev_status)
    _check("tg_gate_mlp_bwd_noalloc", lib().tg_gate_mlp_bwd_noalloc(
        _dtype(H_kept), _ptr(H_kept), M, d, _ptr(W1), _ptr(b1), _ptr(w2), float(temperature), dg, _ptr(dscore),
        _ptr(dW1), _ptr(db1), _ptr(dw2), _ptr(db2), _ptr(dev_status), _stream(stream)))
    return dW1, db1, dw2, db2


def tg_prefill_above_L(H, W1, b1, w2, b2, seqlens, q_len, k, layers, softmax_scale, head_gain=None, flags=0,
                       want_lse=False, out=None, dev_status=None, stream=None, temperature: float = 1.0):
    """The whole gated path above layer L: score -> top-K -> gather -> gated attention per layer.

    layers: list of (Q, K, V) device tensors shaped by the kept count. Returns a dict of the
    outputs (score, kept_idx, cu_kept_dev, H_kept, pos, g, logg, O list, lse list). Pass
    ``out`` (a dict from an earlier call) to reuse its buffers.
    """
    _want(torch.float32, b1=b1, head_gain=head_gain)
    _want(torch.int32, dev_status=dev_status)
    _like("H", H, W1=W1, w2=w2)
    _cuda(H, W1, b1, w2, head_gain, dev_status)
    s = Seqs(seqlens, q_len, k)
    cu = tg_kept_counts(seqlens, q_len, k)
    m = cu[-1]
    n_tok, d = H.shape
    dev = H.device
    nl = len(layers)
    Hq = layers[0][0].shape[1] if nl else 1
    Hkv = layers[0][1].shape[1] if nl else 1
    D = layers[0][0].shape[2] if nl else 64
    if out is None:
        out = {
            "score": torch.empty(n_tok, device=dev, dtype=torch.float32),
            "kept_idx": torch.empty(m, device=dev, dtype=torch.int32),
            "cu_kept_dev": torch.empty(s.B + 1, device=dev, dtype=torch.int32),
            "H_kept": torch.empty(m, d, device=dev, dtype=H.dtype),
            "pos": torch.empty(m, device=dev, dtype=torch.int32),
            "g": torch.empty(m, device=dev, dtype=torch.float32),
            "logg": torch.empty(m, device=dev, dtype=torch.float32),
            "O": [torch.empty_like(q) for (q, _, _) in layers],
            "lse": [torch.empty(Hq, m, device=dev, dtype=torch.float32) if want_lse else None for _ in layers],
        }
    _check_out(out)
    qa = (_VP * max(nl, 1))(*[t[0].data_ptr() for t in layers])
    ka = (_VP * max(nl, 1))(*[t[1].data_ptr() for t in layers])
    va = (_VP * max(nl, 1))(*[t[2].data_ptr() for t in layers])
    oa = (_VP * max(nl, 1))(*[t.data_ptr() for t in out["O"]])
    la = (_VP * max(nl, 1))(*[(t.data_ptr() if t is not None else None) for t in out["lse"]])
    _check("tg_prefill_above_L", lib().tg_prefill_above_L(
        _dtype(H), _ptr(H), H.stride(0), d, _ptr(W1), _ptr(b1), _ptr(w2), float(b2), float(temperature), W1.shape[0],
        s.ref(), nl,
        qa, ka, va, Hq, Hkv, D, float(softmax_scale), _ptr(head_gain), int(flags), _ptr(out["score"]),
        _ptr(out["kept_idx"]), _ptr(out["cu_kept_dev"]), _ptr(out["H_kept"]), _ptr(out["pos"]), _ptr(out["g"]),
        _ptr(out["logg"]), oa, la, _ptr(dev_status), _stream(stream)))
    return out


def tg_prefill_projected(H, W1, b1, w2, b2, seqlens, q_len, k, W_qkv, rope_theta, Hq, Hkv, D, softmax_scale,
                         head_gain=None, flags=0, want_lse=False, out=None, dev_status=None, stream=None,
                         temperature: float = 1.0):
    """The gated path with each above-L layer's own projections: score -> top-K -> kept rows ->
    per layer Q/K/V (rotary at original positions; K and V are the layer's kept-only cache) ->
    gated attention. W_qkv: list of [(Hq + 2 Hkv) D, d] bf16 matrices. Returns a dict with score,
    kept_idx, cu_kept_dev, H_kept, pos, g, logg and per-layer lists Q, K_cache, V_cache, O, lse."""
    _want(torch.float32, b1=b1, head_gain=head_gain)
    _want(torch.int32, dev_status=dev_status)
    _like("H", H, W1=W1, w2=w2, **{f"W_qkv[{i}]": W for i, W in enumerate(W_qkv)})
    n_tok, d = H.shape
    for i, W in enumerate(W_qkv):
        _contig(**{f"W_qkv[{i}]": W})
        _shape(f"W_qkv[{i}]", W, ((Hq + 2 * Hkv) * D, d))
    _cuda(H, W1, b1, w2, head_gain, dev_status, *W_qkv)
    s = Seqs(seqlens, q_len, k)
    cu = tg_kept_counts(seqlens, q_len, k)
    m = cu[-1]
    dev = H.device
    nl = len(W_qkv)
    bf = torch.bfloat16
    if out is None:
        out = {
            "score": torch.empty(n_tok, device=dev, dtype=torch.float32),
            "kept_idx": torch.empty(m, device=dev, dtype=torch.int32),
            "cu_kept_dev": torch.empty(s.B + 1, device=dev, dtype=torch.int32),
            "H_kept": torch.empty(m, d, device=dev, dtype=H.dtype),
            "pos": torch.empty(m, device=dev, dtype=torch.int32),
            "g": torch.empty(m, device=dev, dtype=torch.float32),
            "logg": torch.empty(m, device=dev, dtype=torch.float32),
            "Q": [torch.empty(m, Hq, D, device=dev, dtype=bf) for _ in range(nl)],
            "K_cache": [torch.empty(m, Hkv, D, device=dev, dtype=bf) for _ in range(nl)],
            "V_cache": [torch.empty(m, Hkv, D, device=dev, dtype=bf) for _ in range(nl)],
            "O": [torch.empty(m, Hq, D, device=dev, dtype=bf) for _ in range(nl)],
            "lse": [torch.empty(Hq, m, device=dev, dtype=torch.float32) if want_lse else None for _ in range(nl)],
        }
    _check_out(out)
    arr = lambda ts: (_VP * max(nl, 1))(*[(t.data_ptr() if t is not None else None) for t in ts])
    _check("tg_prefill_projected", lib().tg_prefill_projected(
        _dtype(H), _ptr(H), H.stride(0), d, _ptr(W1), _ptr(b1), _ptr(w2), float(b2), float(temperature), W1.shape[0],
        s.ref(), nl, arr(W_qkv), float(rope_theta), Hq, Hkv, D, float(softmax_scale), _ptr(head_gain), int(flags),
        _ptr(out["score"]), _ptr(out["kept_idx"]), _ptr(out["cu_kept_dev"]), _ptr(out["H_kept"]), _ptr(out["pos"]),
        _ptr(out["g"]), _ptr(out["logg"]), arr(out["Q"]), arr(out["K_cache"]), arr(out["V_cache"]), arr(out["O"]),
        arr(out["lse"]), _ptr(dev_status), _stream(stream)))
    return out


def _check_out(out):
    """The output buffers of the chain have the library's fixed dtypes and are contiguous."""
    _want(torch.float32, score=out["score"], g=out["g"], logg=out["logg"])
    _want(torch.int32, kept_idx=out["kept_idx"], cu_kept_dev=out["cu_kept_dev"], pos=out["pos"])
    for i, t in enumerate(out["lse"]):
        _want(torch.float32, **{f"lse[{i}]": t})


class PreparedChain:
    """The gated path with every C-ABI argument marshalled once, for repeated launches.

    Holds ctypes copies of the pointers and sizes so each call goes straight into the C ABI
    (a few microseconds of host time per launch instead of rebuilding the arguments). The
    tensors passed in must stay alive and keep their storage while this object is used.
    """

    def __init__(self, H, W1, b1, w2, b2, seqlens, q_len, k, layers, softmax_scale, out, head_gain=None, flags=0,
                 dev_status=None, stream=None, temperature: float = 1.0):
        _want(torch.float32, b1=b1, head_gain=head_gain)
        _want(torch.int32, dev_status=dev_status)
        _check_out(out)
        _cuda(H, W1, b1, w2, head_gain, dev_status)
        self._L = lib()
        self._seqs = Seqs(seqlens, q_len, k)
        cu = tg_kept_counts(seqlens, q_len, k)
        self._cu = (ctypes.c_int32 * len(cu))(*cu)
        self._B = len(cu) - 1
        self._stream = _stream(stream)
        self._keep = (H, W1, b1, w2, layers, out, head_gain, dev_status)
        dt = _dtype(H)
        n_tok, d = H.shape
        s = self._stream
        self._score_args = (dt, _ptr(H), H.stride(0), n_tok, d, _ptr(W1), _ptr(b1), _ptr(w2), float(b2),
                            float(temperature), W1.shape[0], _ptr(out["score"]), _ptr(dev_status), s)
        self._select_args = (_ptr(out["score"]), self._seqs.ref(), _ptr(out["kept_idx"]), _ptr(out["cu_kept_dev"]),
                             _ptr(dev_status), s)
        self._gather_args = (dt, _ptr(H), H.stride(0), d, _ptr(out["score"]), _ptr(out["kept_idx"]), self._seqs.ref(),
                             int(flags), _ptr(out["H_kept"]), _ptr(out["pos"]), _ptr(out["g"]), _ptr(out["logg"]),
                             _ptr(dev_status), s)
        self._attn_args = []
        for (q, kk, v), o, l in zip(layers, out["O"], out["lse"]):
            self._attn_args.append((dt, _ptr(q), _ptr(kk), _ptr(v), _ptr(out["logg"]), _ptr(head_gain), _ptr(out["pos"]),
                                    self._cu, self._B, q.shape[1], kk.shape[1], q.shape[2], float(softmax_scale),
                                    int(flags), _ptr(o), _ptr(l), _ptr(dev_status), s))

        nl = len(layers)
        self._arrays = tuple((_VP * max(nl, 1))(*[t[i].data_ptr() for t in layers]) for i in range(3))
        self._o_arr = (_VP * max(nl, 1))(*[t.data_ptr() for t in out["O"]])
        self._lse_arr = (_VP * max(nl, 1))(*[(t.data_ptr() if t is not None else None) for t in out["lse"]])
        Hq = layers[0][0].shape[1] if nl else 1
        Hkv = layers[0][1].shape[1] if nl else 1
        D = layers[0][0].shape[2] if nl else 64
        self._prefill_args = (dt, _ptr(H), H.stride(0), d, _ptr(W1), _ptr(b1), _ptr(w2), float(b2), float(temperature),
                              W1.shape[0],
                              self._seqs.ref(), nl, *self._arrays, Hq, Hkv, D, float(softmax_scale), _ptr(head_gain),
                              int(flags), _ptr(out["score"]), _ptr(out["kept_idx"]), _ptr(out["cu_kept_dev"]),
                              _ptr(out["H_kept"]), _ptr(out["pos"]), _ptr(out["g"]), _ptr(out["logg"]), self._o_arr,
                              self._lse_arr, _ptr(dev_status), s)

    def prefill(self):
        """The whole path through its single C-ABI entry (tg_prefill_above_L)."""
        _check("tg_prefill_above_L", self._L.tg_prefill_above_L(*self._prefill_args))

    def score(self):
        _check("tg_score", self._L.tg_score(*self._score_args))

    def select(self):
        _check("tg_topk_select", self._L.tg_topk_select(*self._select_args))

    def gather(self):
        _check("tg_gather", self._L.tg_gather(*self._gather_args))

    def attention(self, layer=0):
        _check("tg_gated_attn_fwd", self._L.tg_gated_attn_fwd(*self._attn_args[layer]))

    def __call__(self):
        self.score()
        self.select()
        self.gather()
        for i in range(len(self._attn_args)):
            self.attention(i)
