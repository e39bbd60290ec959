"""The allocation-free gate-gradient entry point (tg_gate_mlp_bwd_noalloc), for callers that may
not allocate device memory (a runtime that plans all memory up front, a plugin without access to
its host's allocator, a loop where cudaMalloc's implicit synchronisation is not allowed).

Called through the C ABI twice in a row on the same device, its results must match the
workspace entry point (tg_gate_mlp_bwd) within the bf16 / f32 tolerance of the other tests; the
second call sees the scratch array as the first call left it. A shape whose working memory
exceeds the fixed array is refused before anything runs. This file is collected last so that a
run stopping at its first failure has already run every other test; it also passes alone in a
fresh process (the first call on the device looks the array's address up)."""
import ctypes
import math

import numpy as np
import pytest
import torch

import learned_token_pruning_02_b200 as tg
import tg_inputs as ti
from tg_testutil import TOL, from_dev, max_abs_rel, to_dev

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _case(dtype, M, d, dg, seed):
    g = np.random.default_rng(seed)

    def arr(*shape, s=1.0):
        x = (g.standard_normal(shape) * s).astype(np.float32)
        return to_dev(ti.f32_to_bf16_bits(x) if dtype == "bf16" else x, dtype)

    return (arr(M, d), arr(dg, d, s=1 / math.sqrt(d)), to_dev((g.standard_normal(dg) * 0.1).astype(np.float32), "f32"),
            arr(dg, s=1 / math.sqrt(dg)), to_dev((g.standard_normal(M) * 0.01).astype(np.float32), "f32"))


@pytest.mark.parametrize("dtype,M,d,dg,T", [("bf16", 2176, 2048, 256, 1.0), ("f32", 333, 512, 128, 0.6)])
def test_noalloc_matches_workspace_entry_point_twice(dtype, M, d, dg, T):
    H, W1, b1, w2, ds = _case(dtype, M, d, dg, M)
    ref = tg.tg_gate_mlp_bwd(H, W1, b1, w2, ds, temperature=T)
    torch.cuda.synchronize()
    for call in range(2):
        out = (torch.full((dg, d), 9.0, device="cuda"), torch.full((dg,), 9.0, device="cuda"),
               torch.full((dg,), 9.0, device="cuda"), torch.full((1,), 9.0, device="cuda"))
        got = tg.tg_gate_mlp_bwd_noalloc(H, W1, b1, w2, ds, *out, temperature=T)
        torch.cuda.synchronize()
        for name, a, r in zip(("dW1", "db1", "dw2", "db2"), got, ref):
            err = max_abs_rel(from_dev(a), from_dev(r))
            assert err <= TOL[dtype], (call, name, err)


def test_noalloc_refuses_shapes_beyond_its_scratch():
    L = tg.lib()
    M, d, dg = 1 << 20, 2048, 256
    need = L.tg_gate_mlp_bwd_workspace_size(M, d, dg)
    assert need > 16 << 20
    fake = ctypes.c_void_p(0x1000)
    st = L.tg_gate_mlp_bwd_noalloc(1, fake, M, d, fake, None, fake, 1.0, dg, fake, fake, None, None, None, None,
                                   None)
    assert st == 2  # TG_ERR_UNSUPPORTED, nothing launched
    assert b"scratch" in L.tg_last_error()
