"""The many-sequence top-K (tg_topk_select_stream) against the oracle's topk_select, bit for bit:
kept indices, cu_kept and the status word, on the same cases as the cluster select (edge cases,
ties, NaN, -0, a crowded threshold bin, more sequences than one launch carries, long sequences),
plus the byte-heavy shape of many long sequences; its outputs also equal tg_topk_select's."""
import numpy as np
import pytest
import torch

import learned_token_pruning_02_b200 as tg
import tg_inputs as ti
from oracle import tg_oracle as orc

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = torch.device("cuda")


def _check(s, seqlens, q_len, k):
    sd = torch.from_numpy(np.ascontiguousarray(s, dtype=np.float32)).to(DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    kept, cu = tg.tg_topk_select_stream(sd, seqlens, q_len, k, dev_status=st)
    st_c = torch.zeros(1, dtype=torch.int32, device=DEV)
    kept_c, cu_c = tg.tg_topk_select(sd, seqlens, q_len, k, dev_status=st_c)
    torch.cuda.synchronize()
    ref, ref_cu = orc.topk_select(s, seqlens, q_len, k)
    assert cu.cpu().numpy().tolist() == ref_cu.tolist()
    assert np.array_equal(kept.cpu().numpy(), ref.astype(np.int32))
    assert torch.equal(kept, kept_c) and torch.equal(cu, cu_c)
    assert st.item() == st_c.item()
    return int(st.item())


@pytest.mark.parametrize("case", [
    ((1000,), (10,), (0,)),           # K = 0: only the question tail
    ((1000,), (10,), (990,)),         # K = N - q: everything
    ((1000,), (10,), (5000,)),        # K > N - q
    ((1000,), (0,), (17,)),           # no question
    ((64,), (64,), (8,)),             # question only
    ((0, 5, 0), (0, 2, 0), (3, 1, 3)),  # empty sequences
    ((1,), (0,), (1,)),
    ((16385,), (1,), (16383,)),       # K = n_ctx - 1 over four whole chunks
    ((8193,), (0,), (4096,)),         # a last chunk of one key
    ((40000,), (0,), (40000,)),       # every key kept across ten chunks
    ((262144,), (0,), (1000,)),       # the largest context: 64 chunks
])
def test_select_stream_edge_cases(case):
    seqlens, q_len, k = case
    g = np.random.default_rng(sum(seqlens) + 1)
    s = g.standard_normal(sum(seqlens)).astype(np.float32)
    _check(s, seqlens, q_len, k)


def test_select_stream_ties_nan_negzero():
    g = np.random.default_rng(1)
    n = 50000
    s = g.integers(-2, 3, n).astype(np.float32)  # 5 distinct values: tie groups across every chunk
    s[g.random(n) < 0.01] = np.nan
    s[g.random(n) < 0.05] = -0.0
    s[g.random(n) < 0.01] = -np.inf
    for k in (1, 777, 20000, 49000):
        assert _check(s, (n,), (100,), (k,)) & tg.TG_DEV_NAN_SCORE
    assert _check(np.zeros(40000, np.float32), (40000,), (0,), (12345,)) == 0  # all equal
    s = g.standard_normal(20000).astype(np.float32)
    s[[5, 17777]] = np.nan
    assert _check(s, (20000,), (10,), (19990,)) & tg.TG_DEV_NAN_SCORE  # every context token kept


def test_select_stream_crowded_threshold_bin():
    """Every key shares its top 12 bits, so the whole context lands in the candidate list."""
    g = np.random.default_rng(5)
    for n, ks in ((60000, (1, 3000, 25000, 59000)), (200000, (4096, 150000))):
        s = (1.0 + 0.125 * g.random(n)).astype(np.float32)
        s[g.random(n) < 0.3] = np.float32(1.0625)
        for k in ks:
            assert _check(s, (n,), (64,), (k,)) == 0


def test_select_stream_many_sequences():
    """Ragged sequences at unaligned starts (word-by-word loads) and more of them than one launch."""
    g = np.random.default_rng(2)
    B = 150  # more than the 64 sequences of one launch
    seqlens = tuple(int(x) for x in g.integers(0, 40000, B))
    q_len = tuple(int(g.integers(0, min(n, 300) + 1)) for n in seqlens)
    k = tuple(int(x) for x in g.integers(-5, 20000, B))
    s = np.round(g.standard_normal(sum(seqlens)) * 8).astype(np.float32)
    _check(s, seqlens, q_len, k)


def test_select_stream_byte_heavy_shape():
    """64 sequences of 131072 tokens (question tail 256, K = 4096): the shape of the bench's
    bandwidth instance, with bf16-valued scores (ties)."""
    g = np.random.default_rng(3)
    seqlens, q_len, k = (131072,) * 64, (256,) * 64, (4096,) * 64
    s = ti.bf16_bits_to_f32(ti.f32_to_bf16_bits(g.standard_normal(sum(seqlens)).astype(np.float32)))
    assert _check(s, seqlens, q_len, k) == 0


def test_select_stream_unaligned_score_pointer():
    """Scores that start 4 bytes past a 16-byte boundary load word by word, with the same result."""
    g = np.random.default_rng(9)
    n = 40000
    s = g.standard_normal(n + 1).astype(np.float32)
    sd = torch.from_numpy(s).to(DEV)[1:]
    assert sd.data_ptr() % 16 == 4
    kept, cu = tg.tg_topk_select_stream(sd, (n,), (100,), (1234,))
    torch.cuda.synchronize()
    ref, ref_cu = orc.topk_select(s[1:], (n,), (100,), (1234,))
    assert np.array_equal(kept.cpu().numpy(), ref.astype(np.int32))
    assert cu.cpu().numpy().tolist() == ref_cu.tolist()
