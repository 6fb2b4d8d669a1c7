"""The seeded synthetic inputs follow their stated recipe (CPU only).

Both the oracle and the CUDA path take their inputs from
mla_latent_kv_18_b200/inputs.py; these checks pin the recipe it documents:
determinism per seed, shapes and dtypes, N(0, 1) activations and cache,
N(0, 1)/sqrt(d_c) weights, ragged lengths within their bounds, and page tables
that assign exactly sum ceil(L_b / 64) pages once each (-1 past a sequence's
last page).
"""
import math

import pytest
import torch

from mla_latent_kv_18_b200.inputs import make_inputs, workload


@pytest.mark.parametrize("name,kw", [("tiny", {}),
                                     ("dsv3", dict(batch=3, heads=8, seq_len=300)),
                                     ("ragged", dict(batch=6, heads=4, ragged=(100, 700))),
                                     ("retrofit", dict(batch=2, heads=4, seq_len=200)),
                                     ("prefill", dict(batch=2, n_q=40, heads=4, seq_len=130))])
def test_shapes_dtypes_and_determinism(name, kw):
    w = workload(name, **kw)
    a, b, c = make_inputs(w, seed=7), make_inputs(w, seed=7), make_inputs(w, seed=8)
    for k in a:
        assert torch.equal(a[k], b[k]), k                     # same seed: same bits
    assert not torch.equal(a["q_c"], c["q_c"])                # another seed: other values
    B, P = w.batch, w.page_size
    assert a["q_c"].shape == (B, w.n_q, w.heads, w.d_nope) and a["q_c"].dtype == torch.bfloat16
    assert a["q_r"].shape == (B, w.n_q, w.heads, w.d_rope)
    assert a["w_uk"].shape == (w.heads, w.d_nope, w.d_latent)
    assert a["w_uv"].shape == (w.heads, w.d_latent, w.d_v)
    lens = a["seq_lens"]
    assert lens.dtype == torch.int32 and lens.shape == (B,)
    if w.ragged:
        assert int(lens.min()) >= w.ragged[0] and int(lens.max()) <= w.ragged[1]
    else:
        assert bool((lens == w.seq_len).all())
    pages = [(int(L) + P - 1) // P for L in lens]
    assert a["ckv_pool"].shape == (sum(pages), P, w.d_latent)
    assert a["kr_pool"].shape == (sum(pages), P, w.d_rope)
    table = a["block_table"]
    assert table.shape == (B, max(pages)) and table.dtype == torch.int32
    used = torch.cat([table[i, :n] for i, n in enumerate(pages)])
    assert sorted(used.tolist()) == list(range(sum(pages)))   # every page exactly once
    for i, n in enumerate(pages):
        assert bool((table[i, n:] == -1).all())
    if w.table == "identity":
        assert used.tolist() == list(range(sum(pages)))


def test_value_distributions():
    w = workload("dsv3", batch=4, heads=16, seq_len=2048)
    x = make_inputs(w, seed=0)
    # within 5 standard errors of N(0, 1) for each sample size (plus bf16 rounding of the std)
    def close(v, std):
        n = v.numel()
        m_tol, s_tol = 5.0 * std / math.sqrt(n), 5.0 * std / math.sqrt(2 * n) + 4e-3 * std
        return abs(float(v.mean())) < m_tol and abs(float(v.std()) - std) < s_tol
    for k in ("q_c", "q_r", "ckv_pool", "kr_pool"):
        assert close(x[k].float(), 1.0), k
    for k in ("w_uk", "w_uv"):
        assert close(x[k].float(), 1.0 / math.sqrt(w.d_latent)), k
    # the pages of a permuted table are not in order
    assert x["block_table"][0, :8].tolist() != list(range(8))
