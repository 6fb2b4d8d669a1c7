"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test ties the oracle to something the pages or the mathematics fix:
closed forms printed on the pages, special cases with a textbook answer,
invariants of softmax attention, and brute force on tiny inputs written
independently with numpy/scipy. Together they are chosen so that a dropped
term, a wrong sign, scale or index, an off-by-one mask or a transposed operand
anywhere in the oracle fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from mla_latent_kv_18_b200.inputs import make_inputs, workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "cache_sizes.txt")

# small variants of the five workloads (same head dims, fewer heads/tokens)
SMALL = {
    "tiny": workload("tiny", heads=4),
    "dsv3": workload("dsv3", batch=2, heads=4, seq_len=200),
    "ragged": workload("ragged", batch=3, heads=3, ragged=(65, 190)),
    "retrofit": workload("retrofit", batch=2, heads=4, seq_len=130),
}


def _golden():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = (s.strip() for s in line.split("="))
                vals[k] = float(v)
    return vals


def _rel(a, b):
    return np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300)


def _bf16(x):
    return torch.tensor(np.array(x, dtype=np.float64), dtype=torch.float32).to(torch.bfloat16)


def _f64(t):
    return t.to(torch.float64).numpy()


def _dense_cache(inp):
    """Logical (per-sequence, in token order) c_KV and k_R via numpy indexing."""
    table = inp["block_table"].numpy()
    lens = inp["seq_lens"].numpy()
    ckv, kr = _f64(inp["ckv_pool"]), _f64(inp["kr_pool"])
    P = ckv.shape[1]
    out = []
    for b, L in enumerate(lens):
        t = np.arange(L)
        pages = table[b, t // P]
        out.append((ckv[pages, t % P], kr[pages, t % P]))
    return out


def _numpy_reference(inp, scale):
    """Brute force: dense per-head keys/values, whole-row softmax (scipy)."""
    qc, qr = _f64(inp["q_c"]), _f64(inp["q_r"])
    wuk, wuv = _f64(inp["w_uk"]), _f64(inp["w_uv"])
    B, n_q, H, _ = qc.shape
    out = np.zeros((B, n_q, H, wuv.shape[-1]))
    for b, (c, r) in enumerate(_dense_cache(inp)):
        L = c.shape[0]
        k_nope = np.einsum("sc,hdc->shd", c, wuk)          # path A of the page
        v = np.einsum("sc,hce->she", c, wuv)
        for i in range(n_q):
            vis = L - n_q + i + 1
            s = (np.einsum("hd,shd->hs", qc[b, i], k_nope[:vis])
                 + np.einsum("hj,sj->hs", qr[b, i], r[:vis])) * scale
            p = scipy.special.softmax(s, axis=-1)
            out[b, i] = np.einsum("hs,she->he", p, v[:vis])
    return out


def _run_both(inp, scale=None):
    args = [inp[k] for k in ("q_c", "q_r", "ckv_pool", "kr_pool", "block_table", "seq_lens",
                             "w_uk", "w_uv")]
    dec = oracle.decode_decompress(*args, scale=scale)
    ab, o_lat, lse = oracle.decode_absorbed(*args, scale=scale)
    return dec, ab, o_lat, lse


# ---------------------------------------------------------------------------
# closed forms printed on the pages
# ---------------------------------------------------------------------------

def test_cache_size_closed_forms():
    g = _golden()
    assert 512 + 64 == g["mla_elements_per_token"]
    assert 128 * 128 == g["mha_elements_per_head_block"]
    assert oracle.mla_cache_bytes_per_token(512, 64) == g["mla_bytes_per_token"]
    assert oracle.mla_cache_bytes_per_token(512, 64) / 1024 == 1.125
    assert oracle.mha_cache_bytes_per_token(128, 128) == g["mha_bytes_per_token"]
    comp = 100.0 * (1 - oracle.mla_cache_bytes_per_token(512, 64)
                    / oracle.mha_cache_bytes_per_token(128, 128))
    assert round(comp, 2) == g["compression_percent"]
    tokens = g["total_context"] * g["total_batch"] * g["total_layers"]
    mha = tokens * oracle.mha_cache_bytes_per_token(128, 128) / 2**40
    gqa = tokens * oracle.mha_cache_bytes_per_token(8, 128) / 2**30
    mla = tokens * oracle.mla_cache_bytes_per_token(512, 64) / 2**30
    assert mha == pytest.approx(g["mha_total_tib"], rel=1e-12)
    assert gqa == pytest.approx(g["gqa8_total_gib"], rel=0.03)
    assert mla == pytest.approx(g["mla_total_gib"], rel=0.03)
    # the latent page of 64 tokens is 72 KB ("MLA operator design" §3)
    assert 64 * oracle.mla_cache_bytes_per_token(512, 64) == 72 * 1024
    # "MHA2MLA" §4.2 formulas at its §3.2 dims
    assert oracle.mha_cache_bytes_per_token(32, 128, 1) == g["retrofit_mha_elements_per_token"]
    assert oracle.mla_cache_bytes_per_token(64, 8, 1) == g["retrofit_mla_elements_per_token"]


def test_default_scale_is_page_value():
    # scale = 1/sqrt(dhc + dr) with DeepSeek dims 128 + 64 ("MLA operator design" §4)
    assert oracle.default_scale(128, 64) == 1.0 / math.sqrt(192.0)
    assert oracle.default_scale(120, 8) == 1.0 / math.sqrt(128.0)


# ---------------------------------------------------------------------------
# P1 absorption identity and P4 brute force
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", list(SMALL))
def test_absorption_identity_and_brute_force(name):
    w = SMALL[name]
    inp = make_inputs(w, seed=1)
    dec, ab, o_lat, lse = _run_both(inp)
    assert np.isfinite(dec).all()
    assert _rel(ab, dec) <= 1e-12            # path A == path B (associativity)
    ref = _numpy_reference(inp, oracle.default_scale(w.d_nope, w.d_rope))
    assert _rel(dec, ref) <= 1e-12
    assert np.abs(dec - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_sampled_selection_matches_full():
    inp = make_inputs(SMALL["dsv3"], seed=2)
    args = [inp[k] for k in ("q_c", "q_r", "ckv_pool", "kr_pool", "block_table", "seq_lens",
                             "w_uk", "w_uv")]
    full = oracle.decode_decompress(*args)
    sel = [1, 5, 6]
    part = oracle.decode_decompress(*args, sel=sel)
    flat_f, flat_p = full.reshape(-1, full.shape[-1]), part.reshape(-1, part.shape[-1])
    np.testing.assert_array_equal(flat_p[sel], flat_f[sel])
    assert not flat_p[0].any()


# ---------------------------------------------------------------------------
# special cases
# ---------------------------------------------------------------------------

def test_softmax_weights_sum_to_one():
    # V[t] = c[t] W_UV with W_UV = identity and every c[t] = e_0  =>  out = (sum p) e_0
    w = workload("dsv3", batch=2, heads=3, seq_len=150, d_latent=64, d_v=64)
    inp = make_inputs(w, seed=3)
    ckv = torch.zeros_like(inp["ckv_pool"])
    ckv[..., 0] = 1.0
    inp["ckv_pool"] = ckv
    inp["w_uv"] = _bf16(np.broadcast_to(np.eye(64), (3, 64, 64)))
    # keep the scores non-trivial through the rope part
    dec, ab, _, _ = _run_both(inp)
    assert np.abs(dec[..., 0] - 1.0).max() <= 1e-13
    assert np.abs(dec[..., 1:]).max() == 0.0
    assert np.abs(ab[..., 0] - 1.0).max() <= 1e-13


def test_single_token_returns_its_value():
    w = workload("dsv3", batch=3, heads=4, seq_len=1)
    inp = make_inputs(w, seed=4)
    dec, ab, _, lse = _run_both(inp)
    for b, (c, _r) in enumerate(_dense_cache(inp)):
        v = np.einsum("c,hce->he", c[0], _f64(inp["w_uv"]))
        np.testing.assert_allclose(dec[b, 0], v, rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(ab[b, 0], v, rtol=1e-13, atol=1e-15)


def test_zero_query_gives_mean_value():
    w = SMALL["ragged"]
    inp = make_inputs(w, seed=5)
    inp["q_c"] = torch.zeros_like(inp["q_c"])
    inp["q_r"] = torch.zeros_like(inp["q_r"])
    dec, ab, _, lse = _run_both(inp)
    for b, (c, _r) in enumerate(_dense_cache(inp)):
        mean_v = np.einsum("c,hce->he", c.mean(axis=0), _f64(inp["w_uv"]))
        np.testing.assert_allclose(dec[b, 0], mean_v, rtol=1e-12, atol=1e-14)
        # lse of equal scores 0 over L tokens is log L
        np.testing.assert_allclose(lse[b, 0], math.log(c.shape[0]), rtol=1e-13)


def test_duplicated_tokens_leave_result_unchanged():
    w = workload("dsv3", batch=1, heads=3, seq_len=96)
    inp = make_inputs(w, seed=6)
    dec, _, _, _ = _run_both(inp)
    # same logical sequence with every token repeated twice
    (c, r), = _dense_cache(inp)
    c2, r2 = np.repeat(c, 2, axis=0), np.repeat(r, 2, axis=0)
    L2, P = c2.shape[0], 64
    n_pages = (L2 + P - 1) // P
    pool_c = np.zeros((n_pages * P, c.shape[1]))
    pool_r = np.zeros((n_pages * P, r.shape[1]))
    pool_c[:L2], pool_r[:L2] = c2, r2
    inp2 = dict(inp)
    inp2["ckv_pool"] = _bf16(pool_c.reshape(n_pages, P, -1))
    inp2["kr_pool"] = _bf16(pool_r.reshape(n_pages, P, -1))
    inp2["block_table"] = torch.arange(n_pages, dtype=torch.int32)[None]
    inp2["seq_lens"] = torch.tensor([L2], dtype=torch.int32)
    dec2, _, _, _ = _run_both(inp2)
    np.testing.assert_allclose(dec2, dec, rtol=1e-12, atol=1e-15)


def test_common_score_shift_leaves_result_unchanged():
    # append one rope dimension with q_r = alpha and k_R = 1 for every token:
    # every score moves by scale*alpha, which softmax ignores (fixed scale).
    w = workload("retrofit", batch=2, heads=3, seq_len=100)
    inp = make_inputs(w, seed=7)
    scale = oracle.default_scale(w.d_nope, w.d_rope)
    dec, _, _, _ = _run_both(inp, scale=scale)
    inp2 = dict(inp)
    inp2["q_r"] = torch.cat([inp["q_r"], torch.full_like(inp["q_r"][..., :1], 3.0)], dim=-1)
    inp2["kr_pool"] = torch.cat([inp["kr_pool"], torch.ones_like(inp["kr_pool"][..., :1])], dim=-1)
    dec2, ab2, _, _ = _run_both(inp2, scale=scale)
    np.testing.assert_allclose(dec2, dec, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(ab2, dec, rtol=1e-12, atol=1e-15)


def test_two_token_closed_form_pins_scale():
    # nope part silenced (q_c = 0); rope scores x and 0 => weights are logistic
    # in scale*x with scale = 1/sqrt(192) for the DeepSeek dims.
    w = workload("dsv3", batch=1, heads=2, seq_len=2)
    inp = make_inputs(w, seed=8)
    inp["q_c"] = torch.zeros_like(inp["q_c"])
    qr = torch.zeros_like(inp["q_r"])
    qr[..., 0] = 6.0
    qr[0, 0, 1, 0] = -2.5
    inp["q_r"] = qr
    kr = torch.zeros_like(inp["kr_pool"])
    page = int(inp["block_table"][0, 0])
    kr[page, 0, 0] = 1.0
    inp["kr_pool"] = kr
    dec, ab, _, _ = _run_both(inp)
    (c, _r), = _dense_cache(inp)
    v = np.einsum("sc,hce->she", c, _f64(inp["w_uv"]))
    tau = 1.0 / math.sqrt(192.0)
    for h, x in ((0, 6.0), (1, -2.5)):
        p0 = scipy.special.expit(tau * x)
        expect = p0 * v[0, h] + (1 - p0) * v[1, h]
        np.testing.assert_allclose(dec[0, 0, h], expect, rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(ab[0, 0, h], expect, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("name", ["dsv3", "retrofit"])
def test_rope_argmax_and_mask(name):
    # W_UK = 0 silences the nope part. One visible token gets a rope score 60
    # above all others => the output is its value. A token in the unused tail of
    # the last page gets an even larger score but lies beyond L => ignored.
    w = SMALL[name]
    inp = make_inputs(w, seed=9, seq_lens=[w.seq_len - 5] * w.batch)
    inp["w_uk"] = torch.zeros_like(inp["w_uk"])
    scale = oracle.default_scale(w.d_nope, w.d_rope)
    qr = torch.zeros_like(inp["q_r"])
    qr[..., 0] = 60.0 / scale
    inp["q_r"] = qr
    kr = torch.zeros_like(inp["kr_pool"])
    P = w.page_size
    star = {}
    for b in range(w.batch):
        L = int(inp["seq_lens"][b])
        t_star = (37 * (b + 1)) % (L - w.n_q + 1)          # visible to every query
        pg = int(inp["block_table"][b, t_star // P])
        kr[pg, t_star % P, 0] = 1.0
        tail = L + 2                                         # beyond L, same last page
        pg_t = int(inp["block_table"][b, tail // P])
        kr[pg_t, tail % P, 0] = 2.0
        star[b] = t_star
    inp["kr_pool"] = kr
    dec, ab, _, _ = _run_both(inp, scale=scale)
    for b, (c, _r) in enumerate(_dense_cache(inp)):
        v = np.einsum("c,hce->he", c[star[b]], _f64(inp["w_uv"]))
        for i in range(w.n_q):
            np.testing.assert_allclose(dec[b, i], v, rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(ab[b, i], v, rtol=1e-12, atol=1e-14)


def test_causal_pair_equals_prefix_decode():
    # query 0 of a two-query step sees exactly the prefix of length L-1
    w = SMALL["retrofit"]
    inp = make_inputs(w, seed=10)
    dec, _, _, _ = _run_both(inp)
    single = dict(inp)
    single["q_c"] = inp["q_c"][:, :1].contiguous()
    single["q_r"] = inp["q_r"][:, :1].contiguous()
    single["seq_lens"] = inp["seq_lens"] - 1
    dec0, _, _, _ = _run_both(single, scale=oracle.default_scale(w.d_nope, w.d_rope))
    np.testing.assert_allclose(dec[:, 0], dec0[:, 0], rtol=1e-12, atol=1e-15)
    # and query 1 sees the whole sequence
    last = dict(inp)
    last["q_c"] = inp["q_c"][:, 1:].contiguous()
    last["q_r"] = inp["q_r"][:, 1:].contiguous()
    dec1, _, _, _ = _run_both(last, scale=oracle.default_scale(w.d_nope, w.d_rope))
    np.testing.assert_allclose(dec[:, 1], dec1[:, 0], rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------------------
# paging: gather bits and table invariance
# ---------------------------------------------------------------------------

def test_gather_is_bit_copy():
    w = SMALL["ragged"]
    inp = make_inputs(w, seed=11)
    got = oracle.gather(inp["ckv_pool"], inp["block_table"], inp["seq_lens"], w.page_size)
    bits = inp["ckv_pool"].view(torch.int16).numpy().view(np.uint16)
    table, lens = inp["block_table"].numpy(), inp["seq_lens"].numpy()
    for b, L in enumerate(lens):
        t = np.arange(L)
        np.testing.assert_array_equal(got[b, :L], bits[table[b, t // 64], t % 64])
        assert not got[b, L:].any()


def test_page_permutation_invariance_is_exact():
    w = SMALL["dsv3"]
    inp = make_inputs(w, seed=12)
    dec, ab, o_lat, lse = _run_both(inp)
    g = torch.Generator().manual_seed(99)
    n = inp["ckv_pool"].shape[0]
    perm = torch.randperm(n, generator=g)               # new physical slot of old page k
    inp2 = dict(inp)
    inp2["ckv_pool"] = torch.empty_like(inp["ckv_pool"])
    inp2["kr_pool"] = torch.empty_like(inp["kr_pool"])
    inp2["ckv_pool"][perm] = inp["ckv_pool"]
    inp2["kr_pool"][perm] = inp["kr_pool"]
    tbl = inp["block_table"].clone()
    used = tbl >= 0
    tbl[used] = perm[tbl[used].long()].to(torch.int32)
    inp2["block_table"] = tbl
    dec2, ab2, o_lat2, lse2 = _run_both(inp2)
    np.testing.assert_array_equal(dec2, dec)
    np.testing.assert_array_equal(ab2, ab)
    np.testing.assert_array_equal(lse2, lse)


def test_bad_tables_are_rejected():
    w = SMALL["dsv3"]
    inp = make_inputs(w, seed=13)
    args = lambda d: [d[k] for k in ("q_c", "q_r", "ckv_pool", "kr_pool", "block_table",
                                     "seq_lens", "w_uk", "w_uv")]
    bad = dict(inp)
    bad["block_table"] = inp["block_table"].clone()
    bad["block_table"][0, 1] = inp["ckv_pool"].shape[0]       # page id out of range
    with pytest.raises(ValueError):
        oracle.decode_decompress(*args(bad))
    bad2 = dict(inp)
    bad2["seq_lens"] = inp["seq_lens"].clone()
    bad2["seq_lens"][1] = inp["block_table"].shape[1] * 64 + 1  # beyond the table
    with pytest.raises(ValueError):
        oracle.decode_decompress(*args(bad2))


# ---------------------------------------------------------------------------
# split windows and the log-sum-exp merge
# ---------------------------------------------------------------------------

def test_window_partials_combine_to_full_result():
    w = SMALL["retrofit"]
    inp = make_inputs(w, seed=14)
    scale = oracle.default_scale(w.d_nope, w.d_rope)
    q = torch.cat([inp["q_c"][..., :w.d_latent], inp["q_r"]], dim=-1)  # any bf16 query
    common = (inp["ckv_pool"], inp["kr_pool"], inp["block_table"], inp["seq_lens"], scale)
    o_full, lse_full = oracle.attend_latent(q, *common)
    edges = [0, 17, 64, 64, 100, 500, 1000]      # includes an empty and a past-the-end window
    parts = [oracle.attend_latent(q, *common, t_lo=a, t_hi=b) for a, b in zip(edges, edges[1:])]
    o_part = np.stack([p[0] for p in parts], axis=-2).reshape(-1, len(parts), w.d_latent)
    lse_part = np.stack([p[1] for p in parts], axis=-1).reshape(-1, len(parts))
    assert np.isneginf(lse_part[:, 2]).all() and np.isneginf(lse_part[:, 5]).all()
    o, lse = oracle.combine(o_part, lse_part)
    np.testing.assert_allclose(o, o_full.reshape(-1, w.d_latent), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(lse, lse_full.ravel(), rtol=1e-13)


def test_combine_textbook_cases():
    rng = np.random.default_rng(0)
    o_part = rng.standard_normal((3, 4, 5))
    lse_part = np.array([[0.0, -np.inf, 1.0, 2.0],
                         [-np.inf] * 4,
                         [5.0, 5.0, 5.0, 5.0]])
    o, lse = oracle.combine(o_part, lse_part)
    w0 = scipy.special.softmax(np.array([0.0, 1.0, 2.0]))
    np.testing.assert_allclose(o[0], w0 @ o_part[0, [0, 2, 3]], rtol=1e-14)
    np.testing.assert_allclose(lse[0], scipy.special.logsumexp([0.0, 1.0, 2.0]), rtol=1e-15)
    assert not o[1].any() and np.isneginf(lse[1])
    np.testing.assert_allclose(o[2], o_part[2].mean(axis=0), rtol=1e-14)
    np.testing.assert_allclose(lse[2], 5.0 + math.log(4.0), rtol=1e-15)


# ---------------------------------------------------------------------------
# absorb-in / absorb-out: operand orientation and brute force
# ---------------------------------------------------------------------------

def _onehot_weights(H, rows, cols, rng):
    """W[h][d][c] = 1 where c = perm_h(d) (rows <= cols)."""
    W = np.zeros((H, rows, cols))
    perms = [rng.permutation(cols)[:rows] for _ in range(H)]
    for h in range(H):
        W[h, np.arange(rows), perms[h]] = 1.0
    return W, perms


def test_absorb_q_orientation_and_brute_force():
    rng = np.random.default_rng(1)
    H, d_n, d_c, T = 3, 48, 64, 5
    q = _bf16(rng.standard_normal((T, H, d_n)))
    W, perms = _onehot_weights(H, d_n, d_c, rng)
    got = oracle.absorb_q(q, _bf16(W))
    qd = _f64(q)
    for h in range(H):
        expect = np.zeros((T, d_c))
        expect[:, perms[h]] = qd[:, h]
        np.testing.assert_array_equal(got[:, h], expect)
    Wr = _bf16(rng.standard_normal((H, d_n, d_c)) / 8)
    got = oracle.absorb_q(q, Wr)
    np.testing.assert_allclose(got, np.einsum("thd,hdc->thc", qd, _f64(Wr)), rtol=1e-12,
                               atol=1e-13)


def test_absorb_out_orientation_and_brute_force():
    rng = np.random.default_rng(2)
    H, d_c, d_v, T = 3, 64, 128, 4
    o = _bf16(rng.standard_normal((T, H, d_c)))
    Wt, perms = _onehot_weights(H, d_c, d_v, rng)        # W[h][c][e] = 1 at e = perm_h(c)
    got = oracle.absorb_out(o, _bf16(Wt))
    od = _f64(o)
    for h in range(H):
        expect = np.zeros((T, d_v))
        expect[:, perms[h]] = od[:, h]
        np.testing.assert_array_equal(got[:, h], expect)
    Wr = _bf16(rng.standard_normal((H, d_c, d_v)) / 8)
    got = oracle.absorb_out(o, Wr)
    np.testing.assert_allclose(got, np.einsum("thc,hce->the", od, _f64(Wr)), rtol=1e-12,
                               atol=1e-13)
    # fp64 input path agrees with the bf16 path on bf16-exact values
    np.testing.assert_array_equal(oracle.absorb_out(od, Wr), got)


ROPE_GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "rope_example.txt")


def _kv(path):
    vals = {}
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = (s.strip() for s in line.split("="))
                vals[k] = float(v)
    return vals


def test_rope_worked_example():
    """Hand-worked rotation (tests/golden/rope_example.txt): pins the pairing of
    adjacent channels, the frequency exponent, the sign of the angle and the
    position factor."""
    v = _kv(ROPE_GOLDEN)
    x = torch.tensor([[[1.0, 0.0, 0.0, 1.0]], [[1.0, 0.0, 0.0, 1.0]]], dtype=torch.bfloat16)
    y = oracle.rope(x, [1, 3], theta=10000.0)
    np.testing.assert_allclose(y[0, 0], [v["y0"], v["y1"], v["y2"], v["y3"]], rtol=0, atol=1e-15)
    np.testing.assert_allclose(y[1, 0], [v["z0"], v["z1"], v["z2"], v["z3"]], rtol=0, atol=1e-15)


def test_rope_position_zero_is_identity_and_pair_norms_are_kept():
    g = torch.Generator().manual_seed(5)
    x = torch.randn(5, 3, 8, generator=g).to(torch.bfloat16)
    pos = [0, 1, 7, 1000, 65535]
    y = oracle.rope(x, pos)
    xf = oracle.bf16_bits_to_f64(x).reshape(5, 3, 8)
    assert np.array_equal(y[0], xf[0])
    n_in = xf[..., 0::2] ** 2 + xf[..., 1::2] ** 2
    n_out = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(n_out, n_in, rtol=1e-12, atol=0)


@pytest.mark.parametrize("d_r", [8, 64])
def test_rope_scores_depend_only_on_relative_position(d_r):
    """<R_p x, R_q z> = <R_(p+s) x, R_(q+s) z>: the defining property of a
    rotary embedding (rotations compose by adding angles)."""
    g = torch.Generator().manual_seed(6)
    x = torch.randn(1, 1, d_r, generator=g).to(torch.bfloat16).expand(4, 1, d_r).contiguous()
    z = torch.randn(1, 1, d_r, generator=g).to(torch.bfloat16).expand(4, 1, d_r).contiguous()
    p, q = 17, 5
    for s in (1, 250, 40000):
        rx = oracle.rope(x[:2], [p, p + s])
        rz = oracle.rope(z[:2], [q, q + s])
        d0 = float(np.dot(rx[0, 0], rz[0, 0]))
        d1 = float(np.dot(rx[1, 0], rz[1, 0]))
        assert abs(d0 - d1) <= 1e-9 * max(1.0, abs(d0))
    # and it is not symmetric in p and q: the angle has a direction
    ra, rb = oracle.rope(x[:2], [p, q]), oracle.rope(z[:2], [q, p])
    assert abs(float(np.dot(ra[0, 0], rb[0, 0])) - float(np.dot(ra[1, 0], rb[1, 0]))) > 1e-6


# ---------------------------------------------------------------------------
# decompress branch (prefill): K_nope / V decompression and causal M x L
# ---------------------------------------------------------------------------

def test_decompress_kv_orientation_and_brute_force():
    rng = np.random.default_rng(5)
    w = workload("ragged", batch=2, heads=3, d_nope=48, d_latent=64, d_v=40, ragged=(70, 130))
    inp = make_inputs(w, seed=6)
    W, perms = _onehot_weights(w.heads, w.d_nope, w.d_latent, rng)
    Wv, permv = _onehot_weights(w.heads, w.d_v, w.d_latent, rng)
    wuv = _bf16(np.transpose(Wv, (0, 2, 1)))                 # [H, d_c, d_v]: V[t][e] = c[perm(e)]
    kn, v = oracle.decompress_kv(inp["ckv_pool"], inp["block_table"], inp["seq_lens"], _bf16(W),
                                 wuv)
    for b, (c, _) in enumerate(_dense_cache(inp)):
        L = c.shape[0]
        for h in range(w.heads):
            np.testing.assert_array_equal(kn[b, h, :L], c[:, perms[h]])
            np.testing.assert_array_equal(v[b, h, :L], c[:, permv[h]])
        assert not kn[b, :, L:].any() and not v[b, :, L:].any()
    kn, v = oracle.decompress_kv(inp["ckv_pool"], inp["block_table"], inp["seq_lens"],
                                 inp["w_uk"], inp["w_uv"])
    for b, (c, _) in enumerate(_dense_cache(inp)):
        L = c.shape[0]
        np.testing.assert_allclose(kn[b, :, :L], np.einsum("sc,hdc->hsd", c, _f64(inp["w_uk"])),
                                   rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(v[b, :, :L], np.einsum("sc,hce->hse", c, _f64(inp["w_uv"])),
                                   rtol=1e-12, atol=1e-12)


def _prefill_args(inp):
    return [inp[k] for k in ("q_c", "q_r", "ckv_pool", "kr_pool", "block_table", "seq_lens",
                             "w_uk", "w_uv")]


@pytest.mark.parametrize("M,lens", [(5, (70, 131)), (64, (64, 100)), (130, (130, 130))])
def test_prefill_matches_definition_and_brute_force(M, lens):
    # the decompress-once restatement against the per-output definition (itself pinned
    # above) and against numpy brute force with scipy's softmax / logsumexp
    w = workload("dsv3", batch=2, n_q=M, heads=3, d_nope=32, d_latent=64, d_rope=16, d_v=24)
    inp = make_inputs(w, seed=M, seq_lens=lens)
    out, lse = oracle.prefill_decompress(*_prefill_args(inp))
    dec = oracle.decode_decompress(*_prefill_args(inp))
    np.testing.assert_allclose(out, dec, rtol=1e-12, atol=1e-14)
    scale = oracle.default_scale(w.d_nope, w.d_rope)
    np.testing.assert_allclose(out, _numpy_reference(inp, scale), rtol=1e-10, atol=1e-12)
    qc, qr = _f64(inp["q_c"]), _f64(inp["q_r"])
    for b, (c, r) in enumerate(_dense_cache(inp)):
        L = c.shape[0]
        k_nope = np.einsum("sc,hdc->shd", c, _f64(inp["w_uk"]))
        for i in (0, M // 2, M - 1):
            vis = L - M + i + 1
            s = (np.einsum("hd,shd->hs", qc[b, i], k_nope[:vis])
                 + np.einsum("hj,sj->hs", qr[b, i], r[:vis])) * scale
            np.testing.assert_allclose(lse[b, i], scipy.special.logsumexp(s, axis=-1),
                                       rtol=1e-12, atol=1e-12)


def test_prefill_full_prompt_first_query_returns_first_value():
    # M = L: query 0 sees token 0 only, so out = c_KV[0] W_UV[h] and lse = its score
    w = workload("dsv3", batch=2, n_q=70, heads=3, d_nope=32, d_latent=64, d_rope=16, d_v=24)
    inp = make_inputs(w, seed=3, seq_lens=(70, 70))
    out, lse = oracle.prefill_decompress(*_prefill_args(inp))
    scale = oracle.default_scale(w.d_nope, w.d_rope)
    wuk, wuv = _f64(inp["w_uk"]), _f64(inp["w_uv"])
    qc, qr = _f64(inp["q_c"]), _f64(inp["q_r"])
    for b, (c, r) in enumerate(_dense_cache(inp)):
        np.testing.assert_allclose(out[b, 0], np.einsum("c,hce->he", c[0], wuv), rtol=1e-12,
                                   atol=1e-14)
        s0 = (np.einsum("hd,hdc,c->h", qc[b, 0], wuk, c[0]) + qr[b, 0] @ r[0]) * scale
        np.testing.assert_allclose(lse[b, 0], s0, rtol=1e-12, atol=1e-13)


def test_prefill_zero_query_gives_prefix_means_and_log_counts():
    w = workload("dsv3", batch=1, n_q=40, heads=2, d_nope=32, d_latent=64, d_rope=16, d_v=24)
    inp = make_inputs(w, seed=4, seq_lens=(100,))
    inp["q_c"] = torch.zeros_like(inp["q_c"])
    inp["q_r"] = torch.zeros_like(inp["q_r"])
    out, lse = oracle.prefill_decompress(*_prefill_args(inp))
    (c, _), = _dense_cache(inp)
    v = np.einsum("sc,hce->she", c, _f64(inp["w_uv"]))
    for i in range(40):
        vis = 100 - 40 + i + 1
        np.testing.assert_allclose(out[0, i], v[:vis].mean(axis=0), rtol=1e-12, atol=1e-14)
        assert lse[0, i, 0] == math.log(vis) and lse[0, i, 1] == math.log(vis)


def test_prefill_is_causal():
    # changing the cache at positions > p leaves every query at position <= p unchanged,
    # and changes the later ones
    w = workload("dsv3", batch=1, n_q=50, heads=2, d_nope=32, d_latent=64, d_rope=16, d_v=24)
    inp = make_inputs(w, seed=8, seq_lens=(120,))
    out, lse = oracle.prefill_decompress(*_prefill_args(inp))
    p = 95                                       # query index p - (120 - 50) = 25
    table = inp["block_table"][0]
    ckv, kr = inp["ckv_pool"].clone(), inp["kr_pool"].clone()
    for t in range(p + 1, 120):
        ckv[table[t // 64], t % 64] = -ckv[table[t // 64], t % 64]
        kr[table[t // 64], t % 64] = 2 * kr[table[t // 64], t % 64]
    pert = dict(inp, ckv_pool=ckv, kr_pool=kr)
    out2, lse2 = oracle.prefill_decompress(*_prefill_args(pert))
    i = p - (120 - 50)
    np.testing.assert_array_equal(out2[0, :i + 1], out[0, :i + 1])
    np.testing.assert_array_equal(lse2[0, :i + 1], lse[0, :i + 1])
    assert np.abs(out2[0, i + 1:] - out[0, i + 1:]).min(axis=-1).max() > 0


def test_prefill_sampled_selection_matches_full():
    w = workload("dsv3", batch=2, n_q=20, heads=3, d_nope=32, d_latent=64, d_rope=16, d_v=24)
    inp = make_inputs(w, seed=9, seq_lens=(33, 90))
    out, lse = oracle.prefill_decompress(*_prefill_args(inp))
    sel = [0, 7, 59, 61, 100, 119]
    o2, l2 = oracle.prefill_decompress(*_prefill_args(inp), sel=sel)
    flat_o, flat_l = out.reshape(-1, w.d_v), lse.reshape(-1)
    np.testing.assert_array_equal(o2.reshape(-1, w.d_v)[sel], flat_o[sel])
    np.testing.assert_array_equal(l2.reshape(-1)[sel], flat_l[sel])
    rest = np.setdiff1d(np.arange(flat_l.size), sel)
    assert not o2.reshape(-1, w.d_v)[rest].any() and np.isnan(l2.reshape(-1)[rest]).all()


# ---------------------------------------------------------------------------
# low-precision latent cache: E4M3 codes (OCP 8-bit float) with a per-row scale
# ---------------------------------------------------------------------------

def test_e4m3_values_match_the_format_and_a_library_decoder():
    # landmarks of the format: smallest subnormal 2^-9, smallest normal 2^-6, one,
    # largest finite 448, the NaN code, negative zero
    assert oracle.e4m3_value(0x00) == 0.0 and oracle.e4m3_value(0x01) == 2.0 ** -9
    assert oracle.e4m3_value(0x07) == 7 * 2.0 ** -9 and oracle.e4m3_value(0x08) == 2.0 ** -6
    assert oracle.e4m3_value(0x38) == 1.0 and oracle.e4m3_value(0x7E) == 448.0
    assert math.isnan(oracle.e4m3_value(0x7F)) and math.isnan(oracle.e4m3_value(0xFF))
    assert math.copysign(1.0, oracle.e4m3_value(0x80)) == -1.0
    assert oracle.e4m3_value(0xB8) == -1.0
    # all 256 codes against torch's float8_e4m3fn decoder
    lib = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    lib = lib.float().double().numpy()
    ours = np.array([oracle.e4m3_value(c) for c in range(256)])
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(lib))
    np.testing.assert_array_equal(ours[~np.isnan(ours)], lib[~np.isnan(lib)])


def test_e4m3_encode_rounds_to_nearest_even_and_saturates():
    finite = [c for c in range(256) if c not in (0x7F, 0xFF)]
    for c in finite:                                  # every code is a fixed point
        assert oracle.e4m3_encode(oracle.e4m3_value(c)) == c
    pos = sorted(oracle.e4m3_value(c) for c in range(0x7F))
    for lo, hi in zip(pos, pos[1:]):                  # midpoints go to the even mantissa
        mid = (lo + hi) / 2
        got = oracle.e4m3_value(oracle.e4m3_encode(mid))
        even = lo if (oracle.e4m3_encode(lo) & 1) == 0 else hi
        assert got == even, (lo, hi, got)
    assert oracle.e4m3_encode(1e6) == 0x7E and oracle.e4m3_encode(-500.0) == 0xFE
    for big in (448.0, 455.0, 464.0, 470.0, 479.9):   # beyond the last code: clamp, never NaN
        assert oracle.e4m3_encode(big) == 0x7E and oracle.e4m3_encode(-big) == 0xFE
    assert oracle.e4m3_encode(2.0 ** -11) == 0x00 and oracle.e4m3_encode(-0.0) == 0x80
    # random fp32 values of every magnitude against torch's conversion (which saturates
    # only up to 464; beyond it returns NaN, where ours clamps to 448)
    rng = np.random.default_rng(3)
    y = (rng.standard_normal(20000) * np.exp2(rng.uniform(-12, 9, 20000))).astype(np.float32)
    y = y[np.abs(y) < 464]
    lib = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.e4m3_encode(v) for v in y], dtype=np.uint8)
    np.testing.assert_array_equal(ours, lib)


def test_fp8_row_quantisation_bounds_and_special_rows():
    rng = np.random.default_rng(4)
    x = _bf16(rng.standard_normal((40, 512)) * np.exp2(rng.uniform(-8, 8, (40, 1))))
    x[3] = 0.0                                         # an all-zero row
    codes, scales = oracle.quantize_fp8_rows(x)
    xd = _f64(x)
    amax = np.abs(xd).max(axis=1)
    for r in range(40):
        if amax[r] == 0:
            assert scales[r] == 1.0 and not codes[r].any()
            continue
        assert scales[r] == np.float32(np.float32(amax[r]) / np.float32(448.0))
        # the largest magnitude lands on +-448 and every element within half a code step
        j = int(np.argmax(np.abs(xd[r])))
        assert codes[r, j] & 0x7F == 0x7E
        vals = np.array([oracle.e4m3_value(c) for c in codes[r]])
        y = xd[r] * (np.float32(448.0) / np.float32(amax[r]))
        step = np.exp2(np.maximum(np.floor(np.log2(np.maximum(np.abs(y), 2.0 ** -6))), -6) - 3)
        assert (np.abs(vals - y) <= step / 2 * (1 + 1e-6)).all()
    deq = oracle.dequant_fp8_rows(codes, scales)
    back = _f64(oracle.bf16_from_bits(deq))
    live = amax > 0
    assert not back[~live].any()
    rel = np.abs(back - xd)[live] / np.maximum(np.abs(xd), amax[:, None] * 2.0 ** -6)[live]
    assert rel.max() <= 2.0 ** -4 + 2.0 ** -8      # E4M3 half-step plus the bf16 rounding


def test_fp8_dequant_with_power_of_two_scale_is_exact():
    codes = np.arange(256, dtype=np.uint8).reshape(4, 64)
    codes[codes == 0x7F] = 0x7E
    codes[codes == 0xFF] = 0xFE
    scales = np.array([1.0, 0.5, 2.0 ** -7, 16.0], dtype=np.float32)
    got = _f64(oracle.bf16_from_bits(oracle.dequant_fp8_rows(codes, scales)))
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy() * scales[:, None]
    np.testing.assert_array_equal(got, lib)
    # any scale: the fp32 product rounded to bf16 to nearest even, as torch's conversions do
    rng = np.random.default_rng(6)
    scales = (rng.uniform(0.5, 2.0, 4) * np.exp2(rng.integers(-20, 4, 4))).astype(np.float32)
    got = oracle.dequant_fp8_rows(codes, scales)
    prod = torch.from_numpy(codes).view(torch.float8_e4m3fn).float() * torch.from_numpy(scales)[:, None]
    lib = prod.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, lib)
