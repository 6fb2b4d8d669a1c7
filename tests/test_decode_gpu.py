"""Parity of the CUDA path (through the C ABI) against the fp64 oracle.

Bar (per step and end to end, on bf16 outputs against fp64): max |err| <= 1e-2
and relative L2 error <= 5e-3. Integer/index work (the RoPE copy, the page
gather) is checked bit for bit, through bitwise invariance of the outputs.
Every workload, full-size ones included, is checked on every (batch, query,
head) row against the fp64 absorbed path (itself pinned to the definition), and
on at least eight rows against the definition (decompress K and V per head).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_18_b200.inputs import make_inputs, to_device, workload

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2 = 1e-2, 5e-3


@pytest.fixture(scope="module")
def api():
    from mla_latent_kv_18_b200 import api as _api
    assert torch.cuda.is_available()
    return _api


def _f64(t):
    return t.detach().float().cpu().double().numpy()


def _check(got, ref, what, max_abs=MAX_ABS, rel_l2=REL_L2):
    got, ref = np.asarray(got, dtype=np.float64), np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), what
    err = np.abs(got - ref).max()
    rel = np.linalg.norm((got - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-30)
    assert err <= max_abs and rel <= rel_l2, f"{what}: max abs {err:.3e}, rel L2 {rel:.3e}"
    return err, rel


# Unit of the fp32 accumulation error model for tensor-core sums of exact bf16
# products: 2^-22 (four times the fp32 unit roundoff, so truncating adders fit).
ACC_UNIT = 2.0 ** -22


def acc_bound(x, w, k_len):
    """Worst-case fp32 accumulation error of out[..., h, c] = sum_k x[..., h, k] w[h, k, c]:
    k_len * ACC_UNIT * sum_k |x w| (the standard gamma_K bound)."""
    ax = np.abs(np.asarray(x.float().cpu().double().numpy()))
    aw = np.abs(np.asarray(w.float().cpu().double().numpy()))
    return k_len * ACC_UNIT * np.einsum("...hk,hkc->...hc", ax, aw)


def _check_rounded(got, ref, what, acc=0.0):
    """A bf16 result rounded (to nearest even) from an fp32 value: every element within half a
    bf16 ulp (2^-8 |x|) of the fp32 value x, which is within `acc` (the accumulation error
    bound) of the fp64 value; plus the output bar on relative L2."""
    got, ref = np.asarray(got, dtype=np.float64), np.asarray(ref, dtype=np.float64)
    assert np.isfinite(got).all(), what
    bound = 2.0 ** -8 * (np.abs(ref) + acc) + acc + 1e-30
    worst = (np.abs(got - ref) / bound).max()
    rel = np.linalg.norm((got - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-30)
    assert worst <= 1.0 and rel <= REL_L2, f"{what}: worst err/bound {worst:.3f}, rel L2 {rel:.3e}"


def _check_one_ulp(a, b, what):
    """Two bf16 results rounded from fp32 sums that differ only in summation order: adjacent
    or equal bf16 values, |a - b| <= 2^-7 max(|a|, |b|) (one ulp), with a 1e-6 floor for sums
    that cancel to near zero."""
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    assert np.isfinite(a).all() and np.isfinite(b).all(), what
    bound = 2.0 ** -7 * np.maximum(np.abs(a), np.abs(b)) + 1e-6
    worst = (np.abs(a - b) / bound).max()
    assert worst <= 1.0, f"{what}: worst diff/ulp {worst:.3f}"


def _check_out(got, ref, what):
    """Output bar for large-magnitude outputs: |err| <= 1e-2 + 2^-7 |ref| and rel L2 <= 5e-3."""
    got, ref = np.asarray(got, dtype=np.float64), np.asarray(ref, dtype=np.float64)
    assert np.isfinite(got).all(), what
    worst = (np.abs(got - ref) / (MAX_ABS + 2.0 ** -7 * np.abs(ref))).max()
    rel = np.linalg.norm((got - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-30)
    assert worst <= 1.0 and rel <= REL_L2, f"{what}: worst err/bound {worst:.3f}, rel L2 {rel:.3e}"


def _run(api, inp_d, num_parts=None):
    dims = api.dims_for(inp_d["q_c"], inp_d["q_r"], inp_d["w_uk"], inp_d["w_uv"])
    T = api.tile_tokens(dims)
    lens = inp_d["seq_lens"].cpu()
    total = int(((lens.long() + T - 1) // T).sum())
    if num_parts is None:
        num_parts = api.num_parts_for(dims, total, inp_d["q_c"].device)
    q = api.absorb_q(inp_d["q_c"], inp_d["q_r"], inp_d["w_uk"], dims)
    ws = api.decode_splitkv(q, inp_d["ckv_pool"], inp_d["kr_pool"], inp_d["block_table"],
                            inp_d["seq_lens"], dims, num_parts)
    o_lat, lse = api.combine(ws, inp_d["seq_lens"], inp_d["block_table"].shape[1], dims, num_parts)
    out = api.absorb_out(o_lat, inp_d["w_uv"], dims)
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    return dict(dims=dims, q=q, ws=ws, o_lat=o_lat, lse=lse, out=out, num_parts=num_parts)


def _sample_rows(w, n, seed=0):
    total = w.batch * w.n_q * w.heads
    if n >= total:
        return np.arange(total)
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(total, size=n, replace=False))


def _parity(api, w, n_def_rows, seed=0, inp=None):
    """Every (b, i, h) row of every step against the fp64 oracle, and n_def_rows rows
    (at least 8) end to end against the definition."""
    inp = make_inputs(w, seed=seed) if inp is None else inp
    inp_d = to_device(inp, "cuda")
    r = _run(api, inp_d)
    scale = oracle.default_scale(w.d_nope, w.d_rope)
    D = w.d_latent
    # absorb-in: latent part vs fp64 within half an ulp plus the accumulation bound,
    # RoPE part a bit-exact copy
    q_ref = oracle.absorb_q(inp["q_c"], inp["w_uk"])
    _check_rounded(_f64(r["q"][..., :D]), q_ref, "absorb_q",
                   acc_bound(inp["q_c"], inp["w_uk"], w.d_nope))
    assert torch.equal(r["q"][..., D:].cpu(), inp["q_r"])
    # split-KV + combine on the GPU's own bf16 Q, every row
    o_ref, lse_ref = oracle.attend_latent(r["q"].cpu(), inp["ckv_pool"], inp["kr_pool"],
                                          inp["block_table"], inp["seq_lens"], scale)
    _check(_f64(r["o_lat"]), o_ref, "o_lat")
    assert np.abs(_f64(r["lse"]) - lse_ref).max() <= 1e-3
    # absorb-out on the GPU's own o_lat, every row
    out_ref = oracle.absorb_out(r["o_lat"].cpu(), inp["w_uv"])
    _check(_f64(r["out"]), out_ref, "absorb_out")
    # end to end against the fp64 absorbed path (pinned to the definition), every row ...
    args = [inp[k] for k in ("q_c", "q_r", "ckv_pool", "kr_pool", "block_table", "seq_lens",
                             "w_uk", "w_uv")]
    ab, _, _ = oracle.decode_absorbed(*args)
    _check(_f64(r["out"]), ab, "out vs absorbed")
    # ... and against the definition itself on sampled rows
    sel_def = _sample_rows(w, max(8, n_def_rows), seed + 1)
    dec = oracle.decode_decompress(*args, sel=sel_def)
    _check(_f64(r["out"]).reshape(-1, w.d_v)[sel_def], dec.reshape(-1, w.d_v)[sel_def],
           "out vs decompress")
    return r, inp


def test_parity_tiny(api):
    _parity(api, workload("tiny"), 16)


def test_parity_dsv3(api):
    _parity(api, workload("dsv3"), 16)


def test_parity_ragged(api):
    r, inp = _parity(api, workload("ragged"), 8)
    # the fused combine + absorb-out at 64 tokens (a grid of more than one wave: 32
    # tokens per CTA) on the same full-size partials
    d = to_device(inp, "cuda")
    lse = torch.empty_like(r["lse"])
    fused = api.combine_absorb_out(r["ws"], d["seq_lens"], d["block_table"].shape[1], r["dims"],
                                   r["num_parts"], d["w_uv"], lse_out=lse)
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    assert torch.equal(lse, r["lse"])
    _check_one_ulp(_f64(fused), _f64(r["out"]), "ragged: fused vs unfused")


def test_parity_retrofit(api):
    _parity(api, workload("retrofit"), 16)


@pytest.mark.parametrize("heads", [40, 64])
def test_parity_retrofit_more_than_64_rows(api, heads):
    # n_q * heads = 80 and 128 query rows: one TMEM lane per row (at most 64 rows
    # put each row on two lanes that split the tile's tokens)
    _parity(api, workload("retrofit", batch=3, heads=heads, seq_len=700), 8)


def test_parity_long_context(api):
    r, inp = _parity(api, workload("long"), 8)
    # the fused combine + absorb-out on the same full-size partials (the bench's step)
    d = to_device(inp, "cuda")
    lse = torch.empty_like(r["lse"])
    fused = api.combine_absorb_out(r["ws"], d["seq_lens"], d["block_table"].shape[1], r["dims"],
                                   r["num_parts"], d["w_uv"], lse_out=lse)
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    assert torch.equal(lse, r["lse"])
    _check_one_ulp(_f64(fused), _f64(r["out"]), "long: fused vs unfused")


@pytest.mark.parametrize("name,parts", [("dsv3", 7), ("dsv3", 1), ("retrofit", 5), ("ragged", 13)])
def test_partials_match_oracle_windows(api, name, parts):
    w = workload(name, batch=3, heads=8 if name != "retrofit" else 32,
                 **({"seq_len": 1000} if name != "ragged" else {"ragged": (100, 2000)}))
    inp = make_inputs(w, seed=3)
    r = _run(api, to_device(inp, "cuda"), num_parts=parts)
    dims = r["dims"]
    T = api.tile_tokens(dims)
    lens = inp["seq_lens"].tolist()
    pf, cnt, base, total = api.plan(dims, lens, inp["block_table"].shape[1], parts)
    o_part, lse_part = api.workspace_views(r["ws"], dims, w.batch, parts)
    o_part, lse_part = _f64(o_part), _f64(lse_part)
    n_tiles = [(L + T - 1) // T for L in lens]
    N = sum(n_tiles)
    P = min(parts, N)
    # the plan's cost positions: tiles end to end, SWITCH_COST[T] virtual positions
    # between consecutive non-empty sequences; partition p owns [p C / P, (p+1) C / P)
    W = {64: 8, 128: 3}[T]
    C = N + W * (sum(1 for n in n_tiles if n) - 1)
    scale = oracle.default_scale(w.d_nope, w.d_rope)
    off = 0
    for b in range(w.batch):
        one = {k: (v[b:b + 1] if k not in ("ckv_pool", "kr_pool", "w_uk", "w_uv") else v)
               for k, v in inp.items()}
        for j in range(int(cnt[b])):
            p = int(pf[b]) + j
            t0 = max(p * C // P, off) - off
            t1 = min((p + 1) * C // P, off + n_tiles[b]) - off
            o_ref, lse_ref = oracle.attend_latent(r["q"][b:b + 1].cpu(), one["ckv_pool"],
                                                  one["kr_pool"], one["block_table"],
                                                  one["seq_lens"], scale, t_lo=t0 * T,
                                                  t_hi=t1 * T)
            slot = int(base[b]) + j
            _check(o_part[slot].reshape(1, w.n_q, w.heads, -1), o_ref, f"slot {slot}")
            np.testing.assert_allclose(lse_part[slot].reshape(lse_ref.shape), lse_ref, atol=1e-3)
        off += n_tiles[b] + (W if n_tiles[b] else 0)


@pytest.mark.parametrize("name,parts", [("dsv3", None), ("dsv3", 1), ("dsv3", 74),
                                        ("retrofit", None), ("retrofit", 148)])
def test_edge_lengths(api, name, parts):
    # lengths must be >= n_q (1 for dsv3, 2 for the causal pair of retrofit)
    lens = [1, 2, 63, 64, 65, 127, 128, 129, 200, 3] if name == "dsv3" else \
        [2, 3, 63, 64, 65, 127, 128, 129, 200, 2]
    w = workload(name, batch=len(lens), heads=16 if name == "dsv3" else 32, seq_len=256)
    inp = make_inputs(w, seed=5, seq_lens=lens)
    r = _run(api, to_device(inp, "cuda"), num_parts=parts)
    args = [inp[k] for k in ("q_c", "q_r", "ckv_pool", "kr_pool", "block_table", "seq_lens",
                             "w_uk", "w_uv")]
    ab, o_lat, lse = oracle.decode_absorbed(*args)
    # short sequences average few values, so outputs reach |x| ~ 4 where the bf16
    # rounding of the output alone exceeds 1e-2: bound each element by 1e-2 plus
    # one bf16 ulp of its value
    _check_out(_f64(r["out"]), ab, "out")
    scale = oracle.default_scale(w.d_nope, w.d_rope)
    o_ref, lse_ref = oracle.attend_latent(r["q"].cpu(), inp["ckv_pool"], inp["kr_pool"],
                                          inp["block_table"], inp["seq_lens"], scale)
    _check(_f64(r["o_lat"]), o_ref, "o_lat")


@pytest.mark.parametrize("name,lens,parts", [
    ("dsv3", [1, 63, 65, 100, 127, 129, 200, 257, 64], None),
    ("dsv3", [1, 63, 65, 100, 127, 129, 200, 257, 64], 3),
    ("retrofit", [2, 63, 65, 127, 129, 200, 255, 300, 128], None),
    ("retrofit", [2, 63, 65, 127, 129, 200, 255, 300, 128], 4),
])
def test_nonfinite_page_tails_do_not_leak(api, name, lens, parts):
    """Rows past a sequence's end in its last page hold NaN / +-Inf (an unwritten
    or recycled page slot): every output row still matches the oracle, which
    never reads them."""
    from tail_poison import poison_page_tails
    w = workload(name, batch=len(lens), heads=16 if name == "dsv3" else 32, seq_len=320)
    inp = poison_page_tails(make_inputs(w, seed=19, seq_lens=lens))
    assert not torch.isfinite(inp["ckv_pool"].float()).all()
    r = _run(api, to_device(inp, "cuda"), num_parts=parts)
    args = [inp[k] for k in ("q_c", "q_r", "ckv_pool", "kr_pool", "block_table", "seq_lens",
                             "w_uk", "w_uv")]
    ab, _, _ = oracle.decode_absorbed(*args)
    _check_out(_f64(r["out"]), ab, "out with non-finite page tails")
    scale = oracle.default_scale(w.d_nope, w.d_rope)
    o_ref, lse_ref = oracle.attend_latent(r["q"].cpu(), inp["ckv_pool"], inp["kr_pool"],
                                          inp["block_table"], inp["seq_lens"], scale)
    _check(_f64(r["o_lat"]), o_ref, "o_lat with non-finite page tails")
    assert np.abs(_f64(r["lse"]) - lse_ref).max() <= 1e-3
    # the same cache with finite tails gives bitwise the same results
    clean = _run(api, to_device(make_inputs(w, seed=19, seq_lens=lens), "cuda"), num_parts=parts)
    assert torch.equal(clean["out"], r["out"]) and torch.equal(clean["lse"], r["lse"])


def test_single_token_is_its_value(api):
    w = workload("dsv3", batch=4, heads=32, seq_len=1)
    inp = make_inputs(w, seed=6)
    r = _run(api, to_device(inp, "cuda"))
    # softmax over one token: o_lat is that token's latent (bf16, exact)
    for b in range(w.batch):
        c0 = inp["ckv_pool"][int(inp["block_table"][b, 0]), 0]
        assert torch.equal(r["o_lat"][b, 0].cpu(), c0.expand(w.heads, -1))


def test_page_table_permutation_is_bitwise_invariant(api):
    w = workload("dsv3", batch=4, heads=32, seq_len=777)
    inp = make_inputs(w, seed=7)
    r1 = _run(api, to_device(inp, "cuda"))
    n = inp["ckv_pool"].shape[0]
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(1))
    inp2 = dict(inp)
    inp2["ckv_pool"] = torch.empty_like(inp["ckv_pool"])
    inp2["kr_pool"] = torch.empty_like(inp["kr_pool"])
    inp2["ckv_pool"][perm] = inp["ckv_pool"]
    inp2["kr_pool"][perm] = inp["kr_pool"]
    t = inp["block_table"].clone()
    t[t >= 0] = perm[t[t >= 0].long()].to(torch.int32)
    inp2["block_table"] = t
    r2 = _run(api, to_device(inp2, "cuda"))
    assert torch.equal(r1["out"], r2["out"]) and torch.equal(r1["lse"], r2["lse"])


def test_interleaved_pool_matches_separate_pools(api):
    w = workload("dsv3", batch=3, heads=16, seq_len=300)
    inp = make_inputs(w, seed=8)
    r1 = _run(api, to_device(inp, "cuda"))
    both = torch.cat([inp["ckv_pool"], inp["kr_pool"]], dim=-1).cuda()   # [pages, 64, 576]
    inp_d = to_device(inp, "cuda")
    inp_d["ckv_pool"] = both[..., :512]
    inp_d["kr_pool"] = both[..., 512:]
    r2 = _run(api, inp_d)
    assert torch.equal(r1["out"], r2["out"])


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("dsv3", dict(batch=3, heads=16, seq_len=300)),
                                     ("ragged", dict(batch=6, heads=16, ragged=(1, 700))),
                                     ("retrofit", dict(batch=3, seq_len=250))])
def test_gather_is_bit_exact(api, name, kw):
    """The decode calls' page lookup, written out densely through the same TMA
    pool descriptors, equals the oracle's gather bit for bit: both pools,
    every visible token, nothing written past a sequence's length."""
    w = workload(name, **kw)
    inp = make_inputs(w, seed=12)
    d = to_device(inp, "cuda")
    max_len = int(inp["seq_lens"].max()) + 5
    for pool_name in ("ckv_pool", "kr_pool"):
        got = api.debug_gather(d[pool_name], d["block_table"], d["seq_lens"], max_len)
        assert api.get_device_error() == 0
        ref = oracle.gather(inp[pool_name], inp["block_table"], inp["seq_lens"], 64, max_len)
        assert np.array_equal(got.cpu().view(torch.int16).numpy().view(np.uint16), ref), pool_name


def test_gather_from_interleaved_pool_is_bit_exact(api):
    w = workload("dsv3", batch=3, heads=16, seq_len=300)
    inp = make_inputs(w, seed=13)
    both = torch.cat([inp["ckv_pool"], inp["kr_pool"]], dim=-1).cuda()   # [pages, 64, 576]
    bt, sl = inp["block_table"].cuda(), inp["seq_lens"].cuda()
    for view, pool_name in ((both[..., :512], "ckv_pool"), (both[..., 512:], "kr_pool")):
        got = api.debug_gather(view, bt, sl, 300)
        ref = oracle.gather(inp[pool_name], inp["block_table"], inp["seq_lens"], 64, 300)
        assert np.array_equal(got.cpu().view(torch.int16).numpy().view(np.uint16), ref), pool_name
    assert api.get_device_error() == 0


def test_gather_bad_page_id_sets_device_error(api):
    w = workload("dsv3", batch=2, heads=16, seq_len=300)
    inp = make_inputs(w, seed=14)
    d = to_device(inp, "cuda")
    d["block_table"][1, 3] = -7
    api.debug_gather(d["ckv_pool"], d["block_table"], d["seq_lens"], 300)
    assert api.get_device_error() == 4
    assert api.get_device_error() == 0


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("dsv3", dict(batch=4, seq_len=3000)),
                                     ("dsv3", dict(batch=80, heads=16, seq_len=200)),
                                     ("dsv3", dict(batch=48, heads=128, seq_len=300)),   # 32 tokens per CTA, ragged tail
                                     ("ragged", dict(batch=6, heads=128, ragged=(64, 4000))),
                                     ("retrofit", dict(batch=9, seq_len=700))])
def test_fused_combine_absorb_out(api, name, kw):
    """mla_combine_absorb_out against the oracle's absorb-out of the GPU's own
    merged rows (the same definition, composed) and end to end against the fp64
    absorbed path; its lse equals mla_combine's bit for bit, its output stays
    within one bf16 rounding of mla_combine + mla_absorb_out, and a repeat call
    is bitwise identical."""
    w = workload(name, **kw)
    inp = make_inputs(w, seed=15)
    d = to_device(inp, "cuda")
    r = _run(api, d)
    dims, ws, P = r["dims"], r["ws"], r["num_parts"]
    lse = torch.empty_like(r["lse"])
    out = api.combine_absorb_out(ws, d["seq_lens"], d["block_table"].shape[1], dims, P, d["w_uv"],
                                 lse_out=lse)
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    assert torch.equal(lse, r["lse"])
    out_ref = oracle.absorb_out(r["o_lat"].cpu(), inp["w_uv"])   # fp64 over the same bf16 o_lat
    _check(_f64(out), out_ref, "fused out vs oracle absorb-out")
    _check_one_ulp(_f64(out), _f64(r["out"]), "fused vs unfused")
    args = [inp[k] for k in ("q_c", "q_r", "ckv_pool", "kr_pool", "block_table", "seq_lens",
                             "w_uk", "w_uv")]
    sel = _sample_rows(w, 256, 15)
    ab, _, _ = oracle.decode_absorbed(*args, sel=sel)
    _check(_f64(out).reshape(-1, w.d_v)[sel], ab.reshape(-1, w.d_v)[sel], "fused out vs absorbed")
    again = api.combine_absorb_out(ws, d["seq_lens"], d["block_table"].shape[1], dims, P, d["w_uv"])
    assert torch.equal(again, out)


@pytest.mark.parametrize("name,kw", [("dsv3", dict(batch=3, heads=16, seq_len=300)),
                                     ("retrofit", dict(batch=4, seq_len=900))])
def test_absorb_q_with_rotary_embedding(api, name, kw):
    """mla_absorb_q_rope: the latent part equals mla_absorb_q's bit for bit, the
    RoPE part is the oracle's fp64 rotation within half a bf16 ulp plus the fp32
    rotation's error (large positions included), and position 0 leaves q_r unchanged bit for bit."""
    w = workload(name, **kw)
    inp = make_inputs(w, seed=16)
    d = to_device(inp, "cuda")
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    T = w.batch * w.n_q
    pos = torch.tensor([int(L) - w.n_q + i for L in inp["seq_lens"] for i in range(w.n_q)],
                       dtype=torch.int32)
    pos[: min(4, T)] = torch.tensor([0, 1, 65535, 1_000_003][: min(4, T)], dtype=torch.int32)
    q = api.absorb_q_rope(d["q_c"], d["q_r"], d["w_uk"], dims, pos.cuda())
    q0 = api.absorb_q(d["q_c"], d["q_r"], d["w_uk"], dims)
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    D = w.d_latent
    assert torch.equal(q[..., :D], q0[..., :D])
    ref = oracle.rope(inp["q_r"].reshape(T, w.heads, w.d_rope), pos.numpy())
    # fp32 rotation of a pair: cos and sin rounded to fp32, two products and a sum,
    # each within 2^-24 relative; bounded here by 2^-21 (|x0| + |x1|) per element
    xr = np.abs(_f64(inp["q_r"].reshape(T, w.heads, w.d_rope // 2, 2)))
    acc = np.repeat(2.0 ** -21 * xr.sum(-1, keepdims=True), 2, axis=-1).reshape(ref.shape)
    _check_rounded(_f64(q[..., D:]).reshape(ref.shape), ref, "rotated q_r", acc)
    q_zero = api.absorb_q_rope(d["q_c"], d["q_r"], d["w_uk"], dims, torch.zeros_like(pos).cuda())
    assert torch.equal(q_zero[..., D:].cpu(), inp["q_r"])


def test_absorb_q_rope_negative_position_sets_device_error(api):
    w = workload("dsv3", batch=2, heads=16, seq_len=300)
    d = to_device(make_inputs(w, seed=17), "cuda")
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    api.absorb_q_rope(d["q_c"], d["q_r"], d["w_uk"], dims,
                      torch.tensor([5, -3], dtype=torch.int32, device="cuda"))
    assert api.get_device_error() == 4
    assert api.get_device_error() == 0


def test_repeat_calls_are_bitwise_identical(api):
    w = workload("ragged", batch=8, heads=128, ragged=(500, 5000))
    inp_d = to_device(make_inputs(w, seed=9), "cuda")
    a = _run(api, inp_d)
    b = _run(api, inp_d)
    assert torch.equal(a["out"], b["out"]) and torch.equal(a["o_lat"], b["o_lat"])


def test_empty_batch_is_noop(api):
    import ctypes
    from mla_latent_kv_18_b200 import _binding as b
    d = api.make_dims(128, 1, 128, 512, 64, 128)
    pool = b.MLAPool(0, 0, 0)
    null = ctypes.c_void_p(0)
    assert b.lib.mla_decode_splitkv(ctypes.byref(d), null, ctypes.byref(pool), ctypes.byref(pool),
                                    1, null, 1, null, 0, 1, null, 0, null) == 0
    assert b.lib.mla_combine(ctypes.byref(d), null, 0, null, 1, 0, 1, null, null, null) == 0
    assert b.lib.mla_absorb_q(ctypes.byref(d), null, null, null, null, 0, null) == 0


@pytest.mark.parametrize("name", ["dsv3", "retrofit"])
def test_bad_page_id_sets_device_error(api, name):
    w = workload(name, batch=2, heads=16 if name == "dsv3" else 32, seq_len=300)
    inp = make_inputs(w, seed=10)
    inp_d = to_device(inp, "cuda")
    inp_d["block_table"][1, 2] = inp["ckv_pool"].shape[0] + 5
    dims = api.dims_for(inp_d["q_c"], inp_d["q_r"], inp_d["w_uk"], inp_d["w_uv"])
    q = api.absorb_q(inp_d["q_c"], inp_d["q_r"], inp_d["w_uk"], dims)
    ws = api.decode_splitkv(q, inp_d["ckv_pool"], inp_d["kr_pool"], inp_d["block_table"],
                            inp_d["seq_lens"], dims, 2)
    assert api.get_device_error() == 4
    assert api.get_device_error() == 0          # read clears the word
    # the context is intact: a clean call still works
    _run(api, to_device(inp, "cuda"))


def test_seq_len_beyond_table_sets_device_error(api):
    w = workload("dsv3", batch=2, heads=16, seq_len=300)
    inp_d = to_device(make_inputs(w, seed=11), "cuda")
    inp_d["seq_lens"][0] = inp_d["block_table"].shape[1] * 64 + 1
    dims = api.dims_for(inp_d["q_c"], inp_d["q_r"], inp_d["w_uk"], inp_d["w_uv"])
    q = api.absorb_q(inp_d["q_c"], inp_d["q_r"], inp_d["w_uk"], dims)
    api.decode_splitkv(q, inp_d["ckv_pool"], inp_d["kr_pool"], inp_d["block_table"],
                       inp_d["seq_lens"], dims, 2)
    assert api.get_device_error() == 4


def test_bounded_wait_times_out_cleanly(api):
    api.debug_wait_timeout(20_000_000)      # 20 ms on a barrier nothing completes
    assert api.get_device_error() == 5
    assert api.get_device_error() == 0
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0            # context still usable
