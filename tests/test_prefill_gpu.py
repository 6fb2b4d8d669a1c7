"""Parity of the decompress branch (prefill) through the C ABI against the fp64 oracle.

Bars: the decompressed K_nope / V are bf16 roundings of fp32 sums, so each
element must lie within one bf16 ulp (2^-7 relative) of the fp64 value, and
the rows past a sequence's end must be exactly zero. The attention output
meets the output bar of the decode path (max |err| <= 1e-2, relative L2 <=
5e-3 against fp64) on every query that sees at least 64 keys. The first queries
of a prompt see a handful of keys, so their outputs are close to single V rows
(|x| up to ~4) where the bf16 rounding of the output alone exceeds 1e-2; every
row is therefore also bounded element by element by 1e-2 plus one bf16 ulp of
its value (2^-7 |ref|), as the decode path's short sequences are. The
log-sum-exp is compared within 1e-2: the scores are taken against bf16-rounded
K_nope (relative error <= 2^-9 per element), which moves a score of this workload (|q_c . K_nope| ~ 11, scale 1/sqrt(192)) by a few
1e-3 at most. Full-size prefill (batch 8, prompt 4096, 128 heads) is checked on
sampled (sequence, query, head) rows the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_18_b200.inputs import make_inputs, to_device, workload

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2, LSE_ABS = 1e-2, 5e-3, 1e-2


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


def _check_prefill(got, ref, lens, M, what):
    """Strict bar on queries that see >= 64 keys; 1e-2 + 2^-7 |ref| per element on all."""
    got, ref = np.asarray(got, dtype=np.float64), np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape and np.isfinite(got).all(), what
    vis = np.array([[L - M + i + 1 for i in range(M)] for L in lens])        # [B, M]
    many = vis >= 64
    if many.any():
        _check(got[many], ref[many], what + " (rows seeing >= 64 keys)")
    worst = (np.abs(got - ref) / (MAX_ABS + 2.0 ** -7 * np.abs(ref))).max()
    rel = np.linalg.norm((got - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-30)
    assert worst <= 1.0 and rel <= REL_L2, f"{what}: worst err/bound {worst:.3f}, rel L2 {rel:.3e}"


# Unit of the fp32 accumulation error model for tensor-core sums of exact bf16
# products: 2^-22 (four times the fp32 unit roundoff, so truncating adders fit).
ACC_UNIT = 2.0 ** -22


def _check_rounded(got, ref, what, acc):
    """bf16 rounded (to nearest even) from an fp32 sum: within half a bf16 ulp (2^-8 |x|) of
    the fp32 value x, which is within `acc` (the accumulation error bound) of the fp64 value."""
    got, ref = np.asarray(got, dtype=np.float64), np.asarray(ref, dtype=np.float64)
    assert np.isfinite(got).all(), what
    bound = 2.0 ** -8 * (np.abs(ref) + acc) + acc + 1e-30
    worst = (np.abs(got - ref) / bound).max()
    assert worst <= 1.0, f"{what}: worst err/bound {worst:.3f}"


def _decompress_acc(inp, b, L):
    """gamma_K bounds of the fp32 sums K_nope[h, t, d] = sum_c c[t, c] W_UK[h, d, c] and
    V[h, t, e] = sum_c c[t, c] W_UV[h, c, e] over the d_c = 512 channels of sequence b."""
    t = np.arange(L)
    pages = inp["block_table"][b].long().numpy()[t // 64]
    c = np.abs(inp["ckv_pool"].float().double().numpy()[pages, t % 64])       # [L, d_c]
    wuk = np.abs(inp["w_uk"].float().double().numpy())                         # [H, d_n, d_c]
    wuv = np.abs(inp["w_uv"].float().double().numpy())                         # [H, d_c, d_v]
    K = c.shape[1]
    return (K * ACC_UNIT * np.einsum("tc,hdc->htd", c, wuk),
            K * ACC_UNIT * np.einsum("tc,hce->hte", c, wuv))


def _prefill_w(M, lens, heads=4, seed_batch=None):
    return workload("prefill", batch=len(lens), n_q=M, heads=heads, seq_len=0,
                    ragged=(min(lens), max(lens)))


def _args(inp):
    return [inp[k] for k in ("q_c", "q_r", "ckv_pool", "kr_pool", "block_table", "seq_lens",
                             "w_uk", "w_uv")]


@pytest.mark.parametrize("lens,heads", [((300, 130), 16), ((64, 1), 8), ((777, 256, 129), 3)])
def test_decompress_kv_parity(api, lens, heads):
    w = _prefill_w(1, lens, heads)
    inp = make_inputs(w, seed=sum(lens), seq_lens=lens)
    d = to_device(inp, "cuda")
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    B, max_pages = d["block_table"].shape
    ws = api.decompress_kv(d["ckv_pool"], d["block_table"], d["seq_lens"], d["w_uk"], d["w_uv"],
                           dims)
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    k, v = api.prefill_workspace_views(ws, dims, B, max_pages)
    kn_ref, v_ref = oracle.decompress_kv(inp["ckv_pool"], inp["block_table"], inp["seq_lens"],
                                         inp["w_uk"], inp["w_uv"])
    for b, L in enumerate(lens):
        acc_k, acc_v = _decompress_acc(inp, b, L)
        _check_rounded(_f64(k[b, :, :L]), kn_ref[b, :, :L], f"K_nope seq {b}", acc_k)
        _check_rounded(_f64(v[b, :, :L]), v_ref[b, :, :L], f"V seq {b}", acc_v)
        tail = (L + 127) // 128 * 128
        assert not k[b, :, L:tail].any() and not v[b, :, L:tail].any(), "rows past the end"


@pytest.mark.parametrize("M,lens,heads", [
    (200, (200, 333), 4),          # whole prompt for one sequence, a cached prefix for the other
    (256, (700, 1000), 3),         # a 256-token chunk after a cached prefix (the threshold)
    (130, (130, 130), 5),          # ragged query block (130 = 128 + 2), whole prompt
    (1, (65, 1), 4),               # degenerate: one query; a one-token sequence
    (300, (300, 400, 517), 2),     # three sequences, several key blocks, ragged pages
])
def test_prefill_parity(api, M, lens, heads):
    w = _prefill_w(M, lens, heads)
    inp = make_inputs(w, seed=M + len(lens), seq_lens=lens)
    d = to_device(inp, "cuda")
    out, lse = api.prefill(*_args(d))
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    ref, lse_ref = oracle.prefill_decompress(*_args(inp))
    _check_prefill(_f64(out), ref, lens, M, f"prefill M={M} lens={lens}")
    assert np.abs(_f64(lse) - lse_ref).max() <= LSE_ABS


def test_prefill_with_nonfinite_page_tails(api):
    """Rows past a sequence's end in its last page hold NaN / +-Inf: the decompress
    branch's results are bitwise those of the same cache with finite tails, and
    match the oracle, which never reads them."""
    from tail_poison import poison_page_tails
    M, lens = 130, (130, 333, 200)
    w = _prefill_w(M, lens, 3)
    clean = make_inputs(w, seed=23, seq_lens=lens)
    inp = poison_page_tails(clean)
    assert not torch.isfinite(inp["ckv_pool"].float()).all()
    out, lse = api.prefill(*_args(to_device(inp, "cuda")))
    out0, lse0 = api.prefill(*_args(to_device(clean, "cuda")))
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    assert torch.equal(out, out0) and torch.equal(lse, lse0)
    ref, lse_ref = oracle.prefill_decompress(*_args(inp))
    _check_prefill(_f64(out), ref, lens, M, "prefill with non-finite page tails")
    assert np.abs(_f64(lse) - lse_ref).max() <= LSE_ABS


def test_prefill_split_calls_match_fused_call_bitwise(api):
    lens = (333, 200)
    w = _prefill_w(150, lens, 4)
    d = to_device(make_inputs(w, seed=11, seq_lens=lens), "cuda")
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    ws = api.decompress_kv(d["ckv_pool"], d["block_table"], d["seq_lens"], d["w_uk"], d["w_uv"],
                           dims)
    out1, lse1 = api.prefill_attention(d["q_c"], d["q_r"], d["kr_pool"], d["block_table"],
                                       d["seq_lens"], dims, ws)
    out2, lse2 = api.prefill(*_args(d))
    out3, lse3 = api.prefill(*_args(d))
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)
    assert torch.equal(out2, out3) and torch.equal(lse2, lse3)     # deterministic


def test_prefill_page_placement_is_invisible(api):
    # the same logical cache under another page permutation gives bitwise-equal results
    lens = (260, 190)
    w = _prefill_w(190, lens, 3)
    inp = make_inputs(w, seed=5, seq_lens=lens)
    out1, lse1 = api.prefill(*_args(to_device(inp, "cuda")))
    perm = torch.randperm(inp["ckv_pool"].shape[0], generator=torch.Generator().manual_seed(1))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(perm.numel())
    moved = dict(inp)
    moved["ckv_pool"] = inp["ckv_pool"][perm].contiguous()       # new page j holds old page perm[j]
    moved["kr_pool"] = inp["kr_pool"][perm].contiguous()
    tbl = inp["block_table"].clone()
    tbl[tbl >= 0] = inv[tbl[tbl >= 0].long()].to(torch.int32)
    moved["block_table"] = tbl
    out2, lse2 = api.prefill(*_args(to_device(moved, "cuda")))
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)


def test_attend_routes_by_query_count(api):
    assert api.route(256, 1) == "decompress" and api.route(100, 1) == "absorb"
    assert api.route(1, 128) == "absorb" and api.route(2, 64) == "absorb"
    assert api.route(2, 128) == "decompress"          # 256 query rows: beyond the absorbed kernels
    # one query per sequence (absorbed) and 300 queries (decompressed), same cache
    lens = (400, 310)
    for M in (1, 300):
        w = _prefill_w(M, lens, 8)
        inp = make_inputs(w, seed=M, seq_lens=lens)
        out, lse = api.attend(*_args(to_device(inp, "cuda")))
        torch.cuda.synchronize()
        assert api.get_device_error() == 0
        ref, lse_ref = oracle.prefill_decompress(*_args(inp))
        _check_prefill(_f64(out), ref, lens, M, f"attend M={M}")
        assert np.abs(_f64(lse) - lse_ref).max() <= LSE_ABS


def test_prefill_short_sequence_sets_bounds_error(api):
    # a length below the query count is a data error: recorded, the kernel still ends
    lens = (100, 100)
    w = _prefill_w(100, lens, 2)
    inp = make_inputs(w, seed=2, seq_lens=lens)
    d = to_device(inp, "cuda")
    d["seq_lens"] = torch.tensor([100, 50], dtype=torch.int32, device="cuda")
    api.prefill(*_args(d))
    torch.cuda.synchronize()
    assert api.get_device_error() == 4
    assert api.get_device_error() == 0


def _sample_rows(B, M, H, n_pairs, per_pair, seed):
    rng = np.random.default_rng(seed)
    pairs = rng.choice(B * H, size=n_pairs, replace=False)
    sel = []
    for ph in pairs:
        b, h = divmod(int(ph), H)
        qs = set(rng.choice(M, size=per_pair - 2, replace=False).tolist()) | {0, M - 1}
        sel += [(b * M + i) * H + h for i in sorted(qs)]
    return np.array(sorted(sel), dtype=np.int64)


def test_prefill_full_size_sampled(api):
    # batch 8, prompt 4096, 128 heads: the bench's workload and launch configuration
    w = workload("prefill")
    inp = make_inputs(w, seed=0)
    d = to_device(inp, "cuda")
    out, lse = api.prefill(*_args(d))
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    B, M, H = w.batch, w.n_q, w.heads
    sel = _sample_rows(B, M, H, n_pairs=10, per_pair=4, seed=0)
    ref, lse_ref = oracle.prefill_decompress(*_args(inp), sel=sel)
    got = _f64(out).reshape(-1, w.d_v)[sel]
    want = ref.reshape(-1, w.d_v)[sel]
    vis = (sel // H) % M + 1                                      # M = L: query i sees i + 1 keys
    many = vis >= 64
    _check(got[many], want[many], "prefill full size (sampled rows seeing >= 64 keys)")
    worst = (np.abs(got - want) / (MAX_ABS + 2.0 ** -7 * np.abs(want))).max()
    assert worst <= 1.0, f"prefill full size: worst err/bound {worst:.3f}"
    assert np.abs(_f64(lse).ravel()[sel] - lse_ref.ravel()[sel]).max() <= LSE_ABS
    assert torch.isfinite(out).all()
